"""Fit the polynomial the attention kernel uses for part of its 2^x evaluations.

    python dit_attention_b200/csrc/fit_exp2.py [degree]

Method: 2^x = 2^j * 2^f with j = round(x) and f = x - j in [-1/2, 1/2]
(Cody & Waite style range reduction); 2^f is approximated by a polynomial
p(f) of the given degree with p(0) = 1 exactly, chosen to minimise the
maximum *relative* error on [-1/2, 1/2] by Remez-style exchange on a dense
grid (linear programming would do the same). The coefficients are rounded
to fp32 and the error of the rounded polynomial evaluated in fp32 Horner
form is reported. Output: C initialisers for the kernel.
"""
import sys

import numpy as np


def fit(deg: int, iters: int = 60):
    # unknowns c1..cdeg (c0 = 1); minimise max |p(f)/2^f - 1| with IRLS weights
    f = np.linspace(-0.5, 0.5, 20001)
    y = np.exp2(f)
    A = np.stack([f ** k for k in range(1, deg + 1)], axis=1) / y[:, None]
    b = 1.0 - 1.0 / y                     # want (1 + sum c_k f^k)/y - 1 = 0
    w = np.ones_like(f)
    best = None
    for _ in range(iters):
        sw = np.sqrt(w)
        c, *_ = np.linalg.lstsq(A * sw[:, None], b * sw, rcond=None)
        err = A @ c - b
        m = np.abs(err).max()
        if best is None or m < best[0]:
            best = (m, c)
        w = w * (np.abs(err) / m + 1e-3)   # Lawson's reweighting toward the minimax fit
        w /= w.mean()
    return np.concatenate([[1.0], best[1]])


def eval_fp32(coef32, f32):
    r = np.full_like(f32, coef32[-1])
    for c in coef32[-2::-1]:
        r = (r * f32 + c).astype(np.float32)
    return r


def main():
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 4
    c = fit(deg)
    c32 = c.astype(np.float32)
    f = np.linspace(-0.5, 0.5, 200001).astype(np.float32)
    rel = eval_fp32(c32, f).astype(np.float64) / np.exp2(f.astype(np.float64)) - 1
    print(f"// degree {deg}: max relative error {np.abs(rel).max():.3e} (fp32 Horner, f in [-1/2, 1/2])")
    print("// coefficients c0 .. c%d (fp32 hex, value):" % deg)
    for k, v in enumerate(c32):
        print(f"//   c{k} = {float(v):.9e}  ({np.float32(v).view(np.uint32):#010x})")
    print("{" + ", ".join(f"{float(v):.9e}f" for v in c32) + "}")


if __name__ == "__main__":
    main()
