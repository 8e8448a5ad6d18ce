"""The pins catch plausible mistakes in the oracle.

Each case below plants one mistake in a copy of oracle/oracle.c (a transposed
operand, a wrong sign, a dropped term, a wrong index or exponent), builds it
with the oracle's own recipe, and runs tests/test_oracle_pins.py against it in
a subprocess: at least one pin must fail. The unmodified source, built the
same way, must pass them all. Everything runs on the CPU.
"""
import os
import subprocess
import sys

import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "oracle.c")

MUTANTS = {
    "K transposed in QK^T": ("dot += at(q, qo + d) * at(k, ko + j * D + d);",
                             "dot += at(q, qo + d) * at(k, ko + d * Skv + j);"),
    "V transposed in PV": ("out[d] += p[j] * at(v, ko + j * D + d);",
                           "out[d] += p[j] * at(v, ko + d * Skv + j);"),
    "scale applied twice": ("p[j] = scale * dot;", "p[j] = scale * scale * dot;"),
    "max not subtracted": ("p[j] = exp(p[j] - m);", "p[j] = exp(p[j]);"),
    "normalisation dropped": ("for (int64_t d = 0; d < D; ++d) out[d] /= l;", ""),
    "lse without the max": ("*lse = m + log(l);", "*lse = log(l);"),
    "merge weights swapped": ("(wa * oa[r * D + d] + wb * ob[r * D + d])",
                              "(wb * oa[r * D + d] + wa * ob[r * D + d])"),
    "rope rotation sign": ("row[base[a] + 2 * j] = x0 * c - x1 * s;", "row[base[a] + 2 * j] = x0 * c + x1 * s;"),
    "rope h and w swapped": ("pos[1] = (n / Ww) % Hh;\n    pos[2] = n % Ww;",
                             "pos[1] = n % Ww;\n    pos[2] = (n / Ww) % Hh;"),
    "rope frequency exponent": ("-2.0 * (double)j / (double)width[a]", "-1.0 * (double)j / (double)width[a]"),
    "bwd: delta dropped": ("dS[i * Skv + j] = P[i * Skv + j] * (dS[i * Skv + j] - delta);",
                           "dS[i * Skv + j] = P[i * Skv + j] * dS[i * Skv + j];"),
    "bwd: dK without scale": ("dk[j * D + d] += scale * dS[i * Skv + j] * at(q, qo + i * D + d);",
                              "dk[j * D + d] += dS[i * Skv + j] * at(q, qo + i * D + d);"),
    "block bwd: lse not subtracted": ("const double p = exp(scale * s - lse[i]);", "const double p = exp(scale * s);"),
    "block bwd: delta dropped": ("const double ds = p * (dp - delta);", "const double ds = p * dp;"),
    "bwd: dV uses dS": ("dv[j * D + d] += P[i * Skv + j] * at(dout, doo + i * D + d);",
                        "dv[j * D + d] += dS[i * Skv + j] * at(dout, doo + i * D + d);"),
    "rope bwd: forward rotation used": ("row[base[a] + 2 * j + 1] = c * x1 - s * x0;",
                                        "row[base[a] + 2 * j + 1] = c * x1 + s * x0;"),
    "e4m3 mantissa width": ("double ulp = ldexp(1.0, e - 3);", "double ulp = ldexp(1.0, e - 2);"),
    "e4m3 quantiser scale not inverted": ("inv = 448.0f / amax;", "inv = amax / 448.0f;"),
    "proj: norm over the sum, not the mean": ("ms /= (double)D;", ""),
    "proj: out-proj head and position swapped": ("acc += oracle_bf16_to_f64(O[((b * H + h) * S + s) * D + d]) *",
                                                 "acc += oracle_bf16_to_f64(O[((b * S + s) * H + h) * D + d]) *"),
    "proj: rope on v too": ("                } else {\n                    for (int64_t d = 0; d < D; ++d) o[d] = src[d];",
                            "                } else {\n                    for (int64_t d = 0; d < D; ++d) o[d] = src[d];\n                    rope_row(o, tok % S, Hh, Ww, D, theta, 0);"),
    "rope pair partner index": ("double x1 = row[base[a] + 2 * j + 1];", "double x1 = row[base[a] + j + 1];"),
}


def _run_pins(lib_path):
    env = dict(os.environ, ORACLE_LIB=lib_path)
    res = subprocess.run([sys.executable, "-m", "pytest", os.path.join(ROOT, "tests", "test_oracle_pins.py"),
                          "-x", "-q", "-p", "no:cacheprovider"], cwd=ROOT, env=env, capture_output=True, text=True,
                         timeout=600)
    return res.returncode, res.stdout[-2000:]


def _build(tmp_path, name, text):
    src = tmp_path / f"{name}.c"
    src.write_text(text)
    return oracle.compile_library(str(src), str(tmp_path / f"lib{name}.so"))


def test_unmodified_oracle_passes_its_pins(tmp_path):
    rc, out = _run_pins(_build(tmp_path, "clean", open(SRC).read()))
    assert rc == 0, out


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(tmp_path, name):
    old, new = MUTANTS[name]
    text = open(SRC).read()
    assert text.count(old) == 1, f"mutation target not found once: {old!r}"
    rc, out = _run_pins(_build(tmp_path, "mutant", text.replace(old, new)))
    assert rc != 0, f"no pin caught the planted mistake '{name}'"
