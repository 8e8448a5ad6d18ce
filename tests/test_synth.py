"""The seeded input generator: determinism, distribution, structure."""
import numpy as np

from dit_attention_b200 import synth


def test_splitmix64_reference_values():
    # splitmix64 from state 0: the first outputs of the published generator
    # (Vigna's reference splitmix64.c with x = 0).
    out = synth.splitmix64(np.uint64(0), 0, 3)
    assert [int(v) for v in out] == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]


def test_counter_based_and_deterministic():
    a = synth.normal(7, 1, 1001)
    b = synth.normal(7, 1, 1001)
    np.testing.assert_array_equal(a, b)
    assert not np.array_equal(a, synth.normal(7, 2, 1001))
    key = synth.stream_key(3, 0)
    np.testing.assert_array_equal(synth.splitmix64(key, 10, 5), synth.splitmix64(key, 0, 15)[10:])


def test_normal_moments():
    z = synth.normal(0, 0, 1 << 20)
    assert abs(z.mean()) < 5e-3
    assert abs(z.std() - 1) < 5e-3
    assert abs(np.mean(z ** 4) - 3) < 0.05


def test_rmsnorm_rows():
    x = synth.normal(0, 0, 64 * 128).reshape(64, 128) * 5
    y = synth.rmsnorm_rows(x)
    np.testing.assert_allclose(np.mean(y * y, -1), 1.0 / (1.0 + 1e-6 / np.mean(x * x, -1)), rtol=1e-12)


def test_workload_inputs_structure():
    w = synth.Workload("t", B=1, H=2, D=16, Sq=300, Skv=300, seed=4, q_mult=4.0, spike_mult=8.0,
                       spike_frac=0.01)
    q, k, v = synth.make_inputs(w)
    assert q.shape == (1, 2, 300, 16) and q.dtype == np.uint16
    plain = synth.Workload("t", B=1, H=2, D=16, Sq=300, Skv=300, seed=4)
    q0, k0, v0 = synth.make_inputs(plain)
    np.testing.assert_array_equal(synth.bf16_bits_to_f64(q), 4 * synth.bf16_bits_to_f64(q0))
    kk = synth.bf16_bits_to_f64(k).reshape(2, 300, 16)
    kk0 = synth.bf16_bits_to_f64(k0).reshape(2, 300, 16)
    for bh in range(2):
        rows = synth.spike_rows(4, bh, 300, 3)
        assert len(set(rows.tolist())) == 3
        np.testing.assert_array_equal(kk[bh, rows], 8 * kk0[bh, rows])
        rest = np.setdiff1d(np.arange(300), rows)
        np.testing.assert_array_equal(kk[bh, rest], kk0[bh, rest])
    np.testing.assert_array_equal(v, v0)


def test_named_workloads():
    W = synth.WORKLOADS
    assert W["win77_s31200"].Sq == 20 * 30 * 52 == 31200
    assert W["win25_s10920"].Sq == 7 * 30 * 52 == 10920
    assert W["cross_s31200_kv2072"].Skv == 1560 + 512
    assert W["stress_s10920"].spike_count == 109
    assert abs(W["win77_s31200"].flops - 4 * 40 * 31200 ** 2 * 128) < 1
