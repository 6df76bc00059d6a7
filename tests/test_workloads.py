"""Seeded input generator: determinism, slice independence, bf16 rounding. CPU only."""
import numpy as np

from workloads import PARITY_WORKLOADS, WORKLOADS, bf16_bits, generate, widen


def test_bf16_rounding_ties_to_even_and_exact_widening():
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 1.0 + 2 ** -9], np.float32)
    got = widen(bf16_bits(x), "bf16")
    # 1 + 2^-8 is a tie between 1 and 1 + 2^-7: ties go to the even mantissa (1.0);
    # 1 + 3*2^-8 ties between 1 + 2^-7 and 1 + 2^-6: even is 1 + 2^-6
    np.testing.assert_array_equal(got, np.array([1.0, 1.0, 1.0 + 2 ** -6, -2.5, 1.0], np.float32))
    y = np.random.default_rng(0).standard_normal(1000).astype(np.float32)
    r = widen(bf16_bits(y), "bf16")
    assert np.all(np.abs(r - y) <= np.abs(y) * 2 ** -8)
    np.testing.assert_array_equal(bf16_bits(r), bf16_bits(y))


def test_generation_is_deterministic_and_sliceable():
    w = PARITY_WORKLOADS["p_bf16_blk128"]
    a = generate(w)
    b = generate(w, threads=1)
    for n in "qkv":
        np.testing.assert_array_equal(a[n], b[n])
    part = generate(w, heads=[(1, 1)])
    G = w.G
    np.testing.assert_array_equal(part["k"][1, 1], a["k"][1, 1])
    np.testing.assert_array_equal(part["q"][1, G:2 * G], a["q"][1, G:2 * G])
    assert not part["k"][0].any()


def test_heavy_hitters_are_planted():
    w = PARITY_WORKLOADS["d_bf16_blk16"]
    x = generate(w)
    k = widen(x["k"], "bf16")
    norms = np.linalg.norm(k, axis=-1)
    n_hh = int(np.ceil(w.hh_frac * w.T))
    # planted keys have norm about 4*sqrt(d) + noise; typical keys about sqrt(d)
    big = (norms > 3 * np.sqrt(w.d)).sum(axis=-1)
    assert np.all(big == n_hh)


def test_headline_workload_shapes():
    assert WORKLOADS[3].T == 32768 and WORKLOADS[3].block == 128 and WORKLOADS[3].nb == 256
    assert WORKLOADS[5].Lq == 1 and WORKLOADS[5].nb == 8192 and WORKLOADS[5].B == 16
    assert WORKLOADS[2].nq == 128 and WORKLOADS[1].dtype == "f32"
