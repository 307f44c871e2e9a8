"""The seeded input generator against its published definitions (SplitMix64,
Box-Muller) restated independently in numpy, and the workload recipes."""
import math

import numpy as np

import seeded_inputs as si


def test_u64_stream_matches_numpy_restatement():
    for seed, tid, start in ((25000, 1, 0), (25003, 5, 123456789), (7, 11, 2 ** 40)):
        np.testing.assert_array_equal(si.raw_u64(seed, tid, start, 1000),
                                      si.reference_u64(seed, tid, start, 1000))


def test_splitmix64_first_outputs_of_seed_zero():
    # SplitMix64 seeded with state 0 gives 0xE220A8397B1DCDAF as its first
    # output (Steele, Lea & Flood); check the finaliser and gamma directly
    gamma = np.uint64(0x9E3779B97F4A7C15)
    z = si._mix64_np(np.array([gamma], np.uint64))[0]
    assert int(z) == 0xE220A8397B1DCDAF


def test_normals_match_numpy_restatement():
    got = si.fill(25001, 3, 4097, start=11, dtype="f64")
    want = si.reference_normals(25001, 3, 11, 4097)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


def test_storage_rounding():
    f = si.fill(5, 2, 10000, std=0.1, dtype="f32")
    b = si.fill(5, 2, 10000, std=0.1, dtype="bf16")
    np.testing.assert_array_equal(b, si.f32_to_bf16_bits(f))
    d = si.fill(5, 2, 10000, std=0.1, dtype="f64")
    np.testing.assert_array_equal(f, d.astype(np.float32))


def test_moments_and_lognormal():
    z = si.fill(1, 1, 1_000_000, std=0.5, dtype="f64")
    assert abs(z.mean()) < 3e-3 and abs(z.std() - 0.5) < 3e-3
    t = si.fill(1, 9, 1_000_000, kind="lognormal", mean=0.0, std=0.5, dtype="f64")
    assert (t > 0).all()
    assert abs(np.log(t).mean()) < 3e-3 and abs(np.log(t).std() - 0.5) < 3e-3


def test_slices_are_independent_of_the_split():
    w = si.WORKLOADS["switch_top1_f32"].scaled("tiny", N=16, d=32, d_f=48, E=3)
    full = si.tensor(w, "W_g")
    for e in range(3):
        np.testing.assert_array_equal(si.tensor(w, "W_g", expert=e), full[e])
    whole = si.fill(9, 4, 1000)
    np.testing.assert_array_equal(si.fill(9, 4, 400, start=600), whole[600:])


def test_workload_recipes():
    w = si.WORKLOADS["qwen3_skew_bf16"]
    b = si.tensor(w, "b_r")
    # b_e = 0.5 ln(w_{e+1}), w_r proportional to r^-1.2 over 128 ranks
    H = sum(r ** -1.2 for r in range(1, 129))
    assert abs(b[0] - 0.5 * math.log(1 / H)) < 1e-6
    assert abs(b[127] - 0.5 * math.log(128 ** -1.2 / H)) < 1e-6
    assert (np.diff(b) < 0).all()
    wd = si.WORKLOADS["wdmoe_decode_bf16"]
    lat = si.tensor(wd, "lat")
    assert lat.shape == (64, 8) and lat.dtype == np.float32 and (lat > 0).all()
    small = wd.scaled("s", N=8, d=16, d_f=16)
    x = si.tensor(small, "x")
    assert x.dtype == np.uint16 and x.shape == (8, 16)
    assert si.tensor(si.WORKLOADS["mixtral_bf16"], "b_r") is None
