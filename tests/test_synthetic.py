"""The seeded input generator: published SplitMix64 outputs, determinism, rounding."""
import numpy as np

import synthetic as S


def test_splitmix64_published_sequence():
    # SplitMix64 started from state 0 (Steele, Lea, Flood 2014; the reference C code by Vigna)
    assert [S._mix((i + 1) * S.GOLDEN) for i in range(3)] == [
        0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]


def test_c_draws_match_definition():
    key = S.stream_key(7, 3)
    u = S.uniform_f32(7, 3, 64)
    ref = np.array([(S._mix(key + (i + 1) * S.GOLDEN) >> 11) * 2.0 ** -53 for i in range(64)], np.float32)
    np.testing.assert_array_equal(u, ref)
    # offsets address the same counter stream
    np.testing.assert_array_equal(S.uniform_f32(7, 3, 10, start=20), u[20:30])
    z = S.normal_f32(7, 3, 1 << 16).astype(np.float64)
    assert abs(z.mean()) < 0.02 and abs(z.std() - 1) < 0.02


def test_bf16_rounding_ties_to_even():
    # bf16 spacing is 2^-7 on [1, 2) and 2^-6 on [2, 4)
    x = np.array([1.0, 1.00390625, 1.01171875, np.nextafter(np.float32(1.00390625), np.float32(2)), -2.0078125, 3.0e38], np.float32)
    r = S.round_bf16(x)
    np.testing.assert_array_equal(r[:5], np.array([1.0, 1.0, 1.015625, 1.0078125, -2.0], np.float32))
    assert np.all(S.round_bf16(r) == r)
    assert np.all((r.view(np.uint32) & 0xFFFF) == 0)


def test_workloads_deterministic():
    cfg = S.CONFIGS["tiny_fp32"]
    a = S.make_mel(cfg); b = S.make_mel(cfg)
    np.testing.assert_array_equal(a, b)
    assert a.shape == (1, 128, 200) and a.min() >= -1.5 and a.max() < 1.5
    rg = S.CONFIGS["large_ragged_b64"]
    ln = S.make_lengths(rg)
    assert ln.shape == (64,) and ln.min() >= 500 and ln.max() <= 3000
    med = S.CONFIGS["medium_pool"].replace(n_layers=1)
    w = S.make_weights(med)
    assert np.all(S.round_bf16(w["layers.0.fc1_w"]) == w["layers.0.fc1_w"])
    assert abs(float(w["layers.0.fc1_w"].std()) - 0.02) < 1e-3
    assert abs(float(w["layers.0.ln1_g"].mean()) - 1.0) < 5e-3
