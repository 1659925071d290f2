"""The seeded input generators: determinism, slice consistency, codebook conventions."""
import numpy as np

from compressed_decode_attention_zkv_b200 import inputs as I


def test_kv_slices_are_consistent_and_deterministic():
    wl = I.workload("llama3_8b_32k", B=2, Hkv=2, Hq=8, T=300)
    a = I.kv_tokens(wl, "k", 1, 0, 300)
    b = I.kv_tokens(wl, "k", 1, 120, 300)
    np.testing.assert_array_equal(a[:, 120:], b)
    np.testing.assert_array_equal(a, I.kv_tokens(wl, "k", 1, 0, 300))
    assert a.dtype == np.float16 and a.shape == (2, 300, 128)
    assert not np.array_equal(a, I.kv_tokens(wl, "k", 0, 0, 300))


def test_channel_scales_have_outliers_on_keys_only():
    wl = I.workload("llama3_8b_32k")
    k = I.channel_scales(wl, "k")
    v = I.channel_scales(wl, "v")
    assert k.shape == (8, 128) and np.all(v == 1)
    # eight channels per head carry the x10 gain: they dominate the top of the range
    for h in range(8):
        assert np.sort(k[h])[-8:].min() > 2.0


def test_codebooks_zero_codeword_and_determinism():
    wl = I.workload("tiny", n_cal=1024, kmeans_iters=3)
    c1 = I.train_codebooks(wl, "k")
    c2 = I.train_codebooks(wl, "k")
    assert c1.shape == (1, 2, 256, 128) and c1.dtype == np.float32
    np.testing.assert_array_equal(c1, c2)
    assert np.all(c1[:, :, 0] == 0)
    assert np.all(np.isfinite(c1))


def test_random_codes_and_lengths():
    wl = I.workload("ragged_serving_64")
    lens = I.ragged_lengths(wl)
    assert lens.shape == (64,) and lens.min() >= 1024 and lens.max() <= 16384
    small = I.workload("llama3_8b_32k", B=2, Hkv=2, Hq=4)
    codes = I.random_codes(small, "k", 100)
    assert codes.shape == (2, 2, 100, 4) and codes.dtype == np.uint8


def test_key_smooth_factors_follow_the_oracle_definition():
    """The harness's calibrated lambda (an input of both sides) is the oracle's
    smooth_factors of the same calibration sample, bit for bit."""
    from oracle import zkv_oracle as O
    wl = I.workload("llama3_8b_32k", Hkv=2, n_cal=512)
    lam = I.key_smooth_factors(wl)
    assert lam.shape == (2, wl.d) and lam.dtype == np.float32
    for h in range(2):
        K = I._calibration_sample(wl, "k", h, wl.n_cal, I.SEED_CALIB)
        np.testing.assert_array_equal(lam[h], O.smooth_factors(K))
