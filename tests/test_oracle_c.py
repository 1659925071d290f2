"""The plain C twin of the oracle against the numpy oracle, plus direct pins.

Rotations and working vectors are compared bit for bit on fp16 inputs (every partial sum of the
transform is exact in float64, so evaluation order cannot matter).  Codes are compared exactly;
a difference would only be legitimate at a float64 distance tie broken differently by the two
summation orders, which the numpy oracle's matching walk would report as a near-tie, and none
occurs on these inputs.  Attention agrees to 1e-12 (float64, different summation orders)."""
import numpy as np
import pytest

from compressed_decode_attention_zkv_b200 import inputs as I
from oracle import c_oracle as C
from oracle import zkv_oracle as O


@pytest.fixture(scope="module", autouse=True)
def _built():
    C.lib()


@pytest.mark.parametrize("d", [1, 2, 8, 64, 128, 256])
def test_c_fwht_is_the_sylvester_matrix(d):
    eye = np.eye(d)
    H = C.fwht(eye, 1.0)                     # row j = H e_j = column j of H (H symmetric)
    np.testing.assert_array_equal(H, O.hadamard(d))
    np.testing.assert_array_equal(C.fwht(H, 1.0), d * eye)   # H H^T = d I, exactly
    x = np.random.default_rng(d).standard_normal((5, d)).astype(np.float16)
    np.testing.assert_array_equal(C.fwht(x, 1 / np.sqrt(d)), O.fwht(x, 1 / np.sqrt(d)))


@pytest.mark.parametrize("kind,smooth", [("k", False), ("v", False), ("k", True)])
def test_c_rvq_encode_equals_numpy_oracle(kind, smooth):
    wl = I.workload("tiny", n_cal=1024, kmeans_iters=3)
    books = I.train_codebooks(wl, kind)[0]
    x = I.kv_tokens(wl, kind, 0, 0, 300)[0]
    lam = I.key_smooth_factors(wl)[0] if smooth else None
    z_c, n_c, y_c = C.rvq_encode(x, books, smooth=lam)
    z_o, n_o, y_o, _ = O.rvq_encode(x, books, smooth=lam)
    if not smooth:
        np.testing.assert_array_equal(y_c, y_o)
    walk = O.rvq_match_walk(x, books, z_c, rel_gap=1e-12, smooth=lam)
    assert walk["mismatches"] == 0 and walk["exceptions"] == 0
    np.testing.assert_array_equal(z_c, z_o)
    np.testing.assert_allclose(n_c, n_o, rtol=1e-6, atol=0)


def test_c_greedy_equals_exhaustive_for_one_stage_and_disjoint_blocks():
    rng = np.random.default_rng(5)
    d, K = 8, 6
    # one stage: greedy is the exhaustive optimum
    C1 = rng.standard_normal((1, K, d)).astype(np.float32)
    y = rng.standard_normal(d).astype(np.float32)
    z, _, _ = C.rvq_encode(y[None], C1, rotate=False)
    best, _, _ = O.exhaustive_rvq(y, C1)
    assert tuple(z[0]) == best
    # stages on disjoint coordinate blocks: the objective separates, greedy is optimal
    C2 = np.zeros((2, K, d), np.float32)
    C2[0, :, :4] = rng.standard_normal((K, 4))
    C2[1, :, 4:] = rng.standard_normal((K, 4))
    z, _, _ = C.rvq_encode(y[None], C2, rotate=False)
    best, _, _ = O.exhaustive_rvq(y, C2)
    assert tuple(z[0]) == best


def test_c_rvq_special_cases():
    rng = np.random.default_rng(9)
    books = rng.standard_normal((3, 8, 16)).astype(np.float32)
    books[:, 0] = 0
    books[0, 5] = books[0, 3]                      # duplicate codeword: lower index wins
    x = np.stack([np.zeros(16, np.float32), books[0, 2], books[0, 5]])
    z, n, _ = C.rvq_encode(x, books, rotate=False)
    np.testing.assert_array_equal(z, [[0, 0, 0], [2, 0, 0], [3, 0, 0]])
    assert np.all(n[1:] == 0)
    y = rng.standard_normal((40, 16)).astype(np.float32)
    _, n, _ = C.rvq_encode(y, books, rotate=False)
    assert np.all(np.diff(n, axis=1) <= 0)         # codeword 0 = 0: norms never increase


def _decode_case(seed, d=64, Sk=2, Sv=3, smooth=True):
    rng = np.random.default_rng(seed)
    B, Hq, Hkv, Tcap, Wcap = 3, 4, 2, 40, 6
    q = rng.standard_normal((B, Hq, d)).astype(np.float16)
    kc = rng.integers(0, 16, (B, Hkv, Tcap, Sk)).astype(np.uint8)
    vc = rng.integers(0, 16, (B, Hkv, Tcap, Sv)).astype(np.uint8)
    Ck = (rng.standard_normal((Hkv, Sk, 16, d)) * 0.5).astype(np.float32)
    Cv = rng.standard_normal((Hkv, Sv, 16, d)).astype(np.float32)
    wk = rng.standard_normal((B, Hkv, Wcap, d)).astype(np.float16)
    wv = rng.standard_normal((B, Hkv, Wcap, d)).astype(np.float16)
    comp = np.array([37, 0, 0])
    win = np.array([5, 3, 0])
    lam = np.exp(rng.standard_normal((Hkv, d)) * 0.3).astype(np.float32) if smooth else None
    return (q, kc, vc, comp, Ck, Cv, wk, wv, win), lam


@pytest.mark.parametrize("smooth", [False, True])
def test_c_decode_equals_numpy_oracle(smooth):
    case, lam = _decode_case(3, smooth=smooth)
    o_c, l_c = C.decode_attn(*case, k_smooth=lam)
    o_o, l_o = O.decode_attn(*case, k_smooth=lam)
    np.testing.assert_allclose(o_c, o_o, atol=1e-12, rtol=0)
    fin = np.isfinite(l_o)
    assert np.array_equal(fin, np.isfinite(l_c)) and not fin[2].any()
    np.testing.assert_allclose(l_c[fin], l_o[fin], atol=1e-12, rtol=0)
    assert np.all(o_c[2] == 0)                     # empty context: out = 0, lse = -inf


def test_c_decode_pins():
    rng = np.random.default_rng(4)
    d = 32
    # q = 0: uniform weights, out = mean of the values; one key: out = that value
    Cv = rng.standard_normal((1, 1, 4, d)).astype(np.float32)
    Ck = rng.standard_normal((1, 1, 4, d)).astype(np.float32)
    vc = np.array([0, 1, 2, 3, 1], np.uint8).reshape(1, 1, 5, 1)
    kc = np.array([3, 2, 1, 0, 2], np.uint8).reshape(1, 1, 5, 1)
    none = np.zeros((1, 1, 1, d), np.float16)
    v_rot = O.fwht(Cv[0, 0], 1 / np.sqrt(d))
    out, lse = C.decode_attn(np.zeros((1, 1, d), np.float16), kc, vc, [5], Ck, Cv, none, none,
                             [0])
    np.testing.assert_allclose(out[0, 0], v_rot[[0, 1, 2, 3, 1]].mean(axis=0), atol=1e-13)
    assert lse[0, 0] == pytest.approx(np.log(5.0), abs=1e-13)
    q = rng.standard_normal((1, 1, d)).astype(np.float16)
    out, _ = C.decode_attn(q, kc, vc, [1], Ck, Cv, none, none, [0])
    np.testing.assert_allclose(out[0, 0], v_rot[0], atol=1e-13)


def test_c_lse_merge_equals_one_softmax():
    rng = np.random.default_rng(8)
    s = rng.standard_normal(30) * 3
    V = rng.standard_normal((30, 7))
    q_parts = [(0, 11), (11, 12), (12, 30)]
    parts = []
    for a, b in q_parts:
        p = np.exp(s[a:b] - s[a:b].max())
        parts.append(((p @ V[a:b]) / p.sum(), s[a:b].max() + np.log(p.sum())))
    parts.append((np.zeros(7), -np.inf))
    out, lse = C.lse_merge(parts)
    p = np.exp(s - s.max())
    np.testing.assert_allclose(out, (p @ V) / p.sum(), atol=1e-13)
    assert lse == pytest.approx(s.max() + np.log(p.sum()), abs=1e-13)
    o2, l2 = O.lse_merge(parts)
    np.testing.assert_allclose(out, o2, atol=1e-14)
    out, lse = C.lse_merge([(np.ones(3), -np.inf), (np.ones(3), -np.inf)])
    assert np.all(out == 0) and lse == -np.inf


@pytest.mark.parametrize("m,smooth", [(4, True), (8, False), (2, False)])
def test_c_pq_encode_equals_numpy_oracle(m, smooth):
    wl = I.workload("tiny", n_cal=1024, kmeans_iters=3)
    lam = I.key_smooth_factors(wl)[0] if smooth else None
    book = I.train_pq_codebook(wl, "k", m, smooth=None if lam is None else lam[None])[0]
    x = I.kv_tokens(wl, "k", 0, 0, 200)[0]
    z_c = C.pq_encode(x, book, smooth=lam)
    z_o, _ = O.pq_encode(x, book, smooth=lam)
    walk = O.pq_match_walk(x, book, z_c, rel_gap=1e-12, smooth=lam)
    assert walk["mismatches"] == 0 and walk["exceptions"] == 0
    np.testing.assert_array_equal(z_c, z_o)


@pytest.mark.parametrize("smooth", [False, True])
def test_c_pq_decode_equals_numpy_oracle(smooth):
    rng = np.random.default_rng(12)
    B, Hq, Hkv, d, m, Tcap, Wcap = 2, 6, 2, 32, 4, 30, 5
    kc = rng.integers(0, 256, (B, Hkv, Tcap, d // m)).astype(np.uint8)
    vc = rng.integers(0, 256, (B, Hkv, Tcap, d // m)).astype(np.uint8)
    Ck = (rng.standard_normal((Hkv, 256, m)) * 0.4).astype(np.float32)
    Cv = rng.standard_normal((Hkv, 256, m)).astype(np.float32)
    q = rng.standard_normal((B, Hq, d)).astype(np.float16)
    wk = rng.standard_normal((B, Hkv, Wcap, d)).astype(np.float16)
    wv = rng.standard_normal((B, Hkv, Wcap, d)).astype(np.float16)
    lam = np.exp(rng.standard_normal((Hkv, d)) * 0.3).astype(np.float32) if smooth else None
    case = (q, kc, vc, np.array([30, 7]), Ck, Cv, wk, wv, np.array([0, 5]))
    o_c, l_c = C.pq_decode_attn(*case, k_smooth=lam)
    o_o, l_o = O.pq_decode_attn(*case, k_smooth=lam)
    np.testing.assert_allclose(o_c, o_o, atol=1e-12, rtol=0)
    np.testing.assert_allclose(l_c, l_o, atol=1e-12, rtol=0)
