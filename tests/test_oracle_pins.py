"""Pins of the CPU oracle against what the pages and the mathematics fix (no GPU).

Each test checks the oracle against something other than itself: a hand-worked example, an
independently built matrix, a library routine, a closed form, an invariant, or brute force.
"""
import math
from fractions import Fraction

import numpy as np
import pytest
import scipy.linalg
import torch

from oracle import zkv_oracle as O

GOLDEN = __import__("os").path.join(__import__("os").path.dirname(__file__), "golden")


def _read_fixture(name):
    vals = {}
    with open(f"{GOLDEN}/{name}") as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, rest = line.split(":", 1)
            if "|" in rest:
                vals[key] = np.array([[float(t) for t in part.split()] for part in rest.split("|")])
            else:
                vals[key] = np.array([float(t) for t in rest.split()])
    return vals


# ------------------------------------------------------------------ Hadamard / FWHT

def _sylvester_by_recursion(d):
    H = np.array([[1.0]])
    while H.shape[0] < d:
        H = np.block([[H, H], [H, -H]])
    return H


@pytest.mark.parametrize("d", [1, 2, 4, 8, 16, 64, 128, 256])
def test_hadamard_equals_sylvester_recursion_and_scipy(d):
    H = O.hadamard(d)
    np.testing.assert_array_equal(H, _sylvester_by_recursion(d))
    np.testing.assert_array_equal(H, scipy.linalg.hadamard(d).astype(float))


@pytest.mark.parametrize("d", [4, 64, 128, 256])
def test_hadamard_orthogonality_exact(d):
    H = O.hadamard(d)
    np.testing.assert_array_equal(H @ H.T, d * np.eye(d))


def test_hadamard_rejects_non_power_of_two():
    with pytest.raises(ValueError):
        O.hadamard(12)


@pytest.mark.parametrize("d", [64, 128, 256])
def test_fwht_columns_and_e0(d):
    E = np.eye(d)
    # Transform of basis vectors gives the matrix columns; e0 maps to all ones.
    cols = O.fwht(E, 1.0)
    np.testing.assert_array_equal(cols, _sylvester_by_recursion(d).T)
    np.testing.assert_array_equal(O.fwht(E[0], 1.0), np.ones(d))


@pytest.mark.parametrize("d", [64, 128, 256])
def test_fwht_involution_and_parseval(d):
    rng = np.random.default_rng(5)
    x = rng.standard_normal((7, d))
    s = 1.0 / math.sqrt(d)
    y = O.fwht(x, s)
    np.testing.assert_allclose(O.fwht(y, s), x, atol=1e-12)
    np.testing.assert_allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), rtol=1e-13)


def test_rotation_is_exact_transform_rounded_once():
    # For fp16 inputs: exact integer-rational H x (Fractions), times 1/sqrt(d) in float64,
    # rounded once to float32, must equal the oracle's working vector bit for bit.
    rng = np.random.default_rng(11)
    d = 128
    x = (rng.standard_normal((5, d)) * np.exp(rng.uniform(-8, 6, (5, d)))).astype(np.float16)
    H = _sylvester_by_recursion(d).astype(int)
    s = 1.0 / math.sqrt(d)
    got = O.rotate_to_f32(x)
    for n in range(x.shape[0]):
        fr = [Fraction(float(v)) for v in x[n]]
        for i in range(d):
            exact = sum((fr[j] if H[i, j] > 0 else -fr[j]) for j in range(d))
            want = np.float32(float(exact) * s)
            assert got[n, i] == want


# ------------------------------------------------------------------ greedy RVQ

def test_rvq_hand_example():
    g = _read_fixture("rvq_hand_d4.txt")
    books = np.stack([g["stage0"], g["stage1"]]).astype(np.float32)
    x = g["x"].astype(np.float16)[None]
    codes, norms, y, r = O.rvq_encode(x, books)
    np.testing.assert_array_equal(y[0], g["y"])
    np.testing.assert_array_equal(codes[0], g["codes"])
    np.testing.assert_array_equal(norms[0], g["norms"])
    np.testing.assert_array_equal(O.reconstruct(codes, books)[0], g["xhat_rot"])
    np.testing.assert_allclose(O.reconstruct(codes, books, unrotate=True)[0], g["xhat"],
                               atol=1e-12)


def _tiny_books(rng, S, K, d, zero0=True):
    C = rng.standard_normal((S, K, d)).astype(np.float32)
    if zero0:
        C[:, 0] = 0
    return C


def test_rvq_single_stage_equals_exhaustive():
    rng = np.random.default_rng(1)
    C = _tiny_books(rng, 1, 8, 8)
    y = rng.standard_normal((20, 8)).astype(np.float32)
    codes, _, _, _ = O.rvq_encode(y, C, rotate=False)
    for n in range(20):
        best, _, _ = O.exhaustive_rvq(y[n], C)
        assert codes[n, 0] == best[0]


def test_rvq_disjoint_blocks_greedy_is_joint_optimum():
    # Stage s only moves coordinates of block s, so the distortion separates over stages and
    # the greedy stage-wise choice is the joint optimum over all K^S combinations.
    rng = np.random.default_rng(2)
    S, K, d = 3, 6, 6
    C = np.zeros((S, K, d), np.float32)
    for s in range(S):
        C[s, 1:, 2 * s:2 * s + 2] = rng.standard_normal((K - 1, 2)).astype(np.float32)
    y = rng.standard_normal((15, d)).astype(np.float32)
    codes, _, _, _ = O.rvq_encode(y, C, rotate=False)
    for n in range(15):
        best, best_d, _ = O.exhaustive_rvq(y[n], C)
        assert tuple(int(c) for c in codes[n]) == best
        xh = O.reconstruct(codes[n][None], C)[0]
        assert abs(((y[n] - xh) ** 2).sum() - best_d) < 1e-9


def test_rvq_greedy_is_stagewise_min_and_bounded_by_joint_optimum():
    rng = np.random.default_rng(3)
    S, K, d = 3, 5, 6
    C = _tiny_books(rng, S, K, d)
    y = rng.standard_normal((12, d)).astype(np.float32)
    codes, norms, _, _ = O.rvq_encode(y, C, rotate=False)
    for n in range(12):
        _, best_d, table = O.exhaustive_rvq(y[n], C)
        # Brute-force greedy: at each stage the first combination prefix that minimises the
        # partial distortion, written with explicit loops.
        prefix = []
        r = y[n].astype(np.float32)
        for s in range(S):
            dists = []
            for c in range(K):
                acc = 0.0
                for i in range(d):
                    diff = float(r[i]) - float(C[s, c, i])
                    acc += diff * diff
                dists.append(acc)
            z = min(range(K), key=lambda c: (dists[c], c))
            prefix.append(z)
            r = (r - C[s, z]).astype(np.float32)
        assert tuple(int(c) for c in codes[n]) == tuple(prefix)
        assert table[tuple(prefix)] >= best_d - 1e-12
        assert abs(float(norms[n, -1]) - math.sqrt(float((r.astype(np.float64) ** 2).sum()))) < 1e-6


def test_rvq_norms_never_increase_with_zero_codeword():
    rng = np.random.default_rng(4)
    C = _tiny_books(rng, 6, 32, 16)
    y = (3 * rng.standard_normal((200, 16))).astype(np.float32)
    _, norms, yy, _ = O.rvq_encode(y, C, rotate=False)
    n0 = np.linalg.norm(yy.astype(np.float64), axis=1)
    allnorms = np.concatenate([n0[:, None], norms.astype(np.float64)], axis=1)
    assert np.all(np.diff(allnorms, axis=1) <= 1e-6)


def test_rvq_exact_codeword_then_zeros():
    rng = np.random.default_rng(6)
    C = _tiny_books(rng, 4, 16, 8)
    y = C[0, 9][None].copy()
    codes, norms, _, _ = O.rvq_encode(y, C, rotate=False)
    assert list(codes[0]) == [9, 0, 0, 0]
    assert np.all(norms[0] == 0)


def test_rvq_zero_input_gives_zero_codes():
    rng = np.random.default_rng(7)
    C = _tiny_books(rng, 3, 16, 128)
    codes, norms, _, _ = O.rvq_encode(np.zeros((2, 128), np.float16), C)
    assert np.all(codes == 0) and np.all(norms == 0)


def test_rvq_duplicate_codewords_pick_lowest_index():
    rng = np.random.default_rng(8)
    C = _tiny_books(rng, 1, 8, 4)
    C[0, 5] = C[0, 2]
    y = (C[0, 2] + 1e-3).astype(np.float32)[None]
    codes, _, _, _ = O.rvq_encode(y, C, rotate=False)
    assert codes[0, 0] == 2


def test_reconstruction_plus_residual_is_rotated_input():
    rng = np.random.default_rng(9)
    C = _tiny_books(rng, 4, 64, 128)
    x = rng.standard_normal((50, 128)).astype(np.float16)
    codes, _, y, r = O.rvq_encode(x, C)
    xh = O.reconstruct(codes, C)
    np.testing.assert_allclose(xh + r, y, atol=1e-5)


def test_match_walk_counts_mismatch_and_near_tie():
    rng = np.random.default_rng(10)
    C = _tiny_books(rng, 2, 16, 8)
    y = rng.standard_normal((30, 8)).astype(np.float32)
    codes, _, _, _ = O.rvq_encode(y, C, rotate=False)
    res = O.rvq_match_walk(y, C, codes, rotate=False)
    assert res["mismatches"] == 0 and res["exceptions"] == 0 and res["exact"] == 60
    bad = codes.copy()
    bad[3, 0] = (bad[3, 0] + 1) % 16
    res = O.rvq_match_walk(y, C, bad, rotate=False)
    assert res["mismatches"] >= 1
    # A near tie: codeword 7 moved to within a 1e-7 relative distance of the winner's.
    y1 = y[:1].copy()
    z = int(codes[0, 0])
    alt = 7 if z != 7 else 6
    C2 = C.copy()
    C2[0, alt] = C2[0, z]
    C2[0, alt, 0] += np.float32(1e-6)
    c2, _, _, _ = O.rvq_encode(y1, C2, rotate=False)
    planted = c2.copy()
    planted[0, 0] = alt if c2[0, 0] == z else z
    res = O.rvq_match_walk(y1, C2, planted, rotate=False)
    assert res["exceptions"] == 1 and res["mismatches"] == 0


# ------------------------------------------------------------------ attention and combine

def _rand_decode_case(rng, B=2, Hq=4, Hkv=2, d=64, Tcap=40, Wcap=8, Sk=2, Sv=3, K=16,
                      comp=None, win=None):
    q = rng.standard_normal((B, Hq, d)).astype(np.float16)
    kc = rng.integers(0, K, (B, Hkv, Tcap, Sk)).astype(np.uint8)
    vc = rng.integers(0, K, (B, Hkv, Tcap, Sv)).astype(np.uint8)
    Ck = (rng.standard_normal((Hkv, Sk, K, d)) * 0.7).astype(np.float32)
    Cv = rng.standard_normal((Hkv, Sv, K, d)).astype(np.float32)
    Ck[:, :, 0] = 0
    Cv[:, :, 0] = 0
    wk = rng.standard_normal((B, Hkv, Wcap, d)).astype(np.float16)
    wv = rng.standard_normal((B, Hkv, Wcap, d)).astype(np.float16)
    comp = np.full(B, Tcap) if comp is None else np.asarray(comp)
    win = np.full(B, Wcap) if win is None else np.asarray(win)
    return q, kc, vc, comp, Ck, Cv, wk, wv, win


@pytest.mark.parametrize("comp,win", [([40, 17], [8, 3]), ([0, 40], [8, 8]), ([40, 5], [0, 0]),
                                      ([1, 0], [0, 1])])
def test_decode_direct_equals_lut_form(comp, win):
    rng = np.random.default_rng(20)
    case = _rand_decode_case(rng, comp=comp, win=win)
    o1, l1 = O.decode_attn(*case)
    o2, l2 = O.decode_attn_lut(*case)
    np.testing.assert_allclose(o2, o1, atol=1e-9, rtol=0)
    np.testing.assert_allclose(l2, l1, atol=1e-9, rtol=0)


def test_decode_matches_torch_sdpa_on_explicit_keys():
    # Keys and values built here with explicit loops and scipy's Hadamard, then torch's
    # scaled-dot-product attention in float64.
    rng = np.random.default_rng(21)
    q, kc, vc, comp, Ck, Cv, wk, wv, win = _rand_decode_case(rng, comp=[33, 40], win=[5, 8])
    out, lse = O.decode_attn(q, kc, vc, comp, Ck, Cv, wk, wv, win)
    B, Hq, d = q.shape
    Hkv = kc.shape[1]
    G = Hq // Hkv
    Hn = scipy.linalg.hadamard(d) / math.sqrt(d)
    for b in range(B):
        for h in range(Hq):
            kvh = h // G
            keys, vals = [], []
            for t in range(comp[b]):
                kr = np.zeros(d)
                vr = np.zeros(d)
                for s in range(kc.shape[3]):
                    kr += Ck[kvh, s, kc[b, kvh, t, s]]
                for s in range(vc.shape[3]):
                    vr += Cv[kvh, s, vc[b, kvh, t, s]]
                keys.append(Hn @ kr)
                vals.append(Hn @ vr)
            for t in range(win[b]):
                keys.append(wk[b, kvh, t].astype(np.float64))
                vals.append(wv[b, kvh, t].astype(np.float64))
            Kt = torch.tensor(np.array(keys))[None, None]
            Vt = torch.tensor(np.array(vals))[None, None]
            qt = torch.tensor(q[b, h].astype(np.float64))[None, None, None]
            ref = torch.nn.functional.scaled_dot_product_attention(qt, Kt, Vt)[0, 0, 0].numpy()
            np.testing.assert_allclose(out[b, h], ref, atol=1e-12)
            sc = (np.array(keys) @ q[b, h].astype(np.float64)) / math.sqrt(d)
            assert abs(lse[b, h] - scipy.special.logsumexp(sc)) < 1e-12


def test_decode_hand_example():
    g = _read_fixture("decode_hand_d4.txt")
    d = 4
    q = g["q"].astype(np.float16).reshape(1, 1, d)
    Ck = g["ck"].astype(np.float32).reshape(1, 1, 2, d)
    Cv = g["cv"].astype(np.float32).reshape(1, 1, 2, d)
    kc = g["k_codes"].astype(np.uint8).reshape(1, 1, 2, 1)
    vc = g["v_codes"].astype(np.uint8).reshape(1, 1, 2, 1)
    wk = g["win_k"].astype(np.float16).reshape(1, 1, 1, d)
    wv = g["win_v"].astype(np.float16).reshape(1, 1, 1, d)
    e2 = math.exp(2.0)
    want = np.array([e2 + 4, -e2, e2, -e2]) / (e2 + 2)
    for fn in (O.decode_attn, O.decode_attn_lut):
        out, lse = fn(q, kc, vc, [2], Ck, Cv, wk, wv, [1])
        np.testing.assert_allclose(out[0, 0], want, atol=1e-14)
        assert abs(lse[0, 0] - math.log(e2 + 2)) < 1e-14


def test_decode_zero_query_gives_mean_of_values():
    rng = np.random.default_rng(22)
    q, kc, vc, comp, Ck, Cv, wk, wv, win = _rand_decode_case(rng, comp=[40, 12], win=[8, 2])
    q[:] = 0
    out, lse = O.decode_attn(q, kc, vc, comp, Ck, Cv, wk, wv, win)
    for b in range(2):
        for h in range(4):
            kvh = h // 2
            vals = list(O.reconstruct(vc[b, kvh, :comp[b]], Cv[kvh], unrotate=True))
            vals += list(wv[b, kvh, :win[b]].astype(np.float64))
            np.testing.assert_allclose(out[b, h], np.mean(vals, axis=0), atol=1e-12)
            assert abs(lse[b, h] - math.log(comp[b] + win[b])) < 1e-12


def test_decode_single_token_returns_its_value():
    rng = np.random.default_rng(23)
    q, kc, vc, comp, Ck, Cv, wk, wv, win = _rand_decode_case(rng, comp=[1, 0], win=[0, 1])
    out, _ = O.decode_attn(q, kc, vc, comp, Ck, Cv, wk, wv, win)
    for h in range(4):
        kvh = h // 2
        want = O.reconstruct(vc[0, kvh, :1], Cv[kvh], unrotate=True)[0]
        np.testing.assert_allclose(out[0, h], want, atol=1e-12)
        np.testing.assert_allclose(out[1, h], wv[1, kvh, 0].astype(np.float64), atol=0)


def test_decode_empty_context():
    rng = np.random.default_rng(24)
    case = list(_rand_decode_case(rng, comp=[0, 0], win=[0, 0]))
    for fn in (O.decode_attn, O.decode_attn_lut):
        out, lse = fn(*case)
        assert np.all(out == 0) and np.all(np.isneginf(lse))


def test_lse_merge_equals_softmax_over_concatenation():
    rng = np.random.default_rng(25)
    d = 16
    q = rng.standard_normal(d)
    K = rng.standard_normal((30, d)) * 2
    V = rng.standard_normal((30, d))
    full = O.softmax_attention(q, K, V, 0.25)
    for cuts in ([10], [3, 17], [1, 2, 29], [0, 30]):
        idx = [0] + cuts + [30]
        parts = [O.softmax_attention(q, K[a:b], V[a:b], 0.25) for a, b in zip(idx[:-1], idx[1:])]
        o, l = O.lse_merge(parts)
        np.testing.assert_allclose(o, full[0], atol=1e-12)
        assert abs(l - full[1]) < 1e-12
    # associativity: ((a, b), c) == (a, (b, c))
    pa, pb, pc = (O.softmax_attention(q, K[a:b], V[a:b], 0.25) for a, b in ((0, 9), (9, 20), (20, 30)))
    left = O.lse_merge([O.lse_merge([pa, pb]), pc])
    right = O.lse_merge([pa, O.lse_merge([pb, pc])])
    np.testing.assert_allclose(left[0], right[0], atol=1e-12)
    assert abs(left[1] - right[1]) < 1e-12
    # all-empty parts
    o, l = O.lse_merge([(np.zeros(d), -np.inf), (np.zeros(d), -np.inf)])
    assert np.all(o == 0) and np.isneginf(l)


# ------------------------------------------------------------------ serving step

def test_append_step_window_then_eviction():
    rng = np.random.default_rng(30)
    B, Hkv, Wcap, d, Tcap, S, K = 2, 2, 3, 64, 8, 2, 16
    Ck = _tiny_books(rng, S, K, d)[None].repeat(Hkv, 0)
    Cv = _tiny_books(rng, S, K, d)[None].repeat(Hkv, 0)
    st = dict(k_codes=np.zeros((B, Hkv, Tcap, S), np.uint8),
              v_codes=np.zeros((B, Hkv, Tcap, S), np.uint8),
              comp_len=np.array([0, 5]), win_k=np.zeros((B, Hkv, Wcap, d), np.float16),
              win_v=np.zeros((B, Hkv, Wcap, d), np.float16), win_len=np.array([1, 3]),
              win_head=np.array([0, 1]), Ck=Ck, Cv=Cv)
    st["win_k"][1] = rng.standard_normal((Hkv, Wcap, d))
    st["win_v"][1] = rng.standard_normal((Hkv, Wcap, d))
    nk = rng.standard_normal((B, Hkv, d)).astype(np.float16)
    nv = rng.standard_normal((B, Hkv, d)).astype(np.float16)
    out = O.append_step(st, nk, nv)
    # Sequence 0: window not full -> slot 1, nothing encoded.
    assert out["win_len"][0] == 2 and out["comp_len"][0] == 0
    np.testing.assert_array_equal(out["win_k"][0, :, 1], nk[0])
    # Sequence 1: full -> slot 1 evicted and encoded at position 5.
    assert out["comp_len"][1] == 6 and out["win_head"][1] == 2 and out["win_len"][1] == 3
    for h in range(Hkv):
        zk, _, _, _ = O.rvq_encode(st["win_k"][1, h, 1][None], Ck[h])
        zv, _, _, _ = O.rvq_encode(st["win_v"][1, h, 1][None], Cv[h])
        np.testing.assert_array_equal(out["k_codes"][1, h, 5], zk[0])
        np.testing.assert_array_equal(out["v_codes"][1, h, 5], zv[0])
    np.testing.assert_array_equal(out["win_v"][1, :, 1], nv[1])
    # The caller's state is untouched.
    assert st["comp_len"][1] == 5


def test_append_step_product_vq_encodes_the_evicted_token():
    """With pq=True the evicted token is product-VQ encoded (keys smoothed, values not) to
    position comp_len; the window rule is the RVQ one."""
    rng = np.random.default_rng(32)
    B, Hkv, Wcap, d, m, Tcap = 2, 2, 2, 16, 4, 6
    Ck = rng.standard_normal((Hkv, 256, m)).astype(np.float32)
    Cv = rng.standard_normal((Hkv, 256, m)).astype(np.float32)
    lam = np.exp(rng.standard_normal((Hkv, d)) * 0.3).astype(np.float32)
    st = dict(k_codes=np.zeros((B, Hkv, Tcap, d // m), np.uint8),
              v_codes=np.zeros((B, Hkv, Tcap, d // m), np.uint8), comp_len=np.array([3, 0]),
              win_k=rng.standard_normal((B, Hkv, Wcap, d)).astype(np.float16),
              win_v=rng.standard_normal((B, Hkv, Wcap, d)).astype(np.float16),
              win_len=np.array([2, 1]), win_head=np.array([1, 0]), Ck=Ck, Cv=Cv, k_smooth=lam)
    nk = rng.standard_normal((B, Hkv, d)).astype(np.float16)
    nv = rng.standard_normal((B, Hkv, d)).astype(np.float16)
    out = O.append_step(st, nk, nv, pq=True)
    assert out["comp_len"].tolist() == [4, 0] and out["win_len"].tolist() == [2, 2]
    assert out["win_head"].tolist() == [0, 0]
    for h in range(Hkv):
        zk, _ = O.pq_encode(st["win_k"][0, h, 1][None], Ck[h], smooth=lam[h])
        zv, _ = O.pq_encode(st["win_v"][0, h, 1][None], Cv[h])
        np.testing.assert_array_equal(out["k_codes"][0, h, 3], zk[0])
        np.testing.assert_array_equal(out["v_codes"][0, h, 3], zv[0])
        zk_plain, _ = O.pq_encode(st["win_k"][0, h, 1][None], Ck[h])
        assert not np.array_equal(zk_plain[0], zk[0])   # the smoothing was applied
    np.testing.assert_array_equal(out["win_k"][0, :, 1], nk[0])
    np.testing.assert_array_equal(out["win_v"][1, :, 1], nv[1])
    assert not out["error"]


def test_append_step_at_capacity_leaves_sequence_unchanged():
    rng = np.random.default_rng(31)
    B, Hkv, Wcap, d, Tcap, S, K = 1, 1, 2, 64, 4, 1, 8
    C = _tiny_books(rng, S, K, d)[None]
    st = dict(k_codes=np.zeros((B, Hkv, Tcap, S), np.uint8),
              v_codes=np.zeros((B, Hkv, Tcap, S), np.uint8), comp_len=np.array([Tcap]),
              win_k=rng.standard_normal((B, Hkv, Wcap, d)).astype(np.float16),
              win_v=rng.standard_normal((B, Hkv, Wcap, d)).astype(np.float16),
              win_len=np.array([Wcap]), win_head=np.array([1]), Ck=C, Cv=C)
    out = O.append_step(st, np.ones((B, Hkv, d), np.float16), np.ones((B, Hkv, d), np.float16))
    assert out["error"]
    for k in ("k_codes", "v_codes", "comp_len", "win_k", "win_v", "win_len", "win_head"):
        np.testing.assert_array_equal(out[k], st[k])


# ------------------------------------------------------------------ smooth scaling (VecInfer)

def test_smooth_factors_hand_example():
    # lambda_i = sqrt(max_t |K[t, i]|); an all-zero channel gets 1
    K = np.array([[1.0, -4.0, 0.0, 0.25], [-2.0, 3.0, 0.0, -0.0625]])
    lam = O.smooth_factors(K)
    assert lam.dtype == np.float32
    np.testing.assert_array_equal(lam, np.array([math.sqrt(2.0), 2.0, 1.0, 0.5], np.float32))


def test_smoothing_flattens_channel_ranges():
    # after division by lambda every nonzero channel's largest magnitude is sqrt(max |K_i|)
    rng = np.random.default_rng(40)
    K = rng.standard_normal((300, 16)) * np.exp(rng.standard_normal(16) * 2)
    lam = O.smooth_factors(K).astype(np.float64)
    peak = np.abs(O.smooth_keys(K, lam)).max(axis=0)
    np.testing.assert_allclose(peak, np.sqrt(np.abs(K).max(axis=0)), rtol=1e-6)


def test_smooth_ones_changes_nothing():
    rng = np.random.default_rng(41)
    x = rng.standard_normal((20, 32)).astype(np.float16)
    C = (rng.standard_normal((3, 16, 32)) * 0.5).astype(np.float32)
    a = O.rvq_encode(x, C)
    b = O.rvq_encode(x, C, smooth=np.ones(32, np.float32))
    for u, v in zip(a, b):
        np.testing.assert_array_equal(u, v)
    case = _rand_decode_case(rng, comp=[40, 11], win=[8, 2])
    o1, l1 = O.decode_attn(*case)
    o2, l2 = O.decode_attn(*case, k_smooth=np.ones((2, 64), np.float32))
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)


def test_smoothed_direct_equals_lut_form():
    # the query absorbs lambda exactly: (lambda q) . (H k~ / sqrt d) == q . (lambda H k~ / sqrt d)
    rng = np.random.default_rng(42)
    case = _rand_decode_case(rng, comp=[40, 23], win=[8, 0])
    lam = np.exp(rng.standard_normal((2, 64)) * 0.7).astype(np.float32)
    o1, l1 = O.decode_attn(*case, k_smooth=lam)
    o2, l2 = O.decode_attn_lut(*case, k_smooth=lam)
    np.testing.assert_allclose(o2, o1, atol=1e-9, rtol=0)
    np.testing.assert_allclose(l2, l1, atol=1e-9, rtol=0)
    o0, _ = O.decode_attn(*case)
    assert np.max(np.abs(o0 - o1)) > 1e-3     # lambda really changes the keys


def test_smoothed_encode_decode_recovers_the_original_scores():
    # Codebooks that hold the smoothed, rotated keys exactly (one stage): the decoded scores
    # are q . k of the ORIGINAL keys (to float32 rounding), which fixes the direction of lambda
    rng = np.random.default_rng(43)
    d, n = 64, 5
    keys = (rng.standard_normal((n, d)) * np.exp(rng.standard_normal(d))).astype(np.float16)
    lam = O.smooth_factors(keys)
    y = O.rotate_to_f32(O.smooth_keys(keys, lam))
    Ck = np.zeros((1, 1, 16, d), np.float32)
    Ck[0, 0, 1:1 + n] = y
    codes, _, _, _ = O.rvq_encode(keys, Ck[0], smooth=lam)
    np.testing.assert_array_equal(codes[:, 0], np.arange(1, 1 + n))
    q = rng.standard_normal((1, 1, d)).astype(np.float16)
    kc = np.zeros((1, 1, 16, 1), np.uint8)
    kc[0, 0, :n, 0] = codes[:, 0]
    vc = np.zeros((1, 1, 16, 1), np.uint8)
    Cv = np.zeros((1, 1, 16, d), np.float32)
    wk = np.zeros((1, 1, 1, d), np.float16)
    _, lse = O.decode_attn(q, kc, vc, [n], Ck, Cv, wk, wk, [0], k_smooth=lam[None])
    sc = keys.astype(np.float64) @ q[0, 0].astype(np.float64) / math.sqrt(d)
    assert abs(lse[0, 0] - scipy.special.logsumexp(sc)) < 1e-4
    _, lse_wrong = O.decode_attn(q, kc, vc, [n], Ck, Cv, wk, wk, [0])
    assert abs(lse_wrong[0, 0] - scipy.special.logsumexp(sc)) > 1e-2


# ------------------------------------------------------------------ product VQ (VecInfer)

def test_pq_one_subvector_is_single_stage_vq():
    # m = d: one sub-vector, so product VQ is the first RVQ stage with the same codebook
    rng = np.random.default_rng(50)
    x = rng.standard_normal((40, 16)).astype(np.float16)
    C = (rng.standard_normal((32, 16)) * 0.6).astype(np.float32)
    z, y = O.pq_encode(x, C)
    zr, _, yr, _ = O.rvq_encode(x, C[None])
    np.testing.assert_array_equal(z[:, 0], zr[:, 0])
    np.testing.assert_array_equal(y, yr)


def test_pq_matches_brute_force_per_subvector():
    rng = np.random.default_rng(51)
    d, m, K = 8, 2, 5
    x = rng.standard_normal((12, d)).astype(np.float16)
    C = rng.standard_normal((K, m)).astype(np.float32)
    z, y = O.pq_encode(x, C)
    for n in range(x.shape[0]):
        for j in range(d // m):
            dist = [sum((float(y[n, j * m + i]) - float(C[c, i])) ** 2 for i in range(m))
                    for c in range(K)]
            assert z[n, j] == min(range(K), key=lambda c: (dist[c], c))


def test_pq_exact_codewords_round_trip():
    # codewords cut from the rotated vectors themselves: every sub-vector finds its own piece
    # and the reconstruction rotated back is the input (to float32 rounding)
    rng = np.random.default_rng(52)
    d, m = 32, 4
    x = rng.standard_normal((3, d)).astype(np.float16)
    y = O.rotate_to_f32(x)
    pieces = y.reshape(-1, m)
    C = np.concatenate([np.zeros((1, m), np.float32), pieces])
    z, _ = O.pq_encode(x, C)
    np.testing.assert_array_equal(z.reshape(-1), np.arange(1, 1 + pieces.shape[0]))
    xr = O.pq_reconstruct(z, C, unrotate=True)
    np.testing.assert_allclose(xr, x.astype(np.float64), atol=1e-5)


def test_pq_duplicate_codewords_pick_lowest_index():
    C = np.array([[1.0, 0.0], [0.0, 1.0], [0.0, 1.0]], np.float32)
    y = np.array([[0.1, 0.9, 0.0, 1.2]], np.float32)
    z, _ = O.pq_encode(y, C, rotate=False)
    np.testing.assert_array_equal(z, [[1, 1]])


def test_pq_distortion_is_the_sum_over_subvectors():
    rng = np.random.default_rng(53)
    d, m = 64, 8
    x = rng.standard_normal((25, d)).astype(np.float16)
    C = (rng.standard_normal((64, m)) * 0.4).astype(np.float32)
    z, y = O.pq_encode(x, C)
    err = ((y.astype(np.float64) - O.pq_reconstruct(z, C)) ** 2).sum(axis=1)
    per = np.zeros(x.shape[0])
    for j in range(d // m):
        sub = y[:, j * m:(j + 1) * m].astype(np.float64)
        per += (((sub[:, None, :] - C[None].astype(np.float64)) ** 2).sum(-1)).min(axis=1)
    np.testing.assert_allclose(err, per, rtol=1e-12)


@pytest.mark.parametrize("smooth", [False, True])
def test_pq_direct_equals_lut_form(smooth):
    rng = np.random.default_rng(54)
    B, Hq, Hkv, d, m, Tcap, Wcap = 2, 4, 2, 64, 4, 30, 6
    q = rng.standard_normal((B, Hq, d)).astype(np.float16)
    kc = rng.integers(0, 32, (B, Hkv, Tcap, d // m)).astype(np.uint8)
    vc = rng.integers(0, 32, (B, Hkv, Tcap, d // m)).astype(np.uint8)
    Ck = (rng.standard_normal((Hkv, 32, m)) * 0.7).astype(np.float32)
    Cv = rng.standard_normal((Hkv, 32, m)).astype(np.float32)
    wk = rng.standard_normal((B, Hkv, Wcap, d)).astype(np.float16)
    wv = rng.standard_normal((B, Hkv, Wcap, d)).astype(np.float16)
    lam = np.exp(rng.standard_normal((Hkv, d)) * 0.5).astype(np.float32) if smooth else None
    for comp, win in (([30, 11], [6, 2]), ([0, 30], [6, 0]), ([5, 0], [0, 6])):
        case = (q, kc, vc, np.array(comp), Ck, Cv, wk, wv, np.array(win))
        o1, l1 = O.pq_decode_attn(*case, k_smooth=lam)
        o2, l2 = O.pq_decode_attn_lut(*case, k_smooth=lam)
        np.testing.assert_allclose(o2, o1, atol=1e-9, rtol=0)
        np.testing.assert_allclose(l2, l1, atol=1e-9, rtol=0)


def test_pq_match_walk_counts_exact_near_tie_and_mismatch():
    """Product-VQ match walk on a hand-built case (d = 8, m = 2: four sub-vectors per row).

    Codewords C[c] = (2c, -3c) for c < 14 are far apart; every sub-vector is its codeword plus
    delta = (0.25, 0.125), so its nearest codeword is known by construction.  Two extra
    codewords sit just on the +x side of C[5] and C[3]; the sub-vectors built on C[5] (row 0,
    sub-vector 1) and C[3] (row 4, sub-vector 0) are then nearer to the extra codewords:
      C[14] = C[5] + (1 ulp of 10, 0): D(5) - D(14) ~ 0.5 ulp = 4.8e-7, relative 6.1e-6 < 1e-5;
      C[15] = C[3] + (7.8e-6, 0):       D(3) - D(15) ~ 3.9e-6,         relative 5.0e-5 > 1e-5.
    Planted candidates: 5 at (0, 1) is a near tie (one exception), 3 at (4, 0) is a mismatch,
    13 for 12 at (2, 3) is a plain mismatch.  A near-tie rule applied to the wrong distance, a
    swapped comparison, or a sub-vector index off by one changes the counts or the tuples."""
    C = np.array([(2.0 * c, -3.0 * c) for c in range(16)], np.float32)
    C[14] = (np.nextafter(np.float32(10.0), np.float32(11.0)), -15.0)
    C[15] = (np.float32(6.0) + np.float32(7.8e-6), -9.0)
    z = np.array([[1, 5, 2, 6], [4, 6, 7, 8], [9, 10, 11, 12], [13, 0, 1, 2], [3, 4, 6, 7]])
    x = (C[z] + np.float32([0.25, 0.125])).reshape(5, 8).astype(np.float32)
    oracle = z.copy()
    oracle[0, 1] = 14
    oracle[4, 0] = 15
    zo, _ = O.pq_encode(x, C, rotate=False)
    np.testing.assert_array_equal(zo, oracle)        # the construction's nearest codewords
    res = O.pq_match_walk(x, C, oracle, rotate=False)
    assert (res["exact"], res["exceptions"], res["mismatches"], res["bad"]) == (20, 0, 0, [])
    cand = oracle.copy()
    cand[0, 1] = 5          # near tie
    cand[4, 0] = 3          # gap above 1e-5 relative
    cand[2, 3] = 13         # far
    res = O.pq_match_walk(x, C, cand, rotate=False)
    assert res["exact"] == 17 and res["exceptions"] == 1 and res["mismatches"] == 2
    assert res["bad"] == [(2, 3, 13, 12), (4, 0, 3, 15)]
    # a looser gap turns the second case into an exception too
    res = O.pq_match_walk(x, C, cand, rotate=False, rel_gap=1e-4)
    assert (res["exceptions"], res["mismatches"], res["bad"]) == (2, 1, [(2, 3, 13, 12)])


def test_pq_code_bytes_give_the_stated_bit_rates():
    # 8-bit codes over sub-vectors of 4 (8) dims: 2 (1) bits per element
    x = np.zeros((1, 128), np.float16)
    for m, bits in ((4, 2), (8, 1)):
        z, _ = O.pq_encode(x, np.zeros((256, m), np.float32))
        assert z.dtype == np.uint8 and z.shape[1] * 8 / 128 == bits


# ------------------------------------------------------------------ product VQ, worked examples

def test_pq_encode_hand_example():
    from oracle import c_oracle as C
    g = _read_fixture("pq_encode_hand_d4.txt")
    x = g["x"].astype(np.float16)[None]
    book = g["codebook"].astype(np.float32)
    lam = g["lambda"].astype(np.float32)
    z, y = O.pq_encode(x, book, smooth=lam)
    np.testing.assert_array_equal(y[0], g["y_smoothed"])
    np.testing.assert_array_equal(z[0], g["codes_smoothed"])
    z, y = O.pq_encode(x, book)
    np.testing.assert_array_equal(y[0], g["y_plain"])
    np.testing.assert_array_equal(z[0], g["codes_plain"])
    np.testing.assert_array_equal(C.pq_encode(x, book, smooth=lam)[0], g["codes_smoothed"])
    np.testing.assert_array_equal(C.pq_encode(x, book)[0], g["codes_plain"])


def test_pq_decode_hand_example():
    from oracle import c_oracle as C
    g = _read_fixture("pq_decode_hand_d4.txt")
    d = 4
    q = g["q"].astype(np.float16).reshape(1, 1, d)
    book = g["codebook"].astype(np.float32).reshape(1, 4, 2)
    kc = g["k_codes"].astype(np.uint8).reshape(1, 1, 2, 2)
    vc = g["v_codes"].astype(np.uint8).reshape(1, 1, 2, 2)
    w = np.zeros((1, 1, 1, d), np.float16)
    e2 = math.exp(2.0)
    want = np.array([2 * e2 + 1, 1, 1 - 2 * e2, 1]) / (e2 + 1)
    for fn in (O.pq_decode_attn, O.pq_decode_attn_lut, C.pq_decode_attn):
        out, lse = fn(q, kc, vc, [2], book, book, w, w, [0])
        np.testing.assert_allclose(out[0, 0], want, atol=1e-14)
        assert abs(lse[0, 0] - math.log(e2 + 1)) < 1e-14
