"""GPU parity of the product-VQ (VecInfer) path against the oracle.  Encode: codes equal to the
float64 argmin of every sub-vector except counted near-ties (distance gap below 1e-5
relative), with and without key smoothing, every head dimension and several sub-vector sizes.
Decode: outputs and lse within 2e-3 of the oracle's direct form (reconstruct, rotate back,
softmax attention with the window), across chunk boundaries, 32 and 16 sub-vectors per token,
GQA 1 / 2 / 4 / 6 / 7, smoothing and empty parts.
The file name keeps it after every other GPU test in collection order, so that under
``pytest -x`` a failure here cannot hide the results of the established paths."""
import numpy as np
import pytest
import torch

from compressed_decode_attention_zkv_b200 import build as B
from compressed_decode_attention_zkv_b200 import inputs as I
from compressed_decode_attention_zkv_b200 import zkv
from oracle import zkv_oracle as O

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    B.build()
    zkv.lib()


def _cuda(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


@pytest.mark.parametrize("d,m,kind,smooth", [(128, 4, "k", True), (128, 8, "k", False),
                                             (64, 4, "v", False), (256, 2, "k", True),
                                             (128, 16, "v", False)])
def test_pq_encode_matches_oracle(d, m, kind, smooth):
    wl = I.workload("llama3_8b_32k", B=1, Hkv=2, Hq=8, d=d, T=333, n_cal=1024, kmeans_iters=3)
    lam = I.key_smooth_factors(wl) if smooth else None
    books = I.train_pq_codebook(wl, kind, m, smooth=lam)           # [2][256][m]
    x = I.kv_tokens(wl, kind, 0, 0, wl.T)                         # [Hkv][T][d]
    codes = zkv.pq_encode(_cuda(x).permute(1, 0, 2), _cuda(books),
                          smooth=None if lam is None else _cuda(lam))
    codes = codes[0].cpu().numpy()                                # [T, H, d/m]
    assert codes.shape == (wl.T, 2, d // m)
    for h in range(2):
        walk = O.pq_match_walk(x[h], books[h], codes[:, h],
                               smooth=None if lam is None else lam[h])
        assert walk["mismatches"] == 0, walk["bad"]
        assert walk["exceptions"] <= 2


def test_pq_encode_strided_batch_views():
    # [B, T, H, d] views of a larger buffer, fp32 input without rotation
    rng = np.random.default_rng(7)
    big = rng.standard_normal((2, 50, 3, 64 + 8)).astype(np.float32)
    x = _cuda(big)[..., :64]
    C = rng.standard_normal((3, 256, 4)).astype(np.float32)
    codes = zkv.pq_encode(x, _cuda(C), rotate=False).cpu().numpy()
    for b in range(2):
        for h in range(3):
            want, _ = O.pq_encode(big[b, :, h, :64], C[h], rotate=False)
            np.testing.assert_array_equal(codes[b, :, h], want)


def _pq_case(seed, Bn, Hq, Hkv, d, m, Tcap, comp, Wcap, win, smooth):
    rng = np.random.default_rng(seed)
    nsub = d // m
    kc = rng.integers(0, 256, (Bn, Hkv, Tcap, nsub)).astype(np.uint8)
    vc = rng.integers(0, 256, (Bn, Hkv, Tcap, nsub)).astype(np.uint8)
    Ck = (rng.standard_normal((Hkv, 256, m)) * 0.25).astype(np.float32)
    Cv = rng.standard_normal((Hkv, 256, m)).astype(np.float32)
    q = rng.standard_normal((Bn, Hq, d)).astype(np.float16)
    wk = rng.standard_normal((Bn, Hkv, Wcap, d)).astype(np.float16)
    wv = rng.standard_normal((Bn, Hkv, Wcap, d)).astype(np.float16)
    lam = np.exp(rng.standard_normal((Hkv, d)) * 0.4).astype(np.float32) if smooth else None
    return q, kc, vc, np.asarray(comp, np.int32), Ck, Cv, wk, wv, np.asarray(win, np.int32), lam


@pytest.mark.parametrize("cfg", [
    dict(Bn=3, Hq=8, Hkv=2, d=128, m=4, Tcap=4112, comp=[4100, 0, 2048], Wcap=16,
         win=[16, 5, 0], smooth=True),
    dict(Bn=2, Hq=7, Hkv=1, d=64, m=2, Tcap=4112, comp=[4097, 31], Wcap=8, win=[8, 8],
         smooth=False),
    dict(Bn=1, Hq=4, Hkv=2, d=256, m=8, Tcap=720, comp=[700], Wcap=4, win=[4], smooth=True),
    dict(Bn=2, Hq=2, Hkv=2, d=128, m=4, Tcap=64, comp=[0, 17], Wcap=4, win=[0, 0],
         smooth=False),
    # 16 sub-vectors per token (two tokens per warp step): 1 bit per element at d = 128
    dict(Bn=2, Hq=8, Hkv=2, d=128, m=8, Tcap=2576, comp=[2570, 9], Wcap=8, win=[3, 8],
         smooth=True),
    dict(Bn=1, Hq=6, Hkv=1, d=64, m=4, Tcap=2064, comp=[2051], Wcap=4, win=[2], smooth=False),
])
def test_pq_decode_matches_oracle(cfg):
    q, kc, vc, comp, Ck, Cv, wk, wv, win, lam = _pq_case(200 + cfg["d"], **cfg)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse = zkv.pq_decode_attn(_cuda(q), _cuda(kc), _cuda(vc), _cuda(comp), _cuda(Ck),
                                  _cuda(Cv), _cuda(wk), _cuda(wv), _cuda(win), error_flag=err,
                                  k_smooth=None if lam is None else _cuda(lam))
    out, lse = out.cpu().numpy(), lse.cpu().numpy()
    want_o, want_l = O.pq_decode_attn(q, kc, vc, comp, Ck, Cv, wk, wv, win, k_smooth=lam)
    assert np.max(np.abs(out - want_o)) <= 2e-3
    fin = np.isfinite(want_l)
    assert np.array_equal(fin, np.isfinite(lse))
    assert np.max(np.abs(lse[fin] - want_l[fin]), initial=0.0) <= 2e-3
    assert np.all(out[~fin] == 0)
    assert int(err.item()) == 0


def _pq_state(seed, Bn, Hkv, d, m, Tcap, Wcap, win_len, win_head, comp_len):
    rng = np.random.default_rng(seed)
    nsub = d // m
    return dict(k_codes=rng.integers(0, 256, (Bn, Hkv, Tcap, nsub)).astype(np.uint8),
                v_codes=rng.integers(0, 256, (Bn, Hkv, Tcap, nsub)).astype(np.uint8),
                comp_len=np.array(comp_len), win_len=np.array(win_len),
                win_head=np.array(win_head),
                win_k=rng.standard_normal((Bn, Hkv, Wcap, d)).astype(np.float16),
                win_v=rng.standard_normal((Bn, Hkv, Wcap, d)).astype(np.float16),
                Ck=(rng.standard_normal((Hkv, 256, m)) * 0.5).astype(np.float32),
                Cv=rng.standard_normal((Hkv, 256, m)).astype(np.float32),
                k_smooth=np.exp(rng.standard_normal((Hkv, d)) * 0.3).astype(np.float32))


@pytest.mark.parametrize("d,m", [(128, 4), (64, 2), (256, 16)])
def test_pq_append_steps_match_oracle(d, m):
    """zkv_pq_append against the oracle's append step (product VQ): free slots, evictions with
    smoothed keys, a full prefix (left unchanged and flagged), over several steps."""
    st = _pq_state(300 + d, Bn=5, Hkv=2, d=d, m=m, Tcap=16, Wcap=3, win_len=[0, 2, 3, 3, 3],
                   win_head=[0, 0, 1, 2, 0], comp_len=[0, 4, 7, 15, 16])
    rng = np.random.default_rng(301)
    g = {k: _cuda(v.astype(np.int32) if k in ("comp_len", "win_len", "win_head") else v)
         for k, v in st.items()}
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    for step in range(4):
        nk = rng.standard_normal((5, 2, d)).astype(np.float16)
        nv = rng.standard_normal((5, 2, d)).astype(np.float16)
        zkv.pq_append(_cuda(nk), _cuda(nv), g["win_k"], g["win_v"], g["win_len"], g["win_head"],
                      g["comp_len"], g["k_codes"], g["v_codes"], g["Ck"], g["Cv"],
                      error_flag=err, k_smooth=g["k_smooth"])
        st = O.append_step(st, nk, nv, pq=True)
        for key in ("k_codes", "v_codes", "win_k", "win_v", "comp_len", "win_len", "win_head"):
            np.testing.assert_array_equal(g[key].cpu().numpy(), st[key], err_msg=f"{key} {step}")
    assert st["error"] and int(err.item()) == 1   # the full prefix (ZKV_DEVERR_COMP_LEN)


def test_pq_cache_serving_loop_matches_oracle():
    """PQKVCache: prefill, then step (append + attend) x 5 against the oracle's append step and
    its decode (direct form), with key smoothing; append + attend equals step."""
    rng = np.random.default_rng(310)
    Bn, Hq, Hkv, d, m, W, T0 = 2, 8, 2, 128, 4, 8, 200
    wl = I.workload("llama3_8b_32k", B=Bn, Hq=Hq, Hkv=Hkv, T=T0, W=W, n_cal=1024,
                    kmeans_iters=3)
    lam = I.key_smooth_factors(wl)
    Ck = I.train_pq_codebook(wl, "k", m, smooth=lam)
    Cv = I.train_pq_codebook(wl, "v", m)
    k = np.stack([I.kv_tokens(wl, "k", b, 0, T0) for b in range(Bn)])
    v = np.stack([I.kv_tokens(wl, "v", b, 0, T0) for b in range(Bn)])
    caches = [zkv.PQKVCache(_cuda(Ck), _cuda(Cv), batch=Bn, capacity=T0, window=W, head_dim=d,
                            k_smooth=_cuda(lam)) for _ in range(2)]
    for c in caches:
        c.prefill(_cuda(k), _cuda(v))
    Tc = T0 - W
    Tcap = caches[0].Tcap

    def walk_ok(rows, book, codes, smooth=None):   # float64 argmin up to counted near-ties
        w = O.pq_match_walk(rows, book, codes, smooth=smooth)
        return w["mismatches"] == 0 and w["exceptions"] <= 2

    zk = caches[0].k_codes.cpu().numpy()
    zv = caches[0].v_codes.cpu().numpy()
    for b in range(Bn):
        for h in range(Hkv):
            assert walk_ok(k[b, h, :Tc], Ck[h], zk[b, h, :Tc], smooth=lam[h])
            assert walk_ok(v[b, h, :Tc], Cv[h], zv[b, h, :Tc])
    # the oracle continues from the GPU's (verified) codes
    st = dict(k_codes=zk, v_codes=zv, comp_len=np.full(Bn, Tc), win_len=np.full(Bn, W),
              win_head=np.zeros(Bn, np.int64), win_k=k[:, :, Tc:].copy(),
              win_v=v[:, :, Tc:].copy(), Ck=Ck, Cv=Cv, k_smooth=lam)
    for step in range(5):
        nk = rng.standard_normal((Bn, Hkv, d)).astype(np.float16)
        nv = rng.standard_normal((Bn, Hkv, d)).astype(np.float16)
        q = rng.standard_normal((Bn, Hq, d)).astype(np.float16)
        o1, l1 = caches[0].step(_cuda(nk), _cuda(nv), _cuda(q))
        caches[1].append(_cuda(nk), _cuda(nv))
        o2, l2 = caches[1].attend(_cuda(q))
        assert torch.equal(o1, o2) and torch.equal(l1, l2)
        before = st
        st = O.append_step(st, nk, nv, pq=True)
        gk, gv = caches[0].k_codes.cpu().numpy(), caches[0].v_codes.cpu().numpy()
        for b in range(Bn):   # the evicted token of every sequence, encoded at comp_len
            pos, slot = int(before["comp_len"][b]), int(before["win_head"][b])
            for h in range(Hkv):
                assert walk_ok(before["win_k"][b, h, slot][None], Ck[h], gk[b, h, pos][None],
                               smooth=lam[h])
                assert walk_ok(before["win_v"][b, h, slot][None], Cv[h], gv[b, h, pos][None])
        st["k_codes"], st["v_codes"] = gk, gv
        for key in ("win_k", "win_v", "comp_len", "win_len", "win_head"):
            np.testing.assert_array_equal(getattr(caches[0], key).cpu().numpy(), st[key])
        want_o, want_l = O.pq_decode_attn(q, st["k_codes"], st["v_codes"], st["comp_len"], Ck,
                                          Cv, st["win_k"], st["win_v"], st["win_len"],
                                          k_smooth=lam)
        assert np.max(np.abs(o1.cpu().numpy() - want_o)) <= 2e-3
        assert np.max(np.abs(l1.cpu().numpy() - want_l)) <= 2e-3
    assert int(caches[0].error_flag.item()) == 0
    assert caches[0].memory_bytes() == 2 * Bn * Hkv * (Tcap * d // m + W * d * 2)
