"""GPU parity of the VecInfer smooth scaling (per-channel key factors lambda before the rotation,
absorbed into the query at decode) against the CPU oracle, through the C ABI.

Matching rules as for the unsmoothed path: codes bit-exact except counted near-ties (gap below
1e-5 relative), residual norms within 1e-5 relative where the codes agree, attention outputs and
lse within 2e-3 max-abs."""
import numpy as np
import pytest
import torch

from compressed_decode_attention_zkv_b200 import build as B
from compressed_decode_attention_zkv_b200 import inputs as I
from compressed_decode_attention_zkv_b200 import zkv
from oracle import zkv_oracle as O

pytestmark = pytest.mark.gpu
TOL = 2e-3


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    B.build()
    zkv.lib()


def _cuda(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _smoothed_books(wl):
    lam = I.key_smooth_factors(wl)
    return lam, I.train_codebooks(wl, "k", smooth=lam)


@pytest.mark.parametrize("n_tok,d", [(300, 128), (2600, 128), (2600, 64), (2600, 256)])
def test_smoothed_encode_matches_oracle(n_tok, d):
    """Row-group path (300 x 2 rows), tensor-core path (> 4096 rows, d = 64 / 128), SIMT tile
    path (d = 256)."""
    wl = I.workload("llama3_8b_32k", B=1, Hkv=2, Hq=8, d=d, T=n_tok, n_cal=2048, kmeans_iters=4)
    lam, books = _smoothed_books(wl)
    x = I.kv_tokens(wl, "k", 0, 0, n_tok)                 # [Hkv][T][d]
    codes, norms = zkv.rvq_encode(_cuda(x).permute(1, 0, 2), _cuda(books), smooth=_cuda(lam))
    codes, norms = codes[0].cpu().numpy(), norms[0].cpu().numpy()
    for h in range(2):
        walk = O.rvq_match_walk(x[h], books[h], codes[:, h], smooth=lam[h])
        assert walk["mismatches"] == 0, walk["bad"]
        assert walk["exceptions"] <= max(2, n_tok // 500)
        want_codes, want_norms, _, _ = O.rvq_encode(x[h], books[h], smooth=lam[h])
        same = np.all(codes[:, h] == want_codes, axis=1)
        np.testing.assert_allclose(norms[same, h], want_norms[same], rtol=1e-5, atol=1e-6)
    # and the factors matter: without them the codes differ
    plain, _ = zkv.rvq_encode(_cuda(x).permute(1, 0, 2), _cuda(books))
    assert not np.array_equal(plain[0].cpu().numpy(), codes)


def test_smoothed_decode_matches_oracle():
    rng = np.random.default_rng(61)
    wl = I.workload("llama3_8b_32k", B=3, Hq=8, Hkv=2, T=900, n_cal=2048, kmeans_iters=4)
    lam, Ck = _smoothed_books(wl)
    Cv = I.train_codebooks(wl, "v")
    Tcap, Wcap = 912, 16
    comp = np.array([900, 0, 517])
    win = np.array([16, 5, 0])
    kc = np.zeros((wl.B, wl.Hkv, Tcap, wl.Sk), np.uint8)
    vc = np.zeros((wl.B, wl.Hkv, Tcap, wl.Sv), np.uint8)
    wk = rng.standard_normal((wl.B, wl.Hkv, Wcap, wl.d)).astype(np.float16)
    wv = rng.standard_normal((wl.B, wl.Hkv, Wcap, wl.d)).astype(np.float16)
    for b in range(wl.B):
        xk, xv = I.kv_tokens(wl, "k", b, 0, wl.T), I.kv_tokens(wl, "v", b, 0, wl.T)
        for h in range(wl.Hkv):
            kc[b, h, :comp[b]] = O.rvq_encode(xk[h, :comp[b]], Ck[h], smooth=lam[h])[0]
            vc[b, h, :comp[b]] = O.rvq_encode(xv[h, :comp[b]], Cv[h])[0]
    q = rng.standard_normal((wl.B, wl.Hq, wl.d)).astype(np.float16)
    out, lse = zkv.rvq_decode_attn(_cuda(q), _cuda(kc), _cuda(vc), _cuda(comp.astype(np.int32)),
                                   _cuda(Ck), _cuda(Cv), _cuda(wk), _cuda(wv),
                                   _cuda(win.astype(np.int32)), k_smooth=_cuda(lam))
    want_o, want_l = O.decode_attn(q, kc, vc, comp, Ck, Cv, wk, wv, win, k_smooth=lam)
    out, lse = out.cpu().numpy(), lse.cpu().numpy()
    assert np.max(np.abs(out - want_o)) <= TOL
    fin = np.isfinite(want_l)
    assert np.array_equal(fin, np.isfinite(lse))
    assert np.max(np.abs(lse[fin] - want_l[fin])) <= TOL
    # the unsmoothed oracle is far off: the factors reach the query
    bad_o, _ = O.decode_attn(q, kc, vc, comp, Ck, Cv, wk, wv, win)
    assert np.max(np.abs(out - bad_o)) > 10 * TOL


def test_smoothed_serving_steps_match_oracle():
    """Prepared serving steps with smoothing (the evicted keys are smoothed before encoding,
    the query absorbs the factors) vs the oracle's append step and decode."""
    rng = np.random.default_rng(62)
    wl = I.workload("llama3_8b_32k", B=2, Hq=8, Hkv=2, T=500, W=8, n_cal=2048, kmeans_iters=4)
    lam, Ck = _smoothed_books(wl)
    Cv = I.train_codebooks(wl, "v")
    Tc, Tcap = wl.Tc, (wl.Tc + 16 + 15) // 16 * 16
    zk = np.zeros((wl.B, wl.Hkv, Tcap, wl.Sk), np.uint8)
    zv = np.zeros((wl.B, wl.Hkv, Tcap, wl.Sv), np.uint8)
    wk = np.zeros((wl.B, wl.Hkv, wl.W, wl.d), np.float16)
    wv = np.zeros((wl.B, wl.Hkv, wl.W, wl.d), np.float16)
    for b in range(wl.B):
        xk, xv = I.kv_tokens(wl, "k", b, 0, wl.T), I.kv_tokens(wl, "v", b, 0, wl.T)
        for h in range(wl.Hkv):
            zk[b, h, :Tc] = O.rvq_encode(xk[h, :Tc], Ck[h], smooth=lam[h])[0]
            zv[b, h, :Tc] = O.rvq_encode(xv[h, :Tc], Cv[h])[0]
        wk[b], wv[b] = xk[:, Tc:], xv[:, Tc:]
    st = dict(k_codes=zk, v_codes=zv, comp_len=np.full(wl.B, Tc), win_len=np.full(wl.B, wl.W),
              win_head=np.zeros(wl.B, np.int64), win_k=wk, win_v=wv, Ck=Ck, Cv=Cv, k_smooth=lam)
    g = {k: _cuda(v.astype(np.int32) if k in ("comp_len", "win_len", "win_head") else v)
         for k, v in st.items()}
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    nk_d = torch.zeros((wl.B, wl.Hkv, wl.d), dtype=torch.float16, device="cuda")
    nv_d = torch.zeros_like(nk_d)
    q_d = torch.zeros((wl.B, wl.Hq, wl.d), dtype=torch.float16, device="cuda")
    step = zkv.PreparedServeStep(nk_d, nv_d, q_d, g["win_k"], g["win_v"], g["win_len"],
                                 g["win_head"], g["comp_len"], g["k_codes"], g["v_codes"],
                                 g["Ck"], g["Cv"], max_comp_len=Tcap, error_flag=err,
                                 k_smooth=g["k_smooth"])
    for i in range(3):
        nk = (rng.standard_normal((wl.B, wl.Hkv, wl.d)) * 3).astype(np.float16)
        nv = rng.standard_normal((wl.B, wl.Hkv, wl.d)).astype(np.float16)
        q = rng.standard_normal((wl.B, wl.Hq, wl.d)).astype(np.float16)
        nk_d.copy_(_cuda(nk))
        nv_d.copy_(_cuda(nv))
        q_d.copy_(_cuda(q))
        out, lse = step()
        st = O.append_step(st, nk, nv)
        assert np.array_equal(g["k_codes"].cpu().numpy(), st["k_codes"]), f"step {i}"
        want_o, want_l = O.decode_attn(q, st["k_codes"], st["v_codes"], st["comp_len"], Ck, Cv,
                                       st["win_k"], st["win_v"], st["win_len"], k_smooth=lam)
        assert np.max(np.abs(out.cpu().numpy() - want_o)) <= TOL, f"step {i}"
        assert np.max(np.abs(lse.cpu().numpy() - want_l)) <= TOL, f"step {i}"
    assert int(err.item()) == 0
