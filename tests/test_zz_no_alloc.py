"""The allocation-free decode entry point (zkv_rvq_decode_attn_noalloc): same results as
zkv_rvq_decode_attn with a caller workspace, call after call; oversize shapes refused before
anything runs.  The file name keeps it last in collection so it also runs after every other
test has used the library on the same device."""
import ctypes

import numpy as np
import pytest
import torch

from compressed_decode_attention_zkv_b200 import build as B
from compressed_decode_attention_zkv_b200 import inputs as I
from compressed_decode_attention_zkv_b200 import zkv
from oracle import zkv_oracle as O

TOL = 2e-3
FAKE = 0x7f0000000000   # 256-byte aligned, never dereferenced: the calls below stop in validation


def _case(seed, B_, Hq, Hkv, d, Sk, Sv, Tcap, comp, Wcap, win):
    rng = np.random.default_rng(seed)
    wl = I.workload("llama3_8b_32k", B=B_, Hq=Hq, Hkv=Hkv, d=d, Sk=Sk, Sv=Sv)
    kc = I.random_codes(wl, "k", Tcap, seed=seed, skewed=True)
    vc = I.random_codes(wl, "v", Tcap, seed=seed + 1, skewed=True)
    Ck = (rng.standard_normal((Hkv, Sk, 256, d)) * 0.1).astype(np.float32)
    Cv = (rng.standard_normal((Hkv, Sv, 256, d)) * 0.3).astype(np.float32)
    Ck[:, :, 0] = 0
    Cv[:, :, 0] = 0
    q = rng.standard_normal((B_, Hq, d)).astype(np.float16)
    wk = rng.standard_normal((B_, Hkv, Wcap, d)).astype(np.float16)
    wv = rng.standard_normal((B_, Hkv, Wcap, d)).astype(np.float16)
    return (q, kc, vc, np.asarray(comp, np.int32), Ck, Cv, wk, wv, np.asarray(win, np.int32))


CASE_A = dict(seed=71, B_=3, Hq=8, Hkv=2, d=128, Sk=4, Sv=4, Tcap=5008, comp=[5001, 0, 2222],
              Wcap=16, win=[16, 3, 0])
CASE_B = dict(seed=72, B_=2, Hq=7, Hkv=1, d=64, Sk=2, Sv=3, Tcap=3008, comp=[3000, 17],
              Wcap=8, win=[8, 5])


def _params(**kw):
    base = dict(B=8, Hq=32, Hkv=8, d=128, Sk=4, Sv=4, Tcap=32768, Wcap=128, max_comp_len=32768,
                softmax_scale=0.0, q=FAKE, k_codes=FAKE, v_codes=FAKE, comp_len=FAKE,
                k_codebooks=FAKE, v_codebooks=FAKE, win_k=FAKE, win_v=FAKE, win_len=FAKE,
                out=FAKE)
    base.update(kw)
    return zkv.DecodeParams(**base)


def test_noalloc_refuses_shapes_beyond_the_scratch_array():
    B.build()
    L = zkv.lib()
    # 64 sequences x 16K tokens (the ragged serving batch) need ~36 MiB of workspace
    p = _params(B=64, Tcap=16384, max_comp_len=16384)
    assert L.zkv_decode_workspace_size(ctypes.byref(p)) > zkv.DECODE_SCRATCH_BYTES
    assert L.zkv_rvq_decode_attn_noalloc(ctypes.byref(p), None) == zkv.ZKV_ERR_WORKSPACE
    # 8 x 32K GQA fits
    assert L.zkv_decode_workspace_size(ctypes.byref(_params())) <= zkv.DECODE_SCRATCH_BYTES


@pytest.mark.parametrize("kw,status", [
    (dict(d=96), zkv.ZKV_ERR_UNSUPPORTED),
    (dict(Hq=30), zkv.ZKV_ERR_INVALID_ARG),
    (dict(q=0), zkv.ZKV_ERR_INVALID_ARG),
    (dict(k_codes=FAKE + 4), zkv.ZKV_ERR_INVALID_ARG),
])
def test_noalloc_validates_like_the_workspace_entry_point(kw, status):
    B.build()
    L = zkv.lib()
    p = _params(**kw)
    assert L.zkv_rvq_decode_attn_noalloc(ctypes.byref(p), None) == status
    assert L.zkv_rvq_decode_attn(ctypes.byref(p), ctypes.c_void_p(FAKE), 1 << 30, None) == status


def _cuda(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_call_after_call():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    B.build()
    zkv.lib()
    cases = [_case(**CASE_A), _case(**CASE_B)]
    dev = [[_cuda(x) for x in c] for c in cases]
    # three calls in a row on one stream, no synchronisation between them: A, B, A
    got = [zkv.rvq_decode_attn_noalloc(*dev[i]) for i in (0, 1, 0)]
    torch.cuda.synchronize()
    want = [zkv.rvq_decode_attn(*dev[i]) for i in (0, 1)]
    torch.cuda.synchronize()
    for (o, l), i in zip(got, (0, 1, 0)):
        assert torch.equal(o, want[i][0]), f"out differs on case {i}"
        assert torch.equal(l, want[i][1]), f"lse differs on case {i}"
    # and both agree with the oracle
    for i, c in enumerate(cases):
        wo, wl = O.decode_attn(*c)
        o, l = got[i][0].cpu().numpy(), got[i][1].cpu().numpy()
        assert np.max(np.abs(o - wo)) <= TOL
        fin = np.isfinite(wl)
        assert np.array_equal(fin, np.isfinite(l))
        assert np.max(np.abs(l[fin] - wl[fin]), initial=0.0) <= TOL


@pytest.mark.gpu
def test_noalloc_refusal_raises_a_clear_error_on_device():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    d, Hkv, Tcap = 128, 8, 16384
    q = torch.zeros((64, 32, d), dtype=torch.float16, device="cuda")
    kc = torch.zeros((64, Hkv, Tcap, 4), dtype=torch.uint8, device="cuda")
    cb = torch.zeros((Hkv, 4, 256, d), dtype=torch.float32, device="cuda")
    w = torch.zeros((64, Hkv, 16, d), dtype=torch.float16, device="cuda")
    n = torch.zeros(64, dtype=torch.int32, device="cuda")
    out = torch.full((64, 32, d), float("nan"), dtype=torch.float32, device="cuda")
    lse = torch.full((64, 32), float("nan"), dtype=torch.float32, device="cuda")
    torch.cuda.synchronize()
    with pytest.raises(zkv.ZkvError, match="scratch array holds"):
        zkv.rvq_decode_attn_noalloc(q, kc, kc, n, cb, cb, w, w, n, out=out, lse=lse)
    torch.cuda.synchronize()
    # the refused call launched nothing: the caller's buffers are untouched
    assert torch.isnan(out).all() and torch.isnan(lse).all()
