"""Context-parallel decode emulated on one GPU: every rank's shard is decoded by the library
and the parts are combined by the library's log-sum-exp kernel (zkv_lse_merge); the result
equals the unsharded decode and the oracle.  The combine kernel itself is checked against the
oracle's combine, empty parts included.  (The exchange between ranks is tested on CPU with
gloo in tests/test_multi_rank.py.)"""
import numpy as np
import pytest
import torch

from compressed_decode_attention_zkv_b200 import build as B
from compressed_decode_attention_zkv_b200 import context_parallel as CP
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


def test_lse_merge_matches_oracle_combine():
    rng = np.random.default_rng(101)
    N, rows, d = 4, 37, 128
    po = rng.standard_normal((N, rows, d)).astype(np.float32)
    pl = (rng.standard_normal((N, rows)) * 5).astype(np.float32)
    pl[1, ::3] = -np.inf                  # some parts empty
    pl[:, 5] = -np.inf                    # a row with no keys at all
    packed = np.concatenate([po, pl[..., None]], axis=-1)      # [N, rows, d + 1]
    g = _cuda(packed)
    out, lse = zkv.lse_merge(g[..., :d], g[..., d])
    out, lse = out.cpu().numpy(), lse.cpu().numpy()
    for r in range(rows):
        wo, wl = O.lse_merge([(po[i, r].astype(np.float64), float(pl[i, r])) for i in range(N)])
        np.testing.assert_allclose(out[r], wo, atol=1e-5, rtol=1e-5)
        if np.isneginf(wl):
            assert np.isneginf(lse[r]) and np.all(out[r] == 0)
        else:
            assert abs(lse[r] - wl) <= 1e-5 * max(1.0, abs(wl))


@pytest.mark.parametrize("world", [2, 3])
def test_sharded_decode_plus_combine_equals_unsharded(world):
    rng = np.random.default_rng(100 + world)
    Bn, Hq, Hkv, d, Sk, Sv, Tcap, W = 3, 8, 2, 128, 4, 4, 1024, 16
    kc = rng.integers(0, 256, (Bn, Hkv, Tcap, Sk)).astype(np.uint8)
    vc = rng.integers(0, 256, (Bn, Hkv, Tcap, Sv)).astype(np.uint8)
    Ck = (rng.standard_normal((Hkv, Sk, 256, d)) * 0.1).astype(np.float32)
    Cv = (rng.standard_normal((Hkv, Sv, 256, d)) * 0.3).astype(np.float32)
    Ck[:, :, 0] = 0
    Cv[:, :, 0] = 0
    q = rng.standard_normal((Bn, Hq, d)).astype(np.float16)
    wk = rng.standard_normal((Bn, Hkv, W, d)).astype(np.float16)
    wv = rng.standard_normal((Bn, Hkv, W, d)).astype(np.float16)
    comp = np.array([1024, 333, 1], np.int32)
    win = np.array([16, 0, 7], np.int32)
    g = dict(q=_cuda(q), kc=_cuda(kc), vc=_cuda(vc), comp=_cuda(comp), Ck=_cuda(Ck),
             Cv=_cuda(Cv), wk=_cuda(wk), wv=_cuda(wv), win=_cuda(win))
    full_o, full_l = zkv.rvq_decode_attn(g["q"], g["kc"], g["vc"], g["comp"], g["Ck"], g["Cv"],
                                         g["wk"], g["wv"], g["win"])
    parts = []
    for r in range(world):
        kl, vl, cl = CP.take_shard(g["kc"], g["vc"], g["comp"], r, world)
        wl = g["win"] if r == world - 1 else torch.zeros_like(g["win"])
        o, l = zkv.rvq_decode_attn(g["q"], kl, vl, cl, g["Ck"], g["Cv"], g["wk"], g["wv"], wl)
        parts.append(torch.cat([o, l[..., None]], dim=-1))
    gathered = torch.stack(parts)                             # what the all-gather produces
    out, lse = zkv.lse_merge(gathered[..., :d], gathered[..., d])
    torch.cuda.synchronize()
    # the shards' segments differ from the unsharded call's, so their fixed-point histogram
    # roundings do too (bounded by 2^-15 of each segment's mass)
    assert torch.max(torch.abs(out - full_o)).item() <= 5e-4
    assert torch.max(torch.abs(lse - full_l)).item() <= 5e-4
    want_o, want_l = O.decode_attn(q, kc, vc, comp, Ck, Cv, wk, wv, win)
    assert np.max(np.abs(out.cpu().numpy() - want_o)) <= TOL
    assert np.max(np.abs(lse.cpu().numpy() - want_l)) <= TOL
