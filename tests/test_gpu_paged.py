"""The paged code layout (block table over a page pool) gives bit-identical results to the
contiguous layout, for the decode call and the serving step, and agrees with the oracle; a
block-table entry outside the pool is reported, not followed."""
import numpy as np
import pytest
import torch

from compressed_decode_attention_zkv_b200 import build as B
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


def paginate(codes, P, rng, spare=3):
    """codes [B, Hkv, Tcap, S] -> (pool [n_pages, Hkv, P, S], block table int32 [B, Tcap / P]) with
    the pages shuffled through a larger pool."""
    Bn, Hkv, Tcap, S = codes.shape
    mp = Tcap // P
    n_pages = Bn * mp + spare
    perm = rng.permutation(n_pages)[:Bn * mp].reshape(Bn, mp)
    pool = rng.integers(0, 256, (n_pages, Hkv, P, S)).astype(np.uint8)   # junk in unused pages
    for b in range(Bn):
        for p in range(mp):
            pool[perm[b, p]] = codes[b, :, p * P:(p + 1) * P]
    return pool, perm.astype(np.int32)


def gather(pool, bt, P):
    Bn, mp = bt.shape
    return np.stack([np.concatenate([pool[bt[b, p]] for p in range(mp)], axis=1)
                     for b in range(Bn)])


def _case(seed, Bn, Hq, Hkv, d, Sk, Sv, Tcap, comp, Wcap, win):
    rng = np.random.default_rng(seed)
    kc = rng.integers(0, 256, (Bn, Hkv, Tcap, Sk)).astype(np.uint8)
    vc = rng.integers(0, 256, (Bn, Hkv, Tcap, Sv)).astype(np.uint8)
    Ck = (rng.standard_normal((Hkv, Sk, 256, d)) * 0.1).astype(np.float32)
    Cv = (rng.standard_normal((Hkv, Sv, 256, d)) * 0.3).astype(np.float32)
    Ck[:, :, 0] = 0
    Cv[:, :, 0] = 0
    q = rng.standard_normal((Bn, Hq, d)).astype(np.float16)
    wk = rng.standard_normal((Bn, Hkv, Wcap, d)).astype(np.float16)
    wv = rng.standard_normal((Bn, Hkv, Wcap, d)).astype(np.float16)
    return rng, q, kc, vc, np.asarray(comp, np.int32), Ck, Cv, wk, wv, np.asarray(win, np.int32)


@pytest.mark.parametrize("P,cfg", [
    (32, dict(Bn=3, Hq=8, Hkv=2, d=128, Sk=4, Sv=4, Tcap=2048, comp=[2048, 1000, 31], Wcap=16,
              win=[16, 0, 5])),
    (256, dict(Bn=5, Hq=14, Hkv=2, d=64, Sk=2, Sv=3, Tcap=4096, comp=[4096, 0, 2500, 257, 3],
               Wcap=8, win=[8, 8, 0, 3, 1])),
    (1024, dict(Bn=2, Hq=4, Hkv=4, d=256, Sk=3, Sv=2, Tcap=3072, comp=[3072, 1025], Wcap=4,
                win=[4, 2])),
])
def test_paged_decode_is_bit_identical(P, cfg):
    rng, q, kc, vc, comp, Ck, Cv, wk, wv, win = _case(70 + P, **cfg)
    kpool, bt = paginate(kc, P, rng)
    vpool = np.zeros((kpool.shape[0],) + vc.shape[1:2] + (P, vc.shape[3]), np.uint8)
    for b in range(bt.shape[0]):
        for p in range(bt.shape[1]):
            vpool[bt[b, p]] = vc[b, :, p * P:(p + 1) * P]
    assert np.array_equal(gather(kpool, bt, P), kc) and np.array_equal(gather(vpool, bt, P), vc)
    common = (_cuda(comp), _cuda(Ck), _cuda(Cv), _cuda(wk), _cuda(wv), _cuda(win))
    o1, l1 = zkv.rvq_decode_attn(_cuda(q), _cuda(kc), _cuda(vc), *common)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    o2, l2 = zkv.rvq_decode_attn(_cuda(q), _cuda(kpool), _cuda(vpool), *common,
                                 block_table=_cuda(bt), error_flag=err)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    assert int(err.item()) == 0
    want_o, want_l = O.decode_attn(q, kc, vc, comp, Ck, Cv, wk, wv, win,
                                   pairs=[(b, h) for b in range(q.shape[0]) for h in (0, q.shape[1] - 1)])
    for b in range(q.shape[0]):
        for h in (0, q.shape[1] - 1):
            assert np.max(np.abs(o2[b, h].cpu().numpy() - want_o[b, h])) <= TOL


def test_paged_serving_steps_are_bit_identical():
    P = 64
    rng, q0, kc, vc, comp, Ck, Cv, wk, wv, win = _case(
        80, Bn=4, Hq=8, Hkv=2, d=128, Sk=4, Sv=4, Tcap=512, comp=[500, 63, 0, 511], Wcap=4,
        win=[4, 4, 2, 4])
    kpool, bt = paginate(kc, P, rng)
    vpool = np.zeros((kpool.shape[0], 2, P, 4), np.uint8)
    for b in range(4):
        for p in range(bt.shape[1]):
            vpool[bt[b, p]] = vc[b, :, p * P:(p + 1) * P]
    sides = []
    for paged in (False, True):
        g = dict(kc=_cuda(kpool if paged else kc), vc=_cuda(vpool if paged else vc),
                 comp=_cuda(comp), wl=_cuda(win), wh=_cuda(np.array([1, 0, 0, 3], np.int32)),
                 wk=_cuda(wk), wv=_cuda(wv), err=torch.zeros(1, dtype=torch.int32, device="cuda"),
                 bt=_cuda(bt) if paged else None)
        sides.append(g)
    Ckd, Cvd = _cuda(Ck), _cuda(Cv)
    for step in range(5):
        nk = _cuda(rng.standard_normal((4, 2, 128)).astype(np.float16))
        nv = _cuda(rng.standard_normal((4, 2, 128)).astype(np.float16))
        q = _cuda(rng.standard_normal((4, 8, 128)).astype(np.float16))
        res = []
        for g in sides:
            res.append(zkv.rvq_serve_step(nk, nv, q, g["wk"], g["wv"], g["wl"], g["wh"], g["comp"],
                                          g["kc"], g["vc"], Ckd, Cvd, max_comp_len=512,
                                          error_flag=g["err"], block_table=g["bt"]))
        torch.cuda.synchronize()
        assert torch.equal(res[0][0], res[1][0]) and torch.equal(res[0][1], res[1][1]), step
        a, b = sides
        assert np.array_equal(gather(b["kc"].cpu().numpy(), bt, P), a["kc"].cpu().numpy())
        assert np.array_equal(gather(b["vc"].cpu().numpy(), bt, P), a["vc"].cpu().numpy())
        for key in ("comp", "wl", "wh", "wk", "wv"):
            assert torch.equal(a[key], b[key]), key
    # sequence 3 filled its last page: its next eviction is refused the same way in both
    assert int(sides[0]["err"].item()) == int(sides[1]["err"].item())


def test_block_table_entry_outside_the_pool_is_reported():
    P = 32
    rng, q, kc, vc, comp, Ck, Cv, wk, wv, win = _case(
        90, Bn=2, Hq=4, Hkv=1, d=128, Sk=2, Sv=2, Tcap=128, comp=[128, 64], Wcap=2, win=[2, 2])
    kpool, bt = paginate(kc, P, rng, spare=0)
    vpool = kpool.copy()
    bt_bad = bt.copy()
    bt_bad[0, 1] = kpool.shape[0] + 5          # outside the pool
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    zkv.rvq_decode_attn(_cuda(q), _cuda(kpool), _cuda(vpool), _cuda(comp), _cuda(Ck), _cuda(Cv),
                        _cuda(wk), _cuda(wv), _cuda(win), block_table=_cuda(bt_bad),
                        error_flag=err)
    torch.cuda.synchronize()
    assert int(err.item()) & zkv.ZKV_DEVERR_PAGE
