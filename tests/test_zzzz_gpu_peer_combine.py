"""zkv_lse_merge_peers (the context-parallel exchange and combine in one kernel) on one GPU.

The other ranks are emulated by buffers and flag words that the host prepares BEFORE the
single launch: the kernel under test never waits for another kernel.  It must signal every
rank, see the signals already present, read every "rank's" rows through the pointer tables and
combine them exactly as zkv_lse_merge does; with a signal that never arrives its bounded wait
must run out, report ZKV_DEVERR_TIMEOUT and leave the output unwritten.  (Several GPUs, where
the ranks really run concurrently, are not available here.)  The file name keeps it after
every other GPU test in collection order."""
import pytest
import torch

from compressed_decode_attention_zkv_b200 import build as B
from compressed_decode_attention_zkv_b200 import zkv

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    B.build()
    zkv.lib()


def _ptrs(ts):
    return torch.tensor([t.data_ptr() for t in ts], dtype=torch.int64, device="cuda")


def _ranks(N, rows, d, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    outs = [torch.randn(rows, d, device="cuda", generator=g) for _ in range(N)]
    lses = [torch.randn(rows, device="cuda", generator=g) * 3 for _ in range(N)]
    lses[0][::5] = -float("inf")          # rows where rank 0 has no keys
    for lse in lses:
        lse[3] = -float("inf")            # a row no rank has keys for
    flags = [torch.zeros(N, dtype=torch.int32, device="cuda") for _ in range(N)]
    return outs, lses, flags


@pytest.mark.parametrize("N,rank", [(1, 0), (2, 1), (4, 2)])
def test_peer_combine_equals_the_gathered_combine(N, rank):
    rows, d, epoch = 37, 128, 7
    outs, lses, flags = _ranks(N, rows, d, 10 + N)
    for i in range(N):
        if i != rank:
            flags[rank][i] = epoch          # the other ranks have signalled this epoch
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse = zkv.lse_merge_peers(_ptrs(outs), _ptrs(lses), _ptrs(flags), rank, epoch, rows, d,
                                   error_flag=err)
    want_o, want_l = zkv.lse_merge(torch.stack(outs), torch.stack(lses))
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    torch.testing.assert_close(out, want_o, rtol=0, atol=1e-6)
    assert torch.equal(torch.isinf(lse), torch.isinf(want_l))
    fin = torch.isfinite(want_l)
    torch.testing.assert_close(lse[fin], want_l[fin], rtol=0, atol=1e-6)
    assert torch.all(out[3] == 0) and lse[3].item() == -float("inf")
    for i in range(N):                      # this rank's signal reached every rank's flags
        assert int(flags[i][rank].item()) == epoch


def test_peer_combine_wait_is_bounded_and_reported():
    N, rank, rows, d, epoch = 3, 0, 20, 64, 2
    outs, lses, flags = _ranks(N, rows, d, 20)
    flags[rank][1] = epoch                  # rank 2's signal never arrives
    out = torch.full((rows, d), float("nan"), device="cuda")
    lse = torch.full((rows,), float("nan"), device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    zkv.lse_merge_peers(_ptrs(outs), _ptrs(lses), _ptrs(flags), rank, epoch, rows, d, out=out,
                        lse=lse, error_flag=err, timeout_s=0.005)
    torch.cuda.synchronize()
    assert int(err.item()) & zkv.ZKV_DEVERR_TIMEOUT
    assert torch.isnan(out).all() and torch.isnan(lse).all()   # nothing combined
    for i in range(N):
        assert int(flags[i][rank].item()) == epoch             # the signals still went out
    # the next step, with every signal present, completes normally on the same flags
    flags[rank][1] = epoch + 1
    flags[rank][2] = epoch + 1
    err.zero_()
    out, lse = zkv.lse_merge_peers(_ptrs(outs), _ptrs(lses), _ptrs(flags), rank, epoch + 1,
                                   rows, d, out=out, lse=lse, error_flag=err)
    want_o, _ = zkv.lse_merge(torch.stack(outs), torch.stack(lses))
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    torch.testing.assert_close(out, want_o, rtol=0, atol=1e-6)


def test_peer_exchange_one_rank_end_to_end(tmp_path):
    """PeerExchange on a one-rank NCCL group: torch symmetric memory, the rendezvous, the
    pointer tables and cp_decode_attn's fused path, three steps (both buffer sets).  With one
    rank the combine of a single part returns it unchanged, so the result equals the plain
    decode bit for bit."""
    import datetime

    import numpy as np
    import torch.distributed as dist

    from compressed_decode_attention_zkv_b200 import context_parallel as CP
    if dist.is_initialized():
        pytest.skip("a process group is already initialised in this process")
    store = dist.FileStore(str(tmp_path / "store"), 1)
    dist.init_process_group("nccl", store=store, rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60))
    try:
        rng = np.random.default_rng(400)
        Bn, Hq, Hkv, d, S, Tcap, W = 2, 8, 2, 128, 4, 512, 8
        cu = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()   # noqa: E731
        kc = cu(rng.integers(0, 256, (Bn, Hkv, Tcap, S)).astype(np.uint8))
        vc = cu(rng.integers(0, 256, (Bn, Hkv, Tcap, S)).astype(np.uint8))
        Ck = (rng.standard_normal((Hkv, S, 256, d)) * 0.1).astype(np.float32)
        Cv = (rng.standard_normal((Hkv, S, 256, d)) * 0.3).astype(np.float32)
        Ck[:, :, 0] = 0
        Cv[:, :, 0] = 0
        Ck, Cv = cu(Ck), cu(Cv)
        wk = cu(rng.standard_normal((Bn, Hkv, W, d)).astype(np.float16))
        wv = cu(rng.standard_normal((Bn, Hkv, W, d)).astype(np.float16))
        comp = cu(np.array([500, 37], np.int32))
        win = cu(np.array([W, 3], np.int32))
        try:
            ex = CP.PeerExchange(Bn * Hq, d)
        except (RuntimeError, NotImplementedError, AttributeError) as exc:
            pytest.skip(f"torch symmetric memory unavailable here: {exc}")
        for step in range(3):
            q = cu(rng.standard_normal((Bn, Hq, d)).astype(np.float16))
            out, lse = CP.cp_decode_attn(q, kc, vc, comp, Ck, Cv, wk, wv, win, exchange=ex)
            want_o, want_l = zkv.rvq_decode_attn(q, kc, vc, comp, Ck, Cv, wk, wv, win)
            torch.cuda.synchronize()
            assert torch.equal(out, want_o) and torch.equal(lse, want_l), step
        assert ex.epoch == 3
        del ex
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
