"""Multi-process paths on CPU (world sizes 2 and 3, gloo): the context-parallel decode's sharding and
exchange, and the benchmark's max-over-ranks timing.  No GPU: the context-parallel test runs
the exchange with oracle-backed stand-ins for the library's decode and combine (the GPU test
of those is tests/test_gpu_context_parallel.py)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _init(rank, world, port):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)


def _case():
    rng = np.random.default_rng(123)
    B, Hq, Hkv, d, S, Tcap, W = 3, 4, 2, 64, 3, 96, 8
    q = rng.standard_normal((B, Hq, d)).astype(np.float16)
    kc = rng.integers(0, 32, (B, Hkv, Tcap, S)).astype(np.uint8)
    vc = rng.integers(0, 32, (B, Hkv, Tcap, S)).astype(np.uint8)
    Ck = (rng.standard_normal((Hkv, S, 32, d)) * 0.5).astype(np.float32)
    Cv = rng.standard_normal((Hkv, S, 32, d)).astype(np.float32)
    wk = rng.standard_normal((B, Hkv, W, d)).astype(np.float16)
    wv = rng.standard_normal((B, Hkv, W, d)).astype(np.float16)
    comp = np.array([96, 37, 0], np.int32)
    win = np.array([8, 3, 5], np.int32)
    return q, kc, vc, comp, Ck, Cv, wk, wv, win


def _oracle_decode(q, kc, vc, comp, Ck, Cv, wk, wv, win, **_):
    from oracle import zkv_oracle as O
    o, l = O.decode_attn(*(t.numpy() for t in (q, kc, vc, comp, Ck, Cv, wk, wv, win)))
    return torch.from_numpy(o), torch.from_numpy(l)


def _oracle_merge(part_out, part_lse):
    from oracle import zkv_oracle as O
    N = part_out.shape[0]
    out = torch.empty(part_out.shape[1:], dtype=torch.float64)
    lse = torch.empty(part_lse.shape[1:], dtype=torch.float64)
    for b in range(out.shape[0]):
        for h in range(out.shape[1]):
            o, l = O.lse_merge([(part_out[i, b, h].numpy(), float(part_lse[i, b, h]))
                                for i in range(N)])
            out[b, h] = torch.from_numpy(np.asarray(o))
            lse[b, h] = l
    return out, lse


def _cp_rank(rank, world, port, result):
    from compressed_decode_attention_zkv_b200 import context_parallel as CP
    _init(rank, world, port)
    try:
        q, kc, vc, comp, Ck, Cv, wk, wv, win = (torch.from_numpy(a) for a in _case())
        kl, vl, cl = CP.take_shard(kc, vc, comp, rank, world)
        start, end = CP.shard_bounds(comp, rank, world)
        seen = []

        def decode(*args, **kw):
            seen.append(int(args[8].sum()))   # window tokens this rank attends
            return _oracle_decode(*args, **kw)

        out, lse = CP.cp_decode_attn(q, kl, vl, cl, Ck, Cv, wk, wv, win, decode_fn=decode,
                                     merge_fn=_oracle_merge)
        result[rank] = (out.numpy(), lse.numpy(), seen[0], start.numpy(), end.numpy(),
                        cl.numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_context_parallel_exchange_equals_unsharded_decode(world):
    result = mp.Manager().dict()
    mp.spawn(_cp_rank, args=(world, _free_port(), result), nprocs=world, join=True)
    from oracle import zkv_oracle as O
    q, kc, vc, comp, Ck, Cv, wk, wv, win = _case()
    want_o, want_l = O.decode_attn(q, kc, vc, comp, Ck, Cv, wk, wv, win)
    for r in range(world):
        out, lse, window_tokens, start, end, cl = result[r]
        np.testing.assert_allclose(out, want_o, atol=1e-9, rtol=0)
        fin = np.isfinite(want_l)
        assert np.array_equal(fin, np.isfinite(lse))
        np.testing.assert_allclose(lse[fin], want_l[fin], atol=1e-9, rtol=0)
        # the window is attended on the last rank only; the shards tile every prefix
        assert window_tokens == (int(win.sum()) if r == world - 1 else 0)
        np.testing.assert_array_equal(cl, end - start)
    np.testing.assert_array_equal(result[0][3], 0)
    for r in range(world - 1):
        np.testing.assert_array_equal(result[r][4], result[r + 1][3])
    np.testing.assert_array_equal(result[world - 1][4], comp)


class _FakeSymmMem:
    """Stands in for torch symmetric memory on CPU: plain tensors, and a rendezvous that
    exchanges every rank's data address (meaningless across processes, but enough to check
    the pointer tables the exchange builds)."""

    def empty(self, shape, dtype, device):
        return torch.zeros(shape, dtype=dtype, device=device)

    def rendezvous(self, t, group):
        mine = torch.tensor([t.data_ptr()], dtype=torch.int64)
        every = [torch.zeros(1, dtype=torch.int64) for _ in range(dist.get_world_size(group))]
        dist.all_gather(every, mine, group=group)

        class Handle:
            buffer_ptrs = [int(x) for x in every]
        return Handle()


def _fused_rank(rank, world, port, result):
    """cp_decode_attn with a PeerExchange: the decode writes into this step's slot set and the
    combine (emulated on CPU: gather the slots, oracle combine) receives the right pointer
    tables, epoch and parity, step after step."""
    from compressed_decode_attention_zkv_b200 import context_parallel as CP
    from oracle import zkv_oracle as O
    _init(rank, world, port)
    try:
        q, kc, vc, comp, Ck, Cv, wk, wv, win = (torch.from_numpy(a) for a in _case())
        kl, vl, cl = CP.take_shard(kc, vc, comp, rank, world)
        B, Hq, d = q.shape
        calls = []

        def decode_into(*args, out=None, lse=None, **kw):
            o, l = _oracle_decode(*args)
            out.copy_(o.to(torch.float32))
            lse.copy_(l.to(torch.float32))
            return out, lse

        def merge(out_ptrs, lse_ptrs, flag_ptrs, r, epoch, rows, dd, out=None, lse=None,
                  error_flag=None, timeout_s=None):
            s = epoch & 1
            calls.append((epoch, int(out_ptrs[r]), int(lse_ptrs[r]), int(flag_ptrs[r]),
                          ex.out_buf[s].data_ptr(), ex.lse_buf[s].data_ptr(),
                          ex.flag_buf.data_ptr(), r, rows, dd))
            outs = [torch.zeros(rows, dd) for _ in range(world)]
            lses = [torch.zeros(rows) for _ in range(world)]
            dist.all_gather(outs, ex.out_buf[s].clone())
            dist.all_gather(lses, ex.lse_buf[s].clone())
            o = torch.empty(rows, dd, dtype=torch.float64)
            lo = torch.empty(rows, dtype=torch.float64)
            for i in range(rows):
                oi, li = O.lse_merge([(outs[j][i].numpy(), float(lses[j][i]))
                                      for j in range(world)])
                o[i] = torch.from_numpy(np.asarray(oi))
                lo[i] = li
            return o, lo

        ex = CP.PeerExchange(B * Hq, d, device=torch.device("cpu"), symm_mem=_FakeSymmMem(),
                             merge_fn=merge)
        outs = []
        for _ in range(3):
            out, lse = CP.cp_decode_attn(q, kl, vl, cl, Ck, Cv, wk, wv, win, decode_fn=decode_into,
                                         exchange=ex)
            outs.append((out.numpy(), lse.numpy()))
        result[rank] = (outs, calls)
    finally:
        dist.destroy_process_group()


def test_context_parallel_fused_exchange_bookkeeping():
    world = 2
    result = mp.Manager().dict()
    mp.spawn(_fused_rank, args=(world, _free_port(), result), nprocs=world, join=True)
    from oracle import zkv_oracle as O
    q, kc, vc, comp, Ck, Cv, wk, wv, win = _case()
    want_o, want_l = O.decode_attn(q, kc, vc, comp, Ck, Cv, wk, wv, win)
    fin = np.isfinite(want_l)
    for r in range(world):
        outs, calls = result[r]
        for out, lse in outs:   # every step equals the unsharded decode (float32 partials)
            np.testing.assert_allclose(out, want_o, atol=1e-5, rtol=0)
            assert np.array_equal(fin, np.isfinite(lse))
            np.testing.assert_allclose(lse[fin], want_l[fin], atol=1e-5, rtol=0)
        assert [c[0] for c in calls] == [1, 2, 3]   # one epoch per step
        for epoch, o_ptr, l_ptr, f_ptr, o_slot, l_slot, f_buf, rr, rows, dd in calls:
            # this rank's entry of each table is the slot set of the step's parity
            assert (o_ptr, l_ptr, f_ptr) == (o_slot, l_slot, f_buf)
            assert rr == r and (rows, dd) == (q.shape[0] * q.shape[1], q.shape[2])
        assert calls[0][4] != calls[1][4] and calls[0][4] == calls[2][4]   # sets alternate


def _timing_rank(rank, world, port, result):
    import bench
    _init(rank, world, port)
    try:
        slowest = bench.max_over_ranks(1.0 + rank, world, torch.device("cpu"))
        result[rank] = (slowest, bench.weak_scaling_value(1000, world, slowest))
    finally:
        dist.destroy_process_group()


def test_bench_timing_is_the_slowest_rank_and_value_is_whole_job():
    world = 2
    result = mp.Manager().dict()
    mp.spawn(_timing_rank, args=(world, _free_port(), result), nprocs=world, join=True)
    for r in range(world):
        slowest, value = result[r]
        assert slowest == 2.0
        assert value == pytest.approx(1000 * 2 / 2.0)
