"""Context-parallel decode attention over an RVQ-compressed prefix sharded by tokens.

Passages: VQKV (gist.science summary of arXiv 2603.16435), section 2.3 "Decoding Stage"
(attention reads the codes of the compressed prefix); Differential-KV README, "Decode &
Prefill Innovations" (fp32 log-sum-exp combine of partial results over disjoint key sets).

Each rank of a process group holds one contiguous shard of every sequence's compressed tokens
(an equal split, ``shard_bounds``) in its own code arrays.  A decode step is: the library's
decode attention over the local shard (the fp16 recency window is counted on one rank only),
ONE all-gather of the packed rows (out, lse) [B, Hq, d + 1] over the group (NCCL over NVLink on
GPUs), and the library's log-sum-exp combine (``zkv.lse_merge``) of the gathered parts.  Every
rank ends with the full (out, lse).  This is the only exchange the path has: the shards' partial
attentions are independent until the combine.

With a ``PeerExchange`` the gather and the combine are one kernel (``zkv.lse_merge_peers``):
each rank's decode writes its partial straight into buffers mapped into every rank (torch
symmetric memory), and the kernel signals the peers, waits for their signals (bounded) and
combines every rank's rows read directly from its memory over NVLink -- no gathered copy and
no separate collective.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import zkv


def shard_bounds(comp_len: torch.Tensor, rank: int, world: int):
    """Per sequence, the [start, end) of the compressed tokens rank ``rank`` of ``world`` holds:
    start = floor(c r / N), end = floor(c (r + 1) / N) (int64 tensors on comp_len's device)."""
    c = comp_len.to(torch.int64)
    return (c * rank) // world, (c * (rank + 1)) // world


def take_shard(k_codes: torch.Tensor, v_codes: torch.Tensor, comp_len: torch.Tensor, rank: int,
               world: int, capacity: int | None = None):
    """Copy this rank's shard of full code arrays [B, Hkv, Tcap, S] into local arrays
    [B, Hkv, capacity, S] (capacity rounded up to a multiple of 16; default: the largest shard).
    Returns (k_local, v_local, comp_len_local int32).  For building shards from a prefill or a
    single-GPU cache; a serving deployment prefills each rank's shard directly."""
    start, end = shard_bounds(comp_len, rank, world)
    n = end - start
    cap = int(n.max().item()) if capacity is None else int(capacity)
    cap = max(16, (cap + 15) // 16 * 16)
    B, Hkv, _, Sk = k_codes.shape
    kl = torch.zeros((B, Hkv, cap, Sk), dtype=k_codes.dtype, device=k_codes.device)
    vl = torch.zeros((B, Hkv, cap, v_codes.shape[3]), dtype=v_codes.dtype, device=v_codes.device)
    for b in range(B):
        s, e = int(start[b]), int(end[b])
        kl[b, :, :e - s] = k_codes[b, :, s:e]
        vl[b, :, :e - s] = v_codes[b, :, s:e]
    return kl, vl, n.to(torch.int32)


class PeerExchange:
    """Peer-mapped buffers of the fused exchange for partials of ``rows`` rows of ``d`` floats:
    two sets (alternating by step parity) of out [rows, d] and lse [rows] float32, and one
    int32 flag array [world], allocated as torch symmetric memory and mapped into every rank
    of ``group``.  A step: the local decode writes into ``slots()``, then ``combine()`` runs
    zkv.lse_merge_peers on this step's set.  Alternating the sets by parity is what makes
    reuse safe: a rank rewrites a set only after its previous combine saw every rank's signal
    for the step after the one that last read it.
    ``symm_mem`` / ``merge_fn`` can be replaced (host-side tests without GPUs)."""

    def __init__(self, rows: int, d: int, group=None, device=None, timeout_s: float = 2.0,
                 symm_mem=None, merge_fn=None):
        if symm_mem is None:
            import torch.distributed._symmetric_memory as symm_mem
        self.group = group if group is not None else dist.group.WORLD
        self.world = dist.get_world_size(self.group)
        self.rank = dist.get_rank(self.group)
        if device is None:
            device = torch.device("cuda", torch.cuda.current_device())
        self.rows, self.d, self.timeout_s = rows, d, timeout_s
        self.merge_fn = zkv.lse_merge_peers if merge_fn is None else merge_fn
        enable = getattr(symm_mem, "enable_symm_mem_for_group", None)
        if enable is not None:   # required before a rendezvous by some torch versions
            enable(self.group.group_name)
        self.out_buf = symm_mem.empty((2, rows, d), dtype=torch.float32, device=device)
        self.lse_buf = symm_mem.empty((2, rows), dtype=torch.float32, device=device)
        self.flag_buf = symm_mem.empty((self.world,), dtype=torch.int32, device=device)
        self.flag_buf.zero_()
        addr = [self._peer_addresses(symm_mem, t) for t in (self.out_buf, self.lse_buf,
                                                              self.flag_buf)]
        # pointer tables per parity: rank i's set s of out rows / lse rows, and its flags
        self.out_ptrs = [self._table([a + s * rows * d * 4 for a in addr[0]], device)
                         for s in (0, 1)]
        self.lse_ptrs = [self._table([a + s * rows * 4 for a in addr[1]], device)
                         for s in (0, 1)]
        self.flag_ptrs = self._table(addr[2], device)
        self.epoch = 0
        dist.barrier(group=self.group)   # every rank's flags are zero before anyone signals

    def _peer_addresses(self, symm_mem, t):
        """Every rank's address of tensor t (a symmetric allocation), as mapped here."""
        try:
            hdl = symm_mem.rendezvous(t, self.group)
        except TypeError:
            hdl = symm_mem.rendezvous(t, self.group.group_name)
        base = list(hdl.buffer_ptrs)
        off = t.data_ptr() - base[self.rank]   # t may sit inside a larger symmetric block
        return [b + off for b in base]

    @staticmethod
    def _table(addresses, device):
        return torch.tensor(addresses, dtype=torch.int64, device=device)

    def slots(self):
        """(out [rows, d], lse [rows]) this rank's decode writes for the coming step."""
        s = (self.epoch + 1) & 1
        return self.out_buf[s], self.lse_buf[s]

    def combine(self, out=None, lse=None, error_flag=None):
        """Signal, wait for every rank (bounded) and combine this step's partials: returns
        (out float32 [rows, d], lse float32 [rows])."""
        self.epoch += 1
        s = self.epoch & 1
        return self.merge_fn(self.out_ptrs[s], self.lse_ptrs[s], self.flag_ptrs, self.rank,
                             self.epoch, self.rows, self.d, out=out, lse=lse,
                             error_flag=error_flag, timeout_s=self.timeout_s)


def cp_decode_attn(q, k_codes, v_codes, comp_len, k_codebooks, v_codebooks, win_k, win_v,
                   win_len, group=None, window_rank: int | None = None, decode_fn=None,
                   merge_fn=None, exchange: PeerExchange | None = None, **decode_kw):
    """One context-parallel decode step.  k_codes / v_codes / comp_len: this rank's shard (as
    ``take_shard`` makes it); q, codebooks and window: the same on every rank.  The window is
    attended on ``window_rank`` (default: the last rank) and left out elsewhere.
    ``decode_fn`` / ``merge_fn`` default to the library's zkv.rvq_decode_attn / zkv.lse_merge
    (replaceable so that the exchange logic can be exercised without a GPU).  With
    ``exchange`` (a PeerExchange over B * Hq rows of d) the decode writes into the mapped
    buffers and the gather + combine run as one kernel over peer memory.
    Returns (out float32 [B, Hq, d], lse float32 [B, Hq]) on every rank."""
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    wr = world - 1 if window_rank is None else window_rank
    wl = win_len if rank == wr else torch.zeros_like(win_len)
    decode_fn = zkv.rvq_decode_attn if decode_fn is None else decode_fn
    merge_fn = zkv.lse_merge if merge_fn is None else merge_fn
    if exchange is not None:   # fused: decode into the mapped buffers, one exchange+combine kernel
        B, Hq, d = q.shape
        o_slot, l_slot = exchange.slots()
        decode_fn(q, k_codes, v_codes, comp_len, k_codebooks, v_codebooks, win_k, win_v, wl,
                  out=o_slot.view(B, Hq, d), lse=l_slot.view(B, Hq), **decode_kw)
        out, lse = exchange.combine()
        return out.view(B, Hq, d), lse.view(B, Hq)
    out, lse = decode_fn(q, k_codes, v_codes, comp_len, k_codebooks, v_codebooks, win_k, win_v,
                         wl, **decode_kw)
    d = out.shape[-1]
    packed = torch.cat([out, lse[..., None]], dim=-1).contiguous()   # [B, Hq, d + 1]
    gathered = torch.empty((world,) + tuple(packed.shape), dtype=packed.dtype,
                           device=packed.device)
    if dist.get_backend(group) == "nccl":
        dist.all_gather_into_tensor(gathered, packed, group=group)
    else:
        dist.all_gather(list(gathered.unbind(0)), packed, group=group)
    return merge_fn(gathered[..., :d], gathered[..., d])
