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


def cp_decode_attn(q, k_codes, v_codes, comp_len, k_codebooks, v_codebooks, win_k, win_v,
                   win_len, group=None, window_rank: int | None = None, decode_fn=None,
                   merge_fn=None, **decode_kw):
    """One context-parallel decode step.  k_codes / v_codes / comp_len: this rank's shard (as
    ``take_shard`` makes it); q, codebooks and window: the same on every rank.  The window is
    attended on ``window_rank`` (default: the last rank) and left out elsewhere.
    ``decode_fn`` / ``merge_fn`` default to the library's zkv.rvq_decode_attn / zkv.lse_merge
    (replaceable so that the exchange logic can be exercised without a GPU).
    Returns (out float32 [B, Hq, d], lse float32 [B, Hq]) on every rank."""
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    wr = world - 1 if window_rank is None else window_rank
    wl = win_len if rank == wr else torch.zeros_like(win_len)
    decode_fn = zkv.rvq_decode_attn if decode_fn is None else decode_fn
    merge_fn = zkv.lse_merge if merge_fn is None else merge_fn
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
