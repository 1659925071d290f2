// Per-sequence length update of one serving step (shared by the append call and the fused
// serving step).
//
// Passage: VQKV (gist.science summary of arXiv 2603.16435), section 2.3 "Local Sliding
// Window": the newest tokens stay in the fp16 window; once it is full, each new token evicts
// the oldest one, which joins the compressed prefix.
#pragma once

#include <cstdint>

namespace zkv {

// win_len < Wcap: the new token fills a free slot.  Otherwise the oldest slot (win_head) is
// evicted onto the prefix (comp_len + 1) and reused (win_head advances).  Out-of-range state is
// left unchanged (the encode kernel reports it).
__device__ __forceinline__ void advance_lengths(int b, int64_t Tcap, int64_t Wcap, int32_t* win_len,
                                                int32_t* win_head, int32_t* comp_len) {
  const int64_t wl = win_len[b];
  if (wl < 0 || wl > Wcap) return;
  if (wl < Wcap) {
    win_len[b] = (int32_t)(wl + 1);
    return;
  }
  const int64_t c = comp_len[b], hd = win_head[b];
  if (c < 0 || c >= Tcap || hd < 0 || hd >= Wcap) return;
  comp_len[b] = (int32_t)(c + 1);
  win_head[b] = (int32_t)((hd + 1) % Wcap);
}

}  // namespace zkv
