// zkv_lse_merge: log-sum-exp combine of partial attentions over disjoint key sets.
//
// Passage: Differential-KV README, "Decode & Prefill Innovations" (flash-style fp32 log-sum-exp
// combine of partial attention results).  Used by context-parallel decode, where every rank
// attends over its own shard of each sequence's compressed prefix and the shards' (out, lse)
// are gathered and combined:
//   M = max_i lse_i;  w_i = exp(lse_i - M);  L = sum_i w_i;
//   out = sum_i w_i out_i / L;  lse = M + log L;
// parts with lse = -inf (no keys) carry weight 0; when every part is empty, out = 0 and
// lse = -inf.
#include "zkv_internal.cuh"

namespace zkv {

// One warp per row; every lane recomputes the row's weights (n_parts is small) and owns the
// columns lane, lane + 32, ...
__global__ void __launch_bounds__(256) lse_merge_kernel(zkv_lse_merge_params p) {
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (row >= p.rows) return;
  const float* lse_in = p.part_lse + row * p.lse_row_stride;   // part i at lse_in[i * stride]
  const float* out_in = p.part_out + row * p.out_row_stride;
  float M = -INFINITY;
  for (int64_t i = 0; i < p.n_parts; ++i) M = fmaxf(M, lse_in[i * p.lse_part_stride]);
  float* o = p.out + row * p.d;
  if (M == -INFINITY) {
    for (int e = lane; e < p.d; e += 32) o[e] = 0.f;
    if (lane == 0 && p.lse) p.lse[row] = -INFINITY;
    return;
  }
  float L = 0.f;
  for (int64_t i = 0; i < p.n_parts; ++i) {
    const float l = lse_in[i * p.lse_part_stride];
    L += l == -INFINITY ? 0.f : expf(l - M);
  }
  const float inv = 1.f / L;
  for (int e = lane; e < p.d; e += 32) {
    float acc = 0.f;
    for (int64_t i = 0; i < p.n_parts; ++i) {
      const float l = lse_in[i * p.lse_part_stride];
      if (l == -INFINITY) continue;
      acc = fmaf(expf(l - M), out_in[i * p.out_part_stride + e], acc);
    }
    o[e] = acc * inv;
  }
  if (lane == 0 && p.lse) p.lse[row] = M + logf(L);
}

}  // namespace zkv

using namespace zkv;

extern "C" int zkv_lse_merge(const zkv_lse_merge_params* p, void* stream) {
  if (!p) return ZKV_ERR_INVALID_ARG;
  if (p->n_parts < 1 || p->rows < 0 || p->d < 1 || p->d > 4096) return ZKV_ERR_INVALID_ARG;
  if (p->rows == 0) return ZKV_OK;
  if (!p->part_out || !p->part_lse || !p->out) return ZKV_ERR_INVALID_ARG;
  if ((p->rows + 7) / 8 > 0x7fffffffLL) return ZKV_ERR_UNSUPPORTED;
  lse_merge_kernel<<<(unsigned)((p->rows + 7) / 8), 256, 0,
                     reinterpret_cast<cudaStream_t>(stream)>>>(*p);
  ZKV_CHECK_LAUNCH();
  return ZKV_OK;
}
