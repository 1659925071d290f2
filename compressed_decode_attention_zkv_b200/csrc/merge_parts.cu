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
//
// zkv_lse_merge_peers fuses the exchange into the combine: the kernel signals the peers
// through flag words in their memory, waits (bounded by the global timer) for theirs, and
// reads their partial rows directly over NVLink, so no gather step or gathered copy exists.
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

// ---- the same combine, fused with the exchange over peer memory -------------------------

__device__ __forceinline__ uint32_t ld_acquire_sys_u32(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.sys.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_release_sys_u32(uint32_t* p, uint32_t v) {
  asm volatile("st.release.sys.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// One warp per row, as lse_merge_kernel, after the block has seen every rank's signal.
__global__ void __launch_bounds__(256) lse_merge_peers_kernel(zkv_lse_merge_peers_params p) {
  __shared__ int ready;
  const int tid = threadIdx.x, lane = tid & 31;
  // 1. signal: this rank's partial rows (written by earlier work on this stream) are complete.
  //    Every block stores the same value, so no block depends on another being scheduled.
  if (tid < p.n_ranks) {
    __threadfence_system();
    st_release_sys_u32(p.flags[tid] + p.rank, p.epoch);
  }
  // 2. bounded wait for every rank's signal in this rank's flag array
  if (tid == 0) {
    const uint32_t* mine = p.flags[p.rank];
    const uint64_t t0 = global_timer_ns();
    int ok = 1;
    for (int i = 0; i < p.n_ranks && ok; ++i) {
      while ((int32_t)(ld_acquire_sys_u32(mine + i) - p.epoch) < 0) {
        if (global_timer_ns() - t0 > (uint64_t)p.timeout_ns) {
          ok = 0;
          break;
        }
      }
    }
    if (!ok) set_error(p.error_flag, ZKV_DEVERR_TIMEOUT);
    ready = ok;
  }
  __syncthreads();
  if (!ready) return;
  // 3. combine, reading the peers' rows over NVLink (loads that bypass the caches)
  const int64_t row = (int64_t)blockIdx.x * 8 + (tid >> 5);
  if (row >= p.rows) return;
  float M = -INFINITY;
  for (int i = 0; i < p.n_ranks; ++i) M = fmaxf(M, __ldcv(p.part_lse[i] + row));
  float* o = p.out + row * p.d;
  if (M == -INFINITY) {
    for (int e = lane; e < p.d; e += 32) o[e] = 0.f;
    if (lane == 0 && p.lse) p.lse[row] = -INFINITY;
    return;
  }
  float L = 0.f;
  for (int i = 0; i < p.n_ranks; ++i) {
    const float l = __ldcv(p.part_lse[i] + row);
    L += l == -INFINITY ? 0.f : expf(l - M);
  }
  const float inv = 1.f / L;
  for (int e = lane; e < p.d; e += 32) {
    float acc = 0.f;
    for (int i = 0; i < p.n_ranks; ++i) {
      const float l = __ldcv(p.part_lse[i] + row);
      if (l == -INFINITY) continue;
      acc = fmaf(expf(l - M), __ldcv(p.part_out[i] + row * p.d + e), acc);
    }
    o[e] = acc * inv;
  }
  if (lane == 0 && p.lse) p.lse[row] = M + logf(L);
}

}  // namespace zkv

using namespace zkv;

extern "C" int zkv_lse_merge_peers(const zkv_lse_merge_peers_params* p, void* stream) {
  if (!p) return ZKV_ERR_INVALID_ARG;
  if (p->n_ranks < 1 || p->n_ranks > 64 || p->rank < 0 || p->rank >= p->n_ranks)
    return ZKV_ERR_INVALID_ARG;
  if (p->rows < 0 || p->d < 1 || p->d > 4096 || p->epoch == 0 || p->timeout_ns <= 0)
    return ZKV_ERR_INVALID_ARG;
  if (!p->part_out || !p->part_lse || !p->flags || (p->rows > 0 && !p->out))
    return ZKV_ERR_INVALID_ARG;
  if ((p->rows + 7) / 8 > 0x7fffffffLL) return ZKV_ERR_UNSUPPORTED;
  // one block at least: the signal is sent even when there are no rows to combine
  const unsigned blocks = (unsigned)(p->rows > 0 ? (p->rows + 7) / 8 : 1);
  lse_merge_peers_kernel<<<blocks, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(*p);
  ZKV_CHECK_LAUNCH();
  return ZKV_OK;
}

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
