// Serving-step cache maintenance: window insert, eviction of the oldest window token, RVQ
// encode of the evicted token onto the compressed prefix (sm_100a).
//
// Passages: VQKV (gist.science summary of arXiv 2603.16435), section 2.3 "Local Sliding
// Window" (recent tokens uncompressed, older "middle" tokens compressed to codes); VeloxQuant-
// MLX 0.5.1 "Quick start" (cache.append(k, v) per token, then cache.attend(q)).
//
// Kernel 1 encodes the evicted rows and writes each new token into its window slot; kernel 2
// advances the lengths.  Both read the same pre-step lengths, so their decisions agree.
//
// Kernel 1 is a cluster of 8 CTAs per (group of 8 sequences, kv head, K or V).  CTA k of the
// cluster owns codewords [32k, 32k + 32) of every stage: it copies its slices with cp.async
// into a ring of kAppendNB buffers (up to kAppendNB - 1 stages ahead; all of them when
// S <= kAppendNB) and computes its 32 x 8 float32 distances.  Its candidates
// are the codewords within the rounding margin (the row encoder's bound, taken with this
// slice's largest codeword norm) of its own row minimum: a superset of the slice's codewords
// within the margin of the global minimum, so the exact argmin is always among them.  Each CTA
// publishes, per row, its best (float64 distance, index) and after one cluster barrier every
// CTA reduces the 8 published bests the same way (decided in float64, ties to the lowest
// index).  Within a CTA, warp r decides row r with no block-wide step (lane = local codeword);
// each CTA writes its per-row bests into every CTA of the cluster before the barrier, so the
// reduction after it reads local shared memory.  Every CTA keeps an identical copy of the
// residuals and reads the chosen codeword from its owner's shared memory.
#include <cooperative_groups.h>

#include "encode_rows.cuh"
#include "lengths.cuh"

namespace cg = cooperative_groups;

namespace zkv {

constexpr int kAppendR = 8;        // sequences per cluster
constexpr int kAppendCl = 8;       // CTAs per cluster
constexpr int kAppendCw = kCodebook / kAppendCl;   // codewords per CTA
constexpr int kAppendNB = 4;       // codeword slice buffers (stages in flight)

template <int D>
struct AppendSmem {
  static constexpr int LD = D + 4;            // padded row stride (conflict-free 16-byte reads)
  float cb[kAppendNB][kAppendCw * LD];        // this CTA's codeword slices, ring of stages
  float rows[kAppendR * LD];                  // residuals (identical in every CTA)
  double rn[kAppendR];                        // residual norms
  float dist[kAppendCw][kAppendR];            // float32 distances of this CTA's codewords
  float cnorm[kAppendCw];                     // their squared norms
  // every CTA's per-row best (float64 distance, codeword), written by that CTA into every
  // CTA of the cluster; by stage parity
  double pub_d[2][kAppendCl][kAppendR];
  int pub_c[2][kAppendCl][kAppendR];
  uint8_t code[kAppendR][kMaxStages];
};

template <int D>
__global__ void __cluster_dims__(kAppendCl, 1, 1) __launch_bounds__(256)
    append_cluster_kernel(zkv_append_params p, double rot) {
  constexpr int E = D / 32;
  constexpr int LD = AppendSmem<D>::LD;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  AppendSmem<D>& sm = *reinterpret_cast<AppendSmem<D>*>(smem_raw);
  pdl_trigger();   // the length update may launch now; it waits for this kernel's completion
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = (int)cluster.block_rank();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int kind = blockIdx.z;   // 0 = keys, 1 = values
  const int h = blockIdx.y;
  const int64_t row0 = (int64_t)(blockIdx.x / kAppendCl) * kAppendR;
  const int S = kind ? p.Sv : p.Sk;
  const float* CB = (kind ? p.v_codebooks : p.k_codebooks) + (size_t)h * S * kCodebook * D;
  const __half* win = reinterpret_cast<const __half*>(kind ? p.win_v : p.win_k);
  uint8_t* codes = kind ? p.v_codes : p.k_codes;

  auto row_valid = [&](int64_t j) {   // sequence j evicts a token into a prefix with room
    if (j >= p.B) return false;
    const int64_t wl = p.win_len[j], hd = p.win_head[j], c = p.comp_len[j];
    return wl == p.Wcap && hd >= 0 && hd < p.Wcap && c >= 0 && c < p.Tcap;
  };
  auto load_slice = [&](int s) {      // stage s, codewords [32 rank, 32 rank + 32)
    const float* src = CB + ((size_t)s * kCodebook + (size_t)rank * kAppendCw) * D;
    float* dst = sm.cb[s % kAppendNB];
    for (int f = tid; f < kAppendCw * D / 4; f += 256) {
      const int cl = f / (D / 4), q = f % (D / 4);
      cp_async16(dst + cl * LD + 4 * q, src + (size_t)cl * D + 4 * q);
    }
    cp_async_commit();
  };

  // the first slices; every later one is issued (one commit group per stage) after the cluster
  // barrier of the stage whose buffer it reuses has been passed
  for (int q = 0; q < kAppendNB - 1 && q < S; ++q) load_slice(q);
  // rotated rows (every CTA of the cluster computes the same values)
  if (warp < kAppendR) {
    const int64_t j = row0 + warp;
    double ss = 0.0;
    if (row_valid(j)) {
      double v[E];
      load_row_f64<E>(win, ZKV_DTYPE_F16, ((j * p.Hkv + h) * p.Wcap + p.win_head[j]) * D, lane, v);
      if (kind == 0 && p.k_smooth) {   // keys: x / lambda per channel before the rotation
        const float* l = p.k_smooth + (int64_t)h * D;
#pragma unroll
        for (int q = 0; q < E; ++q) v[q] *= 1.0 / (double)l[q * 32 + lane];
      }
      fwht_warp_f64<D>(v, lane);
#pragma unroll
      for (int q = 0; q < E; ++q) {
        const float y = (float)(v[q] * rot);
        sm.rows[warp * LD + q * 32 + lane] = y;
        ss += (double)y * (double)y;
      }
    } else {
#pragma unroll
      for (int q = 0; q < E; ++q) sm.rows[warp * LD + q * 32 + lane] = 0.f;
    }
    ss = warp_sum_f64(ss);
    if (lane == 0) sm.rn[warp] = sqrt(ss);
  }

  // distance pass: thread = (codeword pair, row half, dimension slice); slice ks holds the
  // 16-byte chunks 4 ks + 32 j of every vector (conflict-free 16-byte reads)
  const int ks = tid & 7, cpair = (tid >> 3) & 15, rhalf = tid >> 7;
  for (int s = 0; s < S; ++s) {
    // groups committed so far: stages 0 .. min(s + NB - 2, S - 1); stage s must be complete
    const int later = (s + kAppendNB - 2 < S - 1 ? s + kAppendNB - 2 : S - 1) - s;
    if (later >= 2) asm volatile("cp.async.wait_group 2;" ::: "memory");
    else if (later == 1) asm volatile("cp.async.wait_group 1;" ::: "memory");
    else asm volatile("cp.async.wait_group 0;" ::: "memory");
    __syncthreads();   // slice s and the residuals are ready
    const float* slice = sm.cb[s % kAppendNB];
    {
      float acc[2][4], cn[2];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        cn[u] = 0.f;
#pragma unroll
        for (int v = 0; v < 4; ++v) acc[u][v] = 0.f;
      }
#pragma unroll
      for (int j = 0; j < D / 32; ++j) {
        const int off = 4 * ks + 32 * j;
        float4 c4[2], x4[4];
#pragma unroll
        for (int u = 0; u < 2; ++u) c4[u] = *reinterpret_cast<const float4*>(slice + (2 * cpair + u) * LD + off);
#pragma unroll
        for (int v = 0; v < 4; ++v) x4[v] = *reinterpret_cast<const float4*>(sm.rows + (4 * rhalf + v) * LD + off);
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          cn[u] = fmaf(c4[u].x, c4[u].x, cn[u]);
          cn[u] = fmaf(c4[u].y, c4[u].y, cn[u]);
          cn[u] = fmaf(c4[u].z, c4[u].z, cn[u]);
          cn[u] = fmaf(c4[u].w, c4[u].w, cn[u]);
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            acc[u][v] = fmaf(x4[v].x, c4[u].x, acc[u][v]);
            acc[u][v] = fmaf(x4[v].y, c4[u].y, acc[u][v]);
            acc[u][v] = fmaf(x4[v].z, c4[u].z, acc[u][v]);
            acc[u][v] = fmaf(x4[v].w, c4[u].w, acc[u][v]);
          }
        }
      }
      // sum over the 8 slices (lanes differing in bits 0-2); the rounding bound used for the
      // margin holds for any summation order
#pragma unroll
      for (int o = 1; o < 8; o <<= 1) {
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          cn[u] += __shfl_xor_sync(0xffffffffu, cn[u], o);
#pragma unroll
          for (int v = 0; v < 4; ++v) acc[u][v] += __shfl_xor_sync(0xffffffffu, acc[u][v], o);
        }
      }
      if (ks == 0) {
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          if (rhalf == 0) sm.cnorm[2 * cpair + u] = cn[u];
#pragma unroll
          for (int v = 0; v < 4; ++v) sm.dist[2 * cpair + u][4 * rhalf + v] = cn[u] - 2.f * acc[u][v];
        }
      }
    }
    __syncthreads();
    // warp r decides row r among this CTA's codewords (lane = local codeword): the row minimum
    // of the float32 distances, the candidates within the margin (taken with this slice's
    // largest codeword norm), their float64 distances, the best (lowest index on ties); it
    // then writes that best into every CTA of the cluster
    static_assert(kAppendCw == 32, "one lane per local codeword");
    if (warp < kAppendR) {
      const int r = warp;
      const float dr = sm.dist[lane][r];
      const float cmax = warp_max_f32(sm.cnorm[lane]);
      const float dmin = warp_min_f32(dr);
      const double thr = (double)dmin + candidate_margin(sm.rn[r], cmax, D);
      unsigned cand = __ballot_sync(0xffffffffu, (double)dr <= thr);
      double bd = DBL_MAX;
      int bc = kCodebook;
      while (cand) {
        const int c = __ffs(cand) - 1;
        cand &= cand - 1u;
        double a = 0.0;
#pragma unroll
        for (int q = 0; q < E; ++q) {
          const int i = q * 32 + lane;
          const double df = (double)sm.rows[r * LD + i] - (double)slice[c * LD + i];
          a = fma(df, df, a);
        }
        a = warp_sum_f64(a);
        const int gc = rank * kAppendCw + c;
        if (a < bd || (a == bd && gc < bc)) {
          bd = a;
          bc = gc;
        }
      }
      if (lane < kAppendCl) {
        AppendSmem<D>* o = cluster.map_shared_rank(&sm, lane);
        o->pub_d[s & 1][rank][r] = bd;
        o->pub_c[s & 1][rank][r] = bc;
      }
    }
    // every CTA's bests have arrived here; every read of stage s-1's slices is done
    cluster.sync();
    // the buffer of stage s-1 is free (its remote reads are done): refill it NB - 1 stages ahead
    if (s + kAppendNB - 1 < S) load_slice(s + kAppendNB - 1);
    // warp r: the cluster's best for row r (min over the 8 published bests, lowest index on
    // ties), then the residual update with that codeword, read from its owner's slice
    if (warp < kAppendR) {
      const int r = warp;
      double bd = lane < kAppendCl ? sm.pub_d[s & 1][lane][r] : DBL_MAX;
      int bc = lane < kAppendCl ? sm.pub_c[s & 1][lane][r] : kCodebook;
#pragma unroll
      for (int o = 1; o < kAppendCl; o <<= 1) {
        const double od = __shfl_xor_sync(0xffffffffu, bd, o);
        const int oc = __shfl_xor_sync(0xffffffffu, bc, o);
        if (od < bd || (od == bd && oc < bc)) {
          bd = od;
          bc = oc;
        }
      }
      // every lane of the warp holds the same choice (lanes 0-7 reduced the same set; the
      // others take lane 0's); non-finite rows match no candidate: never index past the
      // stage's codebook
      bc = __shfl_sync(0xffffffffu, bc, 0);
      const int z = bc < kCodebook ? bc : 0;
      const float* src = cluster.map_shared_rank(&sm.cb[s % kAppendNB][0], z / kAppendCw) + (z % kAppendCw) * LD;
      double ss = 0.0;
#pragma unroll
      for (int q = 0; q < E; ++q) {
        const int i = q * 32 + lane;
        const float nr = sm.rows[r * LD + i] - src[i];
        sm.rows[r * LD + i] = nr;
        ss += (double)nr * (double)nr;
      }
      ss = warp_sum_f64(ss);
      if (lane == 0) {
        sm.rn[r] = sqrt(ss);
        sm.code[r][s] = (uint8_t)z;
      }
    }
  }
  cluster.sync();   // no CTA leaves while another may still read its shared memory
  // Launched as a dependent of the table kernel (the serving step), this kernel completes only
  // after that kernel has: whatever waits for this one then also sees the tables.  Returns at
  // once after a normal launch.
  pdl_wait();
  if (rank != 0) return;
  if (tid < kAppendR) {
    const int64_t j = row0 + tid;
    if (row_valid(j)) {
      const int64_t t = p.comp_len[j];
      uint8_t* c = nullptr;
      if (!p.block_table) {
        c = codes + ((j * p.Hkv + h) * p.Tcap + t) * S;
      } else {   // paged: row (h, t % P) of page block_table[j][t / P]
        const int64_t P = p.page_tokens;
        const int64_t pg = p.block_table[j * p.max_pages + t / P];
        if (pg >= 0 && pg < p.n_pages) c = codes + ((pg * p.Hkv + h) * P + t % P) * S;
        else set_error(p.error_flag, ZKV_DEVERR_PAGE);
      }
      if (c)
        for (int s = 0; s < S; ++s) c[s] = sm.code[tid][s];
    }
  }
  // every CTA read the evicted slots before its first cluster barrier
  if (warp < kAppendR) {
    const int64_t j = row0 + warp;
    if (j >= p.B) return;
    const int64_t wl = p.win_len[j], hd = p.win_head[j], c = p.comp_len[j];
    int64_t slot = -1;
    if (wl >= 0 && wl < p.Wcap) {
      slot = wl;
    } else if (wl == p.Wcap && hd >= 0 && hd < p.Wcap) {
      if (c >= 0 && c < p.Tcap) slot = hd;
      else if (lane == 0 && kind == 0 && h == 0) set_error(p.error_flag, ZKV_DEVERR_COMP_LEN);
    } else if (lane == 0 && kind == 0 && h == 0) {
      set_error(p.error_flag, ZKV_DEVERR_WIN_LEN);
    }
    if (slot < 0) return;
    const __half* src = reinterpret_cast<const __half*>(kind ? p.new_v : p.new_k) + (j * p.Hkv + h) * D;
    __half* dst = reinterpret_cast<__half*>(kind ? p.win_v : p.win_k) + ((j * p.Hkv + h) * p.Wcap + slot) * D;
    for (int i = lane; i < D; i += 32) dst[i] = src[i];
  }
}

__global__ void append_lengths_kernel(int B, int64_t Tcap, int64_t Wcap, int32_t* win_len,
                                      int32_t* win_head, int32_t* comp_len) {
  pdl_wait();   // the encode kernel read the pre-step lengths
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= B) return;
  advance_lengths(b, Tcap, Wcap, win_len, win_head, comp_len);
}

int validate_append(const zkv_append_params* p) {
  if (!p) return ZKV_ERR_INVALID_ARG;
  if (p->B < 1 || p->Hkv < 1 || p->Tcap < 0 || p->Wcap < 1) return ZKV_ERR_INVALID_ARG;
  if (!supported_d(p->d)) return ZKV_ERR_UNSUPPORTED;
  if (p->Sk < 1 || p->Sk > kMaxStages || p->Sv < 1 || p->Sv > kMaxStages) return ZKV_ERR_UNSUPPORTED;
  if (p->Hkv > 65535) return ZKV_ERR_UNSUPPORTED;
  if (!p->new_k || !p->new_v || !p->win_k || !p->win_v || !p->win_len || !p->win_head ||
      !p->comp_len || !p->k_codes || !p->v_codes || !p->k_codebooks || !p->v_codebooks)
    return ZKV_ERR_INVALID_ARG;
  const uintptr_t al = (uintptr_t)p->win_k | (uintptr_t)p->win_v | (uintptr_t)p->k_codebooks |
                       (uintptr_t)p->v_codebooks;
  if (al & 15) return ZKV_ERR_INVALID_ARG;
  return validate_paged(p->block_table, p->page_tokens, p->max_pages, p->n_pages, p->Tcap);
}

// The encode + window-write kernel; with pdl, as a programmatic dependent of the previous
// kernel on the stream (it never reads that kernel's results).
int launch_append_cluster(const zkv_append_params& p, cudaStream_t st, bool pdl) {
  const double rot = 1.0 / std::sqrt((double)p.d);
  const unsigned groups = (unsigned)((p.B + kAppendR - 1) / kAppendR);
  const dim3 grid(groups * kAppendCl, (unsigned)p.Hkv, 2);
  const bool ok =
      ensure_smem_limit(append_cluster_kernel<64>, sizeof(AppendSmem<64>)) == cudaSuccess &&
      ensure_smem_limit(append_cluster_kernel<128>, sizeof(AppendSmem<128>)) == cudaSuccess &&
      ensure_smem_limit(append_cluster_kernel<256>, sizeof(AppendSmem<256>)) == cudaSuccess;
  if (!ok) return ZKV_ERR_CUDA;
  cudaError_t e = cudaSuccess;
  switch (p.d) {
    case 64:
      if (pdl) e = launch_pdl(append_cluster_kernel<64>, grid, dim3(256), sizeof(AppendSmem<64>), st, p, rot);
      else append_cluster_kernel<64><<<grid, 256, sizeof(AppendSmem<64>), st>>>(p, rot);
      break;
    case 128:
      if (pdl) e = launch_pdl(append_cluster_kernel<128>, grid, dim3(256), sizeof(AppendSmem<128>), st, p, rot);
      else append_cluster_kernel<128><<<grid, 256, sizeof(AppendSmem<128>), st>>>(p, rot);
      break;
    default:
      if (pdl) e = launch_pdl(append_cluster_kernel<256>, grid, dim3(256), sizeof(AppendSmem<256>), st, p, rot);
      else append_cluster_kernel<256><<<grid, 256, sizeof(AppendSmem<256>), st>>>(p, rot);
      break;
  }
  if (e != cudaSuccess) return ZKV_ERR_CUDA;
  ZKV_CHECK_LAUNCH();
  return ZKV_OK;
}

}  // namespace zkv

using namespace zkv;

extern "C" int zkv_rvq_append(const zkv_append_params* p, void* stream) {
  const int v = validate_append(p);
  if (v != ZKV_OK) return v;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int rc = launch_append_cluster(*p, st, false);
  if (rc != ZKV_OK) return rc;
  if (launch_pdl(append_lengths_kernel, dim3((p->B + 127) / 128), dim3(128), 0, st, p->B, p->Tcap,
                 p->Wcap, p->win_len, p->win_head, p->comp_len) != cudaSuccess)
    return ZKV_ERR_CUDA;
  return ZKV_OK;
}
