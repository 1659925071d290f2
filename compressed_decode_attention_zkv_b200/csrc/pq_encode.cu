// zkv_pq_encode: product vector quantisation of KV head vectors (sm_100a).
//
// Passage: VeloxQuant-MLX 0.5.1, "VecInfer": the (smoothed, Walsh-Hadamard rotated) vector is
// quantised against a pre-trained K-means codebook by sub-vectors (key_sub_dim 4 or 8 with
// 8-bit codes: 2 or 1 bits per element).  One 256-entry codebook of m-dim sub-vectors per head
// is shared by the d/m consecutive sub-vectors of the rotated vector.
//
// One warp per row: the row is loaded, optionally divided by the smoothing factors, rotated in
// float64 and rounded once to float32 (the same transform as the RVQ encoders), and staged in
// shared memory; lane j then takes sub-vectors j, j + 32, ... and scans the head's codebook
// (broadcast reads from shared memory) with float64 distances, keeping the first minimum
// (lowest index on ties).
//
// zkv_pq_append: the serving-step append of a product-VQ cache.  One block per (group of 8
// sequences, kv head, K or V); warp w takes sequence 8 * group + w: it decides from the
// pre-step lengths whether a token is evicted, encodes the evicted window row exactly as
// zkv_pq_encode does, writes the codes at position comp_len, and writes the new token into the
// window slot.  A second kernel advances the lengths (both read the same pre-step values).
#include "encode_rows.cuh"
#include "lengths.cuh"

namespace zkv {

constexpr int kPqRows = 8;   // rows (warps) per block

// The nearest codeword of the shared codebook cb [256][M] (shared memory) to sub-vector y,
// float64 distances in coordinate order, the first minimum on ties.
template <int M>
__device__ __forceinline__ int pq_nearest(const float* cb, const float* y) {
  double yd[M];
#pragma unroll
  for (int i = 0; i < M; ++i) yd[i] = (double)y[i];
  double best = DBL_MAX;
  int bz = 0;
  for (int c = 0; c < kCodebook; ++c) {
    double dist = 0.0;
#pragma unroll
    for (int i = 0; i < M; ++i) {
      const double df = yd[i] - (double)cb[c * M + i];
      dist = fma(df, df, dist);
    }
    if (dist < best) {
      best = dist;
      bz = c;
    }
  }
  return bz;
}

template <int D, int M>
__global__ void __launch_bounds__(256) pq_encode_kernel(StridedRows map,
                                                        const float* __restrict__ books,
                                                        double rot_scale) {
  constexpr int E = D / 32;
  constexpr int NSUB = D / M;
  __shared__ __align__(16) float cb[kCodebook * M];
  __shared__ __align__(16) float ys[kPqRows][D];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int h = blockIdx.y;
  const float* C = books + (size_t)h * kCodebook * M;
  for (int f = tid; f < kCodebook * M; f += 256) cb[f] = C[f];
  const int64_t j = (int64_t)blockIdx.x * kPqRows + warp;
  const bool ok = map.valid(j, h);
  if (ok) {
    double v[E];
    load_row_f64<E>(map.src(), map.dtype(), map.x_off(j, h), lane, v);
    map.apply_smooth<E>(v, h, lane);
    if (map.do_rotate()) {
      fwht_warp_f64<D>(v, lane);
#pragma unroll
      for (int q = 0; q < E; ++q) v[q] *= rot_scale;
    }
#pragma unroll
    for (int q = 0; q < E; ++q) ys[warp][q * 32 + lane] = (float)v[q];   // element q*32 + lane
  }
  __syncthreads();   // codebook and rows staged
  if (!ok) return;
  const int64_t bb = j / map.n_tok, t = j - bb * map.n_tok;
  uint8_t* out = map.codes + bb * map.c_sb + t * map.c_st + (int64_t)h * map.c_sh;
  for (int s = lane; s < NSUB; s += 32) out[s] = (uint8_t)pq_nearest<M>(cb, &ys[warp][s * M]);
}

template <int D>
static int launch_pq_d(const StridedRows& m, int64_t n_head, int M, const float* books,
                       cudaStream_t st) {
  const dim3 grid((unsigned)((m.n_rows + kPqRows - 1) / kPqRows), (unsigned)n_head);
  const double rot = 1.0 / std::sqrt((double)D);
  switch (M) {
    case 2: pq_encode_kernel<D, 2><<<grid, 256, 0, st>>>(m, books, rot); break;
    case 4: pq_encode_kernel<D, 4><<<grid, 256, 0, st>>>(m, books, rot); break;
    case 8: pq_encode_kernel<D, 8><<<grid, 256, 0, st>>>(m, books, rot); break;
    default: pq_encode_kernel<D, 16><<<grid, 256, 0, st>>>(m, books, rot); break;
  }
  ZKV_CHECK_LAUNCH();
  return ZKV_OK;
}

template <int D, int M>
__global__ void __launch_bounds__(256) pq_append_kernel(zkv_pq_append_params p, double rot) {
  constexpr int E = D / 32;
  constexpr int NSUB = D / M;
  __shared__ __align__(16) float cb[kCodebook * M];
  __shared__ __align__(16) float ys[kPqRows][D];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int kind = blockIdx.z;   // 0 = keys, 1 = values
  const int h = blockIdx.y;
  const float* C = (kind ? p.v_codebook : p.k_codebook) + (size_t)h * kCodebook * M;
  for (int f = tid; f < kCodebook * M; f += 256) cb[f] = C[f];
  const int64_t j = (int64_t)blockIdx.x * kPqRows + warp;
  __half* win = reinterpret_cast<__half*>(kind ? p.win_v : p.win_k);
  int64_t slot = -1, pos = -1;   // window slot written; code position (an eviction)
  if (j < p.B) {
    const int64_t wl = p.win_len[j], hd = p.win_head[j], c = p.comp_len[j];
    const bool report = lane == 0 && kind == 0 && h == 0;   // one report per sequence
    if (wl >= 0 && wl < p.Wcap) {
      slot = wl;
    } else if (wl == p.Wcap) {
      if (c >= 0 && c < p.Tcap && hd >= 0 && hd < p.Wcap) {
        slot = hd;
        pos = c;
      } else if (report) {
        set_error(p.error_flag, ZKV_DEVERR_COMP_LEN);
      }
    } else if (report) {
      set_error(p.error_flag, ZKV_DEVERR_WIN_LEN);
    }
  }
  __half* row = slot >= 0 ? win + ((j * p.Hkv + h) * p.Wcap + slot) * D : nullptr;
  if (pos >= 0) {   // the evicted row: smoothed (keys), rotated in float64, rounded once
    double v[E];
    load_row_f64<E>(row, ZKV_DTYPE_F16, 0, lane, v);
    if (kind == 0 && p.k_smooth) {
      const float* l = p.k_smooth + (int64_t)h * D;
#pragma unroll
      for (int q = 0; q < E; ++q) v[q] *= 1.0 / (double)l[q * 32 + lane];
    }
    fwht_warp_f64<D>(v, lane);
#pragma unroll
    for (int q = 0; q < E; ++q) ys[warp][q * 32 + lane] = (float)(v[q] * rot);
  }
  __syncthreads();   // codebook staged; every evicted row read before the window is written
  if (pos >= 0) {
    uint8_t* out = (kind ? p.v_codes : p.k_codes) + ((j * p.Hkv + h) * p.Tcap + pos) * NSUB;
    for (int s = lane; s < NSUB; s += 32) out[s] = (uint8_t)pq_nearest<M>(cb, &ys[warp][s * M]);
  }
  if (slot >= 0) {
    const __half* src =
        reinterpret_cast<const __half*>(kind ? p.new_v : p.new_k) + (j * p.Hkv + h) * D;
    for (int e = lane; e < D; e += 32) row[e] = src[e];
  }
}

__global__ void pq_append_lengths_kernel(int B, int64_t Tcap, int64_t Wcap, int32_t* win_len,
                                         int32_t* win_head, int32_t* comp_len) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b < B) advance_lengths(b, Tcap, Wcap, win_len, win_head, comp_len);
}

template <int D>
static int launch_pq_append_d(const zkv_pq_append_params& p, cudaStream_t st) {
  const dim3 grid((unsigned)((p.B + kPqRows - 1) / kPqRows), (unsigned)p.Hkv, 2);
  const double rot = 1.0 / std::sqrt((double)D);
  switch (p.m) {
    case 2: pq_append_kernel<D, 2><<<grid, 256, 0, st>>>(p, rot); break;
    case 4: pq_append_kernel<D, 4><<<grid, 256, 0, st>>>(p, rot); break;
    case 8: pq_append_kernel<D, 8><<<grid, 256, 0, st>>>(p, rot); break;
    default: pq_append_kernel<D, 16><<<grid, 256, 0, st>>>(p, rot); break;
  }
  ZKV_CHECK_LAUNCH();
  return ZKV_OK;
}

}  // namespace zkv

using namespace zkv;

extern "C" int zkv_pq_append(const zkv_pq_append_params* p, void* stream) {
  if (!p) return ZKV_ERR_INVALID_ARG;
  if (p->B < 0 || p->Hkv < 1 || p->Tcap < 0 || p->Wcap < 1) return ZKV_ERR_INVALID_ARG;
  if (!supported_d(p->d)) return ZKV_ERR_UNSUPPORTED;
  if (p->m != 2 && p->m != 4 && p->m != 8 && p->m != 16) return ZKV_ERR_UNSUPPORTED;
  if (p->B == 0) return ZKV_OK;
  if (!p->new_k || !p->new_v || !p->win_k || !p->win_v || !p->win_len || !p->win_head ||
      !p->comp_len || !p->k_codes || !p->v_codes || !p->k_codebook || !p->v_codebook)
    return ZKV_ERR_INVALID_ARG;
  if (p->Hkv > 65535 || (p->B + kPqRows - 1) / kPqRows > 0x7fffffffLL) return ZKV_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int rc;
  switch (p->d) {
    case 64: rc = launch_pq_append_d<64>(*p, st); break;
    case 128: rc = launch_pq_append_d<128>(*p, st); break;
    default: rc = launch_pq_append_d<256>(*p, st); break;
  }
  if (rc != ZKV_OK) return rc;
  pq_append_lengths_kernel<<<(p->B + 127) / 128, 128, 0, st>>>(p->B, p->Tcap, p->Wcap, p->win_len,
                                                               p->win_head, p->comp_len);
  ZKV_CHECK_LAUNCH();
  return ZKV_OK;
}

extern "C" int zkv_pq_encode(const zkv_pq_encode_params* p, void* stream) {
  if (!p) return ZKV_ERR_INVALID_ARG;
  if (p->n_batch < 0 || p->n_tok < 0 || p->n_head < 0) return ZKV_ERR_INVALID_ARG;
  if (p->x_dtype != ZKV_DTYPE_F16 && p->x_dtype != ZKV_DTYPE_F32) return ZKV_ERR_INVALID_ARG;
  if (!supported_d(p->d)) return ZKV_ERR_UNSUPPORTED;
  if (p->m != 2 && p->m != 4 && p->m != 8 && p->m != 16) return ZKV_ERR_UNSUPPORTED;
  const int64_t n_rows = p->n_batch * p->n_tok;
  if (n_rows == 0 || p->n_head == 0) return ZKV_OK;
  if (!p->x || !p->codebook || !p->codes) return ZKV_ERR_INVALID_ARG;
  if (p->n_head > 65535 || (n_rows + kPqRows - 1) / kPqRows > 0x7fffffffLL) return ZKV_ERR_INVALID_ARG;
  const int64_t esz = p->x_dtype == ZKV_DTYPE_F16 ? 2 : 4;
  if (((uintptr_t)p->x & 15) || ((p->x_sb * esz) & 15) || ((p->x_st * esz) & 15) ||
      ((p->x_sh * esz) & 15))
    return ZKV_ERR_INVALID_ARG;
  StridedRows m{};
  m.n_tok = p->n_tok;
  m.n_rows = n_rows;
  m.x = p->x;
  m.x_dtype = p->x_dtype;
  m.rotate = p->rotate ? 1 : 0;
  m.x_sb = p->x_sb;
  m.x_st = p->x_st;
  m.x_sh = p->x_sh;
  m.codes = p->codes;
  m.c_sb = p->c_sb;
  m.c_st = p->c_st;
  m.c_sh = p->c_sh;
  m.norms = nullptr;
  m.smooth = p->smooth;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  switch (p->d) {
    case 64: return launch_pq_d<64>(m, p->n_head, p->m, p->codebook, st);
    case 128: return launch_pq_d<128>(m, p->n_head, p->m, p->codebook, st);
    default: return launch_pq_d<256>(m, p->n_head, p->m, p->codebook, st);
  }
}
