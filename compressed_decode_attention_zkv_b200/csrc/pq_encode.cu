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
#include "encode_rows.cuh"

namespace zkv {

constexpr int kPqRows = 8;   // rows (warps) per block

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
  for (int s = lane; s < NSUB; s += 32) {
    double y[M];
#pragma unroll
    for (int i = 0; i < M; ++i) y[i] = (double)ys[warp][s * M + i];
    double best = DBL_MAX;
    int bz = 0;
    for (int c = 0; c < kCodebook; ++c) {
      double dist = 0.0;
#pragma unroll
      for (int i = 0; i < M; ++i) {
        const double df = y[i] - (double)cb[c * M + i];
        dist = fma(df, df, dist);
      }
      if (dist < best) {   // strict: the first minimum wins ties
        best = dist;
        bz = c;
      }
    }
    out[s] = (uint8_t)bz;
  }
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

}  // namespace zkv

using namespace zkv;

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
