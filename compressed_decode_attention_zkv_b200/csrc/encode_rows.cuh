// Row-group RVQ encoder shared by zkv_rvq_encode (small batches) and zkv_rvq_append.
// The decision rule and its rounding-error bound are described in encode.cu.
#pragma once

#include <cfloat>

#include "zkv_internal.cuh"

namespace zkv {

// ------------------------------------------------------------------------------------------
// Row addressing: generic strided (b, t, h) rows of zkv_rvq_encode.
// ------------------------------------------------------------------------------------------
struct StridedRows {
  int64_t n_tok, n_rows;  // n_rows = n_batch * n_tok rows per head
  const void* x;
  int x_dtype, rotate;
  int64_t x_sb, x_st, x_sh;
  uint8_t* codes;
  int64_t c_sb, c_st, c_sh;
  float* norms;
  int64_t n_sb, n_st, n_sh;
  const float* smooth;    // [n_head][d] key smoothing factors or null

  __device__ bool valid(int64_t j, int) const { return j < n_rows; }
  // x / lambda per channel (before the rotation): float64 times the float64 reciprocal
  template <int E>
  __device__ void apply_smooth(double (&v)[E], int h, int lane) const {
    if (!smooth) return;
    const float* l = smooth + (int64_t)h * (E * 32);
#pragma unroll
    for (int q = 0; q < E; ++q) v[q] *= 1.0 / (double)l[q * 32 + lane];
  }
  __device__ const void* src() const { return x; }
  __device__ int dtype() const { return x_dtype; }
  __device__ bool do_rotate() const { return rotate != 0; }
  __device__ int64_t x_off(int64_t j, int h) const {
    const int64_t b = j / n_tok, t = j - b * n_tok;
    return b * x_sb + t * x_st + (int64_t)h * x_sh;
  }
  __device__ void store(int64_t j, int h, int S, const uint8_t* code, const float* nrm) const {
    const int64_t b = j / n_tok, t = j - b * n_tok;
    uint8_t* c = codes + b * c_sb + t * c_st + (int64_t)h * c_sh;
    for (int s = 0; s < S; ++s) c[s] = code[s];
    if (norms) {
      float* n = norms + b * n_sb + t * n_st + (int64_t)h * n_sh;
      for (int s = 0; s < S; ++s) n[s] = nrm[s];
    }
  }
};

__device__ __forceinline__ double candidate_margin(double rnorm, float cn_max, int D) {
  const double u = 1.0 / 16777216.0;
  const double g = (double)D * u / (1.0 - (double)D * u);
  const double a = rnorm * (1.0 + 1e-12);
  const double b = sqrt((double)cn_max) * (1.0 + g) + 1e-30;
  // 2E for the window, and 25 % slack on top.
  return 2.5 * (g + 2.0 * u) * (a + b) * (a + b);
}

// ------------------------------------------------------------------------------------------
// Row-group encoder: R rows of one head per CTA, thread c owns codeword c (256 threads).
// Used for small batches (window evictions, short prefills): few rows, latency matters more
// than codebook reuse.  Each stage's codebook is staged through shared memory in slices of
// KC dims with cp.async (all requests in flight at once).  Slice layout: codeword c's 16-byte
// piece q is stored at position q ^ (c & 7), so the 8 lanes of a 128-bit read phase (8
// consecutive codewords, same q) hit 8 distinct bank groups; the row operands are broadcasts.
// ------------------------------------------------------------------------------------------
template <int D, int R>
struct RowsSmem {
  float r[R][D];
  double rn[R];
  float red_min[8][R];
  float red_cmax[8];
  int cand_count;
  int zsel[R];
  uint16_t cand[R * kCodebook];
  double cand_d[R * kCodebook];
  uint8_t code[R][kMaxStages];
  float nrm[R][kMaxStages];
};

template <int D>
struct RowsSlice {
  static constexpr int KC = D < 128 ? D : 128;   // dims per staged slice
};

template <int D, int R>
constexpr size_t rows_smem_bytes() {
  return ((sizeof(RowsSmem<D, R>) + 15) / 16) * 16 +
         (size_t)kCodebook * RowsSlice<D>::KC * sizeof(float);
}

template <int D, int R, class Map>
__device__ __forceinline__ void encode_rows_body(const Map& map, const float* __restrict__ books,
                                                 int S, double rot_scale, int64_t row0, int h,
                                                 RowsSmem<D, R>& sm, float* cb) {
  constexpr int E = D / 32;
  constexpr int KC = RowsSlice<D>::KC;
  constexpr int NQ = KC / 4;           // 16-byte pieces per codeword slice
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  if (warp < R) {
    const int64_t j = row0 + warp;
    double ss = 0.0;
    if (map.valid(j, h)) {
      double v[E];
      load_row_f64<E>(map.src(), map.dtype(), map.x_off(j, h), lane, v);
      map.apply_smooth<E>(v, h, lane);
      if (map.do_rotate()) {
        fwht_warp_f64<D>(v, lane);
#pragma unroll
        for (int q = 0; q < E; ++q) v[q] *= rot_scale;
      }
#pragma unroll
      for (int q = 0; q < E; ++q) {
        const float y = (float)v[q];
        sm.r[warp][q * 32 + lane] = y;
        ss += (double)y * (double)y;
      }
    } else {
#pragma unroll
      for (int q = 0; q < E; ++q) sm.r[warp][q * 32 + lane] = 0.f;
    }
    ss = warp_sum_f64(ss);
    if (lane == 0) sm.rn[warp] = sqrt(ss);
  }

  const float* CB = books + (size_t)h * S * kCodebook * D;
  for (int s = 0; s < S; ++s) {
    const float* C = CB + (size_t)s * kCodebook * D;
    float acc[R];
#pragma unroll
    for (int r = 0; r < R; ++r) acc[r] = 0.f;
    float cn = 0.f;
    for (int k0 = 0; k0 < D; k0 += KC) {
      __syncthreads();   // previous slice (and the rows) are ready / consumed
      for (int f = tid; f < kCodebook * NQ; f += 256) {
        const int c = f / NQ, q = f % NQ;
        cp_async16(cb + c * KC + 4 * (q ^ (c & 7)), C + (size_t)c * D + k0 + 4 * q);
      }
      cp_async_wait_all();
      __syncthreads();
      const float* row = cb + tid * KC;
      const int sw = tid & 7;
#pragma unroll 4
      for (int q = 0; q < NQ; ++q) {
        const float4 c4 = *reinterpret_cast<const float4*>(row + 4 * (q ^ sw));
        cn = fmaf(c4.x, c4.x, cn);
        cn = fmaf(c4.y, c4.y, cn);
        cn = fmaf(c4.z, c4.z, cn);
        cn = fmaf(c4.w, c4.w, cn);
#pragma unroll
        for (int r = 0; r < R; ++r) {
          const float4 x4 = *reinterpret_cast<const float4*>(&sm.r[r][k0 + 4 * q]);
          acc[r] = fmaf(x4.x, c4.x, acc[r]);
          acc[r] = fmaf(x4.y, c4.y, acc[r]);
          acc[r] = fmaf(x4.z, c4.z, acc[r]);
          acc[r] = fmaf(x4.w, c4.w, acc[r]);
        }
      }
    }
    float dist[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      dist[r] = cn - 2.f * acc[r];
      const float m = warp_min_f32(dist[r]);
      if (lane == 0) sm.red_min[warp][r] = m;
    }
    {
      const float m = warp_max_f32(cn);
      if (lane == 0) sm.red_cmax[warp] = m;
    }
    if (tid == 0) sm.cand_count = 0;
    __syncthreads();

    float cn_max = sm.red_cmax[0];
#pragma unroll
    for (int w = 1; w < 8; ++w) cn_max = fmaxf(cn_max, sm.red_cmax[w]);
#pragma unroll
    for (int r = 0; r < R; ++r) {
      float dmin = sm.red_min[0][r];
#pragma unroll
      for (int w = 1; w < 8; ++w) dmin = fminf(dmin, sm.red_min[w][r]);
      const double thr = (double)dmin + candidate_margin(sm.rn[r], cn_max, D);
      if ((double)dist[r] <= thr) {
        const int k = atomicAdd(&sm.cand_count, 1);
        sm.cand[k] = (uint16_t)((r << 8) | tid);
      }
    }
    __syncthreads();

    // Exact float64 distance of each candidate, one warp per candidate.
    const int nc = sm.cand_count;
    for (int k = warp; k < nc; k += 8) {
      const int r = sm.cand[k] >> 8, c = sm.cand[k] & 255;
      const float* cw = C + (size_t)c * D;
      double a = 0.0;
#pragma unroll
      for (int q = 0; q < E; ++q) {
        const int i = q * 32 + lane;
        // the staged slice holds the whole codeword when KC == D (swizzled 16-byte pieces)
        const float cv = KC == D ? cb[c * KC + 4 * ((i >> 2) ^ (c & 7)) + (i & 3)] : __ldg(cw + i);
        const double df = (double)sm.r[r][i] - (double)cv;
        a = fma(df, df, a);
      }
      a = warp_sum_f64(a);
      if (lane == 0) sm.cand_d[k] = a;
    }
    __syncthreads();
    if (tid < R) {
      double best = DBL_MAX;
      int bc = kCodebook;
      for (int k = 0; k < nc; ++k) {
        if ((sm.cand[k] >> 8) != tid) continue;
        const int c = sm.cand[k] & 255;
        const double dd = sm.cand_d[k];
        if (dd < best || (dd == best && c < bc)) {
          best = dd;
          bc = c;
        }
      }
      // Non-finite rows match no candidate; never index past the stage's codebook.
      sm.zsel[tid] = bc < kCodebook ? bc : 0;
    }
    __syncthreads();

    if (warp < R) {
      const int z = sm.zsel[warp];
      const float* cw = C + (size_t)z * D;
      double ss = 0.0;
#pragma unroll
      for (int q = 0; q < E; ++q) {
        const int i = q * 32 + lane;
        const float nr = sm.r[warp][i] - __ldg(cw + i);
        sm.r[warp][i] = nr;
        ss += (double)nr * (double)nr;
      }
      ss = warp_sum_f64(ss);
      if (lane == 0) {
        const double nn = sqrt(ss);
        sm.rn[warp] = nn;
        sm.code[warp][s] = (uint8_t)z;
        sm.nrm[warp][s] = (float)nn;
      }
    }
    // the next stage's first __syncthreads orders these writes before their use
  }
  __syncthreads();
}

}  // namespace zkv
