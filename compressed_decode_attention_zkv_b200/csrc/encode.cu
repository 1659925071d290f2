// RVQ encode and reconstruction kernels (sm_100a, CUDA cores).
//
// Passage: VQKV (gist.science summary of arXiv 2603.16435), section 2.1 "Residual Simple Vector
// Quantization", "Process": at every stage the nearest codeword of that stage's codebook is
// chosen, subtracted, and the residual is passed to the next stage; "Reconstruction": the sum
// of the chosen codewords.  Rotation first: zerokv-neo "Architecture" (FWHT).
//
// Decision rule implemented here: the stage choice is the argmin of ||r - c||^2 evaluated in
// float64, ties to the lowest index.  The distance of every codeword is first computed in
// float32 in dot-product form, D~_c = ||c||^2 - 2 r.c (sequential FMA accumulation).  A
// rounding-error bound E (below) brackets the exact value, so every codeword within 2E of the
// smallest D~ is a candidate and the true argmin is always among them.  Candidates are then
// re-scored exactly in float64, which makes the choice independent of float32 rounding.
//
// Bound: with u = 2^-24 and g = D u / (1 - D u), sequential float32 FMA accumulation gives
// |fl(r.c) - r.c| <= g ||r|| ||c|| and |fl(||c||^2) - ||c||^2| <= g ||c||^2; the final
// subtraction adds at most u (||c||^2 + 2 ||r|| ||c||)(1 + g).  Altogether
// |D~_c - (||r - c||^2 - ||r||^2)| <= (g + 2u)(||r|| + ||c||)^2 =: E_c <= E(max_c ||c||).
#include "encode_rows.cuh"

#include <cfloat>

namespace zkv {

template <int D, int R>
__global__ void __launch_bounds__(256) encode_rows_kernel(StridedRows map,
                                                          const float* __restrict__ books, int S,
                                                          double rot_scale) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  RowsSmem<D, R>& sm = *reinterpret_cast<RowsSmem<D, R>*>(smem_raw);
  float* cb = reinterpret_cast<float*>(smem_raw + ((sizeof(RowsSmem<D, R>) + 15) / 16) * 16);
  const int h = blockIdx.y;
  const int64_t row0 = (int64_t)blockIdx.x * R;
  encode_rows_body<D, R>(map, books, S, rot_scale, row0, h, sm, cb);
  if (threadIdx.x < R) {
    const int64_t j = row0 + threadIdx.x;
    if (map.valid(j, h)) map.store(j, h, S, sm.code[threadIdx.x], sm.nrm[threadIdx.x]);
  }
}

// ------------------------------------------------------------------------------------------
// Tiled encoder for bulk (prefill) batches: 64 rows of one head per CTA, each stage a
// [64 x D] x [D x 256] float32 product on CUDA cores (8x8 register tiles), codebook staged
// through shared memory in 32-wide slices.
// ------------------------------------------------------------------------------------------
constexpr int kTM = 64;
constexpr int kTPad = kTM + 4;
constexpr int kKC = 32;

template <int D>
struct TileSmem {
  float rT[D][kTPad];         // residual tile, k-major
  float cb[kCodebook][kKC + 1];
  float cn[kCodebook];
  double rn[kTM];
  double part[4][kTM];
  float red[8];
  int zsel[kTM];
  uint8_t code[kTM][kMaxStages];
  float nrm[kTM][kMaxStages];
};

template <int D>
__global__ void __launch_bounds__(256, 2) encode_tile_kernel(StridedRows map,
                                                             const float* __restrict__ books,
                                                             int S, double rot_scale) {
  constexpr int E = D / 32;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  TileSmem<D>& sm = *reinterpret_cast<TileSmem<D>*>(smem_raw);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int h = blockIdx.y;
  const int64_t row0 = (int64_t)blockIdx.x * kTM;

  // Load and rotate 8 rows per warp.
  for (int i = 0; i < 8; ++i) {
    const int row = warp * 8 + i;
    const int64_t j = row0 + row;
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
        sm.rT[q * 32 + lane][row] = y;
        ss += (double)y * (double)y;
      }
    } else {
#pragma unroll
      for (int q = 0; q < E; ++q) sm.rT[q * 32 + lane][row] = 0.f;
    }
    ss = warp_sum_f64(ss);
    if (lane == 0) sm.rn[row] = sqrt(ss);
  }

  const float* CB = books + (size_t)h * S * kCodebook * D;
  for (int s = 0; s < S; ++s) {
    const float* C = CB + (size_t)s * kCodebook * D;
    float acc[8][8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;
    float cnp = 0.f;

    for (int kc = 0; kc < D; kc += kKC) {
      __syncthreads();
      // codebook slice C[c][kc .. kc+31] -> cb[c][0..31]; 8 float4 per thread
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const int f = q * 256 + tid;           // float4 index within the slice
        const int c = f >> 3, kk = (f & 7) * 4;
        const float4 v = __ldg(reinterpret_cast<const float4*>(C + (size_t)c * D + kc + kk));
        sm.cb[c][kk + 0] = v.x;
        sm.cb[c][kk + 1] = v.y;
        sm.cb[c][kk + 2] = v.z;
        sm.cb[c][kk + 3] = v.w;
      }
      __syncthreads();
#pragma unroll 8
      for (int kk = 0; kk < kKC; ++kk) {
        const float b0 = sm.cb[tid][kk];
        cnp = fmaf(b0, b0, cnp);
        const float4 a0 = *reinterpret_cast<const float4*>(&sm.rT[kc + kk][warp * 8]);
        const float4 a1 = *reinterpret_cast<const float4*>(&sm.rT[kc + kk][warp * 8 + 4]);
        const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
        float b[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) b[j] = sm.cb[lane + 32 * j][kk];
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
          for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
      }
    }
    sm.cn[tid] = cnp;
    {
      const float m = warp_max_f32(cnp);
      if (lane == 0) sm.red[warp] = m;
    }
    __syncthreads();
    float cn_max = sm.red[0];
#pragma unroll
    for (int w = 1; w < 8; ++w) cn_max = fmaxf(cn_max, sm.red[w]);
    float cnj[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) cnj[j] = sm.cn[lane + 32 * j];

    for (int i = 0; i < 8; ++i) {
      const int row = warp * 8 + i;
      float dist[8];
      float lmin = FLT_MAX;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        dist[j] = cnj[j] - 2.f * acc[i][j];
        lmin = fminf(lmin, dist[j]);
      }
      const float wmin = warp_min_f32(lmin);
      const double thr = (double)wmin + candidate_margin(sm.rn[row], cn_max, D);
      unsigned mask = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) mask |= ((double)dist[j] <= thr ? 1u : 0u) << j;
      const int cnt = __reduce_add_sync(0xffffffffu, __popc(mask));
      int z;
      if (cnt == 1) {
        const unsigned who = __ballot_sync(0xffffffffu, mask != 0);
        const int src = __ffs(who) - 1;
        const int jj = __ffs(__shfl_sync(0xffffffffu, (int)mask, src)) - 1;
        z = src + 32 * jj;
      } else {
        // Exact float64 re-score of every candidate, warp-cooperative, lowest index on ties.
        double best = DBL_MAX;
        int bz = kCodebook;
        unsigned m = mask;
        while (true) {
          const unsigned who = __ballot_sync(0xffffffffu, m != 0);
          if (!who) break;
          const int src = __ffs(who) - 1;
          const int jj = __ffs(__shfl_sync(0xffffffffu, (int)m, src)) - 1;
          if (lane == src) m &= ~(1u << jj);
          const int c = src + 32 * jj;
          const float* cw = C + (size_t)c * D;
          double a = 0.0;
#pragma unroll
          for (int q = 0; q < E; ++q) {
            const int k = q * 32 + lane;
            const double df = (double)sm.rT[k][row] - (double)__ldg(cw + k);
            a = fma(df, df, a);
          }
          a = warp_sum_f64(a);
          if (a < best || (a == best && c < bz)) {
            best = a;
            bz = c;
          }
        }
        z = bz < kCodebook ? bz : 0;   // non-finite rows match no candidate
      }
      if (lane == 0) sm.zsel[row] = z;
    }
    __syncthreads();

    // Residual update r <- r - C[z] (float32) and its norm (float64).
    {
      const int row = tid & (kTM - 1), kg = tid >> 6;
      constexpr int KQ = D / 4;
      const int z = sm.zsel[row];
      const float* cw = C + (size_t)z * D + kg * KQ;
      double ss = 0.0;
#pragma unroll 4
      for (int q = 0; q < KQ; q += 4) {
        const float4 c4 = __ldg(reinterpret_cast<const float4*>(cw + q));
        const int k = kg * KQ + q;
        float v0 = sm.rT[k + 0][row] - c4.x;
        float v1 = sm.rT[k + 1][row] - c4.y;
        float v2 = sm.rT[k + 2][row] - c4.z;
        float v3 = sm.rT[k + 3][row] - c4.w;
        sm.rT[k + 0][row] = v0;
        sm.rT[k + 1][row] = v1;
        sm.rT[k + 2][row] = v2;
        sm.rT[k + 3][row] = v3;
        ss += (double)v0 * v0 + (double)v1 * v1 + (double)v2 * v2 + (double)v3 * v3;
      }
      sm.part[kg][row] = ss;
    }
    __syncthreads();
    if (tid < kTM) {
      const double nn = sqrt(sm.part[0][tid] + sm.part[1][tid] + sm.part[2][tid] + sm.part[3][tid]);
      sm.rn[tid] = nn;
      sm.code[tid][s] = (uint8_t)sm.zsel[tid];
      sm.nrm[tid][s] = (float)nn;
    }
    // the next stage's first __syncthreads orders these writes before their use
  }
  __syncthreads();
  if (tid < kTM) {
    const int64_t j = row0 + tid;
    if (map.valid(j, h)) map.store(j, h, S, sm.code[tid], sm.nrm[tid]);
  }
}

// ------------------------------------------------------------------------------------------
// Reconstruction: x_hat = sum_s C[h][s][z_s] (float32, s ascending), optionally rotated back.
// One warp per row.
// ------------------------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) reconstruct_kernel(zkv_reconstruct_params p,
                                                          double rot_scale) {
  constexpr int E = D / 32;
  const int lane = threadIdx.x & 31;
  const int64_t n_rows = p.n_batch * p.n_tok;
  const int64_t j = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int h = blockIdx.y;
  if (j >= n_rows) return;
  const int64_t b = j / p.n_tok, t = j - b * p.n_tok;
  const uint8_t* code = p.codes + b * p.c_sb + t * p.c_st + (int64_t)h * p.c_sh;
  float x[E];
#pragma unroll
  for (int q = 0; q < E; ++q) x[q] = 0.f;
  const float* CB = p.codebooks + (size_t)h * p.S * kCodebook * D;
  for (int s = 0; s < p.S; ++s) {
    const float* cw = CB + ((size_t)s * kCodebook + code[s]) * D;
#pragma unroll
    for (int q = 0; q < E; ++q) x[q] += __ldg(cw + q * 32 + lane);
  }
  float* o = p.out + b * p.o_sb + t * p.o_st + (int64_t)h * p.o_sh;
  if (p.unrotate) {
    double v[E];
#pragma unroll
    for (int q = 0; q < E; ++q) v[q] = (double)x[q];
    fwht_warp_f64<D>(v, lane);
#pragma unroll
    for (int q = 0; q < E; ++q) o[q * 32 + lane] = (float)(v[q] * rot_scale);
  } else {
#pragma unroll
    for (int q = 0; q < E; ++q) o[q * 32 + lane] = x[q];
  }
}

// ------------------------------------------------------------------------------------------
// Launchers
// ------------------------------------------------------------------------------------------
int launch_encode_tc(const StridedRows& map, int64_t n_head, int d, int S, const float* books,
                     int* err, cudaStream_t st);   // encode_tc.cu

int launch_encode(const StridedRows& map, int64_t n_head, int d, int S, const float* books,
                  int* err, cudaStream_t st) {
  const double rot = 1.0 / std::sqrt((double)d);
  const int64_t n_rows = map.n_rows;
  if (n_rows * n_head > 4096 && (d == 64 || d == 128)) return launch_encode_tc(map, n_head, d, S, books, err, st);
  if (n_rows * n_head <= 4096) {
    constexpr int R = 8;
    const dim3 grid((unsigned)((n_rows + R - 1) / R), (unsigned)n_head);
    const bool ok = ensure_smem_limit(encode_rows_kernel<64, R>, rows_smem_bytes<64, R>()) == cudaSuccess &&
                    ensure_smem_limit(encode_rows_kernel<128, R>, rows_smem_bytes<128, R>()) == cudaSuccess &&
                    ensure_smem_limit(encode_rows_kernel<256, R>, rows_smem_bytes<256, R>()) == cudaSuccess;
    if (!ok) return ZKV_ERR_CUDA;
    switch (d) {
      case 64: encode_rows_kernel<64, R><<<grid, 256, rows_smem_bytes<64, R>(), st>>>(map, books, S, rot); break;
      case 128: encode_rows_kernel<128, R><<<grid, 256, rows_smem_bytes<128, R>(), st>>>(map, books, S, rot); break;
      case 256: encode_rows_kernel<256, R><<<grid, 256, rows_smem_bytes<256, R>(), st>>>(map, books, S, rot); break;
    }
  } else {
    const bool ok = ensure_smem_limit(encode_tile_kernel<64>, sizeof(TileSmem<64>)) == cudaSuccess &&
                    ensure_smem_limit(encode_tile_kernel<128>, sizeof(TileSmem<128>)) == cudaSuccess &&
                    ensure_smem_limit(encode_tile_kernel<256>, sizeof(TileSmem<256>)) == cudaSuccess;
    if (!ok) return ZKV_ERR_CUDA;
    const dim3 grid((unsigned)((n_rows + kTM - 1) / kTM), (unsigned)n_head);
    switch (d) {
      case 64: encode_tile_kernel<64><<<grid, 256, sizeof(TileSmem<64>), st>>>(map, books, S, rot); break;
      case 128: encode_tile_kernel<128><<<grid, 256, sizeof(TileSmem<128>), st>>>(map, books, S, rot); break;
      case 256: encode_tile_kernel<256><<<grid, 256, sizeof(TileSmem<256>), st>>>(map, books, S, rot); break;
    }
  }
  ZKV_CHECK_LAUNCH();
  return ZKV_OK;
}

}  // namespace zkv

using namespace zkv;

extern "C" int zkv_rvq_encode(const zkv_encode_params* p, void* stream) {
  if (!p) return ZKV_ERR_INVALID_ARG;
  if (p->n_batch < 0 || p->n_tok < 0 || p->n_head < 0) return ZKV_ERR_INVALID_ARG;
  if (p->x_dtype != ZKV_DTYPE_F16 && p->x_dtype != ZKV_DTYPE_F32) return ZKV_ERR_INVALID_ARG;
  if (!supported_d(p->d)) return ZKV_ERR_UNSUPPORTED;
  if (p->S < 1 || p->S > kMaxStages) return ZKV_ERR_UNSUPPORTED;
  const int64_t n_rows = p->n_batch * p->n_tok;
  if (n_rows == 0 || p->n_head == 0) return ZKV_OK;
  if (!p->x || !p->codebooks || !p->codes) return ZKV_ERR_INVALID_ARG;
  if (p->n_head > 65535 || (n_rows + 7) / 8 > 0x7fffffffLL) return ZKV_ERR_INVALID_ARG;
  const int64_t esz = p->x_dtype == ZKV_DTYPE_F16 ? 2 : 4;
  if (((uintptr_t)p->x & 15) || ((uintptr_t)p->codebooks & 15)) return ZKV_ERR_INVALID_ARG;
  if (((p->x_sb * esz) & 15) || ((p->x_st * esz) & 15) || ((p->x_sh * esz) & 15))
    return ZKV_ERR_INVALID_ARG;
  StridedRows m;
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
  m.norms = p->norms;
  m.n_sb = p->n_sb;
  m.n_st = p->n_st;
  m.n_sh = p->n_sh;
  m.smooth = p->smooth;
  return launch_encode(m, p->n_head, p->d, p->S, p->codebooks, p->error_flag,
                       reinterpret_cast<cudaStream_t>(stream));
}

extern "C" int zkv_rvq_reconstruct(const zkv_reconstruct_params* p, void* stream) {
  if (!p) return ZKV_ERR_INVALID_ARG;
  if (p->n_batch < 0 || p->n_tok < 0 || p->n_head < 0) return ZKV_ERR_INVALID_ARG;
  if (!supported_d(p->d)) return ZKV_ERR_UNSUPPORTED;
  if (p->S < 1 || p->S > kMaxStages) return ZKV_ERR_UNSUPPORTED;
  const int64_t n_rows = p->n_batch * p->n_tok;
  if (n_rows == 0 || p->n_head == 0) return ZKV_OK;
  if (!p->codes || !p->codebooks || !p->out) return ZKV_ERR_INVALID_ARG;
  if (p->n_head > 65535 || (n_rows + 7) / 8 > 0x7fffffffLL) return ZKV_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const dim3 grid((unsigned)((n_rows + 7) / 8), (unsigned)p->n_head);
  const double rot = 1.0 / std::sqrt((double)p->d);
  switch (p->d) {
    case 64: reconstruct_kernel<64><<<grid, 256, 0, st>>>(*p, rot); break;
    case 128: reconstruct_kernel<128><<<grid, 256, 0, st>>>(*p, rot); break;
    case 256: reconstruct_kernel<256><<<grid, 256, 0, st>>>(*p, rot); break;
  }
  ZKV_CHECK_LAUNCH();
  return ZKV_OK;
}
