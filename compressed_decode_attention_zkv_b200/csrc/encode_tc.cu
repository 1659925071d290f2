// Tensor-core RVQ encode for bulk batches (sm_100a, tcgen05).
//
// Passage: VQKV (gist.science summary of arXiv 2603.16435), section 2.1 "Residual Simple Vector
// Quantization", "Process": per stage the nearest codeword is chosen and subtracted.  The
// stage's distances are a dense product: for a tile of 128 residual rows and the 256 codewords,
// r.c for all pairs is a [128 x D] x [D x 256] matrix product.
//
// One CTA (512 threads) owns 128 rows of one head for all stages.  The residual tile stays in
// shared memory in the tensor cores' K-major, 128-byte-swizzled operand layout; per stage the
// codebook is copied into the same layout, one thread issues D/8 tcgen05.mma (kind::tf32,
// M = 128, N = 256, K = 8) into a 256-column TMEM accumulator and commits them to an mbarrier,
// and four warps per TMEM lane quarter read 64 columns each of their rows' dot products
// (row = TMEM lane).  The stage's codeword is decided exactly, by three filters that each keep
// the true argmin:
//   1. TF32 distances D1_c = ||c||^2 - 2 (r.c)_tf32.  The MMA uses the top 19 bits of every
//      float32 operand (relative error < 2^-10 per operand, so < 2^-9 + 2^-20 per product) and
//      accumulates in float32 (<= 2^-17 relative over K <= 128 terms): the dot product is off
//      by <= 1.01 * 2^-9 sum_i |r_i c_i| <= 1.01 * 2^-9 ||r|| ||c||.  With the float32 norm
//      (<= 2^-17 ||c||^2) and the final subtraction (<= 2^-24 (||c||^2 + 2 ||r|| ||c||)),
//      |D1_c - (||r-c||^2 - ||r||^2)| <= E1 := 1.02 * 2^-8 ||r|| ||c|| + 2^-16 ||c||^2.
//      Candidates: D1_c <= min D1 + 2 E1(max ||c||).
//   2. For those candidates, the float32 dot form with sequential FMA accumulation (the bound of
//      encode.cu): keep D2_c <= min D2 + 2 E2.
//   3. The survivors' distances ||r - c||^2 in float64, ties to the lowest index.
// The residual update r <- r - C[z] is float32 and the norm float64, as in the other encoders.
#include "encode_rows.cuh"

#include <cfloat>

namespace zkv {

constexpr int kTcM = 128;          // rows per CTA (TMEM lanes)
constexpr int kTcN = 256;          // codewords (TMEM columns)
constexpr int kTcList = 16;        // candidates kept per row after filter 1

template <int D>
struct TcSmem {
  static constexpr int P = D / 32;                    // 128-byte K panels
  float a[P][kTcM * 32];                              // residual tile, swizzled K-major panels
  float b[P][kTcN * 32];                              // codebook stage, swizzled K-major panels
  float cn[kTcN];                                     // ||c||^2 (float32)
  float cmax_w[16];
  double rn[kTcM];                                    // ||r|| (float64)
  double part[4][kTcM];                               // partial residual norms
  float gmin[4][kTcM];                                // per column group row minima (filters 1, 2)
  double gbest[4][kTcM];                              // per column group best float64 distance
  int gbz[4][kTcM];
  int ncand[kTcM];
  int nsurv[kTcM];
  float d2[kTcM][kTcList];                            // filter-2 distances of the candidates
  uint8_t cand[kTcM][kTcList];                        // filter-1 candidates
  uint8_t code[kTcM][kMaxStages];
  float nrm[kTcM][kMaxStages];
  int zsel[kTcM];
  uint64_t mbar;
  uint32_t tmem_base;
};

// Element i of row r inside a swizzled panel (128 bytes per row, 16-byte chunk c of row r at
// position c ^ (r & 7)).
__device__ __forceinline__ int tc_swz(int r, int i) {
  return r * 32 + ((((i >> 2) ^ r) & 7) << 2) + (i & 3);
}
// Start of 16-byte chunk q (0..7) of row r inside a swizzled panel.
__device__ __forceinline__ int tc_chunk(int r, int q) { return r * 32 + ((q ^ r) & 7) * 4; }

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups 1024 bytes apart.
__device__ __forceinline__ uint64_t tc_desc(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);            // start address
  d |= (uint64_t)1u << 16;                            // leading byte offset (unused, 1)
  d |= (uint64_t)(1024u >> 4) << 32;                  // stride byte offset
  d |= (uint64_t)1u << 46;                            // descriptor version
  d |= (uint64_t)2u << 61;                            // 128-byte swizzle
  return d;
}

// Instruction descriptor: D float32, A and B tf32, both K-major, M = 128, N = 256.
constexpr uint32_t kTcIdesc = (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)(kTcN >> 3) << 17) |
                              ((uint32_t)(kTcM >> 4) << 24);

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// 32 consecutive accumulator columns of this thread's TMEM lane.
__device__ __forceinline__ void tc_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
      "%12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, "
      "%30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int k = 0; k < 32; ++k) v[k] = __uint_as_float(r[k]);
}

// Bounded wait for phase `parity` of the MMA mbarrier; false when the limit ran out (the
// caller then reports ZKV_DEVERR_TIMEOUT and stops instead of hanging the device).
__device__ __forceinline__ bool tc_wait(uint32_t mbar, uint32_t parity) {
  for (uint32_t it = 0; it < (1u << 20); ++it) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(mbar), "r"(parity)
        : "memory");
    if (ok) return true;
  }
  return false;
}

// float32 dot-form distance ||c||^2 - 2 r.c of row r and codeword c (sequential-FMA error
// model of encode.cu; four partial sums, the bound holds for any order)
template <int P>
__device__ __forceinline__ float tc_dist32(const float (*a)[kTcM * 32], const float (*b)[kTcN * 32],
                                           const float* cn, int r, int c) {
  float d4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 1
  for (int p = 0; p < P; ++p)
#pragma unroll 4
    for (int q = 0; q < 8; ++q) {
      const float4 x4 = *reinterpret_cast<const float4*>(&a[p][tc_chunk(r, q)]);
      const float4 c4 = *reinterpret_cast<const float4*>(&b[p][tc_chunk(c, q)]);
      d4[0] = fmaf(x4.x, c4.x, d4[0]);
      d4[1] = fmaf(x4.y, c4.y, d4[1]);
      d4[2] = fmaf(x4.z, c4.z, d4[2]);
      d4[3] = fmaf(x4.w, c4.w, d4[3]);
    }
  return cn[c] - 2.f * ((d4[0] + d4[1]) + (d4[2] + d4[3]));
}

// ||r - c||^2 in float64 (four partial sums)
template <int P>
__device__ __forceinline__ double tc_dist64(const float (*a)[kTcM * 32], const float (*b)[kTcN * 32],
                                            int r, int c) {
  double d4[4] = {0.0, 0.0, 0.0, 0.0};
#pragma unroll 1
  for (int p = 0; p < P; ++p)
#pragma unroll 4
    for (int q = 0; q < 8; ++q) {
      const float4 x4 = *reinterpret_cast<const float4*>(&a[p][tc_chunk(r, q)]);
      const float4 c4 = *reinterpret_cast<const float4*>(&b[p][tc_chunk(c, q)]);
      double df;
      df = (double)x4.x - (double)c4.x; d4[0] = fma(df, df, d4[0]);
      df = (double)x4.y - (double)c4.y; d4[1] = fma(df, df, d4[1]);
      df = (double)x4.z - (double)c4.z; d4[2] = fma(df, df, d4[2]);
      df = (double)x4.w - (double)c4.w; d4[3] = fma(df, df, d4[3]);
    }
  return (d4[0] + d4[1]) + (d4[2] + d4[3]);
}

constexpr int kTcThreads = 512;    // 16 warps: 4 per TMEM lane quarter, each 64 columns

template <int D>
__global__ void __launch_bounds__(kTcThreads, 1) encode_tc_kernel(StridedRows map,
                                                                  const float* __restrict__ books,
                                                                  int S, double rot_scale,
                                                                  int* __restrict__ err) {
  constexpr int E = D / 32;          // elements per lane in the row transform
  constexpr int P = TcSmem<D>::P;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  // the operand panels must start on 1024-byte boundaries (swizzle atoms)
  unsigned char* base = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  TcSmem<D>& sm = *reinterpret_cast<TcSmem<D>*>(base);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int h = blockIdx.y;
  const int64_t row0 = (int64_t)blockIdx.x * kTcM;
  const uint32_t mbar = (uint32_t)__cvta_generic_to_shared(&sm.mbar);

  if (warp == 0) {
    const uint32_t slot = (uint32_t)__cvta_generic_to_shared(&sm.tmem_base);
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(slot),
                 "r"((uint32_t)kTcN)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (tid == 0) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(mbar) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }

  // load, rotate and store the rows: warp w handles rows w, w + 16, ..., four at a time
  for (int rb = warp; rb < kTcM; rb += 64) {
    double v[4][E];
    bool ok[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int64_t j = row0 + rb + 16 * u;
      ok[u] = map.valid(j, h);
      if (ok[u]) {
        load_row_f64<E>(map.src(), map.dtype(), map.x_off(j, h), lane, v[u]);
        map.apply_smooth<E>(v[u], h, lane);
      } else {
#pragma unroll
        for (int q = 0; q < E; ++q) v[u][q] = 0.0;
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int row = rb + 16 * u;
      if (ok[u] && map.do_rotate()) {
        fwht_warp_f64<D>(v[u], lane);
#pragma unroll
        for (int q = 0; q < E; ++q) v[u][q] *= rot_scale;
      }
      double ss = 0.0;
#pragma unroll
      for (int q = 0; q < E; ++q) {   // element q*32 + lane lives in panel q
        const float y = (float)v[u][q];
        sm.a[q][tc_swz(row, lane)] = y;
        ss += (double)y * (double)y;
      }
      ss = warp_sum_f64(ss);
      if (lane == 0) sm.rn[row] = sqrt(ss);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  const uint32_t a_base = (uint32_t)__cvta_generic_to_shared(&sm.a[0][0]);
  const uint32_t b_base = (uint32_t)__cvta_generic_to_shared(&sm.b[0][0]);
  // epilogue roles: row r (TMEM lane r = 32 * (warp % 4) + lane), column group g (64 columns)
  const int quarter = warp & 3, g = warp >> 2;
  const int r = quarter * 32 + lane;
  const uint32_t taddr = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(g * 64);

  const float* CB = books + (size_t)h * S * kCodebook * D;
  int stalled = -1;                   // stage whose MMA completion never arrived
  for (int s = 0; s < S; ++s) {
    const float* C = CB + (size_t)s * kCodebook * D;
    // codebook stage -> swizzled panels: chunk f = (codeword n, global chunk gc); a thread's
    // chunks share gc and n & 7, so its destinations and sources advance by fixed strides
    {
      constexpr int CPR = D / 4;                      // chunks per codeword
      constexpr int NSTEP = kTcThreads / CPR;         // codewords per pass
      const int n0 = tid / CPR, gc = tid % CPR;
      float* dst = &sm.b[gc >> 3][tc_chunk(n0, gc & 7)];
      const float* src = C + (size_t)n0 * D + gc * 4;
#pragma unroll 4
      for (int i = 0; i < kTcN / NSTEP; ++i) cp_async16(dst + i * NSTEP * 32, src + (size_t)i * NSTEP * D);
    }
    cp_async_wait_all();
    // residual writes (previous stage) and the copies must be visible to the tensor cores
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (tid == 0) {
#pragma unroll
      for (int k = 0; k < D / 8; ++k) {
        const int p = k >> 2, o = (k & 3) * 32;   // panel, byte offset inside the 128-byte row
        const uint64_t ad = tc_desc(a_base + (uint32_t)(p * kTcM * 128 + o));
        const uint64_t bd = tc_desc(b_base + (uint32_t)(p * kTcN * 128 + o));
        const uint32_t acc = k > 0 ? 1u : 0u;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "setp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}"
            ::"r"(tmem), "l"(ad), "l"(bd), "r"(kTcIdesc), "r"(acc)
            : "memory");
      }
      asm volatile(
          "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(mbar)
          : "memory");
    }
    // codeword norms while the tensor cores run (float32, four partial sums)
    if (tid < kTcN) {
      const int n = tid;
      float c4s[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int p = 0; p < P; ++p)
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const float4 v = *reinterpret_cast<const float4*>(&sm.b[p][tc_chunk(n, q)]);
          c4s[0] = fmaf(v.x, v.x, c4s[0]);
          c4s[1] = fmaf(v.y, v.y, c4s[1]);
          c4s[2] = fmaf(v.z, v.z, c4s[2]);
          c4s[3] = fmaf(v.w, v.w, c4s[3]);
        }
      const float c2 = (c4s[0] + c4s[1]) + (c4s[2] + c4s[3]);
      sm.cn[n] = c2;
      const float m = warp_max_f32(c2);
      if (lane == 0) sm.cmax_w[warp] = m;
    }
    if (tid < kTcM) sm.ncand[tid] = 0;
    __syncthreads();
    float cmax = sm.cmax_w[0];
#pragma unroll
    for (int w = 1; w < kTcN / 32; ++w) cmax = fmaxf(cmax, sm.cmax_w[w]);
    const bool late = !tc_wait(mbar, (uint32_t)(s & 1));
    tc_fence_after();

    // filter 1: TF32 distances of this thread's 64 columns; pass 1 takes the minimum, pass 2
    // (after the row's four minima are combined) re-reads TMEM and lists the candidates
    float m4[4] = {FLT_MAX, FLT_MAX, FLT_MAX, FLT_MAX};
#pragma unroll
    for (int h2 = 0; h2 < 2; ++h2) {
      float dv[32];
      tc_ld32(taddr + 32u * h2, dv);
#pragma unroll
      for (int k = 0; k < 32; k += 4) {
        const float4 c4 = *reinterpret_cast<const float4*>(&sm.cn[g * 64 + 32 * h2 + k]);
        m4[0] = fminf(m4[0], c4.x - 2.f * dv[k + 0]);
        m4[1] = fminf(m4[1], c4.y - 2.f * dv[k + 1]);
        m4[2] = fminf(m4[2], c4.z - 2.f * dv[k + 2]);
        m4[3] = fminf(m4[3], c4.w - 2.f * dv[k + 3]);
      }
    }
    sm.gmin[g][r] = fminf(fminf(m4[0], m4[1]), fminf(m4[2], m4[3]));
    if (__syncthreads_or(late)) {      // uniform: every thread leaves the stage loop together
      stalled = s;
      break;
    }
    const double rn = sm.rn[r];
    {
      // thresholds are compared in float32, rounded up: a superset of the exact comparison
      const float m1 = fminf(fminf(sm.gmin[0][r], sm.gmin[1][r]), fminf(sm.gmin[2][r], sm.gmin[3][r]));
      const double e1 = 1.02 * 0.00390625 * rn * sqrt((double)cmax) + 1.52587890625e-05 * (double)cmax;
      const float thr1 = __double2float_ru((double)m1 + 2.0 * e1);
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        float dv[32];
        tc_ld32(taddr + 32u * h2, dv);
#pragma unroll
        for (int k = 0; k < 32; k += 4) {
          const int c = g * 64 + 32 * h2 + k;
          const float4 c4 = *reinterpret_cast<const float4*>(&sm.cn[c]);
          const float cv[4] = {c4.x, c4.y, c4.z, c4.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            if (cv[e] - 2.f * dv[k + e] <= thr1) {
              const int slot = atomicAdd(&sm.ncand[r], 1);
              if (slot < kTcList) sm.cand[r][slot] = (uint8_t)(c + e);
            }
          }
        }
      }
    }
    if (tid < kTcM) sm.nsurv[tid] = 0;
    tc_fence_before();
    __syncthreads();   // also: every TMEM read of this stage is done
    // filters 2 and 3, each row's candidates split among its four column-group threads.
    // Overflowed lists (never seen in practice) fall back to every codeword.
    const int n1 = sm.ncand[r];
    const bool all = n1 > kTcList;
    const int nl = all ? kTcN : n1;
    if (nl > 1) {
      float m2 = FLT_MAX;
      for (int k = g; k < nl; k += 4) {
        const int c = all ? k : sm.cand[r][k];
        const float d2 = tc_dist32<P>(sm.a, sm.b, sm.cn, r, c);
        if (!all) sm.d2[r][k] = d2;
        m2 = fminf(m2, d2);
      }
      sm.gmin[g][r] = m2;
    }
    __syncthreads();
    float thr2 = 0.f;
    if (nl > 1) {
      const float m2 = fminf(fminf(sm.gmin[0][r], sm.gmin[1][r]), fminf(sm.gmin[2][r], sm.gmin[3][r]));
      thr2 = __double2float_ru((double)m2 + candidate_margin(rn, cmax, D));
      int cnt = 0;
      for (int k = g; k < nl; k += 4) {
        const float d2 = all ? tc_dist32<P>(sm.a, sm.b, sm.cn, r, k) : sm.d2[r][k];
        cnt += d2 <= thr2 ? 1 : 0;
      }
      if (cnt) atomicAdd(&sm.nsurv[r], cnt);
    }
    __syncthreads();
    {
      // one survivor: it is the argmin; several: float64 distances, ties to the lowest index
      double best = DBL_MAX;
      int bz = kCodebook;
      if (nl == 1) {
        if (g == 0) bz = sm.cand[r][0];
      } else if (nl > 1) {
        const bool exact = sm.nsurv[r] > 1;
        for (int k = g; k < nl; k += 4) {
          const int c = all ? k : sm.cand[r][k];
          const float d2 = all ? tc_dist32<P>(sm.a, sm.b, sm.cn, r, k) : sm.d2[r][k];
          if (d2 > thr2) continue;
          const double dd = exact ? tc_dist64<P>(sm.a, sm.b, r, c) : 0.0;
          if (dd < best || (dd == best && c < bz)) {
            best = dd;
            bz = c;
          }
        }
      }
      sm.gbest[g][r] = best;
      sm.gbz[g][r] = bz;
    }
    __syncthreads();
    if (g == 0) {
      double best = sm.gbest[0][r];
      int bz = sm.gbz[0][r];
#pragma unroll
      for (int q = 1; q < 4; ++q) {
        const double dd = sm.gbest[q][r];
        const int c = sm.gbz[q][r];
        if (dd < best || (dd == best && c < bz)) {
          best = dd;
          bz = c;
        }
      }
      sm.zsel[r] = bz < kCodebook ? bz : 0;   // non-finite rows match no candidate
    }
    __syncthreads();
    // residual update r <- r - C[z] (float32): column group g updates panel(s) g, g + 4
    {
      const int z = sm.zsel[r];
      double ss = 0.0;
      for (int p = g; p < P; p += 4) {
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          float4* xp = reinterpret_cast<float4*>(&sm.a[p][tc_chunk(r, q)]);
          const float4 c4 = *reinterpret_cast<const float4*>(&sm.b[p][tc_chunk(z, q)]);
          float4 x4 = *xp;
          x4.x -= c4.x;
          x4.y -= c4.y;
          x4.z -= c4.z;
          x4.w -= c4.w;
          *xp = x4;
          ss += (double)x4.x * x4.x + (double)x4.y * x4.y + (double)x4.z * x4.z + (double)x4.w * x4.w;
        }
      }
      sm.part[g][r] = ss;
    }
    __syncthreads();
    if (g == 0) {
      const double nn = sqrt((sm.part[0][r] + sm.part[1][r]) + (sm.part[2][r] + sm.part[3][r]));
      sm.rn[r] = nn;
      sm.code[r][s] = (uint8_t)sm.zsel[r];
      sm.nrm[r][s] = (float)nn;
    }
    // the next stage's first barrier orders these writes before their use
  }
  if (stalled >= 0) {
    // no codes are stored; one more bounded wait lets the stage's MMAs finish before the
    // accumulator columns are freed
    if (tid == 0 && err != nullptr) atomicOr(err, ZKV_DEVERR_TIMEOUT);
    if (warp == 0) (void)tc_wait(mbar, (uint32_t)(stalled & 1));
  }
  __syncthreads();
  if (g == 0 && stalled < 0) {
    const int64_t j = row0 + r;
    if (map.valid(j, h)) map.store(j, h, S, sm.code[r], sm.nrm[r]);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"((uint32_t)kTcN)
                 : "memory");
  }
}

template <int D>
constexpr size_t tc_smem_bytes() {
  return sizeof(TcSmem<D>) + 1024;   // + alignment of the operand panels
}
static_assert(sizeof(TcSmem<128>) + 1024 <= 227 * 1024, "tensor-core encode tile exceeds shared memory");

int launch_encode_tc(const StridedRows& map, int64_t n_head, int d, int S, const float* books,
                     int* err, cudaStream_t st) {
  const double rot = 1.0 / std::sqrt((double)d);
  const dim3 grid((unsigned)((map.n_rows + kTcM - 1) / kTcM), (unsigned)n_head);
  switch (d) {
    case 64:
      if (ensure_smem_limit(encode_tc_kernel<64>, tc_smem_bytes<64>()) != cudaSuccess) return ZKV_ERR_CUDA;
      encode_tc_kernel<64><<<grid, kTcThreads, tc_smem_bytes<64>(), st>>>(map, books, S, rot, err);
      break;
    case 128:
      if (ensure_smem_limit(encode_tc_kernel<128>, tc_smem_bytes<128>()) != cudaSuccess) return ZKV_ERR_CUDA;
      encode_tc_kernel<128><<<grid, kTcThreads, tc_smem_bytes<128>(), st>>>(map, books, S, rot, err);
      break;
    default:
      return ZKV_ERR_UNSUPPORTED;
  }
  ZKV_CHECK_LAUNCH();
  return ZKV_OK;
}

}  // namespace zkv
