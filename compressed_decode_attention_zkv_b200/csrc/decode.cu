// Compressed decode attention (sm_100a).
//
// Passages: VQKV (gist.science summary of arXiv 2603.16435), section 2.3 "Decoding Stage":
// codes are read directly and keys/values are reconstructed on demand inside the attention
// computation; "Local Sliding Window": recent tokens stay uncompressed.  VeloxQuant-MLX 0.5.1,
// "VecInfer": the Walsh-Hadamard rotation is absorbed into the query (q_tilde . k_tilde =
// q . k).  Differential-KV README, "Decode & Prefill Innovations": flash-style fp32
// log-sum-exp combine of the compressed part with the dense recency window.
//
// Three kernels per call:
//   1. lut_kernel    q_tilde = H q / sqrt(d) (float64, one rounding), per stage
//                    LUT_s[c] = (scale * log2 e) * q_tilde . Ck_s[c] -> workspace; the dense
//                    window attention of every (sequence, kv head); prefix sums of the
//                    compressed lengths that partition the token space among scan CTAs.
//   2. scan_kernel   one CTA per SM walks a contiguous range of the concatenated compressed
//                    tokens of all (sequence, kv head) pairs.  Per pair segment: pass 1 takes
//                    score_t = sum_s LUT_s[zk_{t,s}] (base-2 logits) and their maximum m; pass 2
//                    recomputes the scores, p_t = 2^(score_t - m), and accumulates per-stage
//                    codeword weight histograms W_s[c] = sum over tokens with zv_{t,s} = c of p_t.
//                    sum_t p_t sum_s Cv_s[zv_{t,s}] = sum_s sum_c W_s[c] Cv_s[c]: the value
//                    reconstruction regrouped by codeword.
//   3. merge_kernel  grid (value stage, kv head, sequence): merges the segment histograms by
//                    their maxima, contracts W_s with Cv_s, and the last stage CTA of each
//                    (sequence, kv head) sums the stages, rotates back, and merges with the
//                    window by log-sum-exp.  "Last CTA" is an atomic ticket; no CTA waits.
//
// Shared-memory design of the scan (shared memory bandwidth, not HBM, bounds this kernel):
//  * key tables are replicated per lane group so that the 8 (or 16, 32) lanes of a 128-bit
//    (64-, 32-bit) gather always hit distinct banks;
//  * value histograms use the native shared-memory integer reduction: p is converted to
//    38-bit fixed point (exact to 2^-39 absolute per token, p <= 1 because the segment maximum
//    is known after pass 1) split into two 19-bit halves added with red.shared.add.u32; lanes
//    are mapped to (token slot, stage, head) so one instruction touches 32 distinct banks.
//    Column sums stay below 2^32 because a segment holds at most 8176 tokens per column.
#include "zkv_internal.cuh"

#include <algorithm>
#include <cfloat>
#include <cmath>

namespace zkv {

constexpr int kScanSub = 1024;      // tokens per scan sub-chunk (4 per thread)
constexpr int kScanThreads = 256;
constexpr int kColCap = 8176;       // tokens per histogram column per segment (sum < 2^32)
constexpr size_t kSmemMax = 227 * 1024;

static int sm_count() {
  static int n = 0;
  if (n == 0) {
    int dev = 0, v = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 148;
    n = v;
  }
  return n;
}

static int pow2ceil(int x) { int p = 1; while (p < x) p <<= 1; return p; }
static int pad_heads(int G) { return pow2ceil(G); }
static int pad_stages(int S) { return std::max(2, pow2ceil(S)); }

// Value-side lane mapping: lanes <-> (token slot j, stage s, head g).
struct VMap {
  int combos, J, passes, VW, rounds, codew;
};
static VMap vmap(int SVP, int GP) {
  VMap v;
  v.combos = SVP * GP;
  v.J = v.combos >= 32 ? 1 : 32 / v.combos;
  v.passes = v.combos > 32 ? v.combos / 32 : 1;
  v.VW = 32 * v.passes;
  v.rounds = kScanSub / v.J;
  v.codew = SVP <= 4 ? 1 : 2;
  return v;
}

struct DecodePlan {
  int G, GP, SKP, SVP, Rk, grid;
  int64_t cap, slots;
  size_t scan_smem;
  size_t off_lut, off_pre, off_share, off_pm, off_pl, off_pw, off_wm, off_wl, off_wo, off_so,
      off_cnt, total;
};

static size_t scan_smem_bytes(int Rk, int Sk, int GP, const VMap& v) {
  size_t b = (size_t)Rk * Sk * kCodebook * GP * 4;            // key tables
  b += 2ull * kCodebook * v.VW * 4;                            // value histograms (hi, lo)
  b += (size_t)v.J * GP * (v.rounds + 4) * 4;                   // p staging
  b += (size_t)v.J * (v.rounds + 4) * v.codew * 4;              // value-code staging
  b += (size_t)9 * GP * 4 + 16;                                 // reductions
  return b;
}

static DecodePlan make_plan(const zkv_decode_params* p) {
  DecodePlan pl{};
  pl.G = p->Hq / p->Hkv;
  pl.GP = pad_heads(pl.G);
  pl.SKP = pad_stages(p->Sk);
  pl.SVP = pad_stages(p->Sv);
  const VMap v = vmap(pl.SVP, pl.GP);
  // replication that makes the key gathers conflict-free, reduced until shared memory fits
  int Rk = pl.GP == 1 ? 32 : pl.GP == 2 ? 16 : pl.GP == 4 ? 8 : 4;
  while (Rk > 1 && scan_smem_bytes(Rk, p->Sk, pl.GP, v) > kSmemMax) Rk >>= 1;
  pl.Rk = Rk;
  pl.scan_smem = scan_smem_bytes(Rk, p->Sk, pl.GP, v);
  const int64_t pairs = (int64_t)p->B * p->Hkv;
  pl.cap = (int64_t)kColCap * v.J;
  const int64_t bound = pairs * p->max_comp_len;
  const int sms = sm_count();
  int64_t g1 = (bound + pl.cap - 1) / pl.cap;
  int64_t g2 = std::min<int64_t>(sms, (bound + 1023) / 1024);
  int64_t grid = std::max<int64_t>(1, std::max(g1, g2));
  if (grid > sms) grid = (grid + sms - 1) / sms * sms;
  pl.grid = (int)grid;
  pl.slots = pairs + grid;
  const size_t f = sizeof(float);
  size_t o = 0;
  pl.off_lut = o;   o = align256(o + (size_t)p->B * p->Hq * p->Sk * kCodebook * f);
  pl.off_pre = o;   o = align256(o + (size_t)(pairs + 1) * sizeof(int64_t));
  pl.off_share = o; o = align256(o + sizeof(int64_t));
  pl.off_pm = o;    o = align256(o + (size_t)pl.slots * pl.GP * f);
  pl.off_pl = o;    o = align256(o + (size_t)pl.slots * pl.GP * f);
  pl.off_pw = o;    o = align256(o + (size_t)pl.slots * p->Sv * kCodebook * pl.GP * f);
  pl.off_wm = o;    o = align256(o + (size_t)pairs * pl.GP * f);
  pl.off_wl = o;    o = align256(o + (size_t)pairs * pl.GP * f);
  pl.off_wo = o;    o = align256(o + (size_t)pairs * pl.GP * p->d * f);
  pl.off_so = o;    o = align256(o + (size_t)pairs * p->Sv * pl.GP * p->d * f);
  pl.off_cnt = o;   o = align256(o + (size_t)pairs * sizeof(unsigned));
  pl.total = o;
  return pl;
}

struct DecodeArgs {
  int B, Hq, Hkv, G, d, Sk, Sv, Rk, grid, n_lut_blocks;
  int64_t Tcap, Wcap, max_comp;
  float scale_log2;   // softmax_scale * log2(e)
  double rot;         // 1 / sqrt(d)
  const __half* q;
  const uint8_t* k_codes;
  const uint8_t* v_codes;
  const int32_t* comp_len;
  const float* Ck;
  const float* Cv;
  const __half* win_k;
  const __half* win_v;
  const int32_t* win_len;
  float* out;
  float* lse;
  int32_t* err;
  float* lut;        // [B][Hq][Sk][256]
  int64_t* pre;      // [B*Hkv + 1] exclusive prefix sums of compressed lengths
  int64_t* share;    // tokens per scan CTA
  float* pm;         // [slots][GP] segment maxima
  float* pl;         // [slots][GP] segment sums of p
  float* pw;         // [slots][Sv][256][GP] segment histograms
  float* wm;         // [B*Hkv][GP]
  float* wl;         // [B*Hkv][GP]
  float* wo;         // [B*Hkv][GP][d]
  float* so;         // [B*Hkv][Sv][GP][d]
  unsigned* cnt;     // [B*Hkv]
};

__device__ __forceinline__ int64_t clamp_win_len(const DecodeArgs& a, int b) {
  int64_t w = a.win_len[b];
  if (w < 0 || w > a.Wcap) {
    if (threadIdx.x == 0) set_error(a.err, ZKV_DEVERR_WIN_LEN);
    w = w < 0 ? 0 : a.Wcap;
  }
  return w;
}

// ------------------------------------------------------------------------------------------
// 1. Query rotation + lookup tables; window attention; length prefix sums.
//    1-D grid: [0, n_lut_blocks) tables, then one block per (sequence, kv head) window.
// ------------------------------------------------------------------------------------------
constexpr int kLutC = 64;     // codewords per block
constexpr int kLutH = 32;     // attached query heads per block (b * G + g)

template <int D>
struct LutSmem {
  float qT[D][kLutH + 4];     // rotated queries, k-major
  float cT[D][kLutC + 1];     // codebook slice, k-major
};

template <int D, int GP>
__device__ void window_item(const DecodeArgs& a, int b, int kvh, float* smem) {
  float* qs = smem;                 // [GP][D]   query * scale * log2 e
  float* ps = qs + GP * D;          // [256][GP] probabilities of the current tile
  float* red = ps + 256 * GP;       // [8][GP]
  float* alph = red + 8 * GP;       // [GP]      rescale factor of the current tile
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t pair = (int64_t)b * a.Hkv + kvh;
  const int64_t wl = clamp_win_len(a, b);
  for (int f = tid; f < GP * D; f += 256) {
    const int g = f / D, i = f % D;
    qs[f] = g < a.G ? __half2float(a.q[((int64_t)b * a.Hq + (int64_t)kvh * a.G + g) * D + i]) *
                          a.scale_log2
                    : 0.f;
  }
  float m_run[GP], l_run[GP];
#pragma unroll
  for (int g = 0; g < GP; ++g) { m_run[g] = -INFINITY; l_run[g] = 0.f; }
  constexpr int OPT = (GP * D + 255) / 256;   // output elements (g, i) owned per thread
  float oacc[OPT];
#pragma unroll
  for (int r = 0; r < OPT; ++r) oacc[r] = 0.f;
  __syncthreads();
  const __half* Kb = a.win_k + pair * a.Wcap * D;
  const __half* Vb = a.win_v + pair * a.Wcap * D;
  for (int64_t base = 0; base < wl; base += 256) {
    const int64_t t = base + tid;
    float sc[GP];
#pragma unroll
    for (int g = 0; g < GP; ++g) sc[g] = t < wl ? 0.f : -INFINITY;
    if (t < wl) {
      const __half* kr = Kb + t * D;
      for (int i = 0; i < D; i += 8) {
        const uint4 raw = __ldg(reinterpret_cast<const uint4*>(kr + i));
        const __half2* h2 = reinterpret_cast<const __half2*>(&raw);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 kv = __half22float2(h2[e]);
#pragma unroll
          for (int g = 0; g < GP; ++g) {
            sc[g] = fmaf(qs[g * D + i + 2 * e], kv.x, sc[g]);
            sc[g] = fmaf(qs[g * D + i + 2 * e + 1], kv.y, sc[g]);
          }
        }
      }
    }
#pragma unroll
    for (int g = 0; g < GP; ++g) {
      const float m = warp_max_f32(sc[g]);
      if (lane == 0) red[warp * GP + g] = m;
    }
    __syncthreads();
#pragma unroll
    for (int g = 0; g < GP; ++g) {
      float m = red[g];
#pragma unroll
      for (int w = 1; w < 8; ++w) m = fmaxf(m, red[w * GP + g]);
      const float mn = fmaxf(m_run[g], m);
      const float alpha = m_run[g] == -INFINITY ? 0.f : ex2_approx(m_run[g] - mn);
      l_run[g] *= alpha;
      m_run[g] = mn;
      const float pv = t < wl ? ex2_approx(sc[g] - mn) : 0.f;
      ps[tid * GP + g] = pv;
      l_run[g] += pv;
      if (tid == 0) alph[g] = alpha;
    }
    __syncthreads();
    const int64_t nt = wl - base < 256 ? wl - base : 256;
#pragma unroll
    for (int r = 0; r < OPT; ++r) {
      const int f = tid + 256 * r;
      if (f < GP * D) {
        const int g = f / D, i = f % D;
        float acc = oacc[r] * alph[g];
#pragma unroll 4
        for (int64_t tt = 0; tt < nt; ++tt)
          acc = fmaf(ps[tt * GP + g], __half2float(Vb[(base + tt) * D + i]), acc);
        oacc[r] = acc;
      }
    }
    __syncthreads();
  }
#pragma unroll
  for (int g = 0; g < GP; ++g) {
    const float l = warp_sum_f32(l_run[g]);
    if (lane == 0) red[warp * GP + g] = l;
  }
  __syncthreads();
  if (tid < GP) {
    float l = 0.f;
    for (int w = 0; w < 8; ++w) l += red[w * GP + tid];
    a.wm[pair * GP + tid] = m_run[tid];
    a.wl[pair * GP + tid] = l;
  }
#pragma unroll
  for (int r = 0; r < OPT; ++r) {
    const int f = tid + 256 * r;
    if (f < GP * D) a.wo[pair * GP * D + f] = oacc[r];
  }
}

template <int D, int GP>
__global__ void __launch_bounds__(256) lut_kernel(DecodeArgs a) {
  constexpr int E = D / 32;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if ((int)blockIdx.x >= a.n_lut_blocks) {
    const int pair = blockIdx.x - a.n_lut_blocks;
    window_item<D, GP>(a, pair / a.Hkv, pair % a.Hkv, reinterpret_cast<float*>(smem_raw));
    return;
  }
  if (blockIdx.x == 0) {
    const int npairs = a.B * a.Hkv;
    for (int i = tid; i < npairs; i += blockDim.x) a.cnt[i] = 0u;
    if (tid == 0) {
      int64_t acc = 0;
      a.pre[0] = 0;
      for (int pr = 0; pr < npairs; ++pr) {
        int64_t c = a.comp_len[pr / a.Hkv];
        if (c < 0 || c > a.Tcap) {
          set_error(a.err, ZKV_DEVERR_COMP_LEN);
          c = c < 0 ? 0 : a.Tcap;
        }
        c = c < a.max_comp ? c : a.max_comp;
        acc += c;
        a.pre[pr + 1] = acc;
      }
      int64_t sh = (acc + a.grid - 1) / a.grid;
      sh = (sh + 15) / 16 * 16;
      *a.share = sh < 16 ? 16 : sh;
    }
  }
  LutSmem<D>& sm = *reinterpret_cast<LutSmem<D>*>(smem_raw);
  const int n_hg = (a.B * a.G + kLutH - 1) / kLutH;
  int rest = blockIdx.x;
  const int cblk = rest % (kCodebook / kLutC);
  rest /= kCodebook / kLutC;
  const int s = rest % a.Sk;
  rest /= a.Sk;
  const int hg = rest % n_hg;
  const int kvh = rest / n_hg;
  const int c0 = cblk * kLutC;
  // rotated queries of the attached heads j = b*G + g
  for (int jl = warp; jl < kLutH; jl += 8) {
    const int j = hg * kLutH + jl;
    double v[E];
    if (j < a.B * a.G) {
      const int b = j / a.G, g = j % a.G;
      const int64_t off = ((int64_t)b * a.Hq + (int64_t)kvh * a.G + g) * D;
      load_row_f64<E>(a.q, ZKV_DTYPE_F16, off, lane, v);
      fwht_warp_f64<D>(v, lane);
#pragma unroll
      for (int q = 0; q < E; ++q) sm.qT[q * 32 + lane][jl] = (float)(v[q] * a.rot);
    } else {
#pragma unroll
      for (int q = 0; q < E; ++q) sm.qT[q * 32 + lane][jl] = 0.f;
    }
  }
  // codebook slice C[kvh][s][c0 .. c0+63][:]
  const float* C = a.Ck + (((size_t)kvh * a.Sk + s) * kCodebook + c0) * D;
  for (int f = tid; f < kLutC * D / 4; f += 256) {
    const int c = f / (D / 4), i = (f % (D / 4)) * 4;
    const float4 v = __ldg(reinterpret_cast<const float4*>(C + (size_t)c * D + i));
    sm.cT[i + 0][c] = v.x;
    sm.cT[i + 1][c] = v.y;
    sm.cT[i + 2][c] = v.z;
    sm.cT[i + 3][c] = v.w;
  }
  __syncthreads();
  const int cc = tid & (kLutC - 1), hq = tid >> 6;   // 4 groups of 8 heads
  float acc[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) acc[k] = 0.f;
#pragma unroll 4
  for (int i = 0; i < D; ++i) {
    const float cv = sm.cT[i][cc];
    const float4 q0 = *reinterpret_cast<const float4*>(&sm.qT[i][hq * 8]);
    const float4 q1 = *reinterpret_cast<const float4*>(&sm.qT[i][hq * 8 + 4]);
    acc[0] = fmaf(q0.x, cv, acc[0]);
    acc[1] = fmaf(q0.y, cv, acc[1]);
    acc[2] = fmaf(q0.z, cv, acc[2]);
    acc[3] = fmaf(q0.w, cv, acc[3]);
    acc[4] = fmaf(q1.x, cv, acc[4]);
    acc[5] = fmaf(q1.y, cv, acc[5]);
    acc[6] = fmaf(q1.z, cv, acc[6]);
    acc[7] = fmaf(q1.w, cv, acc[7]);
  }
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const int j = hg * kLutH + hq * 8 + k;
    if (j < a.B * a.G) {
      const int b = j / a.G, g = j % a.G;
      const int64_t h = (int64_t)kvh * a.G + g;
      a.lut[(((int64_t)b * a.Hq + h) * a.Sk + s) * kCodebook + c0 + cc] = acc[k] * a.scale_log2;
    }
  }
}

// ------------------------------------------------------------------------------------------
// 2. Scan of the compressed tokens.
// ------------------------------------------------------------------------------------------

// Codes of one token (S <= 8 bytes, little-endian in up to two words).
template <int SP>
struct Code {
  uint32_t w[SP <= 4 ? 1 : 2];
  __device__ __forceinline__ int byte(int s) const {
    if constexpr (SP <= 4) return (w[0] >> (8 * s)) & 0xff;
    else return (w[s >> 2] >> (8 * (s & 3))) & 0xff;
  }
};

// Codes of the 4 consecutive tokens t0..t0+3 (t0 a multiple of 4, below Tcap).  When S equals
// its padded size SP one naturally aligned vector load covers all four; otherwise byte loads.
template <int SP>
__device__ __forceinline__ void load_codes4(const uint8_t* base, int S, int64_t t0, int64_t tend,
                                            Code<SP> (&out)[4]) {
#pragma unroll
  for (int u = 0; u < 4; ++u) {
#pragma unroll
    for (int q = 0; q < (SP <= 4 ? 1 : 2); ++q) out[u].w[q] = 0u;
  }
  if (t0 >= tend) return;
  if (S == SP) {
    const uint8_t* p = base + t0 * SP;
    if constexpr (SP == 2) {
      const uint2 v = __ldg(reinterpret_cast<const uint2*>(p));
      out[0].w[0] = v.x & 0xffffu; out[1].w[0] = v.x >> 16;
      out[2].w[0] = v.y & 0xffffu; out[3].w[0] = v.y >> 16;
    } else if constexpr (SP == 4) {
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(p));
      out[0].w[0] = v.x; out[1].w[0] = v.y; out[2].w[0] = v.z; out[3].w[0] = v.w;
    } else {
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(p));
      const uint4 u = __ldg(reinterpret_cast<const uint4*>(p + 16));
      out[0].w[0] = v.x; out[0].w[1] = v.y; out[1].w[0] = v.z; out[1].w[1] = v.w;
      out[2].w[0] = u.x; out[2].w[1] = u.y; out[3].w[0] = u.z; out[3].w[1] = u.w;
    }
  } else {
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      if (t0 + u < tend) {
        const uint8_t* p = base + (t0 + u) * S;
#pragma unroll
        for (int s = 0; s < SP; ++s)
          if (s < S) out[u].w[s >> 2] |= (uint32_t)p[s] << (8 * (s & 3));
      }
    }
  }
}

// Key score of one token: sum over stages of the token's table entries (GP heads).
template <int GP, int SKP>
__device__ __forceinline__ void key_score(const float* lut, int Sk, int Rk, int copy, int lane,
                                          const Code<SKP>& kc, float (&sc)[GP]) {
#pragma unroll
  for (int g = 0; g < GP; ++g) sc[g] = 0.f;
#pragma unroll
  for (int s = 0; s < SKP; ++s) {
    if (s < Sk) {
      const int c = kc.byte(s);
      const float* e = lut + ((size_t)(s * kCodebook + c) * Rk + copy) * GP;
      if constexpr (GP == 8) {
        // the two halves are read in lane-dependent order: lanes 4-7 of each 8-lane phase
        // start with the upper half, which puts all 8 lanes of a phase in distinct banks
        const int h0 = (lane >> 2) & 1;
        const float4 v0 = *reinterpret_cast<const float4*>(e + 4 * h0);
        const float4 v1 = *reinterpret_cast<const float4*>(e + 4 * (h0 ^ 1));
        const float4 lo4 = h0 ? v1 : v0, hi4 = h0 ? v0 : v1;
        sc[0] += lo4.x; sc[1] += lo4.y; sc[2] += lo4.z; sc[3] += lo4.w;
        sc[4] += hi4.x; sc[5] += hi4.y; sc[6] += hi4.z; sc[7] += hi4.w;
      } else if constexpr (GP == 4) {
        const float4 v = *reinterpret_cast<const float4*>(e);
        sc[0] += v.x; sc[1] += v.y; sc[2] += v.z; sc[3] += v.w;
      } else if constexpr (GP == 2) {
        const float2 v = *reinterpret_cast<const float2*>(e);
        sc[0] += v.x; sc[1] += v.y;
      } else {
        sc[0] += e[0];
      }
    }
  }
}

__device__ __forceinline__ void red_add_u32(uint32_t* p, uint32_t v) {
  asm volatile("red.shared.add.u32 [%0], %1;" ::"r"((unsigned)__cvta_generic_to_shared(p)), "r"(v)
               : "memory");
}

template <int GP, int SKP, int SVP>
struct ScanCfg {
  static constexpr int COMBOS = SVP * GP;
  static constexpr int J = COMBOS >= 32 ? 1 : 32 / COMBOS;
  static constexpr int PASSES = COMBOS > 32 ? COMBOS / 32 : 1;
  static constexpr int VW = 32 * PASSES;
  static constexpr int ROUNDS = kScanSub / J;
  static constexpr int PR = ROUNDS + 4;          // padded staging row (floats / words)
  static constexpr int CODEW = SVP <= 4 ? 1 : 2;
};

template <int GP, int SKP, int SVP>
__global__ void __launch_bounds__(kScanThreads, 1) scan_kernel(DecodeArgs a) {
  using C = ScanCfg<GP, SKP, SVP>;
  extern __shared__ __align__(16) unsigned char smraw[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int Rk = a.Rk, Sk = a.Sk, Sv = a.Sv, G = a.G;
  float* lut = reinterpret_cast<float*>(smraw);                                 // [Sk][256][Rk][GP]
  uint32_t* vhi = reinterpret_cast<uint32_t*>(lut + (size_t)Rk * Sk * kCodebook * GP);  // [256][VW]
  uint32_t* vlo = vhi + kCodebook * C::VW;
  float* pst = reinterpret_cast<float*>(vlo + kCodebook * C::VW);               // [J][GP][PR]
  uint32_t* cst = reinterpret_cast<uint32_t*>(pst + C::J * GP * C::PR);         // [J][PR][CODEW]
  float* red = reinterpret_cast<float*>(cst + C::J * C::PR * C::CODEW);         // [8][GP]

  const int npairs = a.B * a.Hkv;
  const int64_t share = *a.share;
  const int64_t tot = a.pre[npairs];
  const int64_t lo = (int64_t)blockIdx.x * share;
  const int64_t hi = lo + share < tot ? lo + share : tot;
  if (lo >= hi) return;
  // last pair whose prefix start is <= lo
  int pfirst = 0;
  {
    int l = 0, r = npairs;   // invariant: pre[l] <= lo < pre[r] (pre[npairs] = tot > lo)
    while (r - l > 1) {
      const int m = (l + r) >> 1;
      if (a.pre[m] <= lo) l = m; else r = m;
    }
    pfirst = l;
  }
  const int copy = lane & (Rk - 1);
  // value-side lane roles (PASSES == 1: lane = j * COMBOS + s * GP + g)
  const int vj = C::PASSES == 1 ? lane / C::COMBOS : 0;

  for (int pr = pfirst; pr < npairs && a.pre[pr] < hi; ++pr) {
    const int64_t seg0 = lo > a.pre[pr] ? lo : a.pre[pr];
    const int64_t seg1 = hi < a.pre[pr + 1] ? hi : a.pre[pr + 1];
    if (seg0 >= seg1) continue;
    const int64_t s0 = seg0 - a.pre[pr], s1 = seg1 - a.pre[pr];   // pair-local token range
    const int b = pr / a.Hkv, kvh = pr % a.Hkv;
    const int64_t slot = (int64_t)pr + blockIdx.x;
    const uint8_t* kcb = a.k_codes + (int64_t)pr * a.Tcap * Sk;
    const uint8_t* vcb = a.v_codes + (int64_t)pr * a.Tcap * Sv;

    __syncthreads();   // previous segment's shared memory is free
    {
      const float* src = a.lut + ((int64_t)b * a.Hq + (int64_t)kvh * G) * Sk * kCodebook;
      const int n = Sk * kCodebook * GP;
      for (int f = tid; f < n; f += kScanThreads) {
        const int g = f % GP, sc = f / GP;       // sc = s*256 + c
        const float v = g < G ? __ldg(src + (int64_t)g * Sk * kCodebook + sc) : 0.f;
        float* dst = lut + (size_t)sc * Rk * GP + g;
        for (int cp = 0; cp < Rk; ++cp) dst[cp * GP] = v;
      }
      uint4* z = reinterpret_cast<uint4*>(vhi);
      const int nz = 2 * kCodebook * C::VW / 4;
      for (int f = tid; f < nz; f += kScanThreads) z[f] = make_uint4(0u, 0u, 0u, 0u);
    }
    __syncthreads();

    const int64_t abase = s0 & ~int64_t(3);
    // ---- pass 1: maximum score per head
    float mloc[GP];
#pragma unroll
    for (int g = 0; g < GP; ++g) mloc[g] = -INFINITY;
    for (int64_t base = abase; base < s1; base += kScanSub) {
      const int64_t t0 = base + 4 * tid;
      Code<SKP> kc[4];
      load_codes4<SKP>(kcb, Sk, t0, s1, kc);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int64_t t = t0 + u;
        if (t >= s0 && t < s1) {
          float sc[GP];
          key_score<GP, SKP>(lut, Sk, Rk, copy, lane, kc[u], sc);
#pragma unroll
          for (int g = 0; g < GP; ++g) mloc[g] = fmaxf(mloc[g], sc[g]);
        }
      }
    }
#pragma unroll
    for (int g = 0; g < GP; ++g) {
      const float m = warp_max_f32(mloc[g]);
      if (lane == 0) red[warp * GP + g] = m;
    }
    __syncthreads();
    float mseg[GP];
#pragma unroll
    for (int g = 0; g < GP; ++g) {
      float m = red[g];
#pragma unroll
      for (int w = 1; w < 8; ++w) m = fmaxf(m, red[w * GP + g]);
      mseg[g] = m;
    }

    // ---- pass 2: probabilities and value histograms
    float lacc[GP];
#pragma unroll
    for (int g = 0; g < GP; ++g) lacc[g] = 0.f;
    for (int64_t base = abase; base < s1; base += kScanSub) {
      const int64_t t0 = base + 4 * tid;
      Code<SKP> kc[4];
      Code<SVP> vc[4];
      load_codes4<SKP>(kcb, Sk, t0, s1, kc);
      load_codes4<SVP>(vcb, Sv, t0, s1, vc);
      __syncthreads();   // staging of the previous sub-chunk (and red) has been consumed
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int64_t t = t0 + u;
        const bool ok = t >= s0 && t < s1;
        float p[GP];
        if (ok) {
          float sc[GP];
          key_score<GP, SKP>(lut, Sk, Rk, copy, lane, kc[u], sc);
#pragma unroll
          for (int g = 0; g < GP; ++g) {
            p[g] = ex2_approx(sc[g] - mseg[g]);
            lacc[g] += p[g];
          }
        } else {
#pragma unroll
          for (int g = 0; g < GP; ++g) p[g] = 0.f;
        }
        // staging position: u * 256 + tid  ->  slot j, round k
        const int pos = u * kScanThreads + tid;
        const int j = pos % C::J, k = pos / C::J;
#pragma unroll
        for (int g = 0; g < GP; ++g) pst[(j * GP + g) * C::PR + k] = p[g];
        if constexpr (C::CODEW == 1) {
          cst[j * C::PR + k] = ok ? vc[u].w[0] : 0u;
        } else {
          reinterpret_cast<uint2*>(cst)[j * C::PR + k] =
              ok ? make_uint2(vc[u].w[0], vc[u].w[1]) : make_uint2(0u, 0u);
        }
      }
      __syncthreads();
      // value side: batches of 4 rounds, warp-strided
#pragma unroll
      for (int ps = 0; ps < C::PASSES; ++ps) {
        const int combo = C::PASSES == 1 ? lane % C::COMBOS : ps * 32 + lane;
        const int vs = combo / GP, vg = combo % GP;
        const bool active = vs < Sv && vg < G;
        const int col = ps * 32 + lane;
        const float* prow = pst + (vj * GP + vg) * C::PR;
        for (int bt = warp; bt < C::ROUNDS / 4; bt += 8) {
          const int k0 = bt * 4;
          const float4 pv = *reinterpret_cast<const float4*>(prow + k0);
          uint32_t cw[4];
          if constexpr (C::CODEW == 1) {
            const uint4 c4 = *reinterpret_cast<const uint4*>(cst + vj * C::PR + k0);
            cw[0] = c4.x; cw[1] = c4.y; cw[2] = c4.z; cw[3] = c4.w;
          } else {
            const uint4 c01 = *reinterpret_cast<const uint4*>(cst + 2 * (vj * C::PR + k0));
            const uint4 c23 = *reinterpret_cast<const uint4*>(cst + 2 * (vj * C::PR + k0) + 4);
            const int hw = vs >> 2;
            cw[0] = hw ? c01.y : c01.x; cw[1] = hw ? c01.w : c01.z;
            cw[2] = hw ? c23.y : c23.x; cw[3] = hw ? c23.w : c23.z;
          }
          const float pr4[4] = {pv.x, pv.y, pv.z, pv.w};
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            if (!active || pr4[r] == 0.f) continue;
            const int c = (cw[r] >> (8 * (vs & 3))) & 0xff;
            const unsigned long long fx = __float2ull_rn(pr4[r] * 274877906944.0f);  // p * 2^38
            red_add_u32(vhi + c * C::VW + col, (uint32_t)(fx >> 19));
            red_add_u32(vlo + c * C::VW + col, (uint32_t)(fx & 0x7ffffull));
          }
        }
      }
    }
    // ---- segment partial: maximum, sum of p, histograms in float
#pragma unroll
    for (int g = 0; g < GP; ++g) {
      const float l = warp_sum_f32(lacc[g]);
      if (lane == 0) red[warp * GP + g] = l;
    }
    __syncthreads();   // also: every reduction of this segment has landed
    if (tid < GP) {
      float l = 0.f;
#pragma unroll
      for (int w = 0; w < 8; ++w) l += red[w * GP + tid];
      a.pm[slot * GP + tid] = mseg[tid];
      a.pl[slot * GP + tid] = l;
    }
    {
      float* dst = a.pw + slot * (int64_t)Sv * kCodebook * GP;
      const int n = Sv * kCodebook * GP;
      for (int f = tid; f < n; f += kScanThreads) {
        const int g = f % GP, c = (f / GP) % kCodebook, s = f / (GP * kCodebook);
        const int combo = s * GP + g;
        unsigned long long h = 0, l = 0;
#pragma unroll
        for (int j = 0; j < C::J; ++j) {
          const int col = C::PASSES == 1 ? j * C::COMBOS + combo : combo;
          h += vhi[c * C::VW + col];
          l += vlo[c * C::VW + col];
        }
        dst[f] = (float)((double)h * (1.0 / 524288.0) + (double)l * (1.0 / 274877906944.0));
      }
    }
  }
}

// ------------------------------------------------------------------------------------------
// 3. Merge: segment histograms -> W_s, contraction with Cv_s, stage sum, rotation back,
//    log-sum-exp merge with the window.  grid (Sv, Hkv, B); 256 threads.
// ------------------------------------------------------------------------------------------
template <int D, int GP>
__global__ void __launch_bounds__(256) merge_kernel(DecodeArgs a) {
  constexpr int E = D / 32;
  constexpr int PARTS = 256 / D;   // threads per output element
  extern __shared__ __align__(16) float sm[];
  float* Ws = sm;                              // [256][GP]
  float* oc = Ws + kCodebook * GP;             // [PARTS][GP][D]
  __shared__ float mstar_s[GP], lstar_s[GP];
  __shared__ int is_last;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int s = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int64_t pair = (int64_t)b * a.Hkv + kvh;
  const int64_t share = *a.share;
  const int64_t p0 = a.pre[pair], p1 = a.pre[pair + 1];
  // scan CTAs first..last covered this pair; CTA c wrote its segment to slot pair + c
  const int64_t first = p1 > p0 ? p0 / share : 1, last = p1 > p0 ? (p1 - 1) / share : 0;

  if (tid < GP) {
    float m = -INFINITY, l = 0.f;
    for (int64_t c = first; c <= last; ++c) m = fmaxf(m, a.pm[(pair + c) * GP + tid]);
    for (int64_t c = first; c <= last; ++c)
      l += ex2_approx(a.pm[(pair + c) * GP + tid] - m) * a.pl[(pair + c) * GP + tid];
    mstar_s[tid] = m;
    lstar_s[tid] = l;
  }
  __syncthreads();
  // W_s[c][g] = sum_slots 2^(m_slot - m*) W_slot[s][c][g]
  for (int f = tid; f < kCodebook * GP; f += 256) {
    const int g = f % GP;
    float acc = 0.f;
    for (int64_t c = first; c <= last; ++c) {
      const float w = ex2_approx(a.pm[(pair + c) * GP + g] - mstar_s[g]);
      acc = fmaf(w, a.pw[((pair + c) * a.Sv + s) * kCodebook * GP + f], acc);
    }
    Ws[f] = acc;
  }
  __syncthreads();
  // o_s[g][e] = sum_c W_s[c][g] Cv_s[c][e]
  {
    const int e = tid % D, part = tid / D;
    const float* Cs = a.Cv + ((size_t)kvh * a.Sv + s) * kCodebook * D;
    float acc[GP];
#pragma unroll
    for (int g = 0; g < GP; ++g) acc[g] = 0.f;
#pragma unroll 4
    for (int c = part; c < kCodebook; c += PARTS) {
      const float cv = __ldg(Cs + (size_t)c * D + e);
#pragma unroll
      for (int g = 0; g < GP; ++g) acc[g] = fmaf(Ws[c * GP + g], cv, acc[g]);
    }
    if constexpr (PARTS > 1) {
#pragma unroll
      for (int g = 0; g < GP; ++g) oc[(part * GP + g) * D + e] = acc[g];
      __syncthreads();
      if (part == 0) {
#pragma unroll
        for (int g = 0; g < GP; ++g) {
          float v = acc[g];
          for (int q = 1; q < PARTS; ++q) v += oc[(q * GP + g) * D + e];
          acc[g] = v;
        }
      }
    }
    if (part == 0) {
#pragma unroll
      for (int g = 0; g < GP; ++g) a.so[((pair * a.Sv + s) * GP + g) * D + e] = acc[g];
    }
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    const unsigned ticket = atomicAdd(&a.cnt[pair], 1u);
    is_last = (ticket == (unsigned)a.Sv - 1u);
  }
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  // sum of the stage contributions (rotated domain, unnormalised)
  for (int f = tid; f < GP * D; f += 256) {
    float v = 0.f;
    for (int q = 0; q < a.Sv; ++q) v += __ldcg(a.so + (pair * a.Sv + q) * GP * D + f);
    oc[f] = v;
  }
  __syncthreads();
  // rotate back one head per warp, merge with the window, write out
  for (int g = warp; g < a.G; g += 8) {
    double v[E];
#pragma unroll
    for (int q = 0; q < E; ++q) v[q] = (double)oc[g * D + q * 32 + lane];
    fwht_warp_f64<D>(v, lane);
    const float mc = mstar_s[g], lc = lstar_s[g];
    const float mw = __ldcg(a.wm + pair * GP + g), lw = __ldcg(a.wl + pair * GP + g);
    const float M = fmaxf(mc, mw);
    const float wc = (mc == -INFINITY) ? 0.f : ex2_approx(mc - M);
    const float ww = (mw == -INFINITY) ? 0.f : ex2_approx(mw - M);
    const float L = wc * lc + ww * lw;
    const int64_t h = (int64_t)kvh * a.G + g;
    float* o = a.out + ((int64_t)b * a.Hq + h) * D;
    const float inv = L > 0.f ? 1.f / L : 0.f;
#pragma unroll
    for (int q = 0; q < E; ++q) {
      const int i = q * 32 + lane;
      const float ow = __ldcg(a.wo + (pair * GP + g) * D + i);
      o[i] = (wc * (float)(v[q] * a.rot) + ww * ow) * inv;
    }
    if (lane == 0 && a.lse) {
      a.lse[(int64_t)b * a.Hq + h] = L > 0.f ? (M + log2f(L)) * kLn2 : -INFINITY;
    }
  }
  if (tid == 0) a.cnt[pair] = 0u;
}

// ------------------------------------------------------------------------------------------
// Launch
// ------------------------------------------------------------------------------------------
static inline void trace(void* const* ev, int i, cudaStream_t st) {
  if (ev && ev[i]) cudaEventRecord(reinterpret_cast<cudaEvent_t>(ev[i]), st);
}

template <int GP, int SKP, int SVP>
static int launch_scan(const DecodeArgs& a, size_t smem, cudaStream_t st) {
  if (ensure_smem_limit(scan_kernel<GP, SKP, SVP>, smem) != cudaSuccess) return ZKV_ERR_CUDA;
  scan_kernel<GP, SKP, SVP><<<a.grid, kScanThreads, smem, st>>>(a);
  ZKV_CHECK_LAUNCH();
  return ZKV_OK;
}

template <int GP, int SKP>
static int launch_scan_v(const DecodeArgs& a, int SVP, size_t smem, cudaStream_t st) {
  switch (SVP) {
    case 2: return launch_scan<GP, SKP, 2>(a, smem, st);
    case 4: return launch_scan<GP, SKP, 4>(a, smem, st);
    default: return launch_scan<GP, SKP, 8>(a, smem, st);
  }
}

template <int GP>
static int launch_scan_kv(const DecodeArgs& a, int SKP, int SVP, size_t smem, cudaStream_t st) {
  switch (SKP) {
    case 2: return launch_scan_v<GP, 2>(a, SVP, smem, st);
    case 4: return launch_scan_v<GP, 4>(a, SVP, smem, st);
    default: return launch_scan_v<GP, 8>(a, SVP, smem, st);
  }
}

template <int D, int GP>
static int launch_decode(DecodeArgs a, const DecodePlan& pl, void* const* ev, cudaStream_t st) {
  // 1. tables, window, prefix sums
  trace(ev, 0, st);
  {
    const size_t lut_smem = sizeof(LutSmem<D>);
    const size_t win_smem = ((size_t)GP * D + 256 * GP + 9 * GP) * sizeof(float);
    const size_t smem = lut_smem > win_smem ? lut_smem : win_smem;
    if (ensure_smem_limit(lut_kernel<D, GP>, smem) != cudaSuccess) return ZKV_ERR_CUDA;
    const int n_hg = (a.B * a.G + kLutH - 1) / kLutH;
    a.n_lut_blocks = (kCodebook / kLutC) * a.Sk * a.Hkv * n_hg;
    const int64_t blocks = (int64_t)a.n_lut_blocks + (int64_t)a.B * a.Hkv;
    if (blocks > 0x7fffffff) return ZKV_ERR_UNSUPPORTED;
    lut_kernel<D, GP><<<(unsigned)blocks, 256, smem, st>>>(a);
    ZKV_CHECK_LAUNCH();
  }
  // 2. scan
  trace(ev, 1, st);
  {
    int rc;
    switch (GP) {
      case 1: rc = launch_scan_kv<1>(a, pl.SKP, pl.SVP, pl.scan_smem, st); break;
      case 2: rc = launch_scan_kv<2>(a, pl.SKP, pl.SVP, pl.scan_smem, st); break;
      case 4: rc = launch_scan_kv<4>(a, pl.SKP, pl.SVP, pl.scan_smem, st); break;
      default: rc = launch_scan_kv<8>(a, pl.SKP, pl.SVP, pl.scan_smem, st); break;
    }
    if (rc != ZKV_OK) return rc;
  }
  // 3. merge
  trace(ev, 2, st);
  {
    const size_t smem = ((size_t)kCodebook * GP + (size_t)GP * D * (256 / D > 1 ? 256 / D : 1)) *
                        sizeof(float);
    if (ensure_smem_limit(merge_kernel<D, GP>, smem) != cudaSuccess) return ZKV_ERR_CUDA;
    const dim3 grid((unsigned)a.Sv, (unsigned)a.Hkv, (unsigned)a.B);
    merge_kernel<D, GP><<<grid, 256, smem, st>>>(a);
    ZKV_CHECK_LAUNCH();
  }
  trace(ev, 3, st);
  return ZKV_OK;
}

template <int D>
static int launch_decode_g(const DecodeArgs& a, const DecodePlan& pl, void* const* ev,
                           cudaStream_t st) {
  switch (pl.GP) {
    case 1: return launch_decode<D, 1>(a, pl, ev, st);
    case 2: return launch_decode<D, 2>(a, pl, ev, st);
    case 4: return launch_decode<D, 4>(a, pl, ev, st);
    default: return launch_decode<D, 8>(a, pl, ev, st);
  }
}

// Shapes only (the workspace size query needs no data pointers).
static int validate_decode_shapes(const zkv_decode_params* p) {
  if (!p) return ZKV_ERR_INVALID_ARG;
  if (p->B < 1 || p->Hq < 1 || p->Hkv < 1 || p->Hq % p->Hkv) return ZKV_ERR_INVALID_ARG;
  if (!supported_d(p->d)) return ZKV_ERR_UNSUPPORTED;
  if (p->Sk < 1 || p->Sk > kMaxStages || p->Sv < 1 || p->Sv > kMaxStages) return ZKV_ERR_UNSUPPORTED;
  if (p->Hq / p->Hkv > 8) return ZKV_ERR_UNSUPPORTED;
  if (p->B > 65535 || p->Hkv > 65535 || (int64_t)p->B * p->Hkv > (1 << 24)) return ZKV_ERR_UNSUPPORTED;
  if (p->Tcap < 0 || p->Wcap < 0 || p->max_comp_len < 0 || p->max_comp_len > p->Tcap)
    return ZKV_ERR_INVALID_ARG;
  if (p->Tcap % 16) return ZKV_ERR_INVALID_ARG;
  return ZKV_OK;
}

static int validate_decode(const zkv_decode_params* p) {
  const int v = validate_decode_shapes(p);
  if (v != ZKV_OK) return v;
  if (!p->q || !p->comp_len || !p->win_len || !p->out) return ZKV_ERR_INVALID_ARG;
  if (!p->k_codes || !p->v_codes || !p->k_codebooks || !p->v_codebooks) return ZKV_ERR_INVALID_ARG;
  if (p->Wcap > 0 && (!p->win_k || !p->win_v)) return ZKV_ERR_INVALID_ARG;
  const uintptr_t al = (uintptr_t)p->q | (uintptr_t)p->k_codes | (uintptr_t)p->v_codes |
                       (uintptr_t)p->k_codebooks | (uintptr_t)p->v_codebooks |
                       (uintptr_t)p->win_k | (uintptr_t)p->win_v;
  if (al & 15) return ZKV_ERR_INVALID_ARG;
  return ZKV_OK;
}

}  // namespace zkv

using namespace zkv;

extern "C" size_t zkv_decode_workspace_size(const zkv_decode_params* p) {
  if (validate_decode_shapes(p) != ZKV_OK) return 0;
  return make_plan(p).total;
}

extern "C" int zkv_rvq_decode_attn(const zkv_decode_params* p, void* workspace,
                                   size_t workspace_bytes, void* stream) {
  const int v = validate_decode(p);
  if (v != ZKV_OK) return v;
  const DecodePlan pl = make_plan(p);
  if (!workspace || workspace_bytes < pl.total || ((uintptr_t)workspace & 255))
    return ZKV_ERR_WORKSPACE;
  if (pl.scan_smem > kSmemMax) return ZKV_ERR_UNSUPPORTED;
  unsigned char* ws = reinterpret_cast<unsigned char*>(workspace);
  DecodeArgs a;
  a.B = p->B; a.Hq = p->Hq; a.Hkv = p->Hkv; a.G = pl.G; a.d = p->d; a.Sk = p->Sk; a.Sv = p->Sv;
  a.Rk = pl.Rk; a.grid = pl.grid; a.n_lut_blocks = 0;
  a.Tcap = p->Tcap; a.Wcap = p->Wcap; a.max_comp = p->max_comp_len;
  const float scale = p->softmax_scale > 0.f ? p->softmax_scale : (float)(1.0 / std::sqrt((double)p->d));
  a.scale_log2 = scale * kLog2e;
  a.rot = 1.0 / std::sqrt((double)p->d);
  a.q = reinterpret_cast<const __half*>(p->q);
  a.k_codes = p->k_codes; a.v_codes = p->v_codes; a.comp_len = p->comp_len;
  a.Ck = p->k_codebooks; a.Cv = p->v_codebooks;
  a.win_k = reinterpret_cast<const __half*>(p->win_k);
  a.win_v = reinterpret_cast<const __half*>(p->win_v);
  a.win_len = p->win_len; a.out = p->out; a.lse = p->lse; a.err = p->error_flag;
  a.lut = reinterpret_cast<float*>(ws + pl.off_lut);
  a.pre = reinterpret_cast<int64_t*>(ws + pl.off_pre);
  a.share = reinterpret_cast<int64_t*>(ws + pl.off_share);
  a.pm = reinterpret_cast<float*>(ws + pl.off_pm);
  a.pl = reinterpret_cast<float*>(ws + pl.off_pl);
  a.pw = reinterpret_cast<float*>(ws + pl.off_pw);
  a.wm = reinterpret_cast<float*>(ws + pl.off_wm);
  a.wl = reinterpret_cast<float*>(ws + pl.off_wl);
  a.wo = reinterpret_cast<float*>(ws + pl.off_wo);
  a.so = reinterpret_cast<float*>(ws + pl.off_so);
  a.cnt = reinterpret_cast<unsigned*>(ws + pl.off_cnt);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  switch (p->d) {
    case 64: return launch_decode_g<64>(a, pl, p->trace_events, st);
    case 128: return launch_decode_g<128>(a, pl, p->trace_events, st);
    default: return launch_decode_g<256>(a, pl, p->trace_events, st);
  }
}
