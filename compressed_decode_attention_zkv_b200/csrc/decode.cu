// Compressed decode attention (sm_100a).
//
// Passages: VQKV (gist.science summary of arXiv 2603.16435), section 2.3 "Decoding Stage":
// codes are read directly and keys/values are reconstructed on demand inside the attention
// computation; "Local Sliding Window": recent tokens stay uncompressed.  VeloxQuant-MLX 0.5.1,
// "VecInfer": the Walsh-Hadamard rotation is absorbed into the query (q_tilde . k_tilde =
// q . k).  Differential-KV README, "Decode & Prefill Innovations": flash-style fp32
// log-sum-exp combine of the compressed part with the dense recency window.
//
// Three kernels per call (programmatic dependent launches):
//   1. lut_kernel    q_tilde = H q / sqrt(d) (float32 transform), per stage
//                    LUT_s[c] = (scale * log2 e) * q_tilde . Ck_s[c] -> workspace; one block
//                    computes the prefix sums of the compressed lengths that partition the token
//                    space among scan CTAs; one block per (sequence, kv head) and window part
//                    (64-token parts in a decode call, the whole window in the serving step)
//                    takes the dense attention over its fp16 window rows (partial maximum, sum
//                    and output).
//   2. scan          one CTA per SM walks a contiguous range of the concatenated compressed
//                    tokens of all (sequence, kv head) pairs.  Per pair segment it takes
//                    score_t = sum_s LUT_s[zk_{t,s}] (base-2 logits) against a reference maximum
//                    m, and accumulates p_t = 2^(score_t - m) into per-stage codeword weight
//                    histograms W_s[c] = sum over tokens with zv_{t,s} = c of p_t:
//                    sum_t p_t sum_s Cv_s[zv_{t,s}] = sum_s sum_c W_s[c] Cv_s[c], the value
//                    reconstruction regrouped by codeword.  scan2_kernel (scan_rvq.cuh) serves
//                    1, 2 or 4 stages; scan_kernel below the other stage counts.
//   3. combine_kernel (combine.cuh)  per (pair, value stage, codeword chunk): merges the segment
//                    histograms by their maxima and contracts W_s with its Cv_s codewords; the
//                    block that completes a pair sums the stage outputs, rotates back, and merges
//                    with the window parts by log-sum-exp.
//
// Shared-memory design of scan_kernel (shared memory bandwidth, not HBM, bounds this kernel):
//  * key tables are replicated per lane group so that the 8 (or 16, 32) lanes of a 128-bit
//    (64-, 32-bit) gather always hit distinct banks;
//  * value histograms use the native shared-memory integer reduction: p is converted to
//    38-bit fixed point (exact to 2^-39 absolute per token, p <= 1 relative to the segment's
//    reference) split into two 19-bit halves added with red.shared.add.u32; lanes are mapped to
//    (token slot, stage, head) so one instruction touches 32 distinct banks.  Column sums stay
//    below 2^32 because a segment holds at most 8176 tokens per column.
#include "zkv_internal.cuh"
#include "lengths.cuh"

#include <algorithm>
#include <utility>
#include <type_traits>
#include <cfloat>
#include <cmath>

namespace zkv {

constexpr int kScanSub = 512;       // tokens per scan sub-chunk (1 per thread)
constexpr int kScanThreads = 512;
static_assert(kScanSub == kScanThreads && kScanThreads % 32 == 0, "one token per thread and sub-chunk; 32 per warp");
constexpr int kColCap = 8176;       // tokens per histogram column per segment (sum < 2^32)
constexpr float kHeadroom = 10.f;   // log2 units added to the running maximum on growth
// Setup cost of one scan segment (table fill, histogram zeroing, final fold: about 11K cycles)
// in tokens of the scan loop (about 5.7 cycles per token): the token space is partitioned so
// that tokens + kSegCost x segments is equal across scan CTAs.
constexpr int64_t kSegCost = 1900;
constexpr size_t kSmemMax = 227 * 1024;

// Token-per-thread scan (scan_rvq.cuh).
constexpr int kS2Threads = 512;
constexpr int kS2Fix = 20;                        // value weights as integers of p * 2^20
constexpr float kS2Headroom = 3.f;                // log2 units added to a new reference
constexpr uint32_t kS2KeyRegion = 1u << 16;       // absolute shared address of the key tables
constexpr uint32_t kS2ValRegion = 2u << 16;       // ... of the value histograms
constexpr uint32_t kS2ExvRegion = 3u << 16;       // ... of the listed tokens' value words
constexpr size_t kS2Smem = (size_t(3) << 16) + 32768;   // dynamic shared memory requested
// Set-up cost of one scan segment (table fill, the reference from the first sub-chunk, final
// fold and write: about 8K cycles measured) in tokens of the loop (about 1.3 cycles per token
// and SM).
constexpr int64_t kS2SegCost = 6000;
// tokens of one window part in the decode's table kernel (its K + V tile is 32 KB)
inline int win_tile_part(int d) { return 8192 / d; }


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
  bool scan2;   // the token-per-thread scan (scan_rvq.cuh) serves this shape
  int64_t seg_cost;
  int64_t cap, slots;
  size_t scan_smem;
  size_t off_lut, off_pre, off_bounds, off_ctap, off_vs, off_pfirst, off_plast, off_pm, off_pl, off_pw,
      off_wm, off_wl, off_wo, off_so, off_cnt, total;
  int qc, wparts, wtok;
};

static size_t scan_smem_bytes(int Rk, int Sk, int Sv, int GP, const VMap& v) {
  size_t b = (size_t)Rk * Sk * kCodebook * GP * 4;            // key tables
  b += (size_t)Sv * kCodebook * GP * 4;                         // fp32 master histograms
  b += 2ull * kCodebook * v.VW * 4;                            // value histograms (hi, lo)
  b += 2ull * 2 * v.J * GP * (v.rounds + 4) * 4;                // p staging (2 buffers x hi, lo)
  b += 2ull * v.J * (v.rounds + 4) * v.codew * 4;               // value-code staging (2 buffers)
  b += (size_t)(2 * (kScanThreads / 32) + kScanThreads / 32) * GP * 4 + 16;   // maxima (2), sums
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
  while (Rk > 1 && scan_smem_bytes(Rk, p->Sk, p->Sv, pl.GP, v) > kSmemMax) Rk >>= 1;
  pl.Rk = Rk;
  const int64_t pairs = (int64_t)p->B * p->Hkv;
  const int64_t bound = pairs * p->max_comp_len;
  const int sms = sm_count();
  auto pow124 = [](int s) { return s == 1 || s == 2 || s == 4; };
  pl.scan2 = pow124(p->Sk) && pow124(p->Sv);
  if (pl.scan2) {
    // no column capacity to respect (the integer words are folded on a schedule)
    pl.scan_smem = kS2Smem;
    pl.seg_cost = kS2SegCost;
    pl.cap = 0;
    pl.grid = (int)std::max<int64_t>(1, std::min<int64_t>(sms, (bound + 1023) / 1024));
  } else {
    pl.scan_smem = scan_smem_bytes(Rk, p->Sk, p->Sv, pl.GP, v);
    pl.seg_cost = kSegCost;
    pl.cap = (int64_t)kColCap * v.J;
    // every CTA's virtual share (tokens + kSegCost per pair) stays below the column capacity
    int64_t g1 = (bound + kSegCost * pairs + pl.cap - 1) / pl.cap;
    int64_t g2 = std::min<int64_t>(sms, (bound + 1023) / 1024);
    int64_t grid = std::max<int64_t>(1, std::max(g1, g2));
    if (grid > sms) grid = (grid + sms - 1) / sms * sms;
    pl.grid = (int)grid;
  }
  const int64_t grid = pl.grid;
  pl.slots = pairs + grid;
  const size_t f = sizeof(float);
  size_t o = 0;
  pl.off_lut = o;   o = align256(o + (size_t)pairs * p->Sk * kCodebook * pl.GP * f);
  pl.off_pre = o;   o = align256(o + (size_t)(pairs + 1) * sizeof(int64_t));
  pl.off_bounds = o; o = align256(o + (size_t)(grid + 1) * sizeof(int64_t));
  pl.off_ctap = o;  o = align256(o + (size_t)(grid + 1) * sizeof(int32_t));
  pl.off_vs = o;    o = align256(o + (size_t)(pairs + 1) * sizeof(int64_t));
  pl.off_pfirst = o; o = align256(o + (size_t)pairs * sizeof(int32_t));
  pl.off_plast = o; o = align256(o + (size_t)pairs * sizeof(int32_t));
  pl.off_pm = o;    o = align256(o + (size_t)pl.slots * pl.GP * f);
  pl.off_pl = o;    o = align256(o + (size_t)pl.slots * pl.GP * f);
  pl.off_pw = o;    o = align256(o + (size_t)pl.slots * p->Sv * kCodebook * pl.GP * f);
  // the window in parts of one tile each, one table-kernel block per (pair, part)
  pl.wtok = win_tile_part(p->d);
  pl.wparts = (int)std::max<int64_t>(1, (p->Wcap + pl.wtok - 1) / pl.wtok);
  pl.off_wm = o;    o = align256(o + (size_t)pairs * pl.wparts * pl.GP * f);
  pl.off_wl = o;    o = align256(o + (size_t)pairs * pl.wparts * pl.GP * f);
  pl.off_wo = o;    o = align256(o + (size_t)pairs * pl.wparts * pl.GP * p->d * f);
  // combine blocks: (pair, value stage, chunk of 256 / qc codewords); a chunk's codewords take
  // at most 32 KB of shared memory, and small problems take more chunks (up to 16 or the
  // 32 KB minimum) so that the grid covers the SMs
  {
    int qc = std::max(2, p->d / 32);
    while (qc < 16 && pairs * p->Sv * qc < sms) qc *= 2;
    pl.qc = qc;
  }
  pl.off_so = o;    o = align256(o + (size_t)pairs * p->Sv * pl.qc * pl.GP * p->d * f);
  pl.off_cnt = o;   o = align256(o + (size_t)pairs * sizeof(int32_t));
  pl.total = o;
  return pl;
}

struct DecodeArgs {
  int B, Hq, Hkv, G, GP, d, Sk, Sv, Rk, grid, n_lut_blocks;
  int lut_cpt;        // codewords per table-kernel thread (1 or lut_cpt<D>())
  int64_t seg_cost;   // set-up cost of one scan segment, in tokens (partition weight)
  int qc;             // codeword chunks per value stage in the combine kernel
  // Serving step: the partition uses the lengths after this step's append (predicted from
  // the pre-step state with the append's rule), and scan block 0 stores them.  Null otherwise.
  int32_t* upd_win_len;
  int32_t* upd_win_head;
  int32_t* upd_comp_len;
  // Serving step: the new tokens [B][Hkv][d].  The window attention runs before this step's
  // append and attends to the window that append produces (the new token in the slot it
  // takes).  Null otherwise.
  const __half* new_k;
  const __half* new_v;
  int64_t Tcap, Wcap, max_comp;
  float scale_log2;   // softmax_scale * log2(e)
  double rot;         // 1 / sqrt(d)
  const __half* q;
  const uint8_t* k_codes;   // [B][Hkv][Tcap][Sk], or a page pool [n_pages][Hkv][P][Sk]
  const uint8_t* v_codes;
  const int32_t* bt;        // paged layout: block table [B][max_pages], else null
  int64_t max_pages, n_pages;
  int pshift;               // log2 P (tokens per page)
  const int32_t* comp_len;
  const float* Ck;
  const float* k_smooth;   // [Hkv][d] key smoothing factors (the query is scaled by them) or null
  const float* Cv;
  const __half* win_k;
  const __half* win_v;
  const int32_t* win_len;
  float* out;
  float* lse;
  int32_t* err;
  float* lut;        // [B][Hkv][Sk][256][GP] (heads g >= G unwritten)
  int64_t* pre;      // [B*Hkv + 1] exclusive prefix sums of compressed lengths
  int64_t* bounds;   // [grid + 1] token range of each scan CTA
  int32_t* ctap;     // [grid + 1] the pair holding each CTA's first cut (its first segment's pair
                     // or an earlier one with nothing left at the cut)
  int64_t* vs;       // [B*Hkv + 1] virtual start of each pair (tokens + kSegCost per nonempty pair)
  int32_t* pfirst;   // [B*Hkv] first scan CTA covering the pair (> plast when it has no tokens)
  int32_t* plast;    // [B*Hkv] last scan CTA covering the pair
  float* pm;         // [slots][GP] segment maxima
  float* pl;         // [slots][GP] segment sums of p
  float* pw;         // [slots][Sv][256][GP] segment histograms
  int wparts, wtok;  // window parts per pair, tokens per part (the part is one tile)
  float* wm;         // [B*Hkv][wparts][GP]
  float* wl;         // [B*Hkv][wparts][GP]
  float* wo;         // [B*Hkv][wparts][GP][d]
  float* so;         // [B*Hkv][Sv][qc][GP][d] partial stage outputs
  int32_t* cnt;      // [B*Hkv] finished combine blocks of each pair (zeroed by the table kernel)
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
// 1. Query rotation + lookup tables; length prefix sums (the partition block); the dense
//    window attention (window_item), one block per pair.
// ------------------------------------------------------------------------------------------
constexpr int kLutH = 16;     // attached query heads per table block (b * G + g)
// codewords per table block: 64 per group of 4 heads' threads, and each thread takes lut_cpt of
// them (two up to d = 128: six 16-byte shared loads per 32 FMAs; one at d = 256, where a
// 128-codeword slice would leave one block per SM)
template <int D>
constexpr int lut_cpt() { return D >= 256 ? 1 : 2; }
template <int D>
constexpr int lut_c() { return 64 * lut_cpt<D>(); }

template <int D>
struct LutSmem {
  float qT[D][kLutH + 4];     // rotated queries, k-major
  float cb[lut_c<D>() * D];   // codebook slice, row-major; 16-byte piece q of codeword c at q ^ (c & 7)
};

// Ask the memory system to stage [p, p + bytes) in L2 (no data returned to the SM).  p and
// bytes are rounded outward to 16-byte granules inside [lo, hi), the caller's allocation.
__device__ __forceinline__ void prefetch_l2(const uint8_t* lo, const uint8_t* hi, const uint8_t* p,
                                            int64_t bytes) {
  uintptr_t a = reinterpret_cast<uintptr_t>(p) & ~uintptr_t(15);
  uintptr_t e = (reinterpret_cast<uintptr_t>(p) + bytes + 15) & ~uintptr_t(15);
  if (a < reinterpret_cast<uintptr_t>(lo)) a = reinterpret_cast<uintptr_t>(lo);
  if (e > reinterpret_cast<uintptr_t>(hi)) e = reinterpret_cast<uintptr_t>(hi);
  while (a < e) {
    const uint32_t n = (uint32_t)((e - a) < 65536 ? (e - a) : 65536);
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(a), "r"(n) : "memory");
    a += n;
  }
}

// Dense attention of the GP heads of one (sequence, kv head) over its fp16 window (base-2
// logits, online maximum over tiles).  Each tile's K and V rows (WT tokens) are copied to
// shared memory with cp.async in one round; warps then take tokens and lanes split the head
// dimension.  256 threads.
template <int D>
constexpr int win_tile() { return 16384 / D; }   // tokens per tile: K + V tiles = 64 KB
template <int D>
constexpr int win_tile_part_c() { return 8192 / D; }

// the warps' partial outputs [8][GP][D] reuse the tiles when they fit there
template <int D, int GP, int WT>
constexpr bool win_part_in_tiles() { return (size_t)8 * GP * D * 4 <= (size_t)2 * WT * D * 2; }

template <int D, int GP, int WT = win_tile<D>()>
constexpr size_t window_smem_bytes() {
  return (size_t)2 * WT * D * sizeof(__half) + (size_t)WT * GP * 4 + (size_t)8 * GP * 4 +
         (win_part_in_tiles<D, GP, WT>() ? 0 : (size_t)8 * GP * D * 4);
}

// Part wpart of the window: rows [wpart wtok, (wpart + 1) wtok) of its wl rows; the partial
// (maximum, sum, unnormalised output) goes to slot wpart of the pair's window partials.
template <int D, int GP, int WT = win_tile<D>()>
__device__ void window_item(const DecodeArgs& a, int b, int kvh, int wpart, unsigned char* smem) {
  constexpr int PL = D / 32;        // head dims per lane
  __half* kt = reinterpret_cast<__half*>(smem);                     // [WT][D]
  __half* vt = kt + WT * D;                                         // [WT][D]
  float* sc = reinterpret_cast<float*>(vt + WT * D);                // [WT][GP] scores, then p
  float* red = sc + WT * GP;                                        // [8][GP]
  float* part = win_part_in_tiles<D, GP, WT>() ? reinterpret_cast<float*>(smem)
                                               : red + 8 * GP;      // [8][GP][D], after the tiles
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t pair = (int64_t)b * a.Hkv + kvh;
  // the window's length and, in the serving step, the slot this step's append gives the new
  // token (by the append's rule, from the pre-step state: a free slot, else the oldest one
  // while the prefix has room); the window is a set of rows, so their order does not matter
  int64_t wl, sub = -1;
  if (a.new_k) {
    const int64_t w0 = a.upd_win_len[b], hd = a.upd_win_head[b], c = a.upd_comp_len[b];
    if (w0 >= 0 && w0 < a.Wcap) {
      sub = w0;
      wl = w0 + 1;
    } else if (w0 == a.Wcap && hd >= 0 && hd < a.Wcap) {
      wl = w0;
      if (c >= 0 && c < a.Tcap) sub = hd;
    } else {
      wl = clamp_win_len(a, b);
    }
  } else {
    wl = clamp_win_len(a, b);
  }
  // this part's rows
  const int64_t t0 = (int64_t)wpart * a.wtok;
  const int64_t t1 = wl < t0 + a.wtok ? wl : t0 + a.wtok;
  const __half* Kb = a.win_k + pair * a.Wcap * D;
  const __half* Vb = a.win_v + pair * a.Wcap * D;
  auto stage = [&](int64_t base) {   // rows [base, base + n) as 16-byte pieces
    const int n = (int)(t1 - base < WT ? t1 - base : WT);
    for (int f = tid; f < n * D / 8; f += 256) {
      if (base + f / (D / 8) == sub) continue;
      cp_async16(kt + f * 8, Kb + base * D + f * 8);
      cp_async16(vt + f * 8, Vb + base * D + f * 8);
    }
    if (sub >= base && sub < base + n) {   // the new token (plain loads: no alignment assumed)
      const int64_t ro = (sub - base) * D;
      for (int i = tid; i < D; i += 256) {
        kt[ro + i] = a.new_k[pair * D + i];
        vt[ro + i] = a.new_v[pair * D + i];
      }
    }
  };
  if (t1 > t0) stage(t0);   // in flight while the query is loaded
  float qf[GP][PL];
#pragma unroll
  for (int g = 0; g < GP; ++g)
#pragma unroll
    for (int e = 0; e < PL; ++e)
      qf[g][e] = g < a.G ? __half2float(a.q[((int64_t)b * a.Hq + (int64_t)kvh * a.G + g) * D +
                                            lane * PL + e]) * a.scale_log2
                         : 0.f;
  float m_run[GP], l_run[GP], acc[GP][PL];
#pragma unroll
  for (int g = 0; g < GP; ++g) {
    m_run[g] = -INFINITY;
    l_run[g] = 0.f;
#pragma unroll
    for (int e = 0; e < PL; ++e) acc[g][e] = 0.f;
  }
  for (int64_t base = t0; base < t1; base += WT) {
    const int n = (int)(t1 - base < WT ? t1 - base : WT);
    if (base > t0) stage(base);
    cp_async_wait_all();
    __syncthreads();
    // scores
#pragma unroll 2
    for (int tt = warp; tt < n; tt += 8) {
      const __half* kr = kt + tt * D + lane * PL;
      float kf[PL];
#pragma unroll
      for (int e = 0; e < PL; e += 2) {
        const float2 v = __half22float2(*reinterpret_cast<const __half2*>(kr + e));
        kf[e] = v.x;
        kf[e + 1] = v.y;
      }
      float d[GP];
#pragma unroll
      for (int g = 0; g < GP; ++g) {
        d[g] = 0.f;
#pragma unroll
        for (int e = 0; e < PL; ++e) d[g] = fmaf(qf[g][e], kf[e], d[g]);
      }
      int hd = 0;
      const float tot = TransposeSum<GP, GP, 16>::run(d, lane, hd);
      if ((lane & (32 / GP - 1)) == 0) sc[tt * GP + hd] = tot;
    }
    __syncthreads();
    // tile maximum, probabilities
    float mt[GP];
#pragma unroll
    for (int g = 0; g < GP; ++g) {
      float v = -INFINITY;
      for (int t2 = tid; t2 < n; t2 += 256) v = fmaxf(v, sc[t2 * GP + g]);
      const float m = warp_max_f32(v);
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
      m_run[g] = mn;
      mt[g] = mn;
      l_run[g] *= alpha;
#pragma unroll
      for (int e = 0; e < PL; ++e) acc[g][e] *= alpha;
    }
    for (int t2 = tid; t2 < n; t2 += 256) {
#pragma unroll
      for (int g = 0; g < GP; ++g) {
        const float pv = ex2_approx(sc[t2 * GP + g] - mt[g]);
        sc[t2 * GP + g] = pv;
        l_run[g] += pv;
      }
    }
    __syncthreads();
    // values
#pragma unroll 2
    for (int tt = warp; tt < n; tt += 8) {
      const __half* vr = vt + tt * D + lane * PL;
      float vf[PL];
#pragma unroll
      for (int e = 0; e < PL; e += 2) {
        const float2 v = __half22float2(*reinterpret_cast<const __half2*>(vr + e));
        vf[e] = v.x;
        vf[e + 1] = v.y;
      }
#pragma unroll
      for (int g = 0; g < GP; ++g) {
        const float pv = sc[tt * GP + g];
#pragma unroll
        for (int e = 0; e < PL; ++e) acc[g][e] = fmaf(pv, vf[e], acc[g][e]);
      }
    }
    __syncthreads();   // the tiles and sc are rewritten by the next tile (or by part below)
  }
#pragma unroll
  for (int g = 0; g < GP; ++g) {
#pragma unroll
    for (int e = 0; e < PL; ++e) part[(warp * GP + g) * D + lane * PL + e] = acc[g][e];
    const float l = warp_sum_f32(l_run[g]);
    if (lane == 0) red[warp * GP + g] = l;
  }
  __syncthreads();
  if (tid < GP) {
    float l = 0.f;
    for (int w = 0; w < 8; ++w) l += red[w * GP + tid];
    float mr = 0.f;
#pragma unroll
    for (int g = 0; g < GP; ++g)
      if (g == tid) mr = m_run[g];
    a.wm[(pair * a.wparts + wpart) * GP + tid] = mr;
    a.wl[(pair * a.wparts + wpart) * GP + tid] = l;
  }
  for (int f = tid; f < GP * D; f += 256) {
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) v += part[w * GP * D + f];
    a.wo[(pair * a.wparts + wpart) * GP * D + f] = v;
  }
}

// floor(x * m / d) and ceil(x * m / d) for x, m >= 0 and d > 0, exact.  wide: the product may
// exceed 2^63 (128-bit arithmetic, slow); otherwise 64-bit.
__device__ __forceinline__ int64_t floor_muldiv(int64_t x, int64_t m, int64_t d, bool wide) {
  if (wide) return (int64_t)(((unsigned __int128)(uint64_t)x * (uint64_t)m) / (uint64_t)d);
  return (int64_t)(((uint64_t)x * (uint64_t)m) / (uint64_t)d);
}
__device__ __forceinline__ int64_t ceil_muldiv(int64_t x, int64_t m, int64_t d, bool wide) {
  if (wide)
    return (int64_t)(((unsigned __int128)(uint64_t)x * (uint64_t)m + (uint64_t)(d - 1)) / (uint64_t)d);
  return (int64_t)(((uint64_t)x * (uint64_t)m + (uint64_t)(d - 1)) / (uint64_t)d);
}

// The partition of the compressed token space among the scan CTAs (one block):
// pre = prefix sums of the clamped compressed lengths, vs = prefix sums of the virtual lengths
// len + kSegCost (nonempty pairs).  Scan CTA c covers virtual positions [v_c, v_(c+1)) with
// v_c = floor(V c / grid); a cut inside a pair's kSegCost gap moves to the pair's first token.
// Each pair's thread places the cuts that fall in its virtual range directly (the first cut at
// or after position x is c = ceil(x grid / V)), so no search is needed.
__device__ void partition_block(const DecodeArgs& a) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // exclusive prefix sums of the clamped compressed lengths (pre) and of the virtual lengths
  // len + a.seg_cost * (len > 0) (vs), 256 pairs per round
  __shared__ int64_t warp_tot[2][8];
  __shared__ int64_t carry_s[2];
  const int npairs = a.B * a.Hkv;
  if (tid == 0) {
    carry_s[0] = 0;
    carry_s[1] = 0;
    a.pre[0] = 0;
    a.vs[0] = 0;
  }
  __syncthreads();
  for (int base = 0; base < npairs; base += 256) {
    const int pr = base + tid;
    int64_t c = 0;
    if (pr < npairs) {
      const int b = pr / a.Hkv;
      c = a.comp_len[b];
      if (a.upd_comp_len) {   // this step's append evicts a token onto the prefix
        const int64_t wl = a.upd_win_len[b], hd = a.upd_win_head[b];
        if (wl == a.Wcap && hd >= 0 && hd < a.Wcap && c >= 0 && c < a.Tcap) c += 1;
      }
      if (c < 0 || c > a.Tcap) {
        set_error(a.err, ZKV_DEVERR_COMP_LEN);
        c = c < 0 ? 0 : a.Tcap;
      }
      c = c < a.max_comp ? c : a.max_comp;
    }
    int64_t x = c, y = c > 0 ? c + a.seg_cost : 0;   // inclusive warp scans
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int64_t ux = __shfl_up_sync(0xffffffffu, x, o);
      const int64_t uy = __shfl_up_sync(0xffffffffu, y, o);
      if (lane >= o) {
        x += ux;
        y += uy;
      }
    }
    if (lane == 31) {
      warp_tot[0][warp] = x;
      warp_tot[1][warp] = y;
    }
    __syncthreads();
    int64_t ox = carry_s[0], oy = carry_s[1];
    for (int w = 0; w < warp; ++w) {
      ox += warp_tot[0][w];
      oy += warp_tot[1][w];
    }
    if (pr < npairs) {
      a.pre[pr + 1] = ox + x;
      a.vs[pr + 1] = oy + y;
    }
    __syncthreads();
    if (tid == 255) {
      carry_s[0] = ox + x;
      carry_s[1] = oy + y;
    }
    __syncthreads();
  }
  const int64_t V = carry_s[1], tot = carry_s[0];
  const int grid = a.grid;
  // V <= pairs * (Tcap + a.seg_cost) < 2^53 here; products with grid stay below 2^62 unless the
  // grid is very large
  const bool wide = (double)(V + a.seg_cost + 1) * (double)grid >= 4.0e18;
  if (V == 0) {   // no compressed token at all
    for (int c = tid; c <= grid; c += 256) {
      a.bounds[c] = 0;
      a.ctap[c] = 0;
    }
    for (int k = tid; k < npairs; k += 256) {
      a.pfirst[k] = 1;
      a.plast[k] = 0;
    }
    return;
  }
  if (tid == 0) {
    a.bounds[0] = 0;
    a.bounds[grid] = tot;
    a.ctap[0] = 0;
    a.ctap[grid] = npairs;
  }
  for (int k = tid; k < npairs; k += 256) {
    const int64_t v0 = a.vs[k], v1 = a.vs[k + 1], p0 = a.pre[k], len = a.pre[k + 1] - p0;
    int f = 1, t = 0;   // first / last scan CTA holding the pair's tokens (f > t: none)
    if (len > 0) {
      const int64_t clo = ceil_muldiv(v0, grid, V, wide);   // cuts c in [clo, chi] lie in [v0, v1)
      const int64_t chi = ceil_muldiv(v1, grid, V, wide) - 1;
      for (int64_t c = clo > 1 ? clo : 1; c <= chi && c < grid; ++c) {
        const int64_t off = floor_muldiv(V, c, grid, wide) - v0;
        a.bounds[c] = off < a.seg_cost ? p0 : p0 + (off - a.seg_cost < len ? off - a.seg_cost : len);
        a.ctap[c] = k;
      }
      // the CTA holding the first token: the last cut at or before v0 + a.seg_cost (its bound is
      // p0); the one holding the last token: the last cut before v1
      const int64_t cf = ceil_muldiv(v0 + a.seg_cost + 1, grid, V, wide) - 1;
      f = (int)(cf < chi ? cf : chi);
      t = (int)chi;
    }
    a.pfirst[k] = f;
    a.plast[k] = t;
  }
}

// Table blocks: block = (slice of lut_c codewords, key stage, group of 16 attached query heads,
// kv head); thread (codewords cc + 64 u, head quad hq) forms 4 lut_cpt dot products.  Block
// n_lut_blocks is the partition block; the blocks after it are the window blocks (one per pair
// and window part).
template <int D, int GP>
__global__ void __launch_bounds__(256, GP >= 8 ? 2 : 3) lut_kernel(DecodeArgs a) {
  constexpr int E = D / 32;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  pdl_trigger();   // the next kernel waits for this one before reading the tables
  if ((int)blockIdx.x == a.n_lut_blocks) {
    for (int k = threadIdx.x; k < a.B * a.Hkv; k += blockDim.x) a.cnt[k] = 0;   // combine counters
    partition_block(a);
    return;
  }
  if ((int)blockIdx.x > a.n_lut_blocks) {
    // dense attention over the fp16 window of one (sequence, kv head): it reads only the call's
    // inputs (in the serving step it substitutes the new token for the slot the append gives
    // it), so it runs here, beside the tables
    const int w = (int)blockIdx.x - a.n_lut_blocks - 1;   // (pair, part), part fastest
    const int pair = w / a.wparts;
    if (a.wparts == 1)   // the whole window in one block (64 KB tiles)
      window_item<D, GP>(a, pair / a.Hkv, pair % a.Hkv, 0, smem_raw);
    else                 // one tile-sized part per block
      window_item<D, GP, win_tile_part_c<D>()>(a, pair / a.Hkv, pair % a.Hkv, w % a.wparts, smem_raw);
    return;
  }
  if ((int)blockIdx.x < a.Hkv * a.Sv && tid == 0) {
    // the merge kernel reads every value codebook; stream them into L2 meanwhile
    const uint8_t* cv0 = reinterpret_cast<const uint8_t*>(a.Cv);
    const int64_t bytes = (int64_t)kCodebook * D * sizeof(float);
    const uint8_t* p = cv0 + (int64_t)blockIdx.x * bytes;
    prefetch_l2(p, p + bytes, p, bytes);
  }
  LutSmem<D>& sm = *reinterpret_cast<LutSmem<D>*>(smem_raw);
  const int n_hg = (a.B * a.G + kLutH - 1) / kLutH;
  int rest = blockIdx.x;
  constexpr int CPT = lut_cpt<D>();
  const int cpt = a.lut_cpt, LC = 64 * cpt;
  const int cblk = rest % (kCodebook / LC);
  rest /= kCodebook / LC;
  const int s = rest % a.Sk;
  rest /= a.Sk;
  const int hg = rest % n_hg;
  const int kvh = rest / n_hg;
  const int c0 = cblk * LC;
  // codebook slice C[kvh][s][c0 .. c0 + LC)[:] -> shared memory, in flight during the rotation
  {
    const float* C = a.Ck + (((size_t)kvh * a.Sk + s) * kCodebook + c0) * D;
    for (int f = tid; f < LC * D / 4; f += 256) {
      const int c = f / (D / 4), qq = f % (D / 4);
      cp_async16(sm.cb + c * D + 4 * (qq ^ (c & 7)), C + (size_t)c * D + 4 * qq);
    }
    cp_async_commit();
  }
  // rotated queries of the attached heads j = b*G + g (float32 transform): this warp's rows
  // are loaded first (independent loads), then transformed
  {
    constexpr int NR = kLutH / 8;
    float v[NR][E];
#pragma unroll
    for (int k = 0; k < NR; ++k) {
      const int j = hg * kLutH + warp + 8 * k;
      if (j < a.B * a.G) {
        const int b = j / a.G, g = j % a.G;
        const __half* qr = a.q + ((int64_t)b * a.Hq + (int64_t)kvh * a.G + g) * D + lane;
#pragma unroll
        for (int q = 0; q < E; ++q) v[k][q] = __half2float(qr[q * 32]);
        if (a.k_smooth) {   // the query absorbs the keys' smoothing: lambda * q
          const float* l = a.k_smooth + (int64_t)kvh * D + lane;
#pragma unroll
          for (int q = 0; q < E; ++q) v[k][q] *= l[q * 32];
        }
      } else {
#pragma unroll
        for (int q = 0; q < E; ++q) v[k][q] = 0.f;
      }
    }
    const float rs = (float)a.rot;
#pragma unroll
    for (int k = 0; k < NR; ++k) {
      fwht_warp_f32<D>(v[k], lane);
#pragma unroll
      for (int q = 0; q < E; ++q) sm.qT[q * 32 + lane][warp + 8 * k] = v[k][q] * rs;
    }
  }
  cp_async_wait_all();
  __syncthreads();
  // thread (codewords cc + 64 u for u < CPT, heads 4 hq .. 4 hq + 3): each codeword is read as
  // 16-byte pieces (conflict-free thanks to the swizzle; cc + 64 u has the swizzle of cc), the
  // query columns are broadcasts shared by the thread's codewords; every dot product is
  // accumulated in the same order whatever CPT is
  const int cc = tid & 63, hq = tid / 64;
  const int sw = cc & 7;
  auto dots = [&](auto nu_c) {   // nu codewords per thread (a compile-time count)
    constexpr int NU = decltype(nu_c)::value;
    float acc[NU][4];
#pragma unroll
    for (int u = 0; u < NU; ++u)
#pragma unroll
      for (int k = 0; k < 4; ++k) acc[u][k] = 0.f;
#pragma unroll 4
    for (int qq = 0; qq < D / 4; ++qq) {
      float cv[NU][4];
#pragma unroll
      for (int u = 0; u < NU; ++u) {
        const float4 c4 = *reinterpret_cast<const float4*>(sm.cb + (cc + 64 * u) * D + 4 * (qq ^ sw));
        cv[u][0] = c4.x; cv[u][1] = c4.y; cv[u][2] = c4.z; cv[u][3] = c4.w;
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float4 q4 = *reinterpret_cast<const float4*>(&sm.qT[4 * qq + e][hq * 4]);
#pragma unroll
        for (int u = 0; u < NU; ++u) {
          acc[u][0] = fmaf(q4.x, cv[u][e], acc[u][0]);
          acc[u][1] = fmaf(q4.y, cv[u][e], acc[u][1]);
          acc[u][2] = fmaf(q4.z, cv[u][e], acc[u][2]);
          acc[u][3] = fmaf(q4.w, cv[u][e], acc[u][3]);
        }
      }
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int j = hg * kLutH + hq * 4 + k;
      if (j < a.B * a.G) {
        const int b = j / a.G, g = j % a.G;
#pragma unroll
        for (int u = 0; u < NU; ++u)
          a.lut[((((int64_t)b * a.Hkv + kvh) * a.Sk + s) * kCodebook + c0 + cc + 64 * u) * GP + g] =
              acc[u][k] * a.scale_log2;
      }
    }
  };
  if (CPT > 1 && cpt > 1) dots(std::integral_constant<int, CPT>{});
  else dots(std::integral_constant<int, 1>{});
}

// ------------------------------------------------------------------------------------------
// 2. Scan of the compressed tokens.
// ------------------------------------------------------------------------------------------

// 32-bit shared-memory address operations (the hot loop keeps precomputed addresses).
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ float4 lds128f(uint32_t a) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(a));
  return v;
}
__device__ __forceinline__ float2 lds64f(uint32_t a) {
  float2 v;
  asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(a));
  return v;
}
__device__ __forceinline__ float lds32f(uint32_t a) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(a));
  return v;
}
__device__ __forceinline__ uint4 lds128u(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
  return v;
}
__device__ __forceinline__ void sts32u(uint32_t a, uint32_t v) {
  asm volatile("st.shared.u32 [%0], %1;" ::"r"(a), "r"(v));
}
__device__ __forceinline__ void sts64u(uint32_t a, uint32_t x, uint32_t y) {
  asm volatile("st.shared.v2.u32 [%0], {%1, %2};" ::"r"(a), "r"(x), "r"(y));
}
// hi at a, lo at a + LO_OFF bytes (the lo table follows the hi table)
template <int LO_OFF>
__device__ __forceinline__ void red_pair(uint32_t a, uint32_t hi, uint32_t lo) {
  asm volatile("red.shared.add.u32 [%0], %1;\n\tred.shared.add.u32 [%0+%3], %2;"
               ::"r"(a), "r"(hi), "r"(lo), "n"(LO_OFF));
}

// Codes of one token (S <= 8 bytes, little-endian in up to two words).
template <int SP>
struct Code {
  uint32_t w[SP <= 4 ? 1 : 2];
  __device__ __forceinline__ int byte(int s) const {
    return (int)__byte_perm(w[SP <= 4 ? 0 : (s >> 2)], 0u, 0x4440u | (unsigned)(s & 3));
  }
};

// The code rows of one (sequence, kv head): contiguous (base = the pair's row 0) or, with a
// block table, token t in page bt_row[t / P] at row kvh_off + t % P of that page (base = the
// page pool).  Both layouts give a row address aligned to the row size.
struct PairRows {
  const uint8_t* base;
  const int32_t* bt_row;   // null: contiguous
  int64_t kvh_off;         // kvh * P
};
template <bool PAGED>
__device__ __forceinline__ const uint8_t* pair_row(const DecodeArgs& a, const PairRows& pr,
                                                   uint32_t t, int S) {
  if constexpr (!PAGED) return pr.base + (int64_t)t * S;
  const int64_t pg = __ldg(pr.bt_row + (t >> a.pshift));
  if (pg < 0 || pg >= a.n_pages) {
    set_error(a.err, ZKV_DEVERR_PAGE);
    return nullptr;
  }
  return pr.base + ((pg * a.Hkv << a.pshift) + pr.kvh_off + (t & ((1u << a.pshift) - 1u))) * S;
}

// Codes of token t (0 when t >= tend or its page is invalid).  When S equals its padded size SP
// a single naturally aligned 2-, 4- or 8-byte load reads them; otherwise byte loads.
template <int SP, bool PAGED>
__device__ __forceinline__ Code<SP> load_code1(const DecodeArgs& a, const PairRows& pr, int S,
                                               uint32_t t, uint32_t tend) {
  // t is a pair-local token index (Tcap * S < 2^32 bytes per pair)
  Code<SP> r;
#pragma unroll
  for (int q = 0; q < (SP <= 4 ? 1 : 2); ++q) r.w[q] = 0u;
  if (t >= tend) return r;
  const uint8_t* row = pair_row<PAGED>(a, pr, t, S);
  if (!row) return r;
  if (S == SP) {
    const uint8_t* p = row;
    if constexpr (SP == 2) {
      r.w[0] = __ldg(reinterpret_cast<const unsigned short*>(p));
    } else if constexpr (SP == 4) {
      r.w[0] = __ldg(reinterpret_cast<const unsigned int*>(p));
    } else {
      const uint2 v = __ldg(reinterpret_cast<const uint2*>(p));
      r.w[0] = v.x;
      r.w[1] = v.y;
    }
  } else {
    const uint8_t* p = row;
#pragma unroll
    for (int s = 0; s < SP; ++s)
      if (s < S) r.w[s >> 2] |= (uint32_t)__ldg(p + s) << (8 * (s & 3));
  }
  return r;
}

// Key score of one token: sum over stages of the token's table entries (GP heads).
// sbase[s] is the shared address of this lane's copy of stage s codeword 0; codeword c is
// (c << csh) bytes further.
template <int GP, int SKP>
__device__ __forceinline__ void key_score(const uint32_t (&sbase)[SKP], int Sk, uint32_t csh,
                                          int lane, const Code<SKP>& kc, float (&sc)[GP]) {
#pragma unroll
  for (int g = 0; g < GP; ++g) sc[g] = 0.f;
#pragma unroll
  for (int s = 0; s < SKP; ++s) {
    if (s < Sk) {
      const uint32_t e = sbase[s] + ((uint32_t)kc.byte(s) << csh);
      if constexpr (GP == 8) {
        // the two halves are read in lane-dependent order: lanes 4-7 of each 8-lane phase
        // start with the upper half, which puts all 8 lanes of a phase in distinct banks
        const uint32_t h0 = ((uint32_t)lane >> 2) & 1u;
        const float4 v0 = lds128f(e + 16u * h0);
        const float4 v1 = lds128f(e + 16u * (h0 ^ 1u));
        const float4 lo4 = h0 ? v1 : v0, hi4 = h0 ? v0 : v1;
        sc[0] += lo4.x; sc[1] += lo4.y; sc[2] += lo4.z; sc[3] += lo4.w;
        sc[4] += hi4.x; sc[5] += hi4.y; sc[6] += hi4.z; sc[7] += hi4.w;
      } else if constexpr (GP == 4) {
        const float4 v = lds128f(e);
        sc[0] += v.x; sc[1] += v.y; sc[2] += v.z; sc[3] += v.w;
      } else if constexpr (GP == 2) {
        const float2 v = lds64f(e);
        sc[0] += v.x; sc[1] += v.y;
      } else {
        sc[0] += lds32f(e);
      }
    }
  }
}

// p in [0, 1] as p * 2^38 = hi * 2^19 + lo with hi = round(p * 2^19) in [0, 2^19] and
// lo = round((p * 2^19 - hi) * 2^19) in [-2^18, 2^18] (two's complement).  Each FMA below is
// exact except the roundings to an integer (|error of p * 2^38| <= 1/2); rounding uses the
// 1.5 * 2^23 addend, so only FMA-pipe and integer instructions are involved.
__device__ __forceinline__ void split_fixed38(float p, uint32_t& hi, uint32_t& lo) {
  const float magic = 12582912.0f;                          // 1.5 * 2^23
  const float xr = __fmaf_rn(p, 524288.0f, magic);          // round(p * 2^19) + magic
  hi = __float_as_uint(xr) - 0x4B400000u;
  const float h = __fsub_rn(xr, magic);                     // round(p * 2^19), exact
  const float d = __fmaf_rn(p, 524288.0f, -h);              // p * 2^19 - h, exact
  lo = __float_as_uint(__fmaf_rn(d, 524288.0f, magic)) - 0x4B400000u;
}

// Order-preserving map of a float to an unsigned key (for integer max reductions).
__device__ __forceinline__ uint32_t ord_key(float x) {
  const uint32_t u = __float_as_uint(x);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float ord_val(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
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
  static constexpr int VWSH = PASSES == 1 ? 5 : 6;   // log2(VW)
  static constexpr int ROUNDS = kScanSub / J;
  static constexpr int PR = ROUNDS + 4;          // padded staging row (words)
  static constexpr int CODEW = SVP <= 4 ? 1 : 2;
  static constexpr int NW = kScanThreads / 32;
  static constexpr int BUFW = 2 * J * GP * PR;   // words of one p staging buffer (hi, lo)
  static constexpr int CBUFW = J * PR * CODEW;   // words of one code staging buffer
};

// dst[(s, c, g)] = (master (if any) + histogram value) * scale[g], where the histogram
// value of (s, c, g) is the sum over token slots j of hi * 2^-19 + lo * 2^-38 in column
// j * COMBOS + s * GP + g of code row c.  The integer sums are exact; converting them to
// float32 and adding costs a few roundings, <= 2^-21 relative per entry.  Threads walk the tables row by row (consecutive
// threads, consecutive words: no bank conflicts); the J columns of one (s, g) are combined
// with xor-shuffles (they are COMBOS lanes apart).
template <class C, int GP>
__device__ __forceinline__ void fold_tables(const uint32_t* vhi, const uint32_t* vlo,
                                            const float* master, float* dst, int Sv,
                                            bool has_master, const float (&scale)[GP], int tid) {
  const int lane = tid & 31;
  const int total = kCodebook * C::VW;           // words per table
#pragma unroll 4
  for (int w0 = tid - lane; w0 < total; w0 += kScanThreads) {
    const int wi = w0 + lane;                      // total is a multiple of 32
    const int cc = wi / C::VW, col = wi % C::VW;
    float v = fmaf((float)(int32_t)vlo[wi], 0x1p-38f, (float)vhi[wi] * 0x1p-19f);
    if constexpr (C::PASSES == 1) {
#pragma unroll
      for (int o = C::COMBOS; o < 32; o <<= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    }
    const int combo = C::PASSES == 1 ? col % C::COMBOS : col;
    const int ss = combo / GP, g = combo % GP;
    const bool writer = (C::PASSES == 1 ? col < C::COMBOS : true) && ss < Sv;
    if (writer) {
      float sc = 1.f;
#pragma unroll
      for (int q = 0; q < GP; ++q)
        if (q == g) sc = scale[q];
      const size_t f = ((size_t)ss * kCodebook + cc) * GP + g;
      const float old = has_master ? master[f] : 0.f;
      dst[f] = (old + v) * sc;
    }
  }
}

// The token loop is software-pipelined with one barrier per sub-chunk.  In interval i every
// thread (b) adds the staged p of sub-chunk i-1 to the integer histograms, (c) computes and
// stages the p of sub-chunk i, and (d) gathers the key scores of sub-chunk i+1 and checks
// them against the reference; the interval's barrier ORs those checks.  Staging buffers
// alternate between two copies, so no interval reads what the same interval writes.  When a
// score exceeded the reference (rare: the reference is the maximum so far plus a headroom), the
// next interval first takes the block maxima (a) and, with non-empty histograms, a slow path
// (barrier, fold, barrier, zero, barrier) after (b), uniformly across the block.
template <int GP, int SKP, int SVP, bool PAGED>
__global__ void __launch_bounds__(kScanThreads, 1) scan_kernel(DecodeArgs a) {
  using C = ScanCfg<GP, SKP, SVP>;
  extern __shared__ __align__(16) unsigned char smraw[];
  pdl_wait();   // tables, prefix sums and codes
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (a.upd_comp_len && blockIdx.x == 0) {
    // serving step: the append has read the pre-step lengths; store the new ones (nothing in
    // this kernel reads them)
    for (int b = tid; b < a.B; b += kScanThreads)
      advance_lengths(b, a.Tcap, a.Wcap, a.upd_win_len, a.upd_win_head, a.upd_comp_len);
  }
  const int Rk = a.Rk, Sk = a.Sk, Sv = a.Sv, G = a.G;
  const int ntab = Sv * kCodebook * GP;           // histogram entries (s, c, g)
  float* lut = reinterpret_cast<float*>(smraw);                                 // [Sk][256][Rk][GP]
  float* master = lut + (size_t)Rk * Sk * kCodebook * GP;                       // [Sv][256][GP]
  uint32_t* vhi = reinterpret_cast<uint32_t*>(master + ntab);                   // [256][VW]
  uint32_t* vlo = vhi + kCodebook * C::VW;
  uint32_t* stg = vlo + kCodebook * C::VW;        // [2][hi, lo][J][GP][PR]
  uint32_t* cst = stg + 2 * C::BUFW;              // [2][J][PR][CODEW]
  uint32_t* redk = cst + 2 * C::CBUFW;            // [2][NW][GP] partial maxima (keys)
  float* red = reinterpret_cast<float*>(redk + 2 * C::NW * GP);   // [NW][GP]

  const int npairs = a.B * a.Hkv;
  const int64_t lo = a.bounds[blockIdx.x], hi = a.bounds[blockIdx.x + 1];
  if (lo >= hi) return;
  // last pair whose prefix start is <= lo: block-parallel search, one round of loads per
  // factor of kScanThreads (pre is non-decreasing, so the sampled predicate is a prefix)
  int pfirst = 0;
  {
    int l = 0, r = npairs;   // invariant: pre[l] <= lo < pre[r] (pre[npairs] = tot > lo)
    while (r - l > 1) {
      const int step = (r - l + kScanThreads - 1) / kScanThreads;
      const int k = l + tid * step;
      const int cnt = __syncthreads_count(k < r && a.pre[k] <= lo);
      l = l + (cnt - 1) * step;
      r = l + step < r ? l + step : r;
    }
    pfirst = l;
  }
  const int copy = lane & (Rk - 1);
  const int cshift = __ffs(Rk * GP) - 1;          // Rk * GP is a power of two
  const int sstride = kCodebook * Rk * GP;
  // shared addresses used by the token loop
  uint32_t sbase[SKP];
#pragma unroll
  for (int q = 0; q < SKP; ++q) sbase[q] = smem_u32(lut) + 4u * (uint32_t)(q * sstride + copy * GP);
  const uint32_t csh = (uint32_t)cshift + 2u;
  // value-side lane roles (PASSES == 1: lane = j * COMBOS + s * GP + g)
  const int vj = C::PASSES == 1 ? lane / C::COMBOS : 0;
  // staging slot of this thread's token
  const int sj = tid % C::J, sk = tid / C::J;
  const uint32_t stg_base = smem_u32(stg), cst_base = smem_u32(cst);
  const uint32_t hst_a = stg_base + 4u * (uint32_t)(sj * GP * C::PR + sk);
  const uint32_t cst_a = cst_base + 4u * C::CODEW * (uint32_t)(sj * C::PR + sk);
  const uint32_t vtab_base = smem_u32(vhi);
  const uint32_t redk_a = smem_u32(redk);

  // integer histograms += staged p of one sub-chunk (buffer bf).  Batches of 4 rounds,
  // warp-strided.  Padded heads carry p = 0 and padded stages read code byte 0 of a stage that
  // is never output, so no lane needs masking.
  auto accumulate = [&](int bf) {
#pragma unroll
    for (int ps = 0; ps < C::PASSES; ++ps) {
      const int combo = C::PASSES == 1 ? lane % C::COMBOS : ps * 32 + lane;
      const int vs = combo / GP, vg = combo % GP;
      const uint32_t hrow = stg_base + 4u * (uint32_t)(bf * C::BUFW + (vj * GP + vg) * C::PR);
      const uint32_t lrow = hrow + 4u * (uint32_t)(C::J * GP * C::PR);
      const uint32_t crow = cst_base + 4u * (uint32_t)(bf * C::CBUFW + C::CODEW * vj * C::PR);
      const unsigned sel = 0x4440u | (unsigned)(vs & 3);
      const uint32_t tab = vtab_base + 4u * (uint32_t)(ps * 32 + lane);
      for (int bt = warp; bt < C::ROUNDS / 4; bt += C::NW) {
        const uint32_t k0b = 16u * (uint32_t)bt;   // 4 rounds of 4-byte words
        const uint4 h4 = lds128u(hrow + k0b);
        const uint4 l4 = lds128u(lrow + k0b);
        uint32_t cw[4];
        if constexpr (C::CODEW == 1) {
          const uint4 c4 = lds128u(crow + k0b);
          cw[0] = c4.x; cw[1] = c4.y; cw[2] = c4.z; cw[3] = c4.w;
        } else {
          const uint4 c01 = lds128u(crow + 2u * k0b);
          const uint4 c23 = lds128u(crow + 2u * k0b + 16u);
          const int hw = vs >> 2;
          cw[0] = hw ? c01.y : c01.x; cw[1] = hw ? c01.w : c01.z;
          cw[2] = hw ? c23.y : c23.x; cw[3] = hw ? c23.w : c23.z;
        }
        const uint32_t hh[4] = {h4.x, h4.y, h4.z, h4.w};
        const uint32_t ll[4] = {l4.x, l4.y, l4.z, l4.w};
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const uint32_t adr = tab + (__byte_perm(cw[r], 0u, sel) << (C::VWSH + 2));
          red_pair<kCodebook * C::VW * 4>(adr, hh[r], ll[r]);
        }
      }
    }
  };
  // block maxima of the scores in sc (tokens with okk): warp maxima -> redk, barrier, every
  // lane reads the NW x GP partial maxima (entry w * GP + g in lane (w * GP + g) % 32), folds
  // over w with xor-shuffles and broadcasts each head
  auto block_max = [&](const float (&sc)[GP], bool okk, float (&mn)[GP]) {
#pragma unroll
    for (int g = 0; g < GP; ++g) {
      const uint32_t k = __reduce_max_sync(0xffffffffu, okk ? ord_key(sc[g]) : 0u);
      if (lane == 0) sts32u(redk_a + 4u * (uint32_t)(warp * GP + g), k);
    }
    __syncthreads();
    uint32_t k = 0u;
#pragma unroll
    for (int e = 0; e < C::NW * GP; e += 32)
      if (e + lane < C::NW * GP) {
        uint32_t v;
        asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(redk_a + 4u * (uint32_t)(e + lane)));
        k = max(k, v);
      }
#pragma unroll
    for (int o = GP; o < 32 && o < C::NW * GP; o <<= 1) k = max(k, __shfl_xor_sync(0xffffffffu, k, o));
#pragma unroll
    for (int g = 0; g < GP; ++g) mn[g] = ord_val(__shfl_sync(0xffffffffu, k, g));
  };

  for (int pr = pfirst; pr < npairs && a.pre[pr] < hi; ++pr) {
    const int64_t seg0 = lo > a.pre[pr] ? lo : a.pre[pr];
    const int64_t seg1 = hi < a.pre[pr + 1] ? hi : a.pre[pr + 1];
    if (seg0 >= seg1) continue;
    const int64_t s0 = seg0 - a.pre[pr], s1 = seg1 - a.pre[pr];   // pair-local token range
    const int64_t slot = (int64_t)pr + blockIdx.x;
    PairRows kcb, vcb;
    if constexpr (PAGED) {
      const int b = pr / a.Hkv, kvh = pr - b * a.Hkv;
      kcb = PairRows{a.k_codes, a.bt + (int64_t)b * a.max_pages, (int64_t)kvh << a.pshift};
      vcb = PairRows{a.v_codes, kcb.bt_row, kcb.kvh_off};
    } else {
      kcb = PairRows{a.k_codes + (int64_t)pr * a.Tcap * Sk, nullptr, 0};
      vcb = PairRows{a.v_codes + (int64_t)pr * a.Tcap * Sv, nullptr, 0};
    }
    // the segment's codes stream into L2 while the tables are filled; the per-thread loads
    // below then find them there
    if constexpr (!PAGED) {
      if (tid == 0) {
        const int64_t pbytes_k = (int64_t)a.Tcap * Sk, pbytes_v = (int64_t)a.Tcap * Sv;
        const int64_t a0 = s0 & ~int64_t(15);
        prefetch_l2(kcb.base, kcb.base + pbytes_k, kcb.base + a0 * Sk, (s1 - a0) * Sk);
        prefetch_l2(vcb.base, vcb.base + pbytes_v, vcb.base + a0 * Sv, (s1 - a0) * Sv);
      }
    } else {
      // one thread per page the segment touches (a page's rows of one head are contiguous)
      const int64_t P = int64_t(1) << a.pshift;
      const int64_t p0 = s0 >> a.pshift, np = ((s1 - 1) >> a.pshift) - p0 + 1;
      for (int64_t k = tid; k < np; k += kScanThreads) {
        const int64_t r0 = (p0 + k) * P > s0 ? (p0 + k) * P : s0;
        const int64_t r1 = (p0 + k + 1) * P < s1 ? (p0 + k + 1) * P : s1;
        // page blocks of P * S bytes start 16-byte aligned (P >= 32 is a power of two); the
        // prefetch is rounded outward to 16-byte granules inside the block
        const uint8_t* bk = pair_row<true>(a, kcb, (uint32_t)((p0 + k) * P), Sk);
        const uint8_t* bv = pair_row<true>(a, vcb, (uint32_t)((p0 + k) * P), Sv);
        const int64_t o = r0 - (p0 + k) * P;
        if (bk) prefetch_l2(bk, bk + P * Sk, bk + o * Sk, (r1 - r0) * Sk);
        if (bv) prefetch_l2(bv, bv + P * Sv, bv + o * Sv, (r1 - r0) * Sv);
      }
    }
    const uint32_t u0 = (uint32_t)s0, u1 = (uint32_t)s1;
    const int nsub = (int)((u1 - u0 + kScanSub - 1) / kScanSub);   // same on every thread
    // Token order: warp w owns the contiguous run of nsub * 32 tokens starting at
    // u0 + w * nsub * 32, and sub-chunk i takes block i of every warp's run.  A warp's codes are
    // still one contiguous load per sub-chunk, while each sub-chunk samples the whole segment,
    // so the first sub-chunk's maxima (the initial reference) are close to the segment's and
    // later growth of the reference (a fold) is rare.  The histograms do not depend on order.
    const uint32_t tw = u0 + (uint32_t)(warp * nsub) * 32u + (uint32_t)lane;   // token of sub-chunk 0
    // codes of sub-chunks 0 and 1 in flight during the table fill
    Code<SKP> kc = load_code1<SKP, PAGED>(a, kcb, Sk, tw, u1);
    Code<SVP> vc = load_code1<SVP, PAGED>(a, vcb, Sv, tw, u1);
    Code<SKP> kn = load_code1<SKP, PAGED>(a, kcb, Sk, tw + 32u, u1);
    Code<SVP> vn = load_code1<SVP, PAGED>(a, vcb, Sv, tw + 32u, u1);
    __syncthreads();   // previous segment's shared memory is free
    {
      // zero the histograms, then copy the pair's table entries (s, c) -> every lane-group
      // copy: item f = (entry, copy) with the copy fastest, so consecutive lanes store
      // consecutive GP-wide entries; heads g >= G are zero
      uint4* z = reinterpret_cast<uint4*>(vhi);
      const int nz = 2 * kCodebook * C::VW / 4;
      for (int f = tid; f < nz; f += kScanThreads) z[f] = make_uint4(0u, 0u, 0u, 0u);
      const float* src = a.lut + (int64_t)pr * Sk * kCodebook * GP;
      const int rsh = __ffs(Rk) - 1;
      const int n = Sk * kCodebook * Rk;
      constexpr int NB = GP >= 8 ? 4 : 8;   // items in flight per thread
      for (int f0 = 0; f0 < n; f0 += NB * kScanThreads) {
        float v[NB][GP];
#pragma unroll
        for (int u = 0; u < NB; ++u) {
          const int f = f0 + u * kScanThreads + tid;
          const float* e = src + (int64_t)(f >> rsh) * GP;   // 16-byte aligned for GP >= 4
          if (f < n) {
            if constexpr (GP >= 4) {
#pragma unroll
              for (int g = 0; g < GP; g += 4) {
                const float4 t4 = __ldg(reinterpret_cast<const float4*>(e + g));
                v[u][g] = t4.x; v[u][g + 1] = t4.y; v[u][g + 2] = t4.z; v[u][g + 3] = t4.w;
              }
            } else if constexpr (GP == 2) {
              const float2 t2 = __ldg(reinterpret_cast<const float2*>(e));
              v[u][0] = t2.x; v[u][1] = t2.y;
            } else {
              v[u][0] = __ldg(e);
            }
          }
#pragma unroll
          for (int g = 0; g < GP; ++g)
            if (g >= G) v[u][g] = 0.f;   // padded heads (not written by the table kernel)
        }
#pragma unroll
        for (int u = 0; u < NB; ++u) {
          const int f = f0 + u * kScanThreads + tid;
          if (f < n) {
            float* dst = lut + (size_t)f * GP;   // (sc * Rk + copy) * GP
            if constexpr (GP >= 4) {
#pragma unroll
              for (int g = 0; g < GP; g += 4)
                *reinterpret_cast<float4*>(dst + g) = make_float4(v[u][g], v[u][g + 1], v[u][g + 2], v[u][g + 3]);
            } else if constexpr (GP == 2) {
              *reinterpret_cast<float2*>(dst) = make_float2(v[u][0], v[u][1]);
            } else {
              dst[0] = v[u][0];
            }
          }
        }
      }
    }
    __syncthreads();   // tables and zeroed histograms are ready

    float mref[GP], lacc[GP];
#pragma unroll
    for (int g = 0; g < GP; ++g) {
      mref[g] = -INFINITY;
      lacc[g] = 0.f;
    }
    bool dirty = false, has_master = false;   // uniform across the block
    // prologue: scores of sub-chunk 0 (the reference starts at -inf, so interval 0 grows it)
    float sc[GP];
    key_score<GP, SKP>(sbase, Sk, csh, lane, kc, sc);
    bool over = true;   // uniform: some score of the current sub-chunk exceeds the reference
    for (int i = 0; i < nsub; ++i) {
      const int bf = i & 1;
      const uint32_t t = tw + 32u * (uint32_t)i;
      const bool ok = t < u1;
      // Phase order: even warps (b), (c), (d); odd warps (c), (d), (b) -- half of the block
      // issues the reduction-heavy phase while the other half gathers, so the shared-memory
      // pipe sees a mix.  (c) must precede (d) (it reads this sub-chunk's scores and value
      // codes, which (d) replaces).  A growth of the reference (known from the previous
      // interval's barrier) takes (b) first on every warp, then the fold.
      const bool odd = (warp & 1) != 0;
      if (over) {
        // (a) the block maxima of sub-chunk i set the new reference
        float mn[GP];
        block_max(sc, ok, mn);
        if (i > 0) {
          accumulate(bf ^ 1);
          dirty = true;
        }
        // New reference = maximum + kHeadroom: later sub-chunks rarely exceed it, so folds
        // stay rare.  Precision: the segment's largest p is >= 2^-kHeadroom and its
        // fixed-point error is <= (tokens <= 2^14) * 2^-39 = 2^-25 absolute, i.e.
        // <= 2^(kHeadroom - 25) = 2^-15 relative to the segment's mass.
        float alpha[GP];
#pragma unroll
        for (int g = 0; g < GP; ++g) {
          const float m2 = mn[g] > mref[g] ? mn[g] + kHeadroom : mref[g];
          alpha[g] = mref[g] == -INFINITY ? 0.f : ex2_approx(mref[g] - m2);
          mref[g] = m2;
          lacc[g] *= alpha[g];
        }
        if (dirty) {
          // fold the integer histograms (relative to the old reference) into the fp32
          // master and rescale it to the new reference
          __syncthreads();   // every reduction so far has landed
          fold_tables<C, GP>(vhi, vlo, master, master, Sv, has_master, alpha, tid);
          __syncthreads();
          uint4* z = reinterpret_cast<uint4*>(vhi);
          const int nz = 2 * kCodebook * C::VW / 4;
          for (int f = tid; f < nz; f += kScanThreads) z[f] = make_uint4(0u, 0u, 0u, 0u);
          __syncthreads();
          has_master = true;
          dirty = false;
        }
      } else if (i > 0 && !odd) {
        accumulate(bf ^ 1);   // (b), even warps
      }
      // (c) p of sub-chunk i -> staging buffer bf (every score is <= the reference: p <= 1)
#pragma unroll
      for (int g = 0; g < GP; ++g) {
        uint32_t hv = 0u, lv = 0u;
        if (ok) {
          const float pv = ex2_approx(sc[g] - mref[g]);
          lacc[g] += pv;
          if (g < G) split_fixed38(pv, hv, lv);
        }
        sts32u(hst_a + 4u * (uint32_t)(bf * C::BUFW + g * C::PR), hv);
        sts32u(hst_a + 4u * (uint32_t)(bf * C::BUFW + (C::J * GP + g) * C::PR), lv);   // lo follows hi
      }
      if constexpr (C::CODEW == 1) {
        sts32u(cst_a + 4u * (uint32_t)(bf * C::CBUFW), vc.w[0]);
      } else {
        sts64u(cst_a + 4u * (uint32_t)(bf * C::CBUFW), vc.w[0], vc.w[1]);
      }
      // (d) scores of sub-chunk i+1 and whether any exceeds the reference; codes of
      // sub-chunk i+2 in flight
      bool ex = false;
      if (i + 1 < nsub) {
        kc = kn;
        vc = vn;
        kn = load_code1<SKP, PAGED>(a, kcb, Sk, t + 64u, u1);
        vn = load_code1<SVP, PAGED>(a, vcb, Sv, t + 64u, u1);
        key_score<GP, SKP>(sbase, Sk, csh, lane, kc, sc);
        if (t + 32u < u1) {
#pragma unroll
          for (int g = 0; g < GP; ++g) ex |= sc[g] > mref[g];
        }
      }
      if (!over && i > 0) {
        if (odd) accumulate(bf ^ 1);   // (b), odd warps
        dirty = true;
      }
      over = __syncthreads_or(ex) != 0;
    }
    // histograms += p of the last sub-chunk
    accumulate((nsub - 1) & 1);
    // ---- segment partial: maximum, sum of p, fp32 histograms (master + integer tables)
#pragma unroll
    for (int g = 0; g < GP; ++g) {
      const float l = warp_sum_f32(lacc[g]);
      if (lane == 0) red[warp * GP + g] = l;
    }
    __syncthreads();   // also: every reduction of this segment has landed
    if (tid < GP) {
      float l = 0.f;
#pragma unroll
      for (int w = 0; w < C::NW; ++w) l += red[w * GP + tid];
      float mr = 0.f;
#pragma unroll
      for (int g = 0; g < GP; ++g)
        if (g == tid) mr = mref[g];
      a.pm[slot * GP + tid] = mr;
      a.pl[slot * GP + tid] = l;
    }
    {
      float one[GP];
#pragma unroll
      for (int g = 0; g < GP; ++g) one[g] = 1.f;
      // straight into the segment's slot (the next segment's first barrier orders these reads
      // of the shared tables before they are reused)
      fold_tables<C, GP>(vhi, vlo, master, a.pw + slot * (int64_t)ntab, Sv, has_master, one, tid);
    }
  }
}

#include "scan_rvq.cuh"
#include "combine.cuh"


// ------------------------------------------------------------------------------------------
// 4. Product-VQ decode (VeloxQuant "VecInfer": keys and values quantised by sub-vectors
//    against one shared 256-entry codebook per kv head).  With d / m = 32 sub-vectors a warp's
//    lane j owns sub-vector j of every token: it gathers Ck[zk_j] and Cv[zv_j] from shared
//    memory, forms its partial scores for the GP heads, and the partial scores of TB = 32 / GP
//    tokens are reduced together by one transpose-sum (after it lane L holds the score of
//    token L / GP, head L % GP).  Per head the warp keeps a running maximum; each lane
//    accumulates p * Cv[zv_j] into its m output dims in registers.  No histograms.
//    pq_scan_kernel:     grid (chunks of kPqChunk tokens, pairs); chunk partials -> workspace.
//    pq_finalize_kernel: per pair, the window attention (beside nothing: it is the last kernel),
//                        the log-sum-exp combine of the chunks, rotation back, merge with the
//                        window.
// ------------------------------------------------------------------------------------------
constexpr int kPqChunk = 2048;   // tokens per scan CTA

struct PqArgs {
  int B, Hq, Hkv, G, d, m, n_chunks;
  int64_t Tcap, max_comp;
  float scale_log2;
  double rot;
  const __half* q;
  const uint8_t* k_codes;   // [B][Hkv][Tcap][d/m]
  const uint8_t* v_codes;
  const int32_t* comp_len;
  const float* Ck;          // [Hkv][256][m]
  const float* Cv;
  const float* k_smooth;    // [Hkv][d] or null
  int32_t* err;
  float* cm;                // [pairs][n_chunks][GP] chunk maxima (log2 units)
  float* cl;                // [pairs][n_chunks][GP] chunk sums of p
  float* co;                // [pairs][n_chunks][GP][d] chunk sums of p * v (rotated domain)
};

template <int D, int M, int GP>
__global__ void __launch_bounds__(256) pq_scan_kernel(PqArgs a) {
  constexpr int NSUB = D / M;
  static_assert(NSUB == 32 || NSUB == 16, "one sub-vector per lane of a 32- or 16-lane group");
  constexpr int NH = 32 / NSUB;      // lane groups: each takes its own tokens
  constexpr int TBH = NSUB / GP;     // tokens per group per transpose-sum batch
  constexpr int TB = NH * TBH;       // tokens per batch (32 / GP)
  constexpr int E = D / 32;
  __shared__ __align__(16) float ck[kCodebook * M];
  __shared__ __align__(16) float cv[kCodebook * M];
  __shared__ __align__(16) float qs[GP][D];
  __shared__ float wm[8][GP], wl[8][GP];
  __shared__ __align__(16) float wo[8][GP][D];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int chunk = blockIdx.x;
  const int64_t pair = blockIdx.y;
  const int b = (int)(pair / a.Hkv), kvh = (int)(pair % a.Hkv);
  for (int f = tid; f < kCodebook * M; f += 256) {
    ck[f] = a.Ck[(size_t)kvh * kCodebook * M + f];
    cv[f] = a.Cv[(size_t)kvh * kCodebook * M + f];
  }
  if (warp < GP) {   // q_tilde of head g = warp: H (lambda * q) / sqrt(d), float32
    float v[E];
    const int g = warp;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      float x = 0.f;
      if (g < a.G) {
        x = __half2float(a.q[((int64_t)b * a.Hq + (int64_t)kvh * a.G + g) * D + e * 32 + lane]);
        if (a.k_smooth) x *= a.k_smooth[(int64_t)kvh * D + e * 32 + lane];
      }
      v[e] = x;
    }
    fwht_warp_f32<D>(v, lane);
    const float rs = (float)a.rot;
#pragma unroll
    for (int e = 0; e < E; ++e) qs[g][e * 32 + lane] = v[e] * rs;
  }
  __syncthreads();
  int64_t c = a.comp_len[b];
  if (c < 0 || c > a.Tcap) c = c < 0 ? 0 : a.Tcap;   // (the finalize reports it)
  c = c < a.max_comp ? c : a.max_comp;
  const int64_t t0 = (int64_t)chunk * kPqChunk;
  const int64_t t1 = t0 + kPqChunk < c ? t0 + kPqChunk : c;
  const int64_t n = t1 > t0 ? t1 - t0 : 0;
  // warp w takes the contiguous run [w0, w1) of the chunk
  const int64_t per = (n + 7) / 8;
  const int64_t w0 = t0 + warp * per < t1 ? t0 + warp * per : t1;
  const int64_t w1 = w0 + per < t1 ? w0 + per : t1;
  // lane = (group hh, sub-vector j); group hh takes tokens hh * TBH .. hh * TBH + TBH - 1 of a batch
  const int j = lane % NSUB, hh = lane / NSUB;
  float qr[GP][M];
#pragma unroll
  for (int g = 0; g < GP; ++g)
#pragma unroll
    for (int i = 0; i < M; ++i) qr[g][i] = qs[g][j * M + i];
  const uint8_t* kz = a.k_codes + (pair * a.Tcap) * NSUB + j;
  const uint8_t* vz = a.v_codes + (pair * a.Tcap) * NSUB + j;
  float mrun[GP], acc[GP][M];
#pragma unroll
  for (int g = 0; g < GP; ++g) {
    mrun[g] = -INFINITY;
#pragma unroll
    for (int i = 0; i < M; ++i) acc[g][i] = 0.f;
  }
  float lp = 0.f;   // this lane's share of the sum of p of head lane % GP
  const int gl = lane % GP;
  for (int64_t base = w0; base < w1; base += TB) {
    const int nv = (int)(w1 - base < TB ? w1 - base : TB);
    const int64_t gbase = base + hh * TBH;   // this lane group's first token of the batch
    float x[NSUB];
#pragma unroll
    for (int u = 0; u < TBH; ++u) {
      float kv[M];
      if (hh * TBH + u < nv) {
        const int z = kz[(gbase + u) * NSUB];
#pragma unroll
        for (int i = 0; i < M; ++i) kv[i] = ck[z * M + i];
      } else {
#pragma unroll
        for (int i = 0; i < M; ++i) kv[i] = 0.f;
      }
#pragma unroll
      for (int g = 0; g < GP; ++g) {
        float s = 0.f;
#pragma unroll
        for (int i = 0; i < M; ++i) s = fmaf(qr[g][i], kv[i], s);
        x[u * GP + g] = s;
      }
    }
    // lane L ends with the score of its group's token (L % NSUB) / GP, head L % GP
    int hidx = 0;
    float sc = TransposeSum<NSUB, NSUB, NSUB / 2>::run(x, lane, hidx) * a.scale_log2;   // hidx == j
    const bool ok = hh * TBH + j / GP < nv;
    if (!ok) sc = -INFINITY;
    float bm = sc;   // batch maximum of head lane % GP
#pragma unroll
    for (int o = GP; o < 32; o <<= 1) bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, o));
    float alpha_l = 1.f, mnew_l = 0.f;
#pragma unroll
    for (int g = 0; g < GP; ++g) {
      const float mb = __shfl_sync(0xffffffffu, bm, g);
      const float mn = fmaxf(mrun[g], mb);
      const float alpha = mrun[g] == -INFINITY ? 0.f : ex2_approx(mrun[g] - mn);
#pragma unroll
      for (int i = 0; i < M; ++i) acc[g][i] *= alpha;
      if (g == gl) {
        alpha_l = alpha;
        mnew_l = mn;
      }
      mrun[g] = mn;
    }
    const float p = ok ? ex2_approx(sc - mnew_l) : 0.f;
    lp = lp * alpha_l + p;
#pragma unroll
    for (int u = 0; u < TBH; ++u) {
      // the shuffles run on every lane; a token past the end has p = 0 and reads no codes
      float vv[M];
      if (hh * TBH + u < nv) {
        const int z = vz[(gbase + u) * NSUB];
#pragma unroll
        for (int i = 0; i < M; ++i) vv[i] = cv[z * M + i];
      } else {
#pragma unroll
        for (int i = 0; i < M; ++i) vv[i] = 0.f;
      }
#pragma unroll
      for (int g = 0; g < GP; ++g) {
        const float pg = __shfl_sync(0xffffffffu, p, hh * NSUB + u * GP + g);
#pragma unroll
        for (int i = 0; i < M; ++i) acc[g][i] = fmaf(pg, vv[i], acc[g][i]);
      }
    }
  }
  if constexpr (NH == 2) {   // the two groups hold the same dims for different tokens
#pragma unroll
    for (int g = 0; g < GP; ++g)
#pragma unroll
      for (int i = 0; i < M; ++i) acc[g][i] += __shfl_xor_sync(0xffffffffu, acc[g][i], 16);
  }
  // warp partials: per head the sum of p over the lanes of that head
#pragma unroll
  for (int o = GP; o < 32; o <<= 1) lp += __shfl_xor_sync(0xffffffffu, lp, o);
#pragma unroll
  for (int g = 0; g < GP; ++g) {
    const float l = __shfl_sync(0xffffffffu, lp, g);
    if (lane == 0) {
      wm[warp][g] = mrun[g];
      wl[warp][g] = l;
    }
    if (lane < NSUB) {
#pragma unroll
      for (int i = 0; i < M; ++i) wo[warp][g][j * M + i] = acc[g][i];
    }
  }
  __syncthreads();
  // combine the 8 warps: weight 2^(m_w - M*) (0 for a warp without tokens)
  const int64_t slot = pair * a.n_chunks + chunk;
  for (int f = tid; f < GP * D; f += 256) {
    const int g = f / D, e = f % D;
    float ms = -INFINITY;
#pragma unroll
    for (int w = 0; w < 8; ++w) ms = fmaxf(ms, wm[w][g]);
    float o = 0.f, l = 0.f;
    if (ms != -INFINITY) {
#pragma unroll
      for (int w = 0; w < 8; ++w) {
        const float wt = wm[w][g] == -INFINITY ? 0.f : ex2_approx(wm[w][g] - ms);
        o = fmaf(wt, wo[w][g][e], o);
        l = fmaf(wt, wl[w][g], l);
      }
    }
    a.co[(slot * GP + g) * D + e] = o;
    if (e == 0) {
      a.cm[slot * GP + g] = ms;
      a.cl[slot * GP + g] = l;
    }
  }
}

template <int D, int GP>
__global__ void __launch_bounds__(256) pq_finalize_kernel(PqArgs a, DecodeArgs w) {
  constexpr int E = D / 32;
  extern __shared__ __align__(16) unsigned char win_smem[];
  __shared__ __align__(16) float oc[GP * D];
  __shared__ float ms_s[GP], ls_s[GP];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t pair = blockIdx.x;
  const int b = (int)(pair / a.Hkv), kvh = (int)(pair % a.Hkv);
  window_item<D, GP>(w, b, kvh, 0, win_smem);
  if (tid == 0) {
    const int64_t c = a.comp_len[b];
    if (c < 0 || c > a.Tcap) set_error(a.err, ZKV_DEVERR_COMP_LEN);
  }
  const int64_t s0 = pair * a.n_chunks;
  for (int f = tid; f < GP * D; f += 256) {
    const int g = f / D, e = f % D;
    float m = -INFINITY;
    for (int k = 0; k < a.n_chunks; ++k) m = fmaxf(m, a.cm[(s0 + k) * GP + g]);
    float o = 0.f, l = 0.f;
    if (m != -INFINITY) {
      for (int k = 0; k < a.n_chunks; ++k) {
        const float cmk = a.cm[(s0 + k) * GP + g];
        const float wt = cmk == -INFINITY ? 0.f : ex2_approx(cmk - m);
        o = fmaf(wt, a.co[((s0 + k) * GP + g) * D + e], o);
        l = fmaf(wt, a.cl[(s0 + k) * GP + g], l);
      }
    }
    oc[f] = o;
    if (e == 0) {
      ms_s[g] = m;
      ls_s[g] = l;
    }
  }
  __syncthreads();   // chunk combine and this block's window terms are visible
  for (int g = warp; g < a.G; g += 8) {
    const float mc = ms_s[g], lc = ls_s[g];
    double v[E];   // the compressed part's sum of p * v, rotated back
#pragma unroll
    for (int q = 0; q < E; ++q) v[q] = (double)oc[g * D + q * 32 + lane];
    fwht_warp_f64<D>(v, lane);
    const float mw = w.wm[pair * GP + g], lw = w.wl[pair * GP + g];
    const float M = fmaxf(mc, mw);
    const float wc = (mc == -INFINITY) ? 0.f : ex2_approx(mc - M);
    const float ww = (mw == -INFINITY) ? 0.f : ex2_approx(mw - M);
    const float L = wc * lc + ww * lw;
    const int64_t h = (int64_t)kvh * a.G + g;
    float* o = w.out + ((int64_t)b * a.Hq + h) * D;
    const float inv = L > 0.f ? 1.f / L : 0.f;
#pragma unroll
    for (int q = 0; q < E; ++q) {
      const int i = q * 32 + lane;
      o[i] = (wc * (float)(v[q] * a.rot) + ww * w.wo[(pair * GP + g) * D + i]) * inv;
    }
    if (lane == 0 && w.lse) w.lse[(int64_t)b * a.Hq + h] = L > 0.f ? (M + log2f(L)) * kLn2 : -INFINITY;
  }
}

// ------------------------------------------------------------------------------------------
// Launch
// ------------------------------------------------------------------------------------------
// Under stream capture the record becomes an event node of the graph (so that each replay
// records it and the caller can time the kernels between two events).
static inline void trace(void* const* ev, int i, cudaStream_t st) {
  if (!ev || !ev[i]) return;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(st, &cs) != cudaSuccess) cs = cudaStreamCaptureStatusNone;
  cudaEventRecordWithFlags(reinterpret_cast<cudaEvent_t>(ev[i]), st,
                           cs == cudaStreamCaptureStatusActive ? cudaEventRecordExternal
                                                               : cudaEventRecordDefault);
}

template <int GPH, int SKP, int SVP>
static int launch_scan2(const DecodeArgs& a, cudaStream_t st) {
  auto* k = a.bt ? scan2_kernel<GPH, SKP, SVP, true> : scan2_kernel<GPH, SKP, SVP, false>;
  if (ensure_smem_limit(k, kS2Smem) != cudaSuccess) return ZKV_ERR_CUDA;
  if (launch_pdl(k, dim3(a.grid), dim3(kS2Threads), kS2Smem, st, a) != cudaSuccess)
    return ZKV_ERR_CUDA;
  return ZKV_OK;
}

template <int GPH, int SKP>
static int launch_scan2_v(const DecodeArgs& a, cudaStream_t st) {
  switch (a.Sv) {
    case 1: return launch_scan2<GPH, SKP, 1>(a, st);
    case 2: return launch_scan2<GPH, SKP, 2>(a, st);
    default: return launch_scan2<GPH, SKP, 4>(a, st);
  }
}

template <int GPH>
static int launch_scan2_kv(const DecodeArgs& a, cudaStream_t st) {
  switch (a.Sk) {
    case 1: return launch_scan2_v<GPH, 1>(a, st);
    case 2: return launch_scan2_v<GPH, 2>(a, st);
    default: return launch_scan2_v<GPH, 4>(a, st);
  }
}

template <int GP, int SKP, int SVP>
static int launch_scan(const DecodeArgs& a, size_t smem, cudaStream_t st) {
  // the code layout is a template parameter: the contiguous loop carries no paging logic
  auto* k = a.bt ? scan_kernel<GP, SKP, SVP, true> : scan_kernel<GP, SKP, SVP, false>;
  if (ensure_smem_limit(k, smem) != cudaSuccess) return ZKV_ERR_CUDA;
  if (launch_pdl(k, dim3(a.grid), dim3(kScanThreads), smem, st, a) != cudaSuccess)
    return ZKV_ERR_CUDA;
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

int launch_append_cluster(const zkv_append_params& p, cudaStream_t st, bool pdl);   // append.cu

// ap == nullptr: one decode call.  Otherwise the serving step: the tables (which depend only on
// q and the key codebooks) and the partition (on the lengths this step's append produces) run
// while the evicted tokens are encoded; scan block 0 stores the new lengths.
template <int D, int GP>
static int launch_decode(DecodeArgs a, const DecodePlan& pl, void* const* ev, cudaStream_t st,
                         const zkv_append_params* ap) {
  // 1. tables and partition (with the serving step's encode in between)
  trace(ev, 0, st);
  {
    // a decode call splits each pair's window into tile-sized parts (more, shorter blocks: the
    // scan waits for this kernel); the serving step keeps one block per pair (this kernel runs
    // beside the append, whose clusters need the SMs more)
    if (ap) {
      a.wparts = 1;
      a.wtok = (int)std::min<int64_t>(a.Wcap, 0x7fffffff);
    }
    const size_t smem = std::max(sizeof(LutSmem<D>), a.wparts == 1
                                                         ? window_smem_bytes<D, GP>()
                                                         : window_smem_bytes<D, GP, win_tile_part_c<D>()>());
    if (ensure_smem_limit(lut_kernel<D, GP>, smem) != cudaSuccess) return ZKV_ERR_CUDA;
    const int n_hg = (a.B * a.G + kLutH - 1) / kLutH;
    // two codewords per thread when that still leaves at least 64 table blocks (fewer, longer
    // blocks cost more than they save on small problems)
    a.lut_cpt = lut_cpt<D>() > 1 && (kCodebook / lut_c<D>()) * a.Sk * a.Hkv * n_hg >= 64 ? lut_cpt<D>() : 1;
    a.n_lut_blocks = (kCodebook / (64 * a.lut_cpt)) * a.Sk * a.Hkv * n_hg;
    // + the partition block + one window block per (sequence, kv head, window part)
    const int64_t blocks = (int64_t)a.n_lut_blocks + 1 + (int64_t)a.B * a.Hkv * a.wparts;
    if (blocks > 0x7fffffff) return ZKV_ERR_UNSUPPORTED;
    // a normal launch: the caller's preceding work (which may write q) must be complete, since
    // the table blocks do not wait
    lut_kernel<D, GP><<<(unsigned)blocks, 256, smem, st>>>(a);
    ZKV_CHECK_LAUNCH();
    if (ap) {
      // its completion implies the table kernel's (it waits for it before exiting)
      const int rc = launch_append_cluster(*ap, st, true);
      if (rc != ZKV_OK) return rc;
    }
  }
  // 2. scan
  trace(ev, 1, st);
  if (pl.scan2) {
    // heads in passes of at most four
    const int rc = GP == 1 ? launch_scan2_kv<1>(a, st) : GP == 2 ? launch_scan2_kv<2>(a, st)
                                                                 : launch_scan2_kv<4>(a, st);
    if (rc != ZKV_OK) return rc;
  } else {
    int rc;
    switch (GP) {
      case 1: rc = launch_scan_kv<1>(a, pl.SKP, pl.SVP, pl.scan_smem, st); break;
      case 2: rc = launch_scan_kv<2>(a, pl.SKP, pl.SVP, pl.scan_smem, st); break;
      case 4: rc = launch_scan_kv<4>(a, pl.SKP, pl.SVP, pl.scan_smem, st); break;
      default: rc = launch_scan_kv<8>(a, pl.SKP, pl.SVP, pl.scan_smem, st); break;
    }
    if (rc != ZKV_OK) return rc;
  }
  // 3. value contraction and the final combine with the window partials
  trace(ev, 2, st);
  {
    const size_t smem = combine_smem_bytes(a.grid, GP, D, a.qc);
    auto* k = combine_kernel<D, GP>;
    if (ensure_smem_limit(k, smem) != cudaSuccess) return ZKV_ERR_CUDA;
    const dim3 grid((unsigned)(a.Sv * a.qc), (unsigned)(a.B * a.Hkv));
    if (launch_pdl(k, grid, dim3(256), smem, st, a) != cudaSuccess) return ZKV_ERR_CUDA;
  }
  trace(ev, 3, st);
  return ZKV_OK;
}

template <int D>
static int launch_decode_g(const DecodeArgs& a, const DecodePlan& pl, void* const* ev,
                           cudaStream_t st, const zkv_append_params* ap) {
  switch (pl.GP) {
    case 1: return launch_decode<D, 1>(a, pl, ev, st, ap);
    case 2: return launch_decode<D, 2>(a, pl, ev, st, ap);
    case 4: return launch_decode<D, 4>(a, pl, ev, st, ap);
    default: return launch_decode<D, 8>(a, pl, ev, st, ap);
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
  if (p->Tcap > (int64_t(1) << 28)) return ZKV_ERR_UNSUPPORTED;   // 32-bit in-pair offsets
  return validate_paged(p->block_table, p->page_tokens, p->max_pages, p->n_pages, p->Tcap);
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

namespace zkv {
int validate_append(const zkv_append_params* p);   // append.cu

// Shared by the decode call and the serving step (ap != nullptr).
static int decode_common(const zkv_decode_params* p, void* workspace, size_t workspace_bytes,
                         void* stream, const zkv_append_params* ap) {
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
  a.GP = pl.GP; a.seg_cost = pl.seg_cost;
  a.upd_win_len = ap ? ap->win_len : nullptr;
  a.upd_win_head = ap ? ap->win_head : nullptr;
  a.upd_comp_len = ap ? ap->comp_len : nullptr;
  a.new_k = ap ? reinterpret_cast<const __half*>(ap->new_k) : nullptr;
  a.new_v = ap ? reinterpret_cast<const __half*>(ap->new_v) : nullptr;
  a.Tcap = p->Tcap; a.Wcap = p->Wcap; a.max_comp = p->max_comp_len;
  const float scale = p->softmax_scale > 0.f ? p->softmax_scale : (float)(1.0 / std::sqrt((double)p->d));
  a.scale_log2 = scale * kLog2e;
  a.rot = 1.0 / std::sqrt((double)p->d);
  a.q = reinterpret_cast<const __half*>(p->q);
  a.k_codes = p->k_codes; a.v_codes = p->v_codes; a.comp_len = p->comp_len;
  a.bt = p->block_table; a.max_pages = p->max_pages; a.n_pages = p->n_pages;
  a.pshift = p->block_table ? log2_pow2(p->page_tokens) : 0;
  a.Ck = p->k_codebooks; a.Cv = p->v_codebooks; a.k_smooth = p->k_smooth;
  a.win_k = reinterpret_cast<const __half*>(p->win_k);
  a.win_v = reinterpret_cast<const __half*>(p->win_v);
  a.win_len = p->win_len; a.out = p->out; a.lse = p->lse; a.err = p->error_flag;
  a.lut = reinterpret_cast<float*>(ws + pl.off_lut);
  a.pre = reinterpret_cast<int64_t*>(ws + pl.off_pre);
  a.bounds = reinterpret_cast<int64_t*>(ws + pl.off_bounds);
  a.ctap = reinterpret_cast<int32_t*>(ws + pl.off_ctap);
  a.vs = reinterpret_cast<int64_t*>(ws + pl.off_vs);
  a.pfirst = reinterpret_cast<int32_t*>(ws + pl.off_pfirst);
  a.plast = reinterpret_cast<int32_t*>(ws + pl.off_plast);
  a.pm = reinterpret_cast<float*>(ws + pl.off_pm);
  a.pl = reinterpret_cast<float*>(ws + pl.off_pl);
  a.pw = reinterpret_cast<float*>(ws + pl.off_pw);
  a.wm = reinterpret_cast<float*>(ws + pl.off_wm);
  a.wl = reinterpret_cast<float*>(ws + pl.off_wl);
  a.wo = reinterpret_cast<float*>(ws + pl.off_wo);
  a.wparts = pl.wparts;
  a.wtok = pl.wtok;
  a.so = reinterpret_cast<float*>(ws + pl.off_so);
  a.cnt = reinterpret_cast<int32_t*>(ws + pl.off_cnt);
  a.qc = pl.qc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  switch (p->d) {
    case 64: return launch_decode_g<64>(a, pl, p->trace_events, st, ap);
    case 128: return launch_decode_g<128>(a, pl, p->trace_events, st, ap);
    default: return launch_decode_g<256>(a, pl, p->trace_events, st, ap);
  }
}

}  // namespace zkv

extern "C" int zkv_rvq_decode_attn(const zkv_decode_params* p, void* workspace,
                                   size_t workspace_bytes, void* stream) {
  return decode_common(p, workspace, workspace_bytes, stream, nullptr);
}

extern "C" int zkv_rvq_serve_step(const zkv_append_params* ap, const zkv_decode_params* dp,
                                  void* workspace, size_t workspace_bytes, void* stream) {
  const int va = validate_append(ap);
  if (va != ZKV_OK) return va;
  const int vd = validate_decode(dp);
  if (vd != ZKV_OK) return vd;
  // one cache: the same shapes and the same buffers
  if (ap->B != dp->B || ap->Hkv != dp->Hkv || ap->d != dp->d || ap->Sk != dp->Sk ||
      ap->Sv != dp->Sv || ap->Tcap != dp->Tcap || ap->Wcap != dp->Wcap)
    return ZKV_ERR_INVALID_ARG;
  if (ap->k_codes != dp->k_codes || ap->v_codes != dp->v_codes ||
      ap->k_codebooks != dp->k_codebooks || ap->v_codebooks != dp->v_codebooks ||
      ap->win_k != dp->win_k || ap->win_v != dp->win_v || ap->win_len != dp->win_len ||
      ap->comp_len != dp->comp_len || ap->k_smooth != dp->k_smooth)
    return ZKV_ERR_INVALID_ARG;
  if (ap->block_table != dp->block_table ||
      (ap->block_table && (ap->page_tokens != dp->page_tokens || ap->max_pages != dp->max_pages ||
                           ap->n_pages != dp->n_pages)))
    return ZKV_ERR_INVALID_ARG;
  return decode_common(dp, workspace, workspace_bytes, stream, ap);
}

namespace zkv {
// ------------------------------------------------------------------------------------------
// Product-VQ decode: validation, workspace, launch.
// ------------------------------------------------------------------------------------------
struct PqPlan {
  int G, GP, n_chunks;
  size_t off_cm, off_cl, off_co, off_wm, off_wl, off_wo, total;
};

// Largest padded GQA group of a (d, m) instantiation: the scan holds G*m query values and
// G*m accumulators per lane (registers), and its warp partials take 8*G*d floats of shared
// memory next to the two 256*m codebooks.
constexpr int pq_max_gp(int d, int m) { return d == 256 ? 2 : (m == 8 ? 4 : 8); }

// d / m = 32 (one token per warp step) or 16 (two tokens, one per 16-lane group)
static bool pq_shape_supported(int d, int m, int GP) {
  const bool dm = (d == 64 && (m == 2 || m == 4)) || (d == 128 && (m == 4 || m == 8)) ||
                  (d == 256 && m == 8);
  return dm && GP <= pq_max_gp(d, m);
}

static int validate_pq_shapes(const zkv_pq_decode_params* p) {
  if (!p) return ZKV_ERR_INVALID_ARG;
  if (p->B < 1 || p->Hq < 1 || p->Hkv < 1 || p->Hq % p->Hkv) return ZKV_ERR_INVALID_ARG;
  if (p->Hq / p->Hkv > 8) return ZKV_ERR_UNSUPPORTED;
  if (!pq_shape_supported(p->d, p->m, pad_heads(p->Hq / p->Hkv))) return ZKV_ERR_UNSUPPORTED;
  if (p->B > 65535 || p->Hkv > 65535 || (int64_t)p->B * p->Hkv > 65535) return ZKV_ERR_UNSUPPORTED;
  if (p->Tcap < 0 || p->Wcap < 0 || p->max_comp_len < 0 || p->max_comp_len > p->Tcap)
    return ZKV_ERR_INVALID_ARG;
  if (p->Tcap > (int64_t(1) << 28)) return ZKV_ERR_UNSUPPORTED;
  return ZKV_OK;
}

static PqPlan make_pq_plan(const zkv_pq_decode_params* p) {
  PqPlan pl{};
  pl.G = p->Hq / p->Hkv;
  pl.GP = pad_heads(pl.G);
  pl.n_chunks = (int)std::max<int64_t>(1, (p->max_comp_len + kPqChunk - 1) / kPqChunk);
  const size_t pairs = (size_t)p->B * p->Hkv, f = sizeof(float);
  size_t o = 0;
  pl.off_cm = o; o = align256(o + pairs * pl.n_chunks * pl.GP * f);
  pl.off_cl = o; o = align256(o + pairs * pl.n_chunks * pl.GP * f);
  pl.off_co = o; o = align256(o + pairs * pl.n_chunks * pl.GP * p->d * f);
  pl.off_wm = o; o = align256(o + pairs * pl.GP * f);
  pl.off_wl = o; o = align256(o + pairs * pl.GP * f);
  pl.off_wo = o; o = align256(o + pairs * pl.GP * p->d * f);
  pl.total = o;
  return pl;
}

template <int D, int M, int GP>
static int launch_pq(const PqArgs& a, const DecodeArgs& w, cudaStream_t st) {
  const int pairs = a.B * a.Hkv;
  pq_scan_kernel<D, M, GP><<<dim3((unsigned)a.n_chunks, (unsigned)pairs), 256, 0, st>>>(a);
  ZKV_CHECK_LAUNCH();
  const size_t fsmem = window_smem_bytes<D, GP>();
  if (ensure_smem_limit(pq_finalize_kernel<D, GP>, fsmem) != cudaSuccess) return ZKV_ERR_CUDA;
  pq_finalize_kernel<D, GP><<<(unsigned)pairs, 256, fsmem, st>>>(a, w);
  ZKV_CHECK_LAUNCH();
  return ZKV_OK;
}

template <int D, int M>
static int launch_pq_g(int GP, const PqArgs& a, const DecodeArgs& w, cudaStream_t st) {
  constexpr int kMax = pq_max_gp(D, M);
  switch (GP) {
    case 1: return launch_pq<D, M, 1>(a, w, st);
    case 2: return launch_pq<D, M, 2>(a, w, st);
    case 4: if constexpr (kMax >= 4) return launch_pq<D, M, 4>(a, w, st); else return ZKV_ERR_UNSUPPORTED;
    default: if constexpr (kMax >= 8) return launch_pq<D, M, 8>(a, w, st); else return ZKV_ERR_UNSUPPORTED;
  }
}

}  // namespace zkv

extern "C" size_t zkv_pq_decode_workspace_size(const zkv_pq_decode_params* p) {
  if (validate_pq_shapes(p) != ZKV_OK) return 0;
  return make_pq_plan(p).total;
}

extern "C" int zkv_pq_decode_attn(const zkv_pq_decode_params* p, void* workspace,
                                  size_t workspace_bytes, void* stream) {
  const int v = validate_pq_shapes(p);
  if (v != ZKV_OK) return v;
  if (!p->q || !p->comp_len || !p->win_len || !p->out || !p->k_codes || !p->v_codes ||
      !p->k_codebook || !p->v_codebook)
    return ZKV_ERR_INVALID_ARG;
  if (p->Wcap > 0 && (!p->win_k || !p->win_v)) return ZKV_ERR_INVALID_ARG;
  if (((uintptr_t)p->q | (uintptr_t)p->win_k | (uintptr_t)p->win_v) & 15) return ZKV_ERR_INVALID_ARG;
  const PqPlan pl = make_pq_plan(p);
  if (!workspace || workspace_bytes < pl.total || ((uintptr_t)workspace & 255))
    return ZKV_ERR_WORKSPACE;
  unsigned char* ws = reinterpret_cast<unsigned char*>(workspace);
  const float scale = p->softmax_scale > 0.f ? p->softmax_scale : (float)(1.0 / std::sqrt((double)p->d));
  PqArgs a{};
  a.B = p->B; a.Hq = p->Hq; a.Hkv = p->Hkv; a.G = pl.G; a.d = p->d; a.m = p->m;
  a.n_chunks = pl.n_chunks; a.Tcap = p->Tcap; a.max_comp = p->max_comp_len;
  a.scale_log2 = scale * kLog2e;
  a.rot = 1.0 / std::sqrt((double)p->d);
  a.q = reinterpret_cast<const __half*>(p->q);
  a.k_codes = p->k_codes; a.v_codes = p->v_codes; a.comp_len = p->comp_len;
  a.Ck = p->k_codebook; a.Cv = p->v_codebook; a.k_smooth = p->k_smooth; a.err = p->error_flag;
  a.cm = reinterpret_cast<float*>(ws + pl.off_cm);
  a.cl = reinterpret_cast<float*>(ws + pl.off_cl);
  a.co = reinterpret_cast<float*>(ws + pl.off_co);
  // the window attention and the output go through the decode's own argument block
  DecodeArgs w{};
  w.B = p->B; w.Hq = p->Hq; w.Hkv = p->Hkv; w.G = pl.G; w.d = p->d;
  w.Wcap = p->Wcap; w.Tcap = p->Tcap;
  w.scale_log2 = a.scale_log2; w.rot = a.rot;
  w.q = a.q;
  w.win_k = reinterpret_cast<const __half*>(p->win_k);
  w.win_v = reinterpret_cast<const __half*>(p->win_v);
  w.win_len = p->win_len; w.out = p->out; w.lse = p->lse; w.err = p->error_flag;
  w.wm = reinterpret_cast<float*>(ws + pl.off_wm);
  w.wl = reinterpret_cast<float*>(ws + pl.off_wl);
  w.wo = reinterpret_cast<float*>(ws + pl.off_wo);
  w.wparts = 1;                                 // one part: the whole window, tile by tile
  w.wtok = (int)std::min<int64_t>(p->Wcap, 0x7fffffff);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  switch (p->d * 100 + p->m) {   // the shapes validate_pq_shapes admits
    case 6402: return launch_pq_g<64, 2>(pl.GP, a, w, st);
    case 6404: return launch_pq_g<64, 4>(pl.GP, a, w, st);
    case 12804: return launch_pq_g<128, 4>(pl.GP, a, w, st);
    case 12808: return launch_pq_g<128, 8>(pl.GP, a, w, st);
    default: return launch_pq_g<256, 8>(pl.GP, a, w, st);
  }
}

// ------------------------------------------------------------------------------------------
// Allocation-free variant: the workspace is a fixed module-scope device array.
//
// For callers that cannot hand the library a device buffer: a host program that links only
// this library and the CUDA runtime and keeps no device allocator of its own, or an engine
// that reserves all of its device memory up front and has no pool to carve a per-call
// workspace from.  Such callers get one resident array of ZKV_DECODE_SCRATCH_BYTES per device
// (allocated by the driver when the module loads) instead of a buffer they own.
//
// Nothing in the array has to start at zero: every word a call reads is written earlier in
// the same call.  There is one array per
// device, so calls on one device that overlap in time (two streams, two host threads) race
// on it; the caller orders them.
// ------------------------------------------------------------------------------------------
namespace zkv {

static __device__ __align__(256) unsigned char g_decode_scratch[ZKV_DECODE_SCRATCH_BYTES];

// Device address of g_decode_scratch on the current device.  Looked up at every call (a
// host-side lookup): after a device reset the module loads again, possibly at a new address.
static void* decode_scratch_address() {
  void* a = nullptr;
  if (cudaGetSymbolAddress(&a, g_decode_scratch) != cudaSuccess) return nullptr;
  return a;
}

}  // namespace zkv

extern "C" int zkv_rvq_decode_attn_noalloc(const zkv_decode_params* p, void* stream) {
  const int v = validate_decode(p);
  if (v != ZKV_OK) return v;
  if (make_plan(p).total > (size_t)ZKV_DECODE_SCRATCH_BYTES) return ZKV_ERR_WORKSPACE;
  void* ws = decode_scratch_address();
  if (!ws) return ZKV_ERR_CUDA;
  return zkv_rvq_decode_attn(p, ws, (size_t)ZKV_DECODE_SCRATCH_BYTES, stream);
}
