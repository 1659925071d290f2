// Scan of the compressed tokens, token-per-thread design (sm_100a).  Included by decode.cu.
//
// Passages: VQKV (gist.science summary of arXiv 2603.16435), section 2.3 "Decoding Stage":
// the codes are read directly and keys / values are reconstructed on demand inside attention;
// VeloxQuant-MLX 0.5.1, "VecInfer": the rotation is absorbed into the query, so a key score is
// a sum of per-stage table entries (q_tilde . Ck_s[z_s]).
//
// Every thread takes groups of U consecutive tokens (U = 2 at four heads with packed codes of at
// least two bytes, else 4) of one (sequence, kv head) segment end to end: the key score of each
// token for up to four query heads (one table gather per key stage), p = 2^(score - reference)
// for those heads, and the value side as per-codeword weight histograms W_s[c] += p (one
// shared-memory integer reduction per value stage and head).  No token is staged through shared
// memory and no warp waits for another between tokens: sub-chunks of 512 U tokens run in
// barrier-free runs, and the block meets only between runs.
//
// Shared memory (absolute addresses of the CTA's window; dynamic shared memory begins at 1 KB,
// after the reserved system area, and this kernel asks for everything below 224 KB):
//   [base, 64K)   block scratch: maxima, sums, float32 master histograms, the list of tokens
//                 above the reference (their key code words), its counts, the warps' p sums
//   [64K, 128K)   key tables: 256 rows (codewords) of 256 bytes; row c holds, for every key
//                 stage s and table copy k, the GPH float32 entries of codeword c, stored with
//                 the heads rotated by k mod GPH.  Entry (c, s, k) sits at 64K + 256 c +
//                 (s RK + k) 4 GPH.
//   [128K, 192K)  value histograms: 256 rows of 64 uint32 words; word 8/GPH... see below.
//   [192K, 224K)  the listed tokens' value code words
// Because every row is 256 bytes and each region starts at a multiple of 64 KB, the address
// of a table entry is one byte permutation: [column byte | code byte | region | 0] -- the code
// byte comes straight from the token's packed codes, the other bytes from a per-lane register.
//
// Bank conflicts.  A lane uses table copy k = lane mod RK (so its scores come out with the heads
// rotated by lg = lane mod GPH) and visits the key stages in the order s = (i + lane / RK) mod
// SKP; within one gather instruction the lanes of every shared-memory phase hit distinct banks.
// Value histograms: lane = (lg, ls, r) with ls the value-stage rotation and r a replica index
// (R = 32 / (GPH SVP) replicas).  At step (i, j) the lane adds the p of head (j + lg) mod GPH of
// its token to stage s = (i + ls) mod SVP, codeword z_s, in column ALPHA (j + lg) + s R + r of
// row z_s (ALPHA = 32 / GPH): "virtual head" hv = j + lg runs to 2 GPH - 2 without wrapping, so
// the per-head offset is an immediate; word (s, c, hv, r) counts for head hv mod GPH.  For fixed
// (i, j) the 32 lanes cover 32 distinct banks.  Columns stay below 64: one 256-byte row.
//
// Fixed point.  Each p is added as an integer u = floor(p 2^20 + d), d in [0, 1) a fixed dither
// spread over the lanes of a warp: every score added is <= ref (a larger one
// makes the block raise ref first), so u <= 2^20, and the rounding errors are unbiased in
// aggregate (plain rounding would drop the mass of the many tokens with p below 2^-21).  The sum
// of n rounding errors has a standard deviation near 2^-20 sqrt(n / 12) of the largest p.  A word
// collects at most one u per token of the lanes of its replica, i.e. at most 512 U / R tokens per
// sub-chunk, so a run of at most 8 R / U - 1 sub-chunks cannot take a zero word past 2^32.  The
// words are folded into float32 masters only when the next run could: every word holds at most
// the sum of the u added since the last fold, and every thread keeps the sum of its p, so at
// each run boundary the block knows that bound and shortens the next run, or folds, when the
// bound plus the next run's worst case would pass 2^32.

// Reference: the first sub-chunk's block maximum plus a headroom (kS2Headroom, log2 units).
// Sub-chunks take block i of every warp's contiguous run of the segment, so that first sub-chunk
// samples the whole segment.  A later token whose score is above the reference is listed (its
// code words copied from the registers that hold them) and contributes nothing during its run;
// at the run's end the block takes the listed tokens' maximum plus the headroom as the new
// reference, folds the integer words into the masters rescaled by 2^(old - new), and adds the
// listed tokens.
//
// Output (one slot per (scan CTA, pair)): maxima pm = the reference (log2 units), sums pl, and
// float32 histograms pw[slot][Sv][256][GP] relative to pm -- the partial format the combine
// kernel reads.  Query-head groups larger than four are taken in passes of four heads over the
// same segment.
#pragma once

// (included inside namespace zkv; the kS2* constants are defined beside the plan in decode.cu)

constexpr int ilog2c(int x) { return x <= 1 ? 0 : 1 + ilog2c(x / 2); }

// Compile-time loop: f(std::integral_constant<int, i>) for i = 0 .. N-1, so that register arrays
// indexed by i stay plain registers however large the body is.
template <class F, int... I>
__device__ __forceinline__ void static_for_impl(F&& f, std::integer_sequence<int, I...>) {
  (f(std::integral_constant<int, I>{}), ...);
}
template <int N, class F>
__device__ __forceinline__ void static_for(F&& f) {
  static_for_impl(f, std::make_integer_sequence<int, N>{});
}

template <int GPH, int SKP, int SVP>
struct S2Cfg {
  static_assert(GPH == 1 || GPH == 2 || GPH == 4, "heads per pass");
  static_assert(SKP == 1 || SKP == 2 || SKP == 4, "key stages");
  static_assert(SVP == 1 || SVP == 2 || SVP == 4, "value stages");
  static constexpr int LG = ilog2c(GPH), LSK = ilog2c(SKP), LSV = ilog2c(SVP);
  static constexpr int RK = 64 / (SKP * GPH) < 32 ? 64 / (SKP * GPH) : 32;   // key table copies
  static constexpr int LRK = ilog2c(RK);
  static constexpr int R = 32 / (GPH * SVP);      // value histogram replicas
  static constexpr int ALPHA = 32 / GPH;          // value columns per virtual head
  // tokens per thread and sub-chunk: two for four-head groups with packed codes of at least
  // two bytes (fewer live registers), else four (whole 32-bit code words)
  static constexpr int U = (GPH == 4 && SKP >= 2 && SVP >= 2) ? 2 : 4;
  static constexpr int KW = U * SKP / 4;          // code words of a thread's U tokens
  static constexpr int VW = U * SVP / 4;
  static constexpr int NENT = SVP * kCodebook * GPH;   // histogram entries of one pass
  static constexpr int NE = (NENT + kS2Threads - 1) / kS2Threads;
  // a word takes <= 512 U / R tokens of <= 2^20 each per sub-chunk: runs from a zero word stay
  // below 2^32
  static constexpr int FOLD_EVERY = (8 / U) * R - 1;    // sub-chunks in the longest run
  static constexpr float WSUB = (float)(kS2Threads * U / R) * 1048577.f;   // per word, sub-chunk
  static constexpr int NW = kS2Threads / 32;
  static constexpr int SUBT = kS2Threads * U;    // tokens per sub-chunk
  static constexpr int LCAP = 8192;               // exception list entries
  // sub-chunks per run between block-wide steps: the capacity schedule, and at most one list's
  // worth of scores (a run scores RUN sub-chunks)
  static constexpr int RUN = FOLD_EVERY < LCAP / SUBT - 1 ? FOLD_EVERY : LCAP / SUBT - 1;
  static_assert(RK >= GPH, "every head rotation has its own copy");
};

// 2^x, approximate; results below the smallest normal float flush to zero (such p are far
// below the fixed-point resolution anyway).
__device__ __forceinline__ float ex2_ftz(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ uint32_t prmt_b32(uint32_t a, uint32_t b, uint32_t s) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(s));
  return d;
}
// Two independent float32 additions in one instruction (each rounded as a scalar add).
__device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}
template <int OFF>
__device__ __forceinline__ void red_u32_at(uint32_t a, uint32_t v) {
  // no memory clobber: the histograms are read only after a barrier
  asm volatile("red.shared.add.u32 [%0+%2], %1;" ::"r"(a), "r"(v), "n"(OFF));
}
__device__ __forceinline__ uint4 lds128u_v(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a) : "memory");
  return v;
}
__device__ __forceinline__ void sts128z(uint32_t a) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(a), "r"(0u) : "memory");
}

// Packed codes of a thread's token group t .. t + U - 1 (t a multiple of U, U = 2 or 4; S bytes
// per token) as NW words; zero when t >= tend or the page is invalid.  The group lies inside one
// row block (a pair's Tcap or a page, both multiples of 16 tokens), so one aligned vector load
// reads it.
template <int NW, bool PAGED>
__device__ __forceinline__ void load_group(const DecodeArgs& a, const PairRows& pr, int S,
                                           uint32_t t, uint32_t tend, uint32_t (&w)[NW]) {
#pragma unroll
  for (int q = 0; q < NW; ++q) w[q] = 0u;
  if (t >= tend) return;
  const uint8_t* row = pair_row<PAGED>(a, pr, t, S);
  if (!row) return;
  if constexpr (NW == 1) {
    w[0] = __ldg(reinterpret_cast<const unsigned int*>(row));
  } else if constexpr (NW == 2) {
    const uint2 v = __ldg(reinterpret_cast<const uint2*>(row));
    w[0] = v.x; w[1] = v.y;
  } else {
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(row));
    w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
  }
}

template <int GPH, int SKP, int SVP, bool PAGED>
__global__ void __launch_bounds__(kS2Threads, 1) scan2_kernel(DecodeArgs a) {
  using C = S2Cfg<GPH, SKP, SVP>;
  constexpr int U = C::U;
  constexpr uint32_t KR = kS2KeyRegion, VR = kS2ValRegion;
  extern __shared__ __align__(16) unsigned char smraw[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // the combine kernel may be scheduled now: its blocks take the SMs this grid leaves (every
  // block of this grid is resident, one per SM, by the time all have passed here) and stage
  // their codebook chunks before waiting for this grid's completion
  pdl_trigger();
  const uint32_t sbase = smem_u32(smraw);
  uint32_t dyn;
  asm("mov.u32 %0, %%dynamic_smem_size;" : "=r"(dyn));
  // block scratch at the start of dynamic shared memory
  uint32_t* redk = reinterpret_cast<uint32_t*>(smraw);                    // [2][NW][GPH] maxima
  float* reds = reinterpret_cast<float*>(smraw + 8 * C::NW * GPH);          // [NW][GPH] sums
  float* mst = reinterpret_cast<float*>(smraw + 12 * C::NW * GPH);   // masters [256][SVP][GPH]
  // exception list: the key code words of the tokens whose score exceeded the reference (each
  // shifted so that the token's codes are its low bytes; their value words, likewise, sit at
  // kS2ExvRegion), and its count
  uint32_t* exk = reinterpret_cast<uint32_t*>(smraw + 12 * C::NW * GPH + 4 * C::NE * kS2Threads);
  uint32_t* exn = exk + C::LCAP;                                // [2] counts (runs alternate)
  float* redp = reinterpret_cast<float*>(exn + 4);              // [2][NW] warps' p sums
  constexpr uint32_t XV = kS2ExvRegion;
  const bool fits = sbase + 12u * C::NW * GPH + 4u * C::NE * kS2Threads + 4u * C::LCAP + 16u +
                            8u * C::NW <= KR &&
                    sbase + dyn >= XV + 4u * C::LCAP;
  if (fits) {
    // zero the value histograms (the final fold of every segment leaves them zero again)
    for (uint32_t o = VR + 16u * tid; o < VR + 65536u; o += 16u * kS2Threads) sts128z(o);
  }
  if (fits && tid == 0) {
    // Warm the address translations of this CTA's approximate share of the codes and tables
    // while the previous kernel still runs: a prefetch needs none of its results, and a first
    // touch of a cold page otherwise stalls the segment's first loads for microseconds.
    const int64_t np = (int64_t)a.B * a.Hkv;
    const int64_t pr0 = (int64_t)blockIdx.x * np / gridDim.x;
    if (!a.bt) {
      const int64_t kb = (pr0 * a.Tcap * a.Sk) & ~int64_t(15);
      const int64_t vb = (pr0 * a.Tcap * a.Sv) & ~int64_t(15);
      if (kb + 16 <= np * a.Tcap * a.Sk)
        asm volatile("cp.async.bulk.prefetch.L2.global [%0], 16;" ::"l"(a.k_codes + kb) : "memory");
      if (vb + 16 <= np * a.Tcap * a.Sv)
        asm volatile("cp.async.bulk.prefetch.L2.global [%0], 16;" ::"l"(a.v_codes + vb) : "memory");
    }
    const float* lp = a.lut + pr0 * a.Sk * kCodebook * a.GP;
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], 16;" ::"l"(lp) : "memory");
  }
  pdl_wait();   // tables, prefix sums and codes
  if (a.upd_comp_len && blockIdx.x == 0) {
    // serving step: the append has read the pre-step lengths; store the new ones (nothing in
    // this kernel reads them)
    for (int b = tid; b < a.B; b += kS2Threads)
      advance_lengths(b, a.Tcap, a.Wcap, a.upd_win_len, a.upd_win_head, a.upd_comp_len);
  }
  if (!fits) {
    if (tid == 0) set_error(a.err, ZKV_DEVERR_SMEM);
    return;
  }
  const int Sk = a.Sk, Sv = a.Sv, G = a.G, GP = a.GP;
  const int npairs = a.B * a.Hkv;
  const int64_t lo = a.bounds[blockIdx.x], hi = a.bounds[blockIdx.x + 1];
  // the pair holding this CTA's cut (the partition places it with the cut); lanes hold the
  // prefix starts of the next 32 pairs
  const int pfirst = a.ctap[blockIdx.x];
  if (lo >= hi) return;
  const int64_t pre_l = pfirst + lane <= npairs ? a.pre[pfirst + lane] : INT64_MAX;
  auto pre_at = [&](int pr) -> int64_t {   // a.pre[pr], pr >= pfirst (uniform across the block)
    return pr - pfirst < 32 ? __shfl_sync(0xffffffffu, pre_l, pr - pfirst) : a.pre[pr];
  };
  // ---- per-lane constants
  const uint32_t lg = (uint32_t)lane & (GPH - 1);
  const uint32_t kcopy = (uint32_t)lane & (C::RK - 1);
  const uint32_t lks = ((uint32_t)lane >> C::LRK) & (SKP - 1);
  const uint32_t lvs = ((uint32_t)lane >> C::LG) & (SVP - 1);
  const uint32_t vrep = (uint32_t)lane >> (C::LG + C::LSV);
  // column bytes of stage steps 2h, 2h + 1 in bytes 0, 1; the region in byte 2; 0 in byte 3
  uint32_t kcol[(SKP + 1) / 2], vcol[(SVP + 1) / 2];
#pragma unroll
  for (int h = 0; h < (SKP + 1) / 2; ++h) kcol[h] = (KR >> 16) << 16;
#pragma unroll
  for (int h = 0; h < (SVP + 1) / 2; ++h) vcol[h] = (VR >> 16) << 16;
#pragma unroll
  for (int i = 0; i < SKP; ++i) {
    const uint32_t s = ((uint32_t)i + lks) & (SKP - 1);
    kcol[i >> 1] |= ((s * C::RK + kcopy) * GPH * 4u) << (8 * (i & 1));
  }
#pragma unroll
  for (int i = 0; i < SVP; ++i) {
    const uint32_t s = ((uint32_t)i + lvs) & (SVP - 1);
    vcol[i >> 1] |= (4u * (C::ALPHA * lg + s * C::R + vrep)) << (8 * (i & 1));
  }
  // byte selectors: token u of the group, stage step i -> result [colreg byte i&1 | code byte |
  // colreg byte 2 | colreg byte 3]; the code byte of stage s of token u is byte (u S + s) mod 4 of
  // word (u S) / 4
  uint32_t ksel[4], vsel[4];
#pragma unroll
  for (int q = 0; q < 4 / SKP; ++q)
#pragma unroll
    for (int i = 0; i < SKP; ++i) {
      const uint32_t byte = (uint32_t)(q * SKP) + (((uint32_t)i + lks) & (SKP - 1));
      ksel[q * SKP + i] = (4u + (uint32_t)(i & 1)) | (byte << 4) | (6u << 8) | (7u << 12);
    }
#pragma unroll
  for (int q = 0; q < 4 / SVP; ++q)
#pragma unroll
    for (int i = 0; i < SVP; ++i) {
      const uint32_t byte = (uint32_t)(q * SVP) + (((uint32_t)i + lvs) & (SVP - 1));
      vsel[q * SVP + i] = (4u + (uint32_t)(i & 1)) | (byte << 4) | (6u << 8) | (7u << 12);
    }
  // Dithered rounding: u = floor(p 2^20 + d) with d in [0, 1) fixed per lane and spread evenly
  // over the warp (bit-reversed lane index), so the rounding errors of the tokens have mean zero
  // in aggregate instead of every small p rounding down (computed as round-to-nearest of
  // p 2^20 + d - 1/2).
  const float dith = ((float)(__brev((uint32_t)lane) >> 27) + 0.5f) * (1.f / 32.f) - 0.5f;

  // ---- the pieces of the loop
  // this thread's sum of the p it has added to the words since the last fold (all heads)
  float2 ps2 = make_float2(0.f, 0.f);
  // score of token u of a group, heads rotated by lg; init = -(reference - 20) per rotated head
  auto key_score1 = [&](auto uc, const uint32_t (&wk)[C::KW], const float (&init)[GPH],
                        float (&scu)[GPH]) {
    constexpr int u = decltype(uc)::value;
    static_for<GPH>([&](auto jc) { scu[jc] = init[jc]; });
    static_for<SKP>([&](auto ic) {
      constexpr int i = ic;
      const uint32_t x = prmt_b32(wk[(u * SKP) >> 2], kcol[i >> 1],
                                  ksel[(u & (4 / SKP - 1)) * SKP + i]);
      if constexpr (GPH == 4) {
        const float4 e = lds128f(x);
        const float2 s01 = fadd2(make_float2(scu[0], scu[1]), make_float2(e.x, e.y));
        const float2 s23 = fadd2(make_float2(scu[2], scu[3]), make_float2(e.z, e.w));
        scu[0] = s01.x; scu[1] = s01.y; scu[2] = s23.x; scu[3] = s23.y;
      } else if constexpr (GPH == 2) {
        const float2 e = lds64f(x);
        const float2 s01 = fadd2(make_float2(scu[0], scu[1]), e);
        scu[0] = s01.x; scu[1] = s01.y;
      } else {
        scu[0] += lds32f(x);
      }
    });
  };
  auto key_scores = [&](const uint32_t (&wk)[C::KW], const float (&init)[GPH],
                        float (&sc)[U][GPH]) {
    static_for<U>([&](auto uc) { key_score1(uc, wk, init, sc[uc]); });
  };
  // the value side of token u: p 2^20 = 2^x with x = score - ref + 20, rounded (dithered) to an
  // integer, added to the histograms
  auto value_red1 = [&](auto uc, const uint32_t (&wv)[C::VW], const float (&scu)[GPH]) {
    constexpr int u = decltype(uc)::value;
    // 1.5 * 2^23: adding it rounds [-2^22, 2^22) to an integer held in the low mantissa bits
    const float magic = 12582912.f;
    uint32_t pu[GPH];
    if constexpr (GPH >= 2) {
      static_for<GPH / 2>([&](auto hc) {
        constexpr int j = 2 * hc;
        const float2 pp = make_float2(ex2_ftz(scu[j]), ex2_ftz(scu[j + 1]));
        ps2 = fadd2(ps2, pp);
        float2 e = fadd2(pp, make_float2(dith, dith));
        e = fadd2(e, make_float2(magic, magic));
        pu[j] = __float_as_uint(e.x) - 0x4B400000u;
        pu[j + 1] = __float_as_uint(e.y) - 0x4B400000u;
      });
    } else {
      const float p0 = ex2_ftz(scu[0]);
      ps2.x += p0;
      pu[0] = __float_as_uint((p0 + dith) + magic) - 0x4B400000u;
    }
    static_for<SVP>([&](auto ic) {
      constexpr int i = ic;
      const uint32_t x = prmt_b32(wv[(u * SVP) >> 2], vcol[i >> 1],
                                  vsel[(u & (4 / SVP - 1)) * SVP + i]);
      red_u32_at<0>(x, pu[0]);
      if constexpr (GPH >= 2) red_u32_at<4 * C::ALPHA>(x, pu[1]);
      if constexpr (GPH >= 4) {
        red_u32_at<8 * C::ALPHA>(x, pu[2]);
        red_u32_at<12 * C::ALPHA>(x, pu[3]);
      }
    });
  };
  // tokens of the group outside [s0, s1) get x = -inf (p = 0, never a new maximum)
  auto mask_group = [&](float (&sc)[U][GPH], uint32_t t, uint32_t s0, uint32_t s1) {
    if (t >= s0 && t + U <= s1) return;
    static_for<U>([&](auto uc) {
      if (t + (uint32_t)uc < s0 || t + (uint32_t)uc >= s1)
        static_for<GPH>([&](auto jc) { sc[uc][jc] = -INFINITY; });
    });
  };
  // block maxima per head of per-thread maxima mt (unrotated); one barrier: the two buffers
  // alternate, and two calls are always separated by another barrier
  int rbuf = 0;
  auto block_max_of = [&](const float (&mt)[GPH], float (&m)[GPH]) {
    uint32_t* rk = redk + rbuf * C::NW * GPH;
    rbuf ^= 1;
#pragma unroll
    for (int g = 0; g < GPH; ++g) {
      const uint32_t k = __reduce_max_sync(0xffffffffu, ord_key(mt[g]));
      if (lane == 0) rk[warp * GPH + g] = k;
    }
    __syncthreads();
#pragma unroll
    for (int g = 0; g < GPH; ++g) {
      uint32_t k = 0u;
#pragma unroll
      for (int w = 0; w < C::NW; ++w) k = max(k, rk[w * GPH + g]);
      m[g] = ord_val(k);
    }
  };
  // fold a lane's rotated values x[j] (head (j + lg) mod GPH) into per-head maxima mt[g]
  auto unrotate_max = [&](const float (&x)[GPH], float (&mt)[GPH]) {
#pragma unroll
    for (int j = 0; j < GPH; ++j)
#pragma unroll
      for (int g = 0; g < GPH; ++g)
        if (((uint32_t)j + lg) % GPH == (uint32_t)g) mt[g] = fmaxf(mt[g], x[j]);
  };
  // the reference (minus 20) per head from the lane's rotated score start init = -ref_rot
  auto ref_of = [&](const float (&init)[GPH], float (&refk)[GPH]) {
#pragma unroll
    for (int g = 0; g < GPH; ++g) {
      refk[g] = 0.f;
#pragma unroll
      for (int j = 0; j < GPH; ++j)
        if (((uint32_t)j + lg) % GPH == (uint32_t)g) refk[g] = -init[j];
    }
  };
  // key score (rotated heads, relative to init) of token t from its key word
  auto key_score_w = [&](uint32_t w, uint32_t t, const float (&init)[GPH], float (&x)[GPH]) {
    const uint32_t q = t & (4u / SKP - 1u);   // the token's slot in its 32-bit code word
#pragma unroll
    for (int j = 0; j < GPH; ++j) x[j] = init[j];
#pragma unroll
    for (int i = 0; i < SKP; ++i) {
      const uint32_t byte = q * SKP + (((uint32_t)i + lks) & (SKP - 1));
      const uint32_t sel = (4u + (uint32_t)(i & 1)) | (byte << 4) | (6u << 8) | (7u << 12);
      const uint32_t adr = prmt_b32(w, kcol[i >> 1], sel);
      if constexpr (GPH == 4) {
        const float4 e = lds128f(adr);
        x[0] += e.x; x[1] += e.y; x[2] += e.z; x[3] += e.w;
      } else if constexpr (GPH == 2) {
        const float2 e = lds64f(adr);
        x[0] += e.x; x[1] += e.y;
      } else {
        x[0] += lds32f(adr);
      }
    }
  };
  // the value side of token t with rotated x (relative to the reference - 20), from its value
  // word
  auto value_red_w = [&](uint32_t w, uint32_t t, const float (&x)[GPH]) {
    const uint32_t q = t & (4u / SVP - 1u);
    const float magic = 12582912.f;
    uint32_t pu[GPH];
#pragma unroll
    for (int j = 0; j < GPH; ++j) {
      const float pj = ex2_ftz(x[j]);
      ps2.x += pj;
      pu[j] = __float_as_uint((pj + dith) + magic) - 0x4B400000u;
    }
#pragma unroll
    for (int i = 0; i < SVP; ++i) {
      const uint32_t byte = q * SVP + (((uint32_t)i + lvs) & (SVP - 1));
      const uint32_t sel = (4u + (uint32_t)(i & 1)) | (byte << 4) | (6u << 8) | (7u << 12);
      const uint32_t adr = prmt_b32(w, vcol[i >> 1], sel);
      red_u32_at<0>(adr, pu[0]);
      if constexpr (GPH >= 2) red_u32_at<4 * C::ALPHA>(adr, pu[1]);
      if constexpr (GPH >= 4) {
        red_u32_at<8 * C::ALPHA>(adr, pu[2]);
        red_u32_at<12 * C::ALPHA>(adr, pu[3]);
      }
    }
  };
  // Fold the integer words into the float32 masters mst[(c SVP + s) GPH + g] (each rescaled by
  // its head's factor) and zero them; called by the whole block after a barrier that follows the
  // last reduction.  A row is read as 16 chunks of four words: lane l of warp w takes chunk
  // k = l mod 16 of rows c = 2 w + l / 16 + 32 n (n < 8), so a warp reads two whole rows per
  // instruction, conflict-free.  Chunk k holds columns 4k .. 4k + 3 of virtual head hv = 4k / ALPHA:
  // one stage (R >= 4; the R replicas of an entry fill R / 4 neighbouring chunks) or two stages
  // (R = 2).  Replica sums across chunks and the head's second virtual slot (chunk k + 8, column
  // + 32) are combined with shuffles inside each 16-lane half; the lanes with hv < GPH (and the
  // first chunk of a replica group) own the entries.
  const uint32_t fk = (uint32_t)lane & 15u;                 // chunk
  const uint32_t fhv = (4u * fk) / C::ALPHA;                // its virtual head
  const uint32_t fs0 = ((4u * fk) % C::ALPHA) / C::R;       // its (first) stage
  constexpr int RG = C::R >= 4 ? C::R / 4 : 1;              // chunks per replica group
  const bool fown = fhv < GPH && (fk & (RG - 1)) == 0u;
  // (al: the rescale factor of this lane's head fhv; 1 for a plain capacity fold)
  auto fold = [&](float al) {
#pragma unroll 2
    for (int n = 0; n < 8; ++n) {
      const uint32_t c = 2u * (uint32_t)warp + ((uint32_t)lane >> 4) + 32u * (uint32_t)n;
      const uint32_t adr = VR + 256u * c + 16u * fk;
      const uint4 v = lds128u_v(adr);
      sts128z(adr);
      float v0, v1;
      if constexpr (C::R >= 4) {
        v0 = ((float)v.x + (float)v.y) + ((float)v.z + (float)v.w);
#pragma unroll
        for (int o = 1; o < RG; o <<= 1) v0 += __shfl_xor_sync(0xffffffffu, v0, o);
        v0 += __shfl_xor_sync(0xffffffffu, v0, 8);
        v1 = 0.f;
      } else {
        v0 = (float)v.x + (float)v.y;
        v1 = (float)v.z + (float)v.w;
        v0 += __shfl_xor_sync(0xffffffffu, v0, 8);
        v1 += __shfl_xor_sync(0xffffffffu, v1, 8);
      }
      if (fown) {
        float* mp = mst + ((int)c * SVP + (int)fs0) * GPH + (int)fhv;
        *mp = fmaf(v0, 0x1p-20f, *mp) * al;
        if constexpr (C::R == 2) {
          float* mq = mp + GPH;   // stage fs0 + 1
          *mq = fmaf(v1, 0x1p-20f, *mq) * al;
        }
      }
    }
    ps2 = make_float2(0.f, 0.f);   // the words are zero again
    __syncthreads();
  };

  for (int pr = pfirst; pr < npairs && pre_at(pr) < hi; ++pr) {
    const int64_t pr0 = pre_at(pr), pr1 = pre_at(pr + 1);
    const int64_t seg0 = lo > pr0 ? lo : pr0;
    const int64_t seg1 = hi < pr1 ? hi : pr1;
    if (seg0 >= seg1) continue;
    const uint32_t s0 = (uint32_t)(seg0 - pr0), s1 = (uint32_t)(seg1 - pr0);
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
    const uint32_t a0 = s0 & ~(uint32_t)(U - 1);
    const uint32_t ngrp = (s1 - a0 + U - 1) / U;
    const int nsub = (int)((ngrp + kS2Threads - 1) / kS2Threads);
    // warp w owns the contiguous run of nsub * 32 groups from a0 + 32 U w nsub; sub-chunk i
    // takes block i of every run
    constexpr uint32_t WSTEP = 32u * U;   // tokens of one warp block
    const uint32_t tw = a0 + (uint32_t)U * ((uint32_t)(warp * nsub) * 32u + (uint32_t)lane);
    const int npass = GP / GPH;
    for (int hp = 0; hp < npass; ++hp) {
      uint32_t kn[C::KW], vn[C::VW], vcur[C::VW], kx[C::KW];
      load_group<C::KW, PAGED>(a, kcb, Sk, tw, s1, kx);
      load_group<C::VW, PAGED>(a, vcb, Sv, tw, s1, vcur);
      load_group<C::KW, PAGED>(a, kcb, Sk, tw + WSTEP, s1, kn);
      load_group<C::VW, PAGED>(a, vcb, Sv, tw + WSTEP, s1, vn);
      __syncthreads();   // the previous pass's tables are no longer read
      // ---- key tables of (pair, heads 4 hp ..): item (entry e, copy k), copy fastest; the
      // source entry is the table kernel's [pair][s][c][GP] row; padded heads are zero
      {
        const float* src = a.lut + (int64_t)pr * Sk * kCodebook * GP + hp * 4;
        constexpr int ITEMS = SKP * kCodebook * C::RK;
        constexpr int NB = ITEMS / kS2Threads < 8 ? ITEMS / kS2Threads : 8;   // items in flight per thread
        static_assert(ITEMS % (kS2Threads * NB) == 0, "whole rounds");
#pragma unroll 1
        for (int f0 = 0; f0 < ITEMS; f0 += NB * kS2Threads) {
          float v[NB][GPH];
#pragma unroll
          for (int q = 0; q < NB; ++q) {
            const int f = f0 + q * kS2Threads + tid;
            const int e = f >> C::LRK;              // (c, s) with s fastest
            const int s = e & (SKP - 1), c = e >> C::LSK;
            const float* p = src + ((int64_t)s * kCodebook + c) * GP;
            if constexpr (GPH == 4) {
              const float4 t4 = __ldg(reinterpret_cast<const float4*>(p));
              v[q][0] = t4.x; v[q][1] = t4.y; v[q][2] = t4.z; v[q][3] = t4.w;
            } else if constexpr (GPH == 2) {
              const float2 t2 = __ldg(reinterpret_cast<const float2*>(p));
              v[q][0] = t2.x; v[q][1] = t2.y;
            } else {
              v[q][0] = __ldg(p);
            }
#pragma unroll
            for (int g = 0; g < GPH; ++g)
              if (hp * 4 + g >= G) v[q][g] = 0.f;
          }
#pragma unroll
          for (int q = 0; q < NB; ++q) {
            const int f = f0 + q * kS2Threads + tid;
            const uint32_t k = (uint32_t)f & (C::RK - 1);
            const int e = f >> C::LRK;
            const uint32_t s = (uint32_t)e & (SKP - 1), c = (uint32_t)e >> C::LSK;
            const uint32_t dst = KR + 256u * c + (s * C::RK + k) * GPH * 4u;
            // copy k holds the heads rotated by k mod GPH: o[j] = v[(j + k) mod GPH], built from
            // conditional rotations by 1 and 2 (no indexed register array)
            float o[GPH];
#pragma unroll
            for (int j = 0; j < GPH; ++j) o[j] = v[q][j];
            if constexpr (GPH >= 2) {
              if (k & 1u) {
                const float t0 = o[0];
#pragma unroll
                for (int j = 0; j < GPH - 1; ++j) o[j] = o[j + 1];
                o[GPH - 1] = t0;
              }
            }
            if constexpr (GPH == 4) {
              if (k & 2u) {
                float t = o[0]; o[0] = o[2]; o[2] = t;
                t = o[1]; o[1] = o[3]; o[3] = t;
              }
            }
            if constexpr (GPH == 4) {
              asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "f"(o[0]),
                           "f"(o[1]), "f"(o[2]), "f"(o[3]) : "memory");
            } else if constexpr (GPH == 2) {
              asm volatile("st.shared.v2.f32 [%0], {%1, %2};" ::"r"(dst), "f"(o[0]), "f"(o[1])
                           : "memory");
            } else {
              asm volatile("st.shared.f32 [%0], %1;" ::"r"(dst), "f"(o[0]) : "memory");
            }
          }
        }
      }
      if (tid < 2) exn[tid] = 0u;
      __syncthreads();   // tables ready; histograms are zero; the exception list is empty
#pragma unroll
      for (int k = 0; k < C::NE; ++k) mst[k * kS2Threads + tid] = 0.f;   // (covers NENT)
      ps2 = make_float2(0.f, 0.f);   // the words start at zero
      // init[j] = -(reference - 20) of the lane's rotated head j: the start of every score
      float init[GPH];
      float sc[U][GPH];
#pragma unroll
      for (int j = 0; j < GPH; ++j) init[j] = 0.f;
      key_scores(kx, init, sc);
      mask_group(sc, tw, s0, s1);
      {
        // the reference: the first sub-chunk's block maxima plus the headroom (inline: this
        // runs once per segment, with the scores in registers)
        float mt[GPH];
#pragma unroll
        for (int g = 0; g < GPH; ++g) mt[g] = -INFINITY;
#pragma unroll
        for (int u = 0; u < U; ++u)
#pragma unroll
          for (int j = 0; j < GPH; ++j) {
            const uint32_t g = ((uint32_t)j + lg) & (GPH - 1);
#pragma unroll
            for (int q = 0; q < GPH; ++q)
              if (g == (uint32_t)q) mt[q] = fmaxf(mt[q], sc[u][j]);
          }
        uint32_t* rk = redk + rbuf * C::NW * GPH;
        rbuf ^= 1;
#pragma unroll
        for (int g = 0; g < GPH; ++g) {
          const uint32_t k = __reduce_max_sync(0xffffffffu, ord_key(mt[g]));
          if (lane == 0) rk[warp * GPH + g] = k;
        }
        __syncthreads();
        float m[GPH];
#pragma unroll
        for (int g = 0; g < GPH; ++g) {
          uint32_t k = 0u;
#pragma unroll
          for (int w = 0; w < C::NW; ++w) k = max(k, rk[w * GPH + g]);
          m[g] = ord_val(k) + (kS2Headroom - (float)kS2Fix);
        }
#pragma unroll
        for (int j = 0; j < GPH; ++j) {
          const uint32_t g = ((uint32_t)j + lg) & (GPH - 1);
          float dj = m[0];
#pragma unroll
          for (int q = 1; q < GPH; ++q)
            if (g == (uint32_t)q) dj = m[q];
          init[j] = -dj;
#pragma unroll
          for (int u = 0; u < U; ++u) sc[u][j] -= dj;
        }
      }
      // Runs of sub-chunks with no block-wide step inside: a token whose score exceeds the
      // reference is listed (and contributes nothing in the run).  Between runs the block
      // raises the reference to the listed tokens' maximum plus the headroom when there are any
      // (folding the words rescaled, then adding the listed tokens' weights), and otherwise
      // folds only when the bound on the words says the next run could overflow one.  The list
      // count and the warps' p sums alternate between two buffers, so a boundary with nothing
      // to do costs one barrier.
      int i = 0, run = C::RUN, pb = 0;
      while (true) {
        const int stop = i + run < nsub ? i + run : nsub;
        uint32_t* exc = exn + pb;
        for (; i < stop; ++i) {
          if (i + 1 < nsub) {
            // token by token: the value side of sub-chunk i, then the key side of sub-chunk
            // i + 1 (which takes over token u's score registers)
            const uint32_t t = tw + WSTEP * (uint32_t)(i + 1);
#pragma unroll
            for (int q = 0; q < C::KW; ++q) kx[q] = kn[q];
            uint32_t vx[C::VW];
#pragma unroll
            for (int q = 0; q < C::VW; ++q) vx[q] = vcur[q];
#pragma unroll
            for (int q = 0; q < C::VW; ++q) vcur[q] = vn[q];
            load_group<C::KW, PAGED>(a, kcb, Sk, t + WSTEP, s1, kn);
            load_group<C::VW, PAGED>(a, vcb, Sv, t + WSTEP, s1, vn);
            static_for<U>([&](auto uc) {
              value_red1(uc, vx, sc[uc]);
              key_score1(uc, kx, init, sc[uc]);
            });
            mask_group(sc, t, s0, s1);
            static_for<U>([&](auto uc) {
              float mx = sc[uc][0];
              static_for<GPH>([&](auto jc) { mx = fmaxf(mx, sc[uc][jc]); });
              if (mx > (float)kS2Fix) {   // above the reference: list it, add it later
                constexpr int u = decltype(uc)::value;
                const uint32_t e = atomicAdd(exc, 1u);
                if (e < (uint32_t)C::LCAP) {   // its code words, from the registers
                  exk[e] = kx[(u * SKP) >> 2] >> (8 * ((u * SKP) & 3));
                  const uint32_t vw = vcur[(u * SVP) >> 2] >> (8 * ((u * SVP) & 3));
                  asm volatile("st.shared.u32 [%0], %1;" ::"r"(XV + 4u * e), "r"(vw) : "memory");
                }
                static_for<GPH>([&](auto jc) { sc[uc][jc] = -INFINITY; });
              }
            });
          } else {
            static_for<U>([&](auto uc) { value_red1(uc, vcur, sc[uc]); });
          }
        }
        {   // this warp's p sum since the last fold
          float v = ps2.x + ps2.y;
#pragma unroll
          for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
          if (lane == 0) redp[pb * C::NW + warp] = v;
        }
        __syncthreads();   // the run's reductions, list entries and p sums are complete
        const uint32_t n = *exc;   // (the same for every thread)
        if (n > 0u) {
          // listed tokens (their code words are in the list): their maxima set the new
          // reference.  A thread's first token keeps its value word and score in registers for
          // the second pass.
          float mt[GPH], m[GPH], x[GPH], x0[GPH];
          uint32_t vw0 = 0u;
          auto exv_at = [&](uint32_t e) {
            uint32_t w;
            asm volatile("ld.shared.u32 %0, [%1];" : "=r"(w) : "r"(XV + 4u * e) : "memory");
            return w;
          };
#pragma unroll
          for (int g = 0; g < GPH; ++g) mt[g] = -INFINITY;
          if ((uint32_t)tid < n) {
            vw0 = exv_at((uint32_t)tid);
            key_score_w(exk[tid], 0u, init, x0);
            unrotate_max(x0, mt);
          }
          for (uint32_t e = (uint32_t)tid + kS2Threads; e < n; e += kS2Threads) {
            key_score_w(exk[e], 0u, init, x);
            unrotate_max(x, mt);
          }
          block_max_of(mt, m);
          float refk[GPH], nref[GPH], alpha[GPH], d[GPH];
          ref_of(init, refk);
#pragma unroll
          for (int g = 0; g < GPH; ++g) {
            const float cand = m[g] + refk[g] + (kS2Headroom - (float)kS2Fix);
            nref[g] = fmaxf(refk[g], cand);
            alpha[g] = ex2_approx(refk[g] - nref[g]);
          }
#pragma unroll
          for (int j = 0; j < GPH; ++j) {
            d[j] = 0.f;
#pragma unroll
            for (int g = 0; g < GPH; ++g)
              if (((uint32_t)j + lg) % GPH == (uint32_t)g) d[j] = nref[g] - refk[g];
          }
          {
            float al = alpha[0];   // this lane's head in the fold
#pragma unroll
            for (int g = 1; g < GPH; ++g)
              if (fhv == (uint32_t)g) al = alpha[g];
            fold(al);   // the words so far, rescaled to the new reference (ends with a barrier)
          }
#pragma unroll
          for (int j = 0; j < GPH; ++j) init[j] -= d[j];
          static_for<U>([&](auto uc) {
            static_for<GPH>([&](auto jc) { sc[uc][jc] -= d[jc]; });
          });
          if ((uint32_t)tid < n) {
#pragma unroll
            for (int j = 0; j < GPH; ++j) x0[j] -= d[j];
            value_red_w(vw0, 0u, x0);
          }
          for (uint32_t e = (uint32_t)tid + kS2Threads; e < n; e += kS2Threads) {
            key_score_w(exk[e], 0u, init, x);
            value_red_w(exv_at(e), 0u, x);
          }
          __syncthreads();   // list reads and their reductions are complete
          if (tid == 0) *exc = 0u;
          // the words now hold only the listed tokens (at most ceil(n / SUBT) sub-chunks' worth)
          run = C::RUN - (int)((n + C::SUBT - 1) / C::SUBT);
          if (run < 1) {
            fold(1.f);
            run = C::RUN;
          }
        } else {
          // every word holds at most 2^20 (sum of p) + (its additions) since the last fold; the
          // next run adds at most WSUB per sub-chunk to one word
          float T = 0.f;
#pragma unroll
          for (int w = 0; w < C::NW; ++w) T += redp[pb * C::NW + w];
          const float used = T * 1048576.f * 1.001f + 16777216.f;
          const float avail = (4294967295.f - used) * (1.f / C::WSUB);
          run = avail >= (float)C::RUN ? C::RUN : (avail >= 1.f ? (int)avail : 0);
          if (run < 1 && i < nsub) {
            fold(1.f);
            run = C::RUN;
          }
        }
        pb ^= 1;
        if (i >= nsub) break;
      }
      // ---- segment partial (every reduction has landed: the last run's barrier): the last fold
      // writes the float32 histograms [slot][Sv][256][GP] (relative to the reference) straight
      // from the words and the masters; the owners of stage-0 entries add up the sums of p
      {
        float lsum = 0.f;
#pragma unroll 2
        for (int n8 = 0; n8 < 8; ++n8) {
          const uint32_t c = 2u * (uint32_t)warp + ((uint32_t)lane >> 4) + 32u * (uint32_t)n8;
          const uint32_t adr = VR + 256u * c + 16u * fk;
          const uint4 v = lds128u_v(adr);
          sts128z(adr);
          float v0, v1;
          if constexpr (C::R >= 4) {
            v0 = ((float)v.x + (float)v.y) + ((float)v.z + (float)v.w);
#pragma unroll
            for (int o = 1; o < RG; o <<= 1) v0 += __shfl_xor_sync(0xffffffffu, v0, o);
            v0 += __shfl_xor_sync(0xffffffffu, v0, 8);
            v1 = 0.f;
          } else {
            v0 = (float)v.x + (float)v.y;
            v1 = (float)v.z + (float)v.w;
            v0 += __shfl_xor_sync(0xffffffffu, v0, 8);
            v1 += __shfl_xor_sync(0xffffffffu, v1, 8);
          }
          if (fown) {
            const int mi = ((int)c * SVP + (int)fs0) * GPH + (int)fhv;
            const float w0 = fmaf(v0, 0x1p-20f, mst[mi]);
            a.pw[((slot * Sv + (int)fs0) * kCodebook + (int)c) * GP + hp * 4 + (int)fhv] = w0;
            if (fs0 == 0u) lsum += w0;
            if constexpr (C::R == 2) {
              const float w1 = fmaf(v1, 0x1p-20f, mst[mi + GPH]);
              a.pw[((slot * Sv + (int)fs0 + 1) * kCodebook + (int)c) * GP + hp * 4 + (int)fhv] = w1;
            }
          }
        }
        // the stage-0 owner of head g is chunk g ALPHA / 4 of each 16-lane half
        lsum += __shfl_xor_sync(0xffffffffu, lsum, 16);
        if (lane < 16 && fown && fs0 == 0u) reds[warp * GPH + (int)fhv] = lsum;
        __syncthreads();
        if (tid < GPH) {
          float l = 0.f;
#pragma unroll
          for (int w = 0; w < C::NW; ++w) l += reds[w * GPH + tid];
          a.pl[slot * GP + hp * 4 + tid] = l;
          // thread g < GPH is lane g of warp 0: its rotation is g, so head g is its slot 0
          a.pm[slot * GP + hp * 4 + tid] = (float)kS2Fix - init[0];
        }
      }
    }
  }
}

