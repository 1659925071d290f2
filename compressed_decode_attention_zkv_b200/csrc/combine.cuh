// Value contraction and final combine of the compressed decode (sm_100a).  Included by decode.cu
// (inside namespace zkv, after the scan kernels).
//
// Passages: VQKV (gist.science summary of arXiv 2603.16435), section 2.3 "Decoding Stage": values
// are reconstructed on demand -- here sum_t p_t sum_s Cv_s[z_{t,s}] = sum_s sum_c W_s[c] Cv_s[c],
// the weight histograms W_s of the scan contracted with the value codebooks; Differential-KV
// README, "Decode & Prefill Innovations": the compressed part and the dense window are joined by
// an fp32 log-sum-exp combine.
//
// Grid (Sv * QC, pairs), 256 threads.  Block (s, qc, pair) owns the ncw = 256 / QC codewords
// [qc ncw, (qc + 1) ncw) of value stage s:
//   0. its value-codebook chunk (ncw x d floats) is copied to shared memory before the wait for
//      the scan: it does not depend on it, and the block may start on an SM the scan has left;
//   1. the pair's scan segments (slots) and their maxima pm -> M = max (per head) and the slot
//      weights 2^(pm - M);
//   2. W_s[c] = sum over slots of weight * histogram for the chunk's codewords, the slots split
//      over slices of threads when the chunk has fewer than 256 (codeword, head) items, eight
//      independent loads in flight per thread;
//   3. out_s[g][:] = sum_c W_s[c][g] Cv_s[c][:] from shared memory -> workspace;
//   4. an atomic counter per pair: the block that completes the pair (the last of its blocks)
//      sums the partial outputs (float4 loads, parts split over thread slices and added in a
//      fixed order), rotates them back (H / sqrt(d), float64 transform rounded once), and
//      merges with the window by log-sum-exp (the window's parts merged first, by their
//      maxima).  No block waits for another.
// The window partials come from the table kernel (complete before the scan's, and so before
// this kernel's, wait returns).  Each thread's first eight slot values of step 2 and the
// finishing block's window parts are loaded beside the values they are combined with.
#pragma once

constexpr int kCombineFin = 1024;   // floats of the finishing block's slice buffer

// Dynamic shared memory of a combine block (float offsets, each a multiple of 4): the codebook
// chunk, slot weights, the merged chunk histogram, the slice buffer of step 2, the finishing
// block's output and its slice buffer.
struct CombineSmem {
  int cv, pmv, W, red, ocb, fin, total;
};
__host__ __device__ inline CombineSmem combine_layout(int grid, int GP, int d, int qc) {
  CombineSmem L;
  const int ncw = kCodebook / qc;
  L.cv = 0;
  L.pmv = L.cv + ncw * d;
  L.W = L.pmv + ((grid + 1) * GP + 3) / 4 * 4;
  L.red = L.W + (ncw * GP + 3) / 4 * 4;
  L.ocb = L.red + 256;
  L.fin = L.ocb + GP * d;
  L.total = L.fin + kCombineFin;
  return L;
}
inline size_t combine_smem_bytes(int grid, int GP, int d, int qc) {
  return (size_t)combine_layout(grid, GP, d, qc).total * sizeof(float);
}

template <int D, int GP>
__global__ void __launch_bounds__(256, 4) combine_kernel(DecodeArgs a) {
  constexpr int E = D / 32;
  constexpr int TG = 256 / D;                       // thread groups over the head dimension
  constexpr int HPT = GP >= TG ? GP / TG : 1;       // heads per thread in the contraction
  constexpr int F4 = GP * D / 4;                    // float4 pieces of one partial output
  constexpr int P2 = F4 >= 256 ? 1 : 256 / F4;      // part slices in the finishing sum
  constexpr int J2 = F4 >= 256 ? F4 / 256 : 1;      // pieces per thread in the finishing sum
  static_assert(P2 == 1 || P2 * F4 * 4 <= kCombineFin, "finishing slices fit");
  extern __shared__ __align__(16) float csm[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int QC = a.qc, ncw = kCodebook / QC;
  const int s = (int)blockIdx.x / QC, qc = (int)blockIdx.x % QC;
  const int64_t pair = blockIdx.y;
  const int b = (int)(pair / a.Hkv), kvh = (int)(pair % a.Hkv);
  const int c0 = qc * ncw;
  const CombineSmem L = combine_layout(a.grid, GP, D, QC);
  float* cvs = csm + L.cv;                          // [ncw][D] value codewords
  float* pmv = csm + L.pmv;                         // [n][GP] slot maxima, then weights
  float* W = csm + L.W;                             // [ncw][GP]
  float* red = csm + L.red;                         // [P][I] step-2 slices
  __shared__ float Ms[GP], Ls[GP];
  __shared__ int last_s;
  // 0. the codebook chunk, in flight across the wait
  {
    const float* cv = a.Cv + (((int64_t)kvh * a.Sv + s) * kCodebook + c0) * D;
    for (int f = tid; f < ncw * D / 4; f += 256) cp_async16(cvs + 4 * f, cv + 4 * f);
    cp_async_commit();
  }
  pdl_wait();   // the scan's partials (and, through it, the append and the table kernel)
  const int64_t first = a.pfirst[pair], last = a.plast[pair];
  const int n = last >= first ? (int)(last - first + 1) : 0;
  const int64_t slot0 = pair + first;
  // step 2's item of this thread: f0 = (c, g), g fastest (coalesced slot rows); with I < 256
  // items, thread slice p takes the slots p, p + P, ...  Its first eight slot values are loaded
  // now, beside the maxima (they do not depend on them).
  const int I = ncw * GP;
  const int P = I >= 256 ? 1 : 256 / I;
  const int p = P == 1 ? 0 : tid / I;
  const int64_t stride = (int64_t)a.Sv * kCodebook * GP;   // one slot
  const float* base = a.pw + (slot0 * a.Sv + s) * (int64_t)(kCodebook * GP) + (int64_t)c0 * GP;
  float pv[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int k = p + j * P;
    pv[j] = k < n ? base[(int64_t)k * stride + (P == 1 ? tid : tid % I)] : 0.f;
  }
  // 1. slot maxima -> per-head maximum (warp g) -> weights
  for (int f = tid; f < n * GP; f += 256) pmv[f] = a.pm[slot0 * GP + f];
  __syncthreads();
  if (warp < GP) {
    float m = -INFINITY;
    for (int k = lane; k < n; k += 32) m = fmaxf(m, pmv[k * GP + warp]);
    m = warp_max_f32(m);
    if (lane == 0) Ms[warp] = m;
  }
  __syncthreads();
  for (int f = tid; f < n * GP; f += 256) pmv[f] = ex2_approx(pmv[f] - Ms[f % GP]);
  __syncthreads();
  {
    // 2. merged histogram of the chunk
    for (int f0 = (P == 1 ? tid : tid % I); f0 < I; f0 += 256) {
      const int g = f0 % GP;
      const float* src = base + f0;
      float w = 0.f;
      int k = p;
      if (f0 < 256) {   // the first item: its first eight slots are in pv
#pragma unroll
        for (int j = 0; j < 8; ++j)
          if (p + j * P < n) w = fmaf(pmv[(p + j * P) * GP + g], pv[j], w);
        k = p + 8 * P;
      }
      for (; k + 7 * P < n; k += 8 * P) {   // eight independent loads per round trip
        float v[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) v[j] = src[(int64_t)(k + j * P) * stride];
#pragma unroll
        for (int j = 0; j < 8; ++j) w = fmaf(pmv[(k + j * P) * GP + g], v[j], w);
      }
      for (; k < n; k += P) w = fmaf(pmv[k * GP + g], src[(int64_t)k * stride], w);
      if (P == 1) W[f0] = w;
      else red[p * I + f0] = w;
    }
    if (P > 1) {
      __syncthreads();
      if (tid < I) {
        float w = 0.f;
        for (int q = 0; q < P; ++q) w += red[q * I + tid];
        W[tid] = w;
      }
    }
    cp_async_wait_all();
    __syncthreads();
    // 3. contraction with the chunk's value codewords: thread (e, group) of HPT heads
    const int e = tid % D, grp = tid / D;
    const int gbase = grp * HPT;
    if (gbase < GP) {
      float acc[HPT];
#pragma unroll
      for (int h = 0; h < HPT; ++h) acc[h] = 0.f;
#pragma unroll 8
      for (int c = 0; c < ncw; ++c) {
        const float x = cvs[c * D + e];
#pragma unroll
        for (int h = 0; h < HPT; ++h) acc[h] = fmaf(W[c * GP + gbase + h], x, acc[h]);
      }
#pragma unroll
      for (int h = 0; h < HPT; ++h)
        a.so[(((pair * a.Sv + s) * QC + qc) * GP + gbase + h) * D + e] = acc[h];
    }
  }
  // 4. the block that completes the pair finishes it
  __threadfence();
  __syncthreads();
  if (tid == 0) last_s = atomicAdd(a.cnt + pair, 1) == (int)gridDim.x - 1;
  __syncthreads();
  if (!last_s) return;
  __threadfence();   // the other blocks' partial outputs are visible
  // L = sum over slots of weight * pl (warp g; the weights are this block's, in pmv)
  if (warp < GP) {
    float l = 0.f;
    for (int k = lane; k < n; k += 32) l = fmaf(pmv[k * GP + warp], a.pl[(slot0 + k) * GP + warp], l);
    l = warp_sum_f32(l);
    if (lane == 0) Ls[warp] = l;
  }
  // the window partial of warp g's head: its parts merged by their maxima (log-sum-exp),
  // loaded beside the partial outputs
  float wmg = -INFINITY, wlg = 0.f, wog[E];
#pragma unroll
  for (int q = 0; q < E; ++q) wog[q] = 0.f;
  if (warp < a.G) {
    for (int pt = 0; pt < a.wparts; ++pt) {
      const int64_t wi = (pair * a.wparts + pt) * GP + warp;
      const float mp = a.wm[wi], lp = a.wl[wi];
      float op[E];
#pragma unroll
      for (int q = 0; q < E; ++q) op[q] = a.wo[wi * D + q * 32 + lane];
      const float mn = fmaxf(wmg, mp);
      if (mn == -INFINITY) continue;   // both empty so far
      const float s0 = wmg == -INFINITY ? 0.f : ex2_approx(wmg - mn);
      const float s1 = mp == -INFINITY ? 0.f : ex2_approx(mp - mn);
      wlg = wlg * s0 + lp * s1;
#pragma unroll
      for (int q = 0; q < E; ++q) wog[q] = wog[q] * s0 + op[q] * s1;
      wmg = mn;
    }
  }
  // the sum of the stage / chunk partial outputs (rotated domain, unnormalised): piece f4 of
  // the parts p2, p2 + P2, ... in slice p2, then the slices in order
  float* ocb = csm + L.ocb;   // [GP][D]
  float* fin = csm + L.fin;   // [P2][GP * D]
  {
    const int nparts = a.Sv * QC;
    const float4* so4 = reinterpret_cast<const float4*>(a.so + pair * (int64_t)nparts * GP * D);
    const int p2 = F4 >= 256 ? 0 : tid / F4;
#pragma unroll
    for (int j = 0; j < J2; ++j) {
      const int f4 = (F4 >= 256 ? tid : tid % F4) + j * 256;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      int q = p2;
      for (; q + 7 * P2 < nparts; q += 8 * P2) {
        float4 v[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = so4[(int64_t)(q + i * P2) * F4 + f4];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          acc.x += v[i].x; acc.y += v[i].y; acc.z += v[i].z; acc.w += v[i].w;
        }
      }
      for (; q < nparts; q += P2) {
        const float4 v = so4[(int64_t)q * F4 + f4];
        acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
      }
      if (P2 == 1) reinterpret_cast<float4*>(ocb)[f4] = acc;
      else reinterpret_cast<float4*>(fin)[p2 * F4 + f4] = acc;
    }
    if (P2 > 1) {
      __syncthreads();
      for (int f = tid; f < GP * D; f += 256) {
        float v = 0.f;
        for (int q = 0; q < P2; ++q) v += fin[q * GP * D + f];
        ocb[f] = v;
      }
    }
  }
  __syncthreads();
  if (warp < a.G) {   // G <= 8: one head per warp
    const int g = warp;
    double v[E];
#pragma unroll
    for (int q = 0; q < E; ++q) v[q] = (double)ocb[g * D + q * 32 + lane];
    fwht_warp_f64<D>(v, lane);
    const float mc = Ms[g], lc = Ls[g];
    const float mw = wmg, lw = wlg;
    const float M = fmaxf(mc, mw);
    const float wc = (mc == -INFINITY) ? 0.f : ex2_approx(mc - M);
    const float ww = (mw == -INFINITY) ? 0.f : ex2_approx(mw - M);
    const float Lt = wc * lc + ww * lw;
    const int64_t h = (int64_t)kvh * a.G + g;
    float* o = a.out + ((int64_t)b * a.Hq + h) * D;
    const float inv = Lt > 0.f ? 1.f / Lt : 0.f;
#pragma unroll
    for (int q = 0; q < E; ++q) {
      const int i = q * 32 + lane;
      o[i] = (wc * (float)(v[q] * a.rot) + ww * wog[q]) * inv;
    }
    if (lane == 0 && a.lse) a.lse[(int64_t)b * a.Hq + h] = Lt > 0.f ? (M + log2f(Lt)) * kLn2 : -INFINITY;
  }
  if (tid == 0) a.cnt[pair] = 0;   // ready for the next call
}
