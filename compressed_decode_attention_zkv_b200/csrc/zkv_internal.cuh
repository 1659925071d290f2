// Internal helpers shared by the libzkv kernels (sm_100a).
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "zkv.h"

namespace zkv {

constexpr int kCodebook = ZKV_CODEBOOK_SIZE;   // 256 codewords per stage
constexpr int kMaxStages = 8;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

inline bool supported_d(int d) { return d == 64 || d == 128 || d == 256; }

// Paged code layout (block table): P a power of two in [32, 65536], Tcap = max_pages * P,
// page indices fit int32.  No block table: the contiguous layout, nothing to check.
inline int validate_paged(const int32_t* bt, int64_t P, int64_t max_pages, int64_t n_pages,
                          int64_t Tcap) {
  if (!bt) return ZKV_OK;
  if (P < 32 || P > 65536 || (P & (P - 1))) return ZKV_ERR_INVALID_ARG;
  if (max_pages < 1 || n_pages < 1 || n_pages > 0x7fffffffLL) return ZKV_ERR_INVALID_ARG;
  if (max_pages > (int64_t(1) << 28) / P || max_pages * P != Tcap) return ZKV_ERR_INVALID_ARG;
  return ZKV_OK;
}
inline int log2_pow2(int64_t x) { int s = 0; while ((int64_t(1) << s) < x) ++s; return s; }

#define ZKV_CHECK_LAUNCH()                                   \
  do {                                                       \
    if (cudaGetLastError() != cudaSuccess) return ZKV_ERR_CUDA; \
  } while (0)

// Programmatic dependent launch.  A kernel launched with launch_pdl may start before the
// previous kernel on the stream has finished; pdl_wait() blocks until that kernel has
// completed and its memory is visible (it returns at once for a normal launch).  A kernel's
// blocks all pass their pdl_wait before they exit, so its completion implies the completion of
// everything before it on the stream.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
// Let the next kernel on the stream launch now (its blocks that do not read this kernel's
// results may run concurrently; the others pdl_wait).
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <typename... KArgs, typename... Args>
static inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                                     cudaStream_t st, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// 16-byte asynchronous global -> shared copy (both addresses 16-byte aligned).
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                   (unsigned)__cvta_generic_to_shared(smem_dst)),
               "l"(gmem_src)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
// Commit the copies issued so far and wait for all of this thread's copies.
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

// ------------------------------------------------------------------------------------------
// Walsh-Hadamard transform of one vector held by a warp, float64.
// Lane l holds elements j*32 + l for j < E = D/32 (strided: coalesced loads, conflict-free
// shared-memory stores).  Butterfly pairs (i, i+h) map to (x_i + x_{i+h}, x_i - x_{i+h}) for
// every h = 1, 2, ..., D/2 (Sylvester order): h < 32 pairs lanes l and l^h, h >= 32 pairs the
// lane's own registers j and j ^ (h/32).  For fp16 inputs every partial sum is exact in float64,
// so the result does not depend on the order in which the levels are applied.
// ------------------------------------------------------------------------------------------
template <int D>
__device__ __forceinline__ void fwht_warp_f64(double (&v)[D / 32], int lane) {
  constexpr int E = D / 32;
#pragma unroll
  for (int lm = 1; lm < 32; lm <<= 1) {
    const bool upper = (lane & lm) != 0;
#pragma unroll
    for (int j = 0; j < E; ++j) {
      const double o = __shfl_xor_sync(0xffffffffu, v[j], lm);
      v[j] = upper ? (o - v[j]) : (v[j] + o);
    }
  }
#pragma unroll
  for (int h = 1; h < E; h <<= 1) {
#pragma unroll
    for (int j = 0; j < E; ++j) {
      if ((j & h) == 0) {
        const double a = v[j], b = v[j + h];
        v[j] = a + b;
        v[j + h] = a - b;
      }
    }
  }
}

// The same transform in float32 (each level rounds once), for operands that only feed float32
// arithmetic afterwards (the decode-time query rotation).
template <int D>
__device__ __forceinline__ void fwht_warp_f32(float (&v)[D / 32], int lane) {
  constexpr int E = D / 32;
#pragma unroll
  for (int lm = 1; lm < 32; lm <<= 1) {
    const bool upper = (lane & lm) != 0;
#pragma unroll
    for (int j = 0; j < E; ++j) {
      const float o = __shfl_xor_sync(0xffffffffu, v[j], lm);
      v[j] = upper ? (o - v[j]) : (v[j] + o);
    }
  }
#pragma unroll
  for (int h = 1; h < E; h <<= 1) {
#pragma unroll
    for (int j = 0; j < E; ++j) {
      if ((j & h) == 0) {
        const float a = v[j], b = v[j + h];
        v[j] = a + b;
        v[j + h] = a - b;
      }
    }
  }
}

// Warp sums of NT values per lane in NT - 1 + log2(32 / NT) shuffles (instead of 5 NT): at
// each level a lane keeps half of its live values (x[0 .. N-1]) and sends the other half to its
// partner.  Afterwards every lane holds the full sum of value `h` (accumulated into h).
template <int NT, int N, int O>
struct TransposeSum {
  __device__ __forceinline__ static float run(float (&x)[NT], int lane, int& h) {
    constexpr int H = N / 2;
    const bool up = (lane & O) != 0;
#pragma unroll
    for (int k = 0; k < H; ++k) {
      const float send = up ? x[k] : x[k + H];
      const float keep = up ? x[k + H] : x[k];
      x[k] = keep + __shfl_xor_sync(0xffffffffu, send, O);
    }
    if (up) h += H;
    return TransposeSum<NT, H, O / 2>::run(x, lane, h);
  }
};
template <int NT, int O>
struct TransposeSum<NT, 1, O> {
  __device__ __forceinline__ static float run(float (&x)[NT], int, int&) {
    float v = x[0];
#pragma unroll
    for (int o = O; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
  }
};

// Load the E strided elements (j*32 + lane) of a row (fp16 or fp32) as doubles.
template <int E>
__device__ __forceinline__ void load_row_f64(const void* base, int dtype, int64_t off, int lane,
                                             double (&v)[E]) {
  if (dtype == ZKV_DTYPE_F16) {
    const __half* p = reinterpret_cast<const __half*>(base) + off + lane;
#pragma unroll
    for (int j = 0; j < E; ++j) v[j] = (double)__half2float(p[j * 32]);
  } else {
    const float* p = reinterpret_cast<const float*>(base) + off + lane;
#pragma unroll
    for (int j = 0; j < E; ++j) v[j] = (double)p[j * 32];
  }
}

__device__ __forceinline__ double warp_sum_f64(double x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

__device__ __forceinline__ float warp_sum_f32(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

__device__ __forceinline__ float warp_max_f32(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}

__device__ __forceinline__ float warp_min_f32(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fminf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}

// 2^x via the PTX approximate base-2 exponential (relative error about 2^-22).
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void set_error(int32_t* flag, int bits) {
  if (flag) atomicOr(flag, bits);
}

// Raise a kernel's dynamic shared-memory limit once per (kernel, device); later calls are
// plain launches (so they can be captured into CUDA graphs).  Keyed by the kernel's address:
// every template instantiation has its own entry.
inline cudaError_t ensure_smem_limit_raw(const void* kernel, size_t bytes) {
  struct Entry { const void* fn; int dev; size_t bytes; };
  static std::mutex mu;
  static Entry table[512];
  static int n = 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  int slot = -1;
  for (int i = 0; i < n; ++i)
    if (table[i].fn == kernel && table[i].dev == dev) { slot = i; break; }
  if (slot >= 0 && table[slot].bytes >= bytes) return cudaSuccess;
  const cudaError_t e =
      cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e != cudaSuccess) return e;
  if (slot < 0) {
    if (n == 512) return cudaSuccess;   // table full: the attribute is set, just not cached
    slot = n++;
    table[slot].fn = kernel;
    table[slot].dev = dev;
  }
  table[slot].bytes = bytes;
  return cudaSuccess;
}

template <class F>
inline cudaError_t ensure_smem_limit(F* kernel, size_t bytes) {
  return ensure_smem_limit_raw(reinterpret_cast<const void*>(kernel), bytes);
}

// Round-up helpers for workspace carving.
inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace zkv
