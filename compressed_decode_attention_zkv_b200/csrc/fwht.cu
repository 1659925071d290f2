// zkv_fwht: standalone Walsh-Hadamard transform (one warp per vector, float64 butterflies).
// Passage: zerokv-neo "Architecture" (FWHT energy spreading before quantisation).
#include "zkv_internal.cuh"

namespace zkv {

template <int D>
__global__ void __launch_bounds__(256) fwht_kernel(const void* __restrict__ in, int dtype,
                                                   float* __restrict__ out, int64_t n_vec,
                                                   double scale) {
  constexpr int E = D / 32;
  const int lane = threadIdx.x & 31;
  const int64_t vec = (int64_t)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  if (vec >= n_vec) return;
  double v[E];
  load_row_f64<E>(in, dtype, vec * D, lane, v);
  fwht_warp_f64<D>(v, lane);
  // All loads of this warp precede the stores (the shuffles above are warp-synchronous), so
  // in-place use with F32 input is safe.
  float* o = out + vec * D + lane;
#pragma unroll
  for (int j = 0; j < E; ++j) o[j * 32] = (float)(v[j] * scale);
}

}  // namespace zkv

using namespace zkv;

extern "C" const char* zkv_status_string(int status) {
  switch (status) {
    case ZKV_OK: return "ZKV_OK";
    case ZKV_ERR_INVALID_ARG: return "ZKV_ERR_INVALID_ARG";
    case ZKV_ERR_UNSUPPORTED: return "ZKV_ERR_UNSUPPORTED";
    case ZKV_ERR_WORKSPACE: return "ZKV_ERR_WORKSPACE";
    case ZKV_ERR_CUDA: return "ZKV_ERR_CUDA";
    default: return "ZKV_ERR_UNKNOWN";
  }
}

extern "C" int zkv_version(void) { return ZKV_VERSION; }

extern "C" int zkv_fwht(const void* in, int in_dtype, float* out, int64_t n_vec, int d,
                        float scale, void* stream) {
  if (n_vec < 0) return ZKV_ERR_INVALID_ARG;
  if (in_dtype != ZKV_DTYPE_F16 && in_dtype != ZKV_DTYPE_F32) return ZKV_ERR_INVALID_ARG;
  if (!supported_d(d)) return ZKV_ERR_UNSUPPORTED;
  if (n_vec == 0) return ZKV_OK;
  if (!in || !out) return ZKV_ERR_INVALID_ARG;
  if (in_dtype == ZKV_DTYPE_F16 && (const void*)out == in) return ZKV_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int warps = 8;
  const int64_t blocks = (n_vec + warps - 1) / warps;
  if (blocks > 0x7fffffffLL) return ZKV_ERR_INVALID_ARG;
  const double s = (double)scale;
  switch (d) {
    case 64: fwht_kernel<64><<<(unsigned)blocks, warps * 32, 0, st>>>(in, in_dtype, out, n_vec, s); break;
    case 128: fwht_kernel<128><<<(unsigned)blocks, warps * 32, 0, st>>>(in, in_dtype, out, n_vec, s); break;
    case 256: fwht_kernel<256><<<(unsigned)blocks, warps * 32, 0, st>>>(in, in_dtype, out, n_vec, s); break;
  }
  ZKV_CHECK_LAUNCH();
  return ZKV_OK;
}
