// Serving-step cache maintenance: window insert, eviction of the oldest window token, RVQ
// encode of the evicted token onto the compressed prefix (sm_100a).
//
// Passages: VQKV (gist.science summary of arXiv 2603.16435), section 2.3 "Local Sliding
// Window" (recent tokens uncompressed, older "middle" tokens compressed to codes); VeloxQuant-
// MLX 0.5.1 "Quick start" (cache.append(k, v) per token, then cache.attend(q)).
//
// Kernel 1 (grid: sequence groups x kv heads x {K, V}) encodes the evicted rows with the
// row-group encoder and writes the new token into its slot; kernel 2 advances the lengths.
// Both read the same pre-step lengths, so their decisions agree.
#include "encode_rows.cuh"

namespace zkv {

struct AppendRows {
  int B, Hkv, d;
  int64_t Tcap, Wcap;
  const __half* win;
  uint8_t* codes;
  const int32_t* win_len;
  const int32_t* win_head;
  const int32_t* comp_len;

  // Row j (a sequence) is encoded iff its window is full and the prefix has room.
  __device__ bool valid(int64_t j, int) const {
    if (j >= B) return false;
    const int64_t wl = win_len[j], hd = win_head[j], c = comp_len[j];
    return wl == Wcap && hd >= 0 && hd < Wcap && c >= 0 && c < Tcap;
  }
  __device__ const void* src() const { return win; }
  __device__ int dtype() const { return ZKV_DTYPE_F16; }
  __device__ bool do_rotate() const { return true; }
  __device__ int64_t x_off(int64_t j, int h) const {
    return (((int64_t)j * Hkv + h) * Wcap + win_head[j]) * d;
  }
  __device__ void store(int64_t j, int h, int S, const uint8_t* code, const float*) const {
    uint8_t* c = codes + (((int64_t)j * Hkv + h) * Tcap + comp_len[j]) * S;
    for (int s = 0; s < S; ++s) c[s] = code[s];
  }
};

constexpr int kAppendR = 8;

template <int D>
__global__ void __launch_bounds__(256) append_encode_kernel(zkv_append_params p, double rot) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  RowsSmem<D, kAppendR>& sm = *reinterpret_cast<RowsSmem<D, kAppendR>*>(smem_raw);
  float* cb = reinterpret_cast<float*>(smem_raw + ((sizeof(RowsSmem<D, kAppendR>) + 15) / 16) * 16);
  const int kind = blockIdx.z;   // 0 = keys, 1 = values
  const int h = blockIdx.y;
  const int64_t row0 = (int64_t)blockIdx.x * kAppendR;
  AppendRows map;
  map.B = p.B;
  map.Hkv = p.Hkv;
  map.d = D;
  map.Tcap = p.Tcap;
  map.Wcap = p.Wcap;
  map.win = reinterpret_cast<const __half*>(kind ? p.win_v : p.win_k);
  map.codes = kind ? p.v_codes : p.k_codes;
  map.win_len = p.win_len;
  map.win_head = p.win_head;
  map.comp_len = p.comp_len;
  const int S = kind ? p.Sv : p.Sk;
  const float* books = kind ? p.v_codebooks : p.k_codebooks;
  encode_rows_body<D, kAppendR>(map, books, S, rot, row0, h, sm, cb);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid < kAppendR) {
    const int64_t j = row0 + tid;
    if (map.valid(j, h)) map.store(j, h, S, sm.code[tid], sm.nrm[tid]);
  }
  __syncthreads();   // every read of an evicted slot precedes the overwrite below
  if (warp < kAppendR) {
    const int64_t j = row0 + warp;
    if (j >= p.B) return;
    const int64_t wl = p.win_len[j], hd = p.win_head[j], c = p.comp_len[j];
    int64_t slot = -1;
    if (wl >= 0 && wl < p.Wcap) {
      slot = wl;
    } else if (wl == p.Wcap && hd >= 0 && hd < p.Wcap) {
      if (c >= 0 && c < p.Tcap) slot = hd;
      else if (lane == 0 && kind == 0 && h == 0) set_error(p.error_flag, ZKV_DEVERR_COMP_LEN);
    } else if (lane == 0 && kind == 0 && h == 0) {
      set_error(p.error_flag, ZKV_DEVERR_WIN_LEN);
    }
    if (slot < 0) return;
    const __half* src = reinterpret_cast<const __half*>(kind ? p.new_v : p.new_k) +
                        ((int64_t)j * p.Hkv + h) * D;
    __half* dst = reinterpret_cast<__half*>(kind ? p.win_v : p.win_k) +
                  (((int64_t)j * p.Hkv + h) * p.Wcap + slot) * D;
    for (int i = lane; i < D; i += 32) dst[i] = src[i];
  }
}

__global__ void append_lengths_kernel(int B, int64_t Tcap, int64_t Wcap, int32_t* win_len,
                                      int32_t* win_head, int32_t* comp_len) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= B) return;
  const int64_t wl = win_len[b];
  if (wl < 0 || wl > Wcap) return;
  if (wl < Wcap) {
    win_len[b] = (int32_t)(wl + 1);
    return;
  }
  const int64_t c = comp_len[b], hd = win_head[b];
  if (c < 0 || c >= Tcap || hd < 0 || hd >= Wcap) return;
  comp_len[b] = (int32_t)(c + 1);
  win_head[b] = (int32_t)((hd + 1) % Wcap);
}

}  // namespace zkv

using namespace zkv;

extern "C" int zkv_rvq_append(const zkv_append_params* p, void* stream) {
  if (!p) return ZKV_ERR_INVALID_ARG;
  if (p->B < 1 || p->Hkv < 1 || p->Tcap < 0 || p->Wcap < 1) return ZKV_ERR_INVALID_ARG;
  if (!supported_d(p->d)) return ZKV_ERR_UNSUPPORTED;
  if (p->Sk < 1 || p->Sk > kMaxStages || p->Sv < 1 || p->Sv > kMaxStages) return ZKV_ERR_UNSUPPORTED;
  if (p->Hkv > 65535) return ZKV_ERR_UNSUPPORTED;
  if (!p->new_k || !p->new_v || !p->win_k || !p->win_v || !p->win_len || !p->win_head ||
      !p->comp_len || !p->k_codes || !p->v_codes || !p->k_codebooks || !p->v_codebooks)
    return ZKV_ERR_INVALID_ARG;
  const uintptr_t al = (uintptr_t)p->win_k | (uintptr_t)p->win_v | (uintptr_t)p->k_codebooks |
                       (uintptr_t)p->v_codebooks;
  if (al & 15) return ZKV_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const double rot = 1.0 / std::sqrt((double)p->d);
  const dim3 grid((unsigned)((p->B + kAppendR - 1) / kAppendR), (unsigned)p->Hkv, 2);
  const bool ok =
      ensure_smem_limit(append_encode_kernel<64>, rows_smem_bytes<64, kAppendR>()) == cudaSuccess &&
      ensure_smem_limit(append_encode_kernel<128>, rows_smem_bytes<128, kAppendR>()) == cudaSuccess &&
      ensure_smem_limit(append_encode_kernel<256>, rows_smem_bytes<256, kAppendR>()) == cudaSuccess;
  if (!ok) return ZKV_ERR_CUDA;
  switch (p->d) {
    case 64: append_encode_kernel<64><<<grid, 256, rows_smem_bytes<64, kAppendR>(), st>>>(*p, rot); break;
    case 128: append_encode_kernel<128><<<grid, 256, rows_smem_bytes<128, kAppendR>(), st>>>(*p, rot); break;
    default: append_encode_kernel<256><<<grid, 256, rows_smem_bytes<256, kAppendR>(), st>>>(*p, rot); break;
  }
  ZKV_CHECK_LAUNCH();
  append_lengths_kernel<<<(p->B + 127) / 128, 128, 0, st>>>(p->B, p->Tcap, p->Wcap, p->win_len,
                                                           p->win_head, p->comp_len);
  ZKV_CHECK_LAUNCH();
  return ZKV_OK;
}
