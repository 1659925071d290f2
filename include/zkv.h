/*
 * zkv.h -- C ABI of libzkv: RVQ KV-cache encode and compressed decode attention on B200.
 *
 * The method (web pages this library follows):
 *   - "VQKV: High-Fidelity and High-Ratio Cache Compression via Vector-Quantization"
 *     (gist.science summary of arXiv 2603.16435), section 2.1 "Residual Simple Vector
 *     Quantization": greedy residual stages and reconstruction x_hat = sum_s Q_s[z_s];
 *     section 2.3 "Inference Integration": codes stored at prefill, on-demand reconstruction
 *     inside attention at decode, a local window of recent tokens kept uncompressed.
 *   - "zerokv-neo 4.0.0", "Architecture": FWHT energy spreading before quantisation.
 *   - "VeloxQuant-MLX 0.5.1", "VecInfer": Walsh-Hadamard rotation absorbed into the query.
 *   - "Differential-KV", "Decode & Prefill Innovations": flash-style fp32 log-sum-exp combine
 *     of the compressed part with a dense recency window.
 *
 * Conventions shared by every entry point:
 *   - All tensor pointers are DEVICE pointers owned by the caller.  The library allocates
 *     nothing per call.  Its state between calls is the CUDA runtime's (loaded kernels and
 *     their attributes) plus one fixed device array per device, the scratch workspace of
 *     zkv_rvq_decode_attn_noalloc (below); every other call works only in the caller's
 *     buffers.  fp16 tensors are passed as uint16_t bit patterns (IEEE binary16).
 *   - Every call is asynchronous on `stream` (a cudaStream_t passed as void*; NULL = legacy
 *     default stream).  Argument validation is synchronous and happens before any launch; a
 *     failed validation returns an error and launches nothing.  A launch failure returns
 *     ZKV_ERR_CUDA.  No C++ exception crosses this boundary.
 *   - Codebooks hold K = 256 float32 codewords per stage in the ROTATED domain
 *     (y = H_d x / sqrt(d), Sylvester-ordered Hadamard), layout [n_head][S][256][d].  Codeword
 *     0 of every stage should be the zero vector (then residual norms never increase).
 *   - Head dimension d must be 64, 128 or 256; stage counts 1..8.
 *   - GQA: query head h reads kv head h / (Hq / Hkv).
 *   - Device-side conditions that cannot be checked on the host (a length beyond capacity)
 *     are reported by OR-ing ZKV_DEVERR_* bits into an optional caller-owned device word
 *     (`error_flag`, may be NULL); the offending sequence is clamped or skipped, never read
 *     or written out of bounds.  No kernel waits on another.  The tensor-core encoder's wait
 *     for its own matrix-multiply completion is bounded: if it ever ran out, that tile's codes
 *     are not written and ZKV_DEVERR_TIMEOUT is set instead of the device hanging.
 */
#ifndef ZKV_H
#define ZKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes returned by every entry point. */
typedef enum {
  ZKV_OK = 0,
  ZKV_ERR_INVALID_ARG = 1, /* null pointer, negative size, inconsistent shapes, misalignment */
  ZKV_ERR_UNSUPPORTED = 2, /* d not in {64,128,256}, S not in 1..8, GQA group > 8, ...     */
  ZKV_ERR_WORKSPACE = 3,   /* workspace missing or smaller than the size query returned     */
  ZKV_ERR_CUDA = 4         /* a CUDA launch or attribute call failed                        */
} zkv_status;

/* Bits OR-ed into a caller's device error word. */
#define ZKV_DEVERR_COMP_LEN 1   /* comp_len[b] > Tcap (clamped) or append at Tcap (skipped) */
#define ZKV_DEVERR_WIN_LEN 2    /* win_len[b] > Wcap (clamped)                              */
#define ZKV_DEVERR_TIMEOUT 4    /* a bounded on-chip wait ran out (results of that tile absent) */
#define ZKV_DEVERR_PAGE 8       /* a block-table entry outside [0, n_pages): its tokens read as code
                                   0 (decode) / the append writes nothing for that sequence      */
#define ZKV_DEVERR_SMEM 16      /* the decode scan's shared-memory layout did not fit the CTA's
                                   shared window (its partial results are absent)               */

#define ZKV_DTYPE_F16 0
#define ZKV_DTYPE_F32 1

#define ZKV_CODEBOOK_SIZE 256

/* Human-readable name of a status code (static string). */
const char* zkv_status_string(int status);

/* Library ABI version (major * 100 + minor): 1.01 adds the serving step, the paged layout,
 * key smoothing, product VQ and the context-parallel combines to 1.00's encode / decode. */
#define ZKV_VERSION 101
int zkv_version(void);

/*
 * zkv_fwht -- Walsh-Hadamard transform of n_vec vectors of length d.
 * Passage: zerokv-neo "Architecture" (FWHT energy spreading); VeloxQuant "Highlights"
 * (O(d log d) Hadamard rotation).
 *   out[n][i] = float32( scale * sum_j H_d[i][j] * in[n][j] ),  H_d Sylvester-ordered (+-1).
 * The sum is accumulated in float64 (exact for fp16 inputs), multiplied by `scale` in float64
 * and rounded once to float32.  scale = 1/sqrt(d) gives the orthonormal, self-inverse rotation.
 *   in      device, [n_vec][d], dtype ZKV_DTYPE_F16 or ZKV_DTYPE_F32, contiguous rows
 *   out     device, [n_vec][d] float32; may alias `in` only when in_dtype is F32
 *   n_vec   >= 0 (0 launches nothing); d in {64,128,256}
 * Errors: INVALID_ARG (null with n_vec>0, bad dtype), UNSUPPORTED (d), CUDA.
 */
int zkv_fwht(const void* in, int in_dtype, float* out, int64_t n_vec, int d, float scale,
             void* stream);

/*
 * zkv_rvq_encode -- greedy residual vector quantisation of KV head vectors.
 * Passage: VQKV section 2.1 "Process" steps 1-4 (nearest codeword per stage, residual passed
 * on), section 2.3 "Prefilling Stage" (store only integer codes); rotation: zerokv-neo
 * "Architecture".
 * Rows are addressed as (b, t, h) for b < n_batch, t < n_tok, h < n_head.  For each row:
 *   y = rotate ? float32(H_d x / sqrt(d)) : x        (float64 accumulate, one rounding)
 *   r = y; for s in 0..S-1:
 *     z_s = argmin_c ||r - C[h][s][c]||^2   decided in float64, ties -> lowest c
 *     r   = r - C[h][s][z_s]                 (float32, elementwise)
 *     norms[s] = float32(||r||_2)            (float64 accumulate)
 * Layouts (strides in ELEMENTS of each tensor's type; the innermost index is contiguous):
 *   x      fp16 or fp32 (x_dtype), element (b,t,h,i) at x[b*x_sb + t*x_st + h*x_sh + i]
 *   codes  uint8, code s of (b,t,h) at codes[b*c_sb + t*c_st + h*c_sh + s]
 *   norms  float32 or NULL, norm s of (b,t,h) at norms[b*n_sb + t*n_st + n_sh*h + s]
 *   codebooks float32 [n_head][S][256][d]
 * Alignment: x rows 16-byte aligned (x base and strides multiples of 8 fp16 / 4 fp32 elements).
 * error_flag: optional device int32 that receives ZKV_DEVERR_TIMEOUT (see the conventions above).
 * smooth: optional float32 [n_head][d] per-channel key smoothing factors lambda (VeloxQuant
 *   "VecInfer": lambda_i = sqrt(max |K_i|) calibrated offline): each row is multiplied by
 *   1/lambda (float64 reciprocal, float64 product) before the rotation.  NULL: no smoothing.
 *   Decode must then be given the same factors (zkv_decode_params.k_smooth).
 * Errors: INVALID_ARG, UNSUPPORTED (d, S), CUDA.
 */
typedef struct {
  int64_t n_batch, n_tok, n_head;
  int d, S;
  int rotate;   /* 1: apply the Hadamard rotation first; 0: x is already rotated */
  int x_dtype;  /* ZKV_DTYPE_F16 or ZKV_DTYPE_F32 */
  const void* x;
  int64_t x_sb, x_st, x_sh;
  const float* codebooks;
  uint8_t* codes;
  int64_t c_sb, c_st, c_sh;
  float* norms;
  int64_t n_sb, n_st, n_sh;
  int32_t* error_flag;
  const float* smooth;
} zkv_encode_params;

int zkv_rvq_encode(const zkv_encode_params* p, void* stream);

/*
 * zkv_rvq_reconstruct -- x_hat = sum_s C[h][s][z_s] (float32, s ascending), optionally
 * rotated back: out = H_d x_hat / sqrt(d) (float64 transform, one rounding).
 * Passage: VQKV section 2.1 "Reconstruction".  Same row addressing as zkv_rvq_encode; `out`
 * is float32 with strides o_sb, o_st, o_sh (elements) and contiguous d.
 */
typedef struct {
  int64_t n_batch, n_tok, n_head;
  int d, S;
  int unrotate;
  const uint8_t* codes;
  int64_t c_sb, c_st, c_sh;
  const float* codebooks;
  float* out;
  int64_t o_sb, o_st, o_sh;
} zkv_reconstruct_params;

int zkv_rvq_reconstruct(const zkv_reconstruct_params* p, void* stream);

/*
 * zkv_rvq_decode_attn -- one decode step of attention over an RVQ-compressed prefix plus an
 * fp16 recency window, for every (sequence, query head) in one call.
 * Passages: VQKV section 2.3 "Decoding Stage" (on-demand reconstruction inside attention;
 * local sliding window); VeloxQuant "VecInfer" (q_tilde . k_tilde = q . k: the rotation is
 * applied to the query); Differential-KV "Flash-Style LSE Combine" (fp32 log-sum-exp merge).
 * Computes, for b < B, h < Hq, kvh = h / (Hq/Hkv):
 *   keys   = { H (sum_s Ck[kvh][s][zk[b][kvh][t][s]]) / sqrt(d) : t < comp_len[b] }
 *            U { win_k[b][kvh][w] : w < win_len[b] }                (values likewise)
 *   out[b][h] = softmax(softmax_scale * q[b][h] . keys) . values    (float32)
 *   lse[b][h] = natural log of sum exp(softmax_scale * q . k)        (float32, may be NULL)
 * An empty context gives out = 0 and lse = -inf.
 * Internally: q_tilde = H q / sqrt(d); per-stage tables LUT_s[c] = q_tilde . Ck_s[c]; scores
 * are sums of table entries; values are accumulated as per-codeword weight histograms that are
 * contracted with Cv once per (sequence, kv head); window and compressed part are joined by
 * the log-sum-exp combine.
 * Layouts:
 *   q        fp16  [B][Hq][d]
 *   k_codes  uint8 [B][Hkv][Tcap][Sk]      v_codes uint8 [B][Hkv][Tcap][Sv]
 *   comp_len int32 [B] (device)             compressed tokens of each sequence, <= Tcap
 *   k_codebooks float32 [Hkv][Sk][256][d]   v_codebooks float32 [Hkv][Sv][256][d]
 *   win_k, win_v fp16 [B][Hkv][Wcap][d]     slots 0..win_len[b]-1 are valid (any order)
 *   win_len  int32 [B] (device), <= Wcap
 *   out      float32 [B][Hq][d]             lse float32 [B][Hq] or NULL
 * max_comp_len: host-side upper bound on every comp_len[b] (<= Tcap); it sizes the launch.
 *   Tokens beyond it are not read.
 * softmax_scale: <= 0 selects 1/sqrt(d).
 * The first call on a device sets kernel shared-memory attributes; make it before capturing
 * calls into a CUDA graph.
 * Workspace: device buffer of at least zkv_decode_workspace_size(p) bytes, 256-byte aligned,
 *   no initial contents required; it must not be shared by calls that run concurrently.
 * Errors: INVALID_ARG, UNSUPPORTED (d, S, Hq/Hkv > 8, or a GQA group of 5..8 with Sv > 4,
 *         whose value histograms do not fit in one SM's shared memory), WORKSPACE, CUDA.
 */
typedef struct {
  int B, Hq, Hkv, d, Sk, Sv;
  int64_t Tcap, Wcap;
  int64_t max_comp_len;
  float softmax_scale;
  const uint16_t* q;
  const uint8_t* k_codes;
  const uint8_t* v_codes;
  const int32_t* comp_len;
  const float* k_codebooks;
  const float* v_codebooks;
  const uint16_t* win_k;
  const uint16_t* win_v;
  const int32_t* win_len;
  float* out;
  float* lse;
  int32_t* error_flag;
  /* Optional tracing: NULL, or 4 cudaEvent_t handles (as void*) recorded on `stream` before
   * the lookup-table kernel, before the scan kernel, before the combine kernel and after it.
   * While `stream` is being captured into a CUDA graph they become event-record nodes of the
   * graph (recorded at every replay). */
  void* const* trace_events;
  /* Optional float32 [Hkv][d]: the per-channel smoothing factors the compressed keys were
   * encoded with (zkv_encode_params.smooth).  The query is multiplied by them before its
   * rotation, so q_tilde . k_tilde = q . k (VeloxQuant "VecInfer").  The window keys are raw.
   * NULL: no smoothing. */
  const float* k_smooth;
  /* Optional paged code layout (serving with fixed token blocks): block_table int32
   * [B][max_pages] maps a sequence's page p (its tokens [p P, (p+1) P)) to a page of the pools;
   * k_codes / v_codes are then pools [n_pages][Hkv][P][Sk | Sv] (page index outermost, every
   * kv head's P rows contiguous inside a page), P = page_tokens a power of two in [32, 65536],
   * and Tcap must equal max_pages * P (the per-sequence capacity).  Pages need not be distinct
   * across sequences that never write them.  NULL: the contiguous layout above. */
  const int32_t* block_table;
  int64_t page_tokens, max_pages, n_pages;
} zkv_decode_params;

/* Workspace bytes for a call with these shapes (data pointers are not read); 0 if the shapes
 * are invalid or unsupported. */
size_t zkv_decode_workspace_size(const zkv_decode_params* p);
int zkv_rvq_decode_attn(const zkv_decode_params* p, void* workspace, size_t workspace_bytes,
                        void* stream);

/*
 * zkv_rvq_decode_attn_noalloc -- zkv_rvq_decode_attn without a caller workspace.  The web
 * pages have no counterpart: this is a library convenience for callers that cannot allocate
 * device memory per call (a host program with no device allocator of its own, or an engine
 * whose device memory is fully reserved up front).
 * Computes exactly what zkv_rvq_decode_attn computes, with the same parameters, layouts and
 * errors, using as workspace a device array inside this library of ZKV_DECODE_SCRATCH_BYTES
 * bytes (one per device, allocated when the library's device code is loaded; nothing is
 * allocated or freed by the call).
 *   - A call whose zkv_decode_workspace_size(p) exceeds ZKV_DECODE_SCRATCH_BYTES returns
 *     ZKV_ERR_WORKSPACE and launches nothing (8 x 32K-token GQA batches need about 6.6 MiB;
 *     64 sequences x 16K tokens need about 36 MiB and are refused).
 *   - Nothing in the array must start at zero: each call writes every word it reads.
 *   - There is ONE array per device: calls on the same device that overlap in time (different
 *     streams or host threads) race on it and give wrong results.  Order them (same stream,
 *     or events).  Calls on different devices do not interact.
 *   - Every call looks up the array's device address on the host (so it stays right after a
 *     device reset).  The first call on each device loads the library's device code and sets
 *     kernel attributes; make that first call before any stream capture.
 * Errors: as zkv_rvq_decode_attn; ZKV_ERR_CUDA if the array's address cannot be obtained.
 */
#define ZKV_DECODE_SCRATCH_BYTES (8u << 20)
int zkv_rvq_decode_attn_noalloc(const zkv_decode_params* p, void* stream);

/*
 * zkv_rvq_append -- one serving step of cache maintenance: each sequence's new token enters
 * the fp16 window; when the window is full, its oldest token is evicted, RVQ-encoded (same
 * rule as zkv_rvq_encode, rotate = 1) and appended to the compressed prefix.
 * Passages: VQKV section 2.3 "Local Sliding Window" (recent tokens uncompressed, middle tokens
 * compressed); VeloxQuant "Quick start" (cache.append then cache.attend).
 * Per sequence b (device-side state, updated in place):
 *   if win_len[b] < Wcap:  slot = win_len[b]; win_len[b] += 1
 *   else: slot = win_head[b]; encode win_k/win_v[b][:][slot] into k_codes/v_codes at position
 *         comp_len[b]; comp_len[b] += 1; win_head[b] = (slot + 1) % Wcap
 *   win_k[b][:][slot] = new_k[b]; win_v[b][:][slot] = new_v[b]
 * If comp_len[b] == Tcap when an eviction is due, sequence b is left unchanged and
 * ZKV_DEVERR_COMP_LEN is set.  Layouts as in zkv_rvq_decode_attn; new_k/new_v fp16 [B][Hkv][d];
 * win_head int32 [B].  No workspace.  Two kernels are launched (encode+write, then the length
 * update), so the state is consistent for any later work on the same stream.
 */
typedef struct {
  int B, Hkv, d, Sk, Sv;
  int64_t Tcap, Wcap;
  const uint16_t* new_k;
  const uint16_t* new_v;
  uint16_t* win_k;
  uint16_t* win_v;
  int32_t* win_len;
  int32_t* win_head;
  int32_t* comp_len;
  uint8_t* k_codes;
  uint8_t* v_codes;
  const float* k_codebooks;
  const float* v_codebooks;
  int32_t* error_flag;
  const float* k_smooth;   /* optional [Hkv][d]: evicted keys are smoothed as in zkv_rvq_encode */
  /* optional paged layout, as in zkv_decode_params (the evicted token's codes go to page
   * block_table[b][comp_len[b] / P]) */
  const int32_t* block_table;
  int64_t page_tokens, max_pages, n_pages;
} zkv_append_params;

int zkv_rvq_append(const zkv_append_params* p, void* stream);

/*
 * zkv_rvq_serve_step -- one whole decode step of a serving loop: zkv_rvq_append(ap) followed
 * by zkv_rvq_decode_attn(dp) on the updated cache, in one call.
 * Passages: VeloxQuant "Quick start" (cache.append(k, v), then cache.attend(q)); VQKV section
 * 2.3 "Local Sliding Window" and "Decoding Stage".
 * Results are identical to the two calls made in that order.  The library overlaps the
 * decode's lookup-table construction (which needs only q and the key codebooks), its partition
 * of the token space (computed from the lengths the append will produce) and its window
 * attention (over the window the append will produce: the pre-step rows with the new token in
 * the slot the append gives it) with the encode of the evicted tokens; the new lengths are
 * stored by the decode's scan kernel.
 * ap and dp describe one cache: B, Hkv, d, Sk, Sv, Tcap and Wcap must be equal, and so must
 * k_codes, v_codes, k_codebooks, v_codebooks, win_k, win_v, win_len, comp_len, k_smooth and the
 * paged layout (block_table, page_tokens, max_pages, n_pages) (else
 * ZKV_ERR_INVALID_ARG).  dp->comp_len and dp->win_len are read after the update, so
 * dp->max_comp_len must allow for the new token.  workspace: as zkv_rvq_decode_attn
 * (zkv_decode_workspace_size(dp)); dp->trace_events: as zkv_rvq_decode_attn, where the first
 * interval covers the tables, the encode and the length update.
 * Errors: those of zkv_rvq_append and zkv_rvq_decode_attn; validation of both happens before
 * any launch.
 */
int zkv_rvq_serve_step(const zkv_append_params* ap, const zkv_decode_params* dp,
                       void* workspace, size_t workspace_bytes, void* stream);

/*
 * zkv_pq_encode -- product vector quantisation of KV head vectors (VecInfer).
 * Passage: VeloxQuant "VecInfer" (smooth scaling + Walsh-Hadamard dual transform, then a
 * pre-trained K-means codebook over sub-vectors; key_sub_dim 4 or 8 with 8-bit codes).
 * Rows are addressed as in zkv_rvq_encode.  For each row:
 *   y = rotate ? float32(H_d (x / lambda) / sqrt(d)) : x / lambda   (lambda = smooth, or 1)
 *   z_j = argmin_c ||y[j m : (j+1) m] - C[h][c]||^2 for j < d / m  (float64, ties -> lowest c)
 * Layouts: x as in zkv_rvq_encode; codebook float32 [n_head][256][m] (one codebook per head,
 * shared by the sub-vectors); codes uint8, code j of (b,t,h) at
 * codes[b*c_sb + t*c_st + h*c_sh + j] (d / m contiguous bytes); smooth float32 [n_head][d] or
 * NULL.  d in {64, 128, 256}, m in {2, 4, 8, 16}.
 * Errors: INVALID_ARG, UNSUPPORTED (d, m), CUDA.
 */
typedef struct {
  int64_t n_batch, n_tok, n_head;
  int d, m;
  int rotate;
  int x_dtype;
  const void* x;
  int64_t x_sb, x_st, x_sh;
  const float* codebook;
  uint8_t* codes;
  int64_t c_sb, c_st, c_sh;
  const float* smooth;
} zkv_pq_encode_params;

int zkv_pq_encode(const zkv_pq_encode_params* p, void* stream);

/*
 * zkv_pq_append -- one serving step of cache maintenance for a product-VQ cache: each
 * sequence's new token enters the fp16 window; when the window is full its oldest token is
 * evicted, product-VQ encoded (as zkv_pq_encode with rotate = 1; keys smoothed by k_smooth
 * when given) and appended to the compressed prefix.
 * Passages: VeloxQuant "VecInfer" (product VQ of the smoothed, rotated vectors) and "Quick
 * start" (cache.append then cache.attend); VQKV section 2.3 "Local Sliding Window".
 * Per sequence b, the window rule of zkv_rvq_append:
 *   if win_len[b] < Wcap:  slot = win_len[b]; win_len[b] += 1
 *   else: slot = win_head[b]; encode win_k/win_v[b][:][slot] into k_codes/v_codes at position
 *         comp_len[b]; comp_len[b] += 1; win_head[b] = (slot + 1) % Wcap
 *   win_k[b][:][slot] = new_k[b]; win_v[b][:][slot] = new_v[b]
 * If comp_len[b] == Tcap when an eviction is due, sequence b is left unchanged and
 * ZKV_DEVERR_COMP_LEN is set (ZKV_DEVERR_WIN_LEN for a window length outside 0..Wcap).
 * Layouts: codes uint8 [B][Hkv][Tcap][d / m]; codebooks float32 [Hkv][256][m]; window fp16
 * [B][Hkv][Wcap][d]; new_k / new_v fp16 [B][Hkv][d]; lengths int32 [B]; k_smooth float32
 * [Hkv][d] or NULL.  d in {64, 128, 256}, m in {2, 4, 8, 16}, Wcap >= 1.  Two kernels are
 * launched (encode + window write, then the length update).  No workspace.
 * Errors: INVALID_ARG, UNSUPPORTED (d, m), CUDA.
 */
typedef struct {
  int B, Hkv, d, m;
  int64_t Tcap, Wcap;
  const uint16_t* new_k;
  const uint16_t* new_v;
  uint16_t* win_k;
  uint16_t* win_v;
  int32_t* win_len;
  int32_t* win_head;
  int32_t* comp_len;
  uint8_t* k_codes;
  uint8_t* v_codes;
  const float* k_codebook;
  const float* v_codebook;
  int32_t* error_flag;
  const float* k_smooth;
} zkv_pq_append_params;

int zkv_pq_append(const zkv_pq_append_params* p, void* stream);

/*
 * zkv_pq_decode_attn -- decode attention over a product-VQ compressed prefix (zkv_pq_encode's
 * codes, keys and values) plus the fp16 recency window.
 * Passages: VeloxQuant "VecInfer" (product VQ with the dual transform absorbed into the query);
 * VQKV section 2.3 "Decoding Stage" and "Local Sliding Window"; Differential-KV "Flash-Style
 * LSE Combine".
 * Computes what zkv_rvq_decode_attn computes with the keys / values reconstructed as
 *   k_t = lambda * H concat_j Ck[kvh][zk_{t,j}] / sqrt(d),  v_t = H concat_j Cv[kvh][zv_{t,j}] / sqrt(d)
 * (lambda = k_smooth, or 1).  Internally lane j of a warp (of each 16-lane half when d / m = 16)
 * owns sub-vector j of its tokens (the scores of 32 / GP tokens are reduced together), per head
 * a running maximum, the values accumulated per lane: no histograms.
 * Shapes: d / m = 32 or 16 -- (d, m) in {(64, 2), (64, 4), (128, 4), (128, 8), (256, 8)}, i.e.
 * 2 or 1 code bits per element at d = 128; Hq / Hkv <= 8, <= 4 at (128, 8), <= 2 at d = 256.  Layouts: k_codes / v_codes uint8 [B][Hkv][Tcap][d / m]; k_codebook / v_codebook
 * float32 [Hkv][256][m]; the rest as zkv_rvq_decode_attn.  Workspace:
 * zkv_pq_decode_workspace_size(p) bytes, 256-byte aligned.  Two kernels are launched.
 * Errors: INVALID_ARG, UNSUPPORTED (shapes), WORKSPACE, CUDA; device-side length errors as in
 * zkv_rvq_decode_attn.
 */
typedef struct {
  int B, Hq, Hkv, d, m;
  int64_t Tcap, Wcap, max_comp_len;
  float softmax_scale;
  const uint16_t* q;
  const uint8_t* k_codes;
  const uint8_t* v_codes;
  const int32_t* comp_len;
  const float* k_codebook;
  const float* v_codebook;
  const uint16_t* win_k;
  const uint16_t* win_v;
  const int32_t* win_len;
  float* out;
  float* lse;
  int32_t* error_flag;
  const float* k_smooth;
} zkv_pq_decode_params;

size_t zkv_pq_decode_workspace_size(const zkv_pq_decode_params* p);
int zkv_pq_decode_attn(const zkv_pq_decode_params* p, void* workspace, size_t workspace_bytes,
                       void* stream);

/*
 * zkv_lse_merge -- log-sum-exp combine of partial attention results over disjoint key sets
 * (context-parallel decode: every rank attends over its shard of each compressed prefix, the
 * shards' (out, lse) are gathered and combined).
 * Passage: Differential-KV "Decode & Prefill Innovations" (fp32 log-sum-exp combine).
 * For each row r:  M = max_i lse[i][r];  w_i = exp(lse[i][r] - M);  L = sum_i w_i;
 *   out[r] = sum_i w_i part_out[i][r] / L;  lse_out[r] = M + log L   (float32)
 * A part with lse = -inf (no keys) has weight 0; a row whose parts are all empty gets out = 0,
 * lse = -inf.  Layouts (strides in floats): part_out element (i, r, e) at
 * part_out[i * out_part_stride + r * out_row_stride + e]; part_lse element (i, r) at
 * part_lse[i * lse_part_stride + r * lse_row_stride] (natural log, as zkv_rvq_decode_attn
 * writes it) -- so a gathered [n_parts][rows][d + 1] buffer of packed (out, lse) rows is read in
 * place; out float32 [rows][d] contiguous, lse [rows] (may be NULL).
 * Errors: INVALID_ARG (n_parts < 1, d not in 1..4096, null pointers with rows > 0), CUDA.
 */
typedef struct {
  int64_t n_parts, rows;
  int d;
  const float* part_out;
  int64_t out_part_stride, out_row_stride;
  const float* part_lse;
  int64_t lse_part_stride, lse_row_stride;
  float* out;
  float* lse;
} zkv_lse_merge_params;

int zkv_lse_merge(const zkv_lse_merge_params* p, void* stream);

/*
 * zkv_lse_merge_peers -- the context-parallel exchange and the log-sum-exp combine as ONE
 * kernel over peer memory (in place of an all-gather followed by zkv_lse_merge).
 * Passage: Differential-KV "Decode & Prefill Innovations" (fp32 log-sum-exp combine of
 * partial attentions over disjoint key sets).
 * Every rank's decode has written its partial (out [rows][d], lse [rows]) into buffers that
 * every rank can address (symmetric / IPC-mapped device memory).  The kernel, on rank `rank`
 * of n_ranks:
 *   1. signals: stores `epoch` into word `rank` of every rank's flag array (release, system
 *      scope; every block stores the same value, so no block waits for another to run);
 *   2. waits until every word of its own flag array has reached `epoch` (acquire, system
 *      scope), for at most timeout_ns nanoseconds of the device's global timer;
 *   3. reads every rank's rows straight from that rank's memory (cache-bypassing loads over
 *      NVLink) and combines them exactly as zkv_lse_merge.
 * If the wait runs out, ZKV_DEVERR_TIMEOUT is OR-ed into error_flag and the blocks that timed
 * out leave their rows of out / lse unwritten; nothing hangs.
 * Arguments: part_out / part_lse / flags are DEVICE arrays of n_ranks device pointers
 * (rank i's out rows, lse rows and flag array of n_ranks uint32 words, as mapped in this
 * process); epoch >= 1, one more than the previous call's on the same flags (flags start at
 * 0; compared modulo 2^32).  A rank's out / lse buffers must not be rewritten until every
 * rank has passed the next call's wait: alternating two buffer sets by epoch parity gives
 * exactly that.  out float32 [rows][d], lse [rows] (may be NULL).  d in 1..4096,
 * 1 <= n_ranks <= 64, 0 <= rank < n_ranks.
 * Errors: INVALID_ARG, CUDA.
 */
typedef struct {
  int n_ranks, rank;
  int64_t rows;
  int d;
  const float* const* part_out;
  const float* const* part_lse;
  uint32_t* const* flags;
  uint32_t epoch;
  int64_t timeout_ns;
  float* out;
  float* lse;
  int32_t* error_flag;
} zkv_lse_merge_peers_params;

int zkv_lse_merge_peers(const zkv_lse_merge_peers_params* p, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* ZKV_H */
