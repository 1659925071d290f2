"""Thin ctypes binding of libzkv (include/zkv.h): argument marshalling only.

Every computation runs in the library's CUDA kernels; PyTorch supplies device memory and the
current CUDA stream.  If the library is missing or a call fails, an exception is raised -- there
is no fallback path.

Entry points (same names as the C ABI):
  fwht, rvq_encode, rvq_reconstruct, decode_workspace_size, rvq_decode_attn,
  rvq_decode_attn_noalloc, rvq_append
plus PreparedAppend / PreparedDecode (the same calls with their arguments marshalled once)
and ``RVQKVCache``, a small owner of one layer's compressed cache built on them
(prefill -> append -> attend, the append/attend cache interface of the VeloxQuant-MLX page).
"""
from __future__ import annotations

import ctypes
import math
import os
from ctypes import POINTER, c_float, c_int, c_int64, c_size_t, c_void_p

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libzkv.so")

ZKV_OK, ZKV_ERR_INVALID_ARG, ZKV_ERR_UNSUPPORTED, ZKV_ERR_WORKSPACE, ZKV_ERR_CUDA = range(5)
ZKV_DEVERR_COMP_LEN = 1
ZKV_DEVERR_WIN_LEN = 2
ZKV_DEVERR_TIMEOUT = 4
ZKV_DEVERR_PAGE = 8
ZKV_DEVERR_SMEM = 16
ZKV_DTYPE_F16, ZKV_DTYPE_F32 = 0, 1
CODEBOOK_SIZE = 256
DECODE_SCRATCH_BYTES = 8 << 20   # ZKV_DECODE_SCRATCH_BYTES: the no-allocation decode's array


class ZkvError(RuntimeError):
    def __init__(self, fn: str, status: int, detail: str = ""):
        super().__init__(f"{fn} failed: {status_string(status)} ({status})"
                         + (f": {detail}" if detail else ""))
        self.status = status


class EncodeParams(ctypes.Structure):
    _fields_ = [("n_batch", c_int64), ("n_tok", c_int64), ("n_head", c_int64),
                ("d", c_int), ("S", c_int), ("rotate", c_int), ("x_dtype", c_int),
                ("x", c_void_p), ("x_sb", c_int64), ("x_st", c_int64), ("x_sh", c_int64),
                ("codebooks", c_void_p),
                ("codes", c_void_p), ("c_sb", c_int64), ("c_st", c_int64), ("c_sh", c_int64),
                ("norms", c_void_p), ("n_sb", c_int64), ("n_st", c_int64), ("n_sh", c_int64),
                ("error_flag", c_void_p), ("smooth", c_void_p)]


class ReconstructParams(ctypes.Structure):
    _fields_ = [("n_batch", c_int64), ("n_tok", c_int64), ("n_head", c_int64),
                ("d", c_int), ("S", c_int), ("unrotate", c_int),
                ("codes", c_void_p), ("c_sb", c_int64), ("c_st", c_int64), ("c_sh", c_int64),
                ("codebooks", c_void_p),
                ("out", c_void_p), ("o_sb", c_int64), ("o_st", c_int64), ("o_sh", c_int64)]


class DecodeParams(ctypes.Structure):
    _fields_ = [("B", c_int), ("Hq", c_int), ("Hkv", c_int), ("d", c_int), ("Sk", c_int),
                ("Sv", c_int), ("Tcap", c_int64), ("Wcap", c_int64), ("max_comp_len", c_int64),
                ("softmax_scale", c_float),
                ("q", c_void_p), ("k_codes", c_void_p), ("v_codes", c_void_p),
                ("comp_len", c_void_p), ("k_codebooks", c_void_p), ("v_codebooks", c_void_p),
                ("win_k", c_void_p), ("win_v", c_void_p), ("win_len", c_void_p),
                ("out", c_void_p), ("lse", c_void_p), ("error_flag", c_void_p),
                ("trace_events", c_void_p), ("k_smooth", c_void_p),
                ("block_table", c_void_p), ("page_tokens", c_int64), ("max_pages", c_int64),
                ("n_pages", c_int64)]


class AppendParams(ctypes.Structure):
    _fields_ = [("B", c_int), ("Hkv", c_int), ("d", c_int), ("Sk", c_int), ("Sv", c_int),
                ("Tcap", c_int64), ("Wcap", c_int64),
                ("new_k", c_void_p), ("new_v", c_void_p), ("win_k", c_void_p),
                ("win_v", c_void_p), ("win_len", c_void_p), ("win_head", c_void_p),
                ("comp_len", c_void_p), ("k_codes", c_void_p), ("v_codes", c_void_p),
                ("k_codebooks", c_void_p), ("v_codebooks", c_void_p), ("error_flag", c_void_p),
                ("k_smooth", c_void_p), ("block_table", c_void_p), ("page_tokens", c_int64),
                ("max_pages", c_int64), ("n_pages", c_int64)]


class PQEncodeParams(ctypes.Structure):
    _fields_ = [("n_batch", c_int64), ("n_tok", c_int64), ("n_head", c_int64),
                ("d", c_int), ("m", c_int), ("rotate", c_int), ("x_dtype", c_int),
                ("x", c_void_p), ("x_sb", c_int64), ("x_st", c_int64), ("x_sh", c_int64),
                ("codebook", c_void_p),
                ("codes", c_void_p), ("c_sb", c_int64), ("c_st", c_int64), ("c_sh", c_int64),
                ("smooth", c_void_p)]


class PQDecodeParams(ctypes.Structure):
    _fields_ = [("B", c_int), ("Hq", c_int), ("Hkv", c_int), ("d", c_int), ("m", c_int),
                ("Tcap", c_int64), ("Wcap", c_int64), ("max_comp_len", c_int64),
                ("softmax_scale", c_float),
                ("q", c_void_p), ("k_codes", c_void_p), ("v_codes", c_void_p),
                ("comp_len", c_void_p), ("k_codebook", c_void_p), ("v_codebook", c_void_p),
                ("win_k", c_void_p), ("win_v", c_void_p), ("win_len", c_void_p),
                ("out", c_void_p), ("lse", c_void_p), ("error_flag", c_void_p),
                ("k_smooth", c_void_p)]


class PQAppendParams(ctypes.Structure):
    _fields_ = [("B", c_int), ("Hkv", c_int), ("d", c_int), ("m", c_int),
                ("Tcap", c_int64), ("Wcap", c_int64),
                ("new_k", c_void_p), ("new_v", c_void_p), ("win_k", c_void_p),
                ("win_v", c_void_p), ("win_len", c_void_p), ("win_head", c_void_p),
                ("comp_len", c_void_p), ("k_codes", c_void_p), ("v_codes", c_void_p),
                ("k_codebook", c_void_p), ("v_codebook", c_void_p), ("error_flag", c_void_p),
                ("k_smooth", c_void_p)]


class MergeParams(ctypes.Structure):
    _fields_ = [("n_parts", c_int64), ("rows", c_int64), ("d", c_int),
                ("part_out", c_void_p), ("out_part_stride", c_int64), ("out_row_stride", c_int64),
                ("part_lse", c_void_p), ("lse_part_stride", c_int64), ("lse_row_stride", c_int64),
                ("out", c_void_p), ("lse", c_void_p)]


class MergePeersParams(ctypes.Structure):
    _fields_ = [("n_ranks", c_int), ("rank", c_int), ("rows", c_int64), ("d", c_int),
                ("part_out", c_void_p), ("part_lse", c_void_p), ("flags", c_void_p),
                ("epoch", ctypes.c_uint32), ("timeout_ns", c_int64),
                ("out", c_void_p), ("lse", c_void_p), ("error_flag", c_void_p)]


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded libzkv.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libzkv.so not found at {LIB_PATH}; build it with "
                              "`python -m compressed_decode_attention_zkv_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        L.zkv_status_string.restype = ctypes.c_char_p
        L.zkv_status_string.argtypes = [c_int]
        L.zkv_version.restype = c_int
        L.zkv_fwht.restype = c_int
        L.zkv_fwht.argtypes = [c_void_p, c_int, c_void_p, c_int64, c_int, c_float, c_void_p]
        L.zkv_rvq_encode.restype = c_int
        L.zkv_rvq_encode.argtypes = [POINTER(EncodeParams), c_void_p]
        L.zkv_rvq_reconstruct.restype = c_int
        L.zkv_rvq_reconstruct.argtypes = [POINTER(ReconstructParams), c_void_p]
        L.zkv_decode_workspace_size.restype = c_size_t
        L.zkv_decode_workspace_size.argtypes = [POINTER(DecodeParams)]
        L.zkv_rvq_decode_attn.restype = c_int
        L.zkv_rvq_decode_attn.argtypes = [POINTER(DecodeParams), c_void_p, c_size_t, c_void_p]
        L.zkv_rvq_decode_attn_noalloc.restype = c_int
        L.zkv_rvq_decode_attn_noalloc.argtypes = [POINTER(DecodeParams), c_void_p]
        L.zkv_rvq_append.restype = c_int
        L.zkv_rvq_append.argtypes = [POINTER(AppendParams), c_void_p]
        L.zkv_pq_encode.restype = c_int
        L.zkv_pq_encode.argtypes = [POINTER(PQEncodeParams), c_void_p]
        L.zkv_pq_append.restype = c_int
        L.zkv_pq_append.argtypes = [POINTER(PQAppendParams), c_void_p]
        L.zkv_pq_decode_workspace_size.restype = c_size_t
        L.zkv_pq_decode_workspace_size.argtypes = [POINTER(PQDecodeParams)]
        L.zkv_pq_decode_attn.restype = c_int
        L.zkv_pq_decode_attn.argtypes = [POINTER(PQDecodeParams), c_void_p, c_size_t, c_void_p]
        L.zkv_lse_merge_peers.restype = c_int
        L.zkv_lse_merge_peers.argtypes = [POINTER(MergePeersParams), c_void_p]
        L.zkv_lse_merge.restype = c_int
        L.zkv_lse_merge.argtypes = [POINTER(MergeParams), c_void_p]
        L.zkv_rvq_serve_step.restype = c_int
        L.zkv_rvq_serve_step.argtypes = [POINTER(AppendParams), POINTER(DecodeParams), c_void_p,
                                         c_size_t, c_void_p]
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().zkv_status_string(int(status)).decode()


def _check(fn: str, status: int):
    if status != ZKV_OK:
        raise ZkvError(fn, status)


def _stream() -> int:
    return torch.cuda.current_stream().cuda_stream


def _ptr(t):
    return None if t is None else t.data_ptr()


def _code_layout(k_codes, block_table):
    """(Hkv, Tcap, Sk, paged fields) of a contiguous [B, Hkv, Tcap, Sk] code array, or of a page
    pool [n_pages, Hkv, P, Sk] with an int32 [B, max_pages] block table."""
    if block_table is None:
        _, Hkv, Tcap, Sk = k_codes.shape
        return Hkv, Tcap, Sk, dict(block_table=None, page_tokens=0, max_pages=0, n_pages=0)
    _need(block_table, "block_table", torch.int32)
    n_pages, Hkv, P, Sk = k_codes.shape
    max_pages = block_table.shape[1]
    return Hkv, max_pages * P, Sk, dict(block_table=_ptr(block_table), page_tokens=P,
                                        max_pages=max_pages, n_pages=n_pages)


def _smooth_ptr(lam, heads: int, d: int, name: str) -> int | None:
    """Pointer of a float32 [heads, d] contiguous CUDA tensor of smoothing factors (or None)."""
    if lam is None:
        return None
    _need(lam, name, torch.float32)
    if tuple(lam.shape) != (heads, d):
        raise ValueError(f"{name} must be [{heads}, {d}], got {tuple(lam.shape)}")
    return _ptr(lam)


def _need(t: torch.Tensor, name: str, dtype, contiguous=True):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if contiguous and not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


# --------------------------------------------------------------------------------------------
# Entry points
# --------------------------------------------------------------------------------------------

def fwht(x: torch.Tensor, scale: float, out: torch.Tensor | None = None) -> torch.Tensor:
    """out = float32(scale * H_d x) for every row of x ([..., d], fp16 or fp32)."""
    if x.dtype not in (torch.float16, torch.float32):
        raise TypeError("x must be fp16 or fp32")
    _need(x, "x", x.dtype)
    d = x.shape[-1]
    if out is None:
        out = torch.empty(x.shape, dtype=torch.float32, device=x.device)
    _need(out, "out", torch.float32)
    dt = ZKV_DTYPE_F16 if x.dtype == torch.float16 else ZKV_DTYPE_F32
    _check("zkv_fwht", lib().zkv_fwht(_ptr(x), dt, _ptr(out), x.numel() // d, d,
                                      float(scale), _stream()))
    return out


def _as4(t: torch.Tensor, name: str) -> torch.Tensor:
    if t.dim() == 2:
        return t[None, :, None, :]
    if t.dim() == 3:
        return t[None]
    if t.dim() == 4:
        return t
    raise ValueError(f"{name} must be [N, X], [T, H, X] or [B, T, H, X]")


def rvq_encode(x: torch.Tensor, codebooks: torch.Tensor, codes: torch.Tensor | None = None,
               norms: torch.Tensor | None = None, rotate: bool = True,
               with_norms: bool = True, error_flag: torch.Tensor | None = None,
               smooth: torch.Tensor | None = None):
    """Greedy RVQ of x rows.  x: [B, T, H, d] view (any strides, d contiguous), or [T, H, d],
    or [N, d] (one head).  codebooks: [H, S, 256, d] float32 contiguous.  error_flag: optional
    int32 device word that receives ZKV_DEVERR_TIMEOUT.  smooth: optional float32 [H, d] key
    smoothing factors (rows are divided by them before the rotation).
    Returns (codes uint8 [B, T, H, S] view, norms float32 [B, T, H, S] or None)."""
    if x.dtype not in (torch.float16, torch.float32):
        raise TypeError("x must be fp16 or fp32")
    _need(x, "x", x.dtype, contiguous=False)
    _need(codebooks, "codebooks", torch.float32)
    x4 = _as4(x, "x")
    if x4.stride(-1) != 1:
        raise ValueError("x rows must be contiguous")
    Bn, T, H, d = x4.shape
    S = codebooks.shape[1]
    if codebooks.shape != (H, S, CODEBOOK_SIZE, d):
        raise ValueError(f"codebooks must be [H={H}, S, 256, d={d}], got {tuple(codebooks.shape)}")
    if codes is None:
        codes = torch.empty((Bn, T, H, S), dtype=torch.uint8, device=x.device)
    if norms is None and with_norms:
        norms = torch.empty((Bn, T, H, S), dtype=torch.float32, device=x.device)
    _need(codes, "codes", torch.uint8, contiguous=False)
    c4 = _as4(codes, "codes")
    if c4.shape != (Bn, T, H, S) or c4.stride(-1) != 1:
        raise ValueError("codes must be a [B, T, H, S] view with contiguous S")
    p = EncodeParams(n_batch=Bn, n_tok=T, n_head=H, d=d, S=S, rotate=int(bool(rotate)),
                     x_dtype=ZKV_DTYPE_F16 if x.dtype == torch.float16 else ZKV_DTYPE_F32,
                     x=_ptr(x4), x_sb=x4.stride(0), x_st=x4.stride(1), x_sh=x4.stride(2),
                     codebooks=_ptr(codebooks), codes=_ptr(c4), c_sb=c4.stride(0),
                     c_st=c4.stride(1), c_sh=c4.stride(2))
    if norms is not None:
        _need(norms, "norms", torch.float32, contiguous=False)
        n4 = _as4(norms, "norms")
        if n4.shape != (Bn, T, H, S) or n4.stride(-1) != 1:
            raise ValueError("norms must be a [B, T, H, S] view with contiguous S")
        p.norms, p.n_sb, p.n_st, p.n_sh = _ptr(n4), n4.stride(0), n4.stride(1), n4.stride(2)
    if error_flag is not None:
        _need(error_flag, "error_flag", torch.int32)
        p.error_flag = _ptr(error_flag)
    p.smooth = _smooth_ptr(smooth, H, d, "smooth")
    _check("zkv_rvq_encode", lib().zkv_rvq_encode(ctypes.byref(p), _stream()))
    return codes, norms


def rvq_reconstruct(codes: torch.Tensor, codebooks: torch.Tensor, unrotate: bool = False,
                    out: torch.Tensor | None = None) -> torch.Tensor:
    """x_hat = sum_s C[h][s][z_s] for codes [B, T, H, S] (views allowed); returns float32
    [B, T, H, d] (rotated back by H/sqrt(d) when ``unrotate``)."""
    _need(codes, "codes", torch.uint8, contiguous=False)
    _need(codebooks, "codebooks", torch.float32)
    c4 = _as4(codes, "codes")
    Bn, T, H, S = c4.shape
    d = codebooks.shape[-1]
    if codebooks.shape != (H, S, CODEBOOK_SIZE, d):
        raise ValueError("codebooks must be [H, S, 256, d]")
    if out is None:
        out = torch.empty((Bn, T, H, d), dtype=torch.float32, device=codes.device)
    _need(out, "out", torch.float32, contiguous=False)
    o4 = _as4(out, "out")
    p = ReconstructParams(n_batch=Bn, n_tok=T, n_head=H, d=d, S=S, unrotate=int(bool(unrotate)),
                          codes=_ptr(c4), c_sb=c4.stride(0), c_st=c4.stride(1), c_sh=c4.stride(2),
                          codebooks=_ptr(codebooks), out=_ptr(o4), o_sb=o4.stride(0),
                          o_st=o4.stride(1), o_sh=o4.stride(2))
    _check("zkv_rvq_reconstruct", lib().zkv_rvq_reconstruct(ctypes.byref(p), _stream()))
    return out


def _decode_params(q, k_codes, v_codes, comp_len, k_codebooks, v_codebooks, win_k, win_v,
                   win_len, out, lse, max_comp_len, softmax_scale, error_flag,
                   k_smooth=None, block_table=None) -> DecodeParams:
    _need(q, "q", torch.float16)
    _need(k_codes, "k_codes", torch.uint8)
    _need(v_codes, "v_codes", torch.uint8)
    _need(comp_len, "comp_len", torch.int32)
    _need(win_len, "win_len", torch.int32)
    _need(k_codebooks, "k_codebooks", torch.float32)
    _need(v_codebooks, "v_codebooks", torch.float32)
    _need(win_k, "win_k", torch.float16)
    _need(win_v, "win_v", torch.float16)
    B, Hq, d = q.shape
    Hkv, Tcap, Sk, paged = _code_layout(k_codes, block_table)
    Sv = v_codes.shape[3]
    Wcap = win_k.shape[2]
    if out is not None:
        _need(out, "out", torch.float32)
    if lse is not None:
        _need(lse, "lse", torch.float32)
    if error_flag is not None:
        _need(error_flag, "error_flag", torch.int32)
    return DecodeParams(B=B, Hq=Hq, Hkv=Hkv, d=d, Sk=Sk, Sv=Sv, Tcap=Tcap, Wcap=Wcap,
                        max_comp_len=Tcap if max_comp_len is None else int(max_comp_len),
                        softmax_scale=0.0 if softmax_scale is None else float(softmax_scale),
                        q=_ptr(q), k_codes=_ptr(k_codes), v_codes=_ptr(v_codes),
                        comp_len=_ptr(comp_len), k_codebooks=_ptr(k_codebooks),
                        v_codebooks=_ptr(v_codebooks), win_k=_ptr(win_k), win_v=_ptr(win_v),
                        win_len=_ptr(win_len), out=_ptr(out), lse=_ptr(lse),
                        error_flag=_ptr(error_flag),
                        k_smooth=_smooth_ptr(k_smooth, Hkv, d, "k_smooth"), **paged)


def decode_workspace_size(q, k_codes, v_codes, comp_len, k_codebooks, v_codebooks, win_k,
                          win_v, win_len, max_comp_len=None, block_table=None) -> int:
    p = _decode_params(q, k_codes, v_codes, comp_len, k_codebooks, v_codebooks, win_k, win_v,
                       win_len, None, None, max_comp_len, None, None, None, block_table)
    n = lib().zkv_decode_workspace_size(ctypes.byref(p))
    if n == 0:
        raise ZkvError("zkv_decode_workspace_size", ZKV_ERR_INVALID_ARG)
    return n


def rvq_decode_attn(q, k_codes, v_codes, comp_len, k_codebooks, v_codebooks, win_k, win_v,
                    win_len, out=None, lse=None, max_comp_len=None, softmax_scale=None,
                    workspace: torch.Tensor | None = None, error_flag=None, trace_events=None,
                    k_smooth=None, block_table=None):
    """Decode attention over the compressed prefix plus the fp16 window (see include/zkv.h).
    ``trace_events``: optional 4 torch.cuda.Event(enable_timing=True) recorded before the
    table, scan and combine kernels and after the last one (graph nodes under capture).  ``k_smooth``: the [Hkv, d] key
    smoothing factors the prefix was encoded with.  ``block_table``: int32 [B, max_pages] for
    the paged layout (k_codes / v_codes are then page pools [n_pages, Hkv, P, S]).
    Returns (out float32 [B, Hq, d], lse float32 [B, Hq])."""
    B, Hq, d = q.shape
    if out is None:
        out = torch.empty((B, Hq, d), dtype=torch.float32, device=q.device)
    if lse is None:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    p = _decode_params(q, k_codes, v_codes, comp_len, k_codebooks, v_codebooks, win_k, win_v,
                       win_len, out, lse, max_comp_len, softmax_scale, error_flag, k_smooth,
                       block_table)
    ev_arr = None
    if trace_events is not None:
        if len(trace_events) != 4:
            raise ValueError("trace_events needs 4 events")
        ev_arr = (c_void_p * 4)(*[e.cuda_event for e in trace_events])
        p.trace_events = ctypes.cast(ev_arr, c_void_p)
    need = lib().zkv_decode_workspace_size(ctypes.byref(p))
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    _need(workspace, "workspace", torch.uint8)
    _check("zkv_rvq_decode_attn",
           lib().zkv_rvq_decode_attn(ctypes.byref(p), _ptr(workspace), workspace.numel(),
                                     _stream()))
    return out, lse


def rvq_decode_attn_noalloc(q, k_codes, v_codes, comp_len, k_codebooks, v_codebooks, win_k,
                            win_v, win_len, out=None, lse=None, max_comp_len=None,
                            softmax_scale=None, error_flag=None, k_smooth=None):
    """rvq_decode_attn with the library's fixed device scratch array as workspace
    (zkv_rvq_decode_attn_noalloc).  Calls on one device must not overlap in time.  Raises
    ZkvError(ZKV_ERR_WORKSPACE) when the shapes need more than DECODE_SCRATCH_BYTES."""
    B, Hq, d = q.shape
    if out is None:
        out = torch.empty((B, Hq, d), dtype=torch.float32, device=q.device)
    if lse is None:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    p = _decode_params(q, k_codes, v_codes, comp_len, k_codebooks, v_codebooks, win_k, win_v,
                       win_len, out, lse, max_comp_len, softmax_scale, error_flag, k_smooth)
    status = lib().zkv_rvq_decode_attn_noalloc(ctypes.byref(p), _stream())
    if status == ZKV_ERR_WORKSPACE:
        need = lib().zkv_decode_workspace_size(ctypes.byref(p))
        raise ZkvError("zkv_rvq_decode_attn_noalloc", status,
                       f"these shapes need {need} bytes of workspace; the library's scratch "
                       f"array holds {DECODE_SCRATCH_BYTES}; use rvq_decode_attn")
    _check("zkv_rvq_decode_attn_noalloc", status)
    return out, lse


def _append_params(new_k, new_v, win_k, win_v, win_len, win_head, comp_len, k_codes, v_codes,
                   k_codebooks, v_codebooks, error_flag, k_smooth=None, block_table=None):
    _need(new_k, "new_k", torch.float16)
    _need(new_v, "new_v", torch.float16)
    for n, t in (("win_k", win_k), ("win_v", win_v)):
        _need(t, n, torch.float16)
    for n, t in (("win_len", win_len), ("win_head", win_head), ("comp_len", comp_len)):
        _need(t, n, torch.int32)
    _need(k_codes, "k_codes", torch.uint8)
    _need(v_codes, "v_codes", torch.uint8)
    _need(k_codebooks, "k_codebooks", torch.float32)
    _need(v_codebooks, "v_codebooks", torch.float32)
    if error_flag is not None:
        _need(error_flag, "error_flag", torch.int32)
    B = new_k.shape[0]
    Hkv, Tcap, Sk, paged = _code_layout(k_codes, block_table)
    return AppendParams(B=B, Hkv=Hkv, d=new_k.shape[-1], Sk=Sk, Sv=v_codes.shape[3], Tcap=Tcap,
                        Wcap=win_k.shape[2], new_k=_ptr(new_k), new_v=_ptr(new_v),
                        win_k=_ptr(win_k), win_v=_ptr(win_v), win_len=_ptr(win_len),
                        win_head=_ptr(win_head), comp_len=_ptr(comp_len), k_codes=_ptr(k_codes),
                        v_codes=_ptr(v_codes), k_codebooks=_ptr(k_codebooks),
                        v_codebooks=_ptr(v_codebooks), error_flag=_ptr(error_flag),
                        k_smooth=_smooth_ptr(k_smooth, Hkv, new_k.shape[-1], "k_smooth"),
                        **paged)


def rvq_append(new_k, new_v, win_k, win_v, win_len, win_head, comp_len, k_codes, v_codes,
               k_codebooks, v_codebooks, error_flag=None, k_smooth=None, block_table=None):
    """One serving step of cache maintenance (see include/zkv.h); state updated in place."""
    p = _append_params(new_k, new_v, win_k, win_v, win_len, win_head, comp_len, k_codes,
                       v_codes, k_codebooks, v_codebooks, error_flag, k_smooth, block_table)
    _check("zkv_rvq_append", lib().zkv_rvq_append(ctypes.byref(p), _stream()))


class PreparedAppend:
    """rvq_append with its arguments validated and marshalled once.  The tensors must keep their
    storage (their contents may change between calls); calling the object runs one serving
    step on the current stream with no per-call Python work beyond the library call."""

    def __init__(self, new_k, new_v, win_k, win_v, win_len, win_head, comp_len, k_codes,
                 v_codes, k_codebooks, v_codebooks, error_flag=None, k_smooth=None):
        self._keep = (new_k, new_v, win_k, win_v, win_len, win_head, comp_len, k_codes, v_codes,
                      k_codebooks, v_codebooks, error_flag, k_smooth)
        self._p = _append_params(new_k, new_v, win_k, win_v, win_len, win_head, comp_len,
                                 k_codes, v_codes, k_codebooks, v_codebooks, error_flag, k_smooth)
        self._ref = ctypes.byref(self._p)
        self._fn = lib().zkv_rvq_append

    def __call__(self):
        st = self._fn(self._ref, torch.cuda.current_stream().cuda_stream)
        if st != ZKV_OK:
            raise ZkvError("zkv_rvq_append", st)


class PreparedServeStep:
    """One serving step (append of the new tokens, then decode attention of q over the updated
    cache) as a single library call, zkv_rvq_serve_step, with its arguments marshalled once.
    The tensors must keep their storage; max_comp_len must stay an upper bound of every
    comp_len after the step.  Calling it runs the step on the current stream and returns
    (out, lse)."""

    def __init__(self, new_k, new_v, q, win_k, win_v, win_len, win_head, comp_len, k_codes,
                 v_codes, k_codebooks, v_codebooks, out=None, lse=None, max_comp_len=None,
                 softmax_scale=None, workspace: torch.Tensor | None = None, error_flag=None,
                 trace_events=None, k_smooth=None, block_table=None):
        B, Hq, d = q.shape
        if out is None:
            out = torch.empty((B, Hq, d), dtype=torch.float32, device=q.device)
        if lse is None:
            lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
        self._pa = _append_params(new_k, new_v, win_k, win_v, win_len, win_head, comp_len,
                                  k_codes, v_codes, k_codebooks, v_codebooks, error_flag,
                                  k_smooth, block_table)
        self._pd = _decode_params(q, k_codes, v_codes, comp_len, k_codebooks, v_codebooks, win_k,
                                  win_v, win_len, out, lse, max_comp_len, softmax_scale,
                                  error_flag, k_smooth, block_table)
        self._ev = None
        if trace_events is not None:   # recorded before the tables, the scan, the combine, and last
            if len(trace_events) != 4:
                raise ValueError("trace_events needs 4 events")
            self._ev = (c_void_p * 4)(*[e.cuda_event for e in trace_events])
            self._pd.trace_events = ctypes.cast(self._ev, c_void_p)
        need = lib().zkv_decode_workspace_size(ctypes.byref(self._pd))
        if need == 0:
            raise ZkvError("zkv_decode_workspace_size", ZKV_ERR_INVALID_ARG)
        if workspace is None:
            workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
        _need(workspace, "workspace", torch.uint8)
        if workspace.numel() < need:
            raise ZkvError("zkv_rvq_serve_step", ZKV_ERR_WORKSPACE,
                           f"workspace holds {workspace.numel()} bytes, {need} needed")
        self.out, self.lse = out, lse
        self._keep = (new_k, new_v, q, win_k, win_v, win_len, win_head, comp_len, k_codes,
                      v_codes, k_codebooks, v_codebooks, workspace, error_flag, k_smooth,
                      block_table)
        self._refa, self._refd = ctypes.byref(self._pa), ctypes.byref(self._pd)
        self._ws = ctypes.c_void_p(workspace.data_ptr())
        self._wsn = ctypes.c_size_t(workspace.numel())
        self._fn = lib().zkv_rvq_serve_step

    def __call__(self):
        st = self._fn(self._refa, self._refd, self._ws, self._wsn,
                      torch.cuda.current_stream().cuda_stream)
        if st != ZKV_OK:
            raise ZkvError("zkv_rvq_serve_step", st)
        return self.out, self.lse


def rvq_serve_step(new_k, new_v, q, win_k, win_v, win_len, win_head, comp_len, k_codes, v_codes,
                   k_codebooks, v_codebooks, out=None, lse=None, max_comp_len=None,
                   softmax_scale=None, workspace=None, error_flag=None, trace_events=None,
                   k_smooth=None, block_table=None):
    """rvq_append(new_k, new_v, ...) then rvq_decode_attn(q, ...) on the updated cache, in one
    library call (see include/zkv.h).  Returns (out, lse)."""
    if max_comp_len is None:
        max_comp_len = _code_layout(k_codes, block_table)[1]
    return PreparedServeStep(new_k, new_v, q, win_k, win_v, win_len, win_head, comp_len,
                             k_codes, v_codes, k_codebooks, v_codebooks, out, lse, max_comp_len,
                             softmax_scale, workspace, error_flag, trace_events, k_smooth,
                             block_table)()


class PreparedDecode:
    """rvq_decode_attn with its arguments validated and marshalled once (workspace included).
    The tensors must keep their storage; max_comp_len must stay an upper bound of every
    comp_len for as long as the object is used.  Calling it runs one decode step on the current
    stream and returns (out, lse)."""

    def __init__(self, q, k_codes, v_codes, comp_len, k_codebooks, v_codebooks, win_k, win_v,
                 win_len, out=None, lse=None, max_comp_len=None, softmax_scale=None,
                 workspace: torch.Tensor | None = None, error_flag=None, k_smooth=None):
        B, Hq, d = q.shape
        if out is None:
            out = torch.empty((B, Hq, d), dtype=torch.float32, device=q.device)
        if lse is None:
            lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
        self._p = _decode_params(q, k_codes, v_codes, comp_len, k_codebooks, v_codebooks, win_k,
                                 win_v, win_len, out, lse, max_comp_len, softmax_scale,
                                 error_flag, k_smooth)
        need = lib().zkv_decode_workspace_size(ctypes.byref(self._p))
        if need == 0:
            raise ZkvError("zkv_decode_workspace_size", ZKV_ERR_INVALID_ARG)
        if workspace is None:
            workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
        _need(workspace, "workspace", torch.uint8)
        if workspace.numel() < need:
            raise ZkvError("zkv_rvq_decode_attn", ZKV_ERR_WORKSPACE,
                           f"workspace holds {workspace.numel()} bytes, {need} needed")
        self.out, self.lse = out, lse
        self._keep = (q, k_codes, v_codes, comp_len, k_codebooks, v_codebooks, win_k, win_v,
                      win_len, workspace, error_flag, k_smooth)
        self._ref = ctypes.byref(self._p)
        self._ws = ctypes.c_void_p(workspace.data_ptr())
        self._wsn = ctypes.c_size_t(workspace.numel())
        self._fn = lib().zkv_rvq_decode_attn

    def __call__(self):
        st = self._fn(self._ref, self._ws, self._wsn, torch.cuda.current_stream().cuda_stream)
        if st != ZKV_OK:
            raise ZkvError("zkv_rvq_decode_attn", st)
        return self.out, self.lse


# --------------------------------------------------------------------------------------------
# A layer's compressed cache
# --------------------------------------------------------------------------------------------

def pq_encode(x: torch.Tensor, codebook: torch.Tensor, codes: torch.Tensor | None = None,
              rotate: bool = True, smooth: torch.Tensor | None = None) -> torch.Tensor:
    """Product VQ (VecInfer) of x rows.  x: [B, T, H, d] view (any strides, d contiguous), or
    [T, H, d], or [N, d] (one head).  codebook: [H, 256, m] float32 contiguous (shared by the d/m
    sub-vectors of a head).  smooth: optional [H, d] key smoothing factors.
    Returns codes uint8 [B, T, H, d/m] (a view when ``codes`` is given)."""
    if x.dtype not in (torch.float16, torch.float32):
        raise TypeError("x must be fp16 or fp32")
    _need(x, "x", x.dtype, contiguous=False)
    _need(codebook, "codebook", torch.float32)
    x4 = _as4(x, "x")
    if x4.stride(-1) != 1:
        raise ValueError("x rows must be contiguous")
    Bn, T, H, d = x4.shape
    if codebook.dim() != 3 or codebook.shape[0] != H or codebook.shape[1] != CODEBOOK_SIZE:
        raise ValueError(f"codebook must be [H={H}, 256, m], got {tuple(codebook.shape)}")
    m = codebook.shape[2]
    if d % m:
        raise ValueError("d must be a multiple of the sub-vector size")
    if codes is None:
        codes = torch.empty((Bn, T, H, d // m), dtype=torch.uint8, device=x.device)
    _need(codes, "codes", torch.uint8, contiguous=False)
    c4 = _as4(codes, "codes")
    if c4.shape != (Bn, T, H, d // m) or c4.stride(-1) != 1:
        raise ValueError("codes must be a [B, T, H, d/m] view with contiguous sub-vector codes")
    p = PQEncodeParams(n_batch=Bn, n_tok=T, n_head=H, d=d, m=m, rotate=int(bool(rotate)),
                       x_dtype=ZKV_DTYPE_F16 if x.dtype == torch.float16 else ZKV_DTYPE_F32,
                       x=_ptr(x4), x_sb=x4.stride(0), x_st=x4.stride(1), x_sh=x4.stride(2),
                       codebook=_ptr(codebook), codes=_ptr(c4), c_sb=c4.stride(0),
                       c_st=c4.stride(1), c_sh=c4.stride(2),
                       smooth=_smooth_ptr(smooth, H, d, "smooth"))
    _check("zkv_pq_encode", lib().zkv_pq_encode(ctypes.byref(p), _stream()))
    return codes


def pq_append(new_k, new_v, win_k, win_v, win_len, win_head, comp_len, k_codes, v_codes,
              k_codebook, v_codebook, error_flag=None, k_smooth=None):
    """One serving step of cache maintenance for a product-VQ cache (see include/zkv.h):
    the new token enters the window, a full window's oldest token is product-VQ encoded onto
    the prefix.  State updated in place.  codes uint8 [B, Hkv, Tcap, d/m]; codebooks float32
    [Hkv, 256, m]."""
    _need(new_k, "new_k", torch.float16)
    _need(new_v, "new_v", torch.float16)
    for n, t in (("win_k", win_k), ("win_v", win_v)):
        _need(t, n, torch.float16)
    for n, t in (("win_len", win_len), ("win_head", win_head), ("comp_len", comp_len)):
        _need(t, n, torch.int32)
    for n, t in (("k_codes", k_codes), ("v_codes", v_codes)):
        _need(t, n, torch.uint8)
    for n, t in (("k_codebook", k_codebook), ("v_codebook", v_codebook)):
        _need(t, n, torch.float32)
    if error_flag is not None:
        _need(error_flag, "error_flag", torch.int32)
    B, Hkv, d = new_k.shape
    _, _, Tcap, nsub = k_codes.shape
    m = k_codebook.shape[-1]
    if nsub * m != d or tuple(v_codes.shape) != tuple(k_codes.shape):
        raise ValueError("codes must be [B, Hkv, Tcap, d/m] for K and V")
    if tuple(new_v.shape) != (B, Hkv, d) or win_k.shape[:2] != (B, Hkv):
        raise ValueError("new tokens [B, Hkv, d] and window [B, Hkv, Wcap, d] must agree")
    p = PQAppendParams(B=B, Hkv=Hkv, d=d, m=m, Tcap=Tcap, Wcap=win_k.shape[2],
                       new_k=_ptr(new_k), new_v=_ptr(new_v), win_k=_ptr(win_k),
                       win_v=_ptr(win_v), win_len=_ptr(win_len), win_head=_ptr(win_head),
                       comp_len=_ptr(comp_len), k_codes=_ptr(k_codes), v_codes=_ptr(v_codes),
                       k_codebook=_ptr(k_codebook), v_codebook=_ptr(v_codebook),
                       error_flag=_ptr(error_flag),
                       k_smooth=_smooth_ptr(k_smooth, Hkv, d, "k_smooth"))
    _check("zkv_pq_append", lib().zkv_pq_append(ctypes.byref(p), _stream()))


def pq_decode_workspace_size(q, k_codes, k_codebook, win_k, max_comp_len=None) -> int:
    """Bytes of device workspace zkv_pq_decode_attn needs for these shapes (see include/zkv.h);
    pass a buffer of this size as ``workspace`` to keep allocation out of a timed loop."""
    B, Hq, d = q.shape
    _, Hkv, Tcap, _ = k_codes.shape
    p = PQDecodeParams(B=B, Hq=Hq, Hkv=Hkv, d=d, m=k_codebook.shape[-1], Tcap=Tcap,
                       Wcap=win_k.shape[2],
                       max_comp_len=Tcap if max_comp_len is None else int(max_comp_len))
    need = lib().zkv_pq_decode_workspace_size(ctypes.byref(p))
    if need == 0:
        raise ZkvError("zkv_pq_decode_workspace_size", ZKV_ERR_UNSUPPORTED)
    return int(need)


def pq_decode_attn(q, k_codes, v_codes, comp_len, k_codebook, v_codebook, win_k, win_v, win_len,
                   out=None, lse=None, max_comp_len=None, softmax_scale=None,
                   workspace: torch.Tensor | None = None, error_flag=None, k_smooth=None):
    """Decode attention over product-VQ codes (see include/zkv.h).  k_codes / v_codes uint8
    [B, Hkv, Tcap, d/m]; k_codebook / v_codebook float32 [Hkv, 256, m].
    Returns (out float32 [B, Hq, d], lse float32 [B, Hq])."""
    _need(q, "q", torch.float16)
    for n, t in (("k_codes", k_codes), ("v_codes", v_codes)):
        _need(t, n, torch.uint8)
    for n, t in (("comp_len", comp_len), ("win_len", win_len)):
        _need(t, n, torch.int32)
    for n, t in (("k_codebook", k_codebook), ("v_codebook", v_codebook)):
        _need(t, n, torch.float32)
    _need(win_k, "win_k", torch.float16)
    _need(win_v, "win_v", torch.float16)
    B, Hq, d = q.shape
    _, Hkv, Tcap, nsub = k_codes.shape
    m = k_codebook.shape[-1]
    if nsub * m != d or tuple(v_codes.shape) != tuple(k_codes.shape):
        raise ValueError("codes must be [B, Hkv, Tcap, d/m] for K and V")
    if out is None:
        out = torch.empty((B, Hq, d), dtype=torch.float32, device=q.device)
    if lse is None:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    _need(out, "out", torch.float32)
    _need(lse, "lse", torch.float32)
    if error_flag is not None:
        _need(error_flag, "error_flag", torch.int32)
    p = PQDecodeParams(B=B, Hq=Hq, Hkv=Hkv, d=d, m=m, Tcap=Tcap, Wcap=win_k.shape[2],
                       max_comp_len=Tcap if max_comp_len is None else int(max_comp_len),
                       softmax_scale=0.0 if softmax_scale is None else float(softmax_scale),
                       q=_ptr(q), k_codes=_ptr(k_codes), v_codes=_ptr(v_codes),
                       comp_len=_ptr(comp_len), k_codebook=_ptr(k_codebook),
                       v_codebook=_ptr(v_codebook), win_k=_ptr(win_k), win_v=_ptr(win_v),
                       win_len=_ptr(win_len), out=_ptr(out), lse=_ptr(lse),
                       error_flag=_ptr(error_flag),
                       k_smooth=_smooth_ptr(k_smooth, Hkv, d, "k_smooth"))
    need = lib().zkv_pq_decode_workspace_size(ctypes.byref(p))
    if need == 0:
        raise ZkvError("zkv_pq_decode_workspace_size", ZKV_ERR_UNSUPPORTED)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    _need(workspace, "workspace", torch.uint8)
    _check("zkv_pq_decode_attn",
           lib().zkv_pq_decode_attn(ctypes.byref(p), _ptr(workspace), workspace.numel(),
                                    _stream()))
    return out, lse


def lse_merge(part_out: torch.Tensor, part_lse: torch.Tensor, out=None, lse=None):
    """Log-sum-exp combine of N partial attentions over disjoint key sets (see include/zkv.h).
    part_out float32 [N, ..., d] and part_lse float32 [N, ...] may be views (any part and row
    strides, d contiguous; e.g. the two halves of a gathered [N, ..., d + 1] buffer of packed
    rows).  Returns (out float32 [..., d], lse float32 [...])."""
    _need(part_out, "part_out", torch.float32, contiguous=False)
    _need(part_lse, "part_lse", torch.float32, contiguous=False)
    N, d = part_out.shape[0], part_out.shape[-1]
    lead = tuple(part_out.shape[1:-1])
    if tuple(part_lse.shape) != (N,) + lead:
        raise ValueError("part_lse must be [N, ...] matching part_out [N, ..., d]")
    po = part_out.reshape(N, -1, d) if part_out.dim() != 3 else part_out
    pl = part_lse.reshape(N, -1) if part_lse.dim() != 2 else part_lse
    if po.stride(-1) != 1:
        raise ValueError("part_out rows must be contiguous")
    rows = po.shape[1]
    if out is None:
        out = torch.empty(lead + (d,), dtype=torch.float32, device=part_out.device)
    if lse is None:
        lse = torch.empty(lead, dtype=torch.float32, device=part_out.device)
    _need(out, "out", torch.float32)
    _need(lse, "lse", torch.float32)
    p = MergeParams(n_parts=N, rows=rows, d=d, part_out=_ptr(po), out_part_stride=po.stride(0),
                    out_row_stride=po.stride(1), part_lse=_ptr(pl), lse_part_stride=pl.stride(0),
                    lse_row_stride=pl.stride(1), out=_ptr(out), lse=_ptr(lse))
    _check("zkv_lse_merge", lib().zkv_lse_merge(ctypes.byref(p), _stream()))
    return out, lse


def lse_merge_peers(part_out_ptrs: torch.Tensor, part_lse_ptrs: torch.Tensor,
                    flag_ptrs: torch.Tensor, rank: int, epoch: int, rows: int, d: int,
                    out: torch.Tensor | None = None, lse: torch.Tensor | None = None,
                    error_flag: torch.Tensor | None = None, timeout_s: float = 2.0):
    """The context-parallel exchange and combine in one kernel over peer memory (see
    include/zkv.h).  part_out_ptrs / part_lse_ptrs / flag_ptrs: int64 CUDA tensors [n_ranks]
    holding every rank's out-rows / lse-rows / flag-array device addresses as mapped in this
    process.  Returns (out float32 [rows, d], lse float32 [rows])."""
    for n, t in (("part_out_ptrs", part_out_ptrs), ("part_lse_ptrs", part_lse_ptrs),
                 ("flag_ptrs", flag_ptrs)):
        _need(t, n, torch.int64)
    n = part_out_ptrs.numel()
    if part_lse_ptrs.numel() != n or flag_ptrs.numel() != n:
        raise ValueError("one out, lse and flag address per rank")
    dev = part_out_ptrs.device
    if out is None:
        out = torch.empty((rows, d), dtype=torch.float32, device=dev)
    if lse is None:
        lse = torch.empty((rows,), dtype=torch.float32, device=dev)
    _need(out, "out", torch.float32)
    _need(lse, "lse", torch.float32)
    if error_flag is not None:
        _need(error_flag, "error_flag", torch.int32)
    p = MergePeersParams(n_ranks=n, rank=rank, rows=rows, d=d, part_out=_ptr(part_out_ptrs),
                         part_lse=_ptr(part_lse_ptrs), flags=_ptr(flag_ptrs),
                         epoch=epoch & 0xFFFFFFFF, timeout_ns=int(timeout_s * 1e9),
                         out=_ptr(out), lse=_ptr(lse), error_flag=_ptr(error_flag))
    _check("zkv_lse_merge_peers", lib().zkv_lse_merge_peers(ctypes.byref(p), _stream()))
    return out, lse


class RVQKVCache:
    """Compressed KV cache of one attention layer: RVQ codes for old tokens, an fp16 window for
    the newest ones.  prefill() encodes a prompt, append() inserts one token per sequence
    (evicting and encoding the oldest window token when the window is full), attend() runs one
    decode step of attention, step() does both in one library call.  All state lives on the GPU; lengths never leave the device.
    k_smooth: optional float32 [Hkv, d] key smoothing factors (the key codebooks must have been
    trained on smoothed keys)."""

    def __init__(self, k_codebooks: torch.Tensor, v_codebooks: torch.Tensor, batch: int,
                 capacity: int, window: int, device="cuda", k_smooth: torch.Tensor | None = None):
        Hkv, Sk, _, d = k_codebooks.shape
        Sv = v_codebooks.shape[1]
        self.Ck, self.Cv = k_codebooks.contiguous(), v_codebooks.contiguous()
        self.k_smooth = None if k_smooth is None else k_smooth.contiguous()
        self.B, self.Hkv, self.d, self.Sk, self.Sv = batch, Hkv, d, Sk, Sv
        self.Tcap = (capacity + 15) // 16 * 16
        self.Wcap = window
        dev = torch.device(device)
        self.k_codes = torch.zeros((batch, Hkv, self.Tcap, Sk), dtype=torch.uint8, device=dev)
        self.v_codes = torch.zeros((batch, Hkv, self.Tcap, Sv), dtype=torch.uint8, device=dev)
        self.win_k = torch.zeros((batch, Hkv, window, d), dtype=torch.float16, device=dev)
        self.win_v = torch.zeros((batch, Hkv, window, d), dtype=torch.float16, device=dev)
        self.comp_len = torch.zeros(batch, dtype=torch.int32, device=dev)
        self.win_len = torch.zeros(batch, dtype=torch.int32, device=dev)
        self.win_head = torch.zeros(batch, dtype=torch.int32, device=dev)
        self.error_flag = torch.zeros(1, dtype=torch.int32, device=dev)
        self.max_comp_len = 0      # host-side bound used to size decode launches
        self._ws = None

    def prefill(self, k: torch.Tensor, v: torch.Tensor):
        """k, v: fp16 [B, Hkv, T, d] (same T for every sequence).  The last min(T, window)
        tokens go to the window, the rest are encoded."""
        T = k.shape[2]
        W = min(T, self.Wcap)
        Tc = T - W
        if Tc > self.Tcap:
            raise ValueError("prompt longer than capacity + window")
        if Tc > 0:
            rvq_encode(k[:, :, :Tc].permute(0, 2, 1, 3), self.Ck,
                       codes=self.k_codes[:, :, :Tc].permute(0, 2, 1, 3), with_norms=False,
                       smooth=self.k_smooth)
            rvq_encode(v[:, :, :Tc].permute(0, 2, 1, 3), self.Cv,
                       codes=self.v_codes[:, :, :Tc].permute(0, 2, 1, 3), with_norms=False)
        self.win_k[:, :, :W].copy_(k[:, :, Tc:])
        self.win_v[:, :, :W].copy_(v[:, :, Tc:])
        self.comp_len.fill_(Tc)
        self.win_len.fill_(W)
        self.win_head.zero_()
        self.max_comp_len = Tc

    def append(self, k_new: torch.Tensor, v_new: torch.Tensor):
        """k_new, v_new: fp16 [B, Hkv, d]."""
        rvq_append(k_new.contiguous(), v_new.contiguous(), self.win_k, self.win_v, self.win_len,
                   self.win_head, self.comp_len, self.k_codes, self.v_codes, self.Ck, self.Cv,
                   self.error_flag, self.k_smooth)
        self.max_comp_len = min(self.max_comp_len + 1, self.Tcap)

    def attend(self, q: torch.Tensor, softmax_scale=None, out=None, lse=None):
        """q: fp16 [B, Hq, d] -> (out float32 [B, Hq, d], lse float32 [B, Hq])."""
        args = (q, self.k_codes, self.v_codes, self.comp_len, self.Ck, self.Cv, self.win_k,
                self.win_v, self.win_len)
        need = decode_workspace_size(*args, max_comp_len=self.max_comp_len)
        if self._ws is None or self._ws.numel() < need:
            self._ws = torch.empty(need, dtype=torch.uint8, device=q.device)
        return rvq_decode_attn(*args, out=out, lse=lse, max_comp_len=self.max_comp_len,
                               softmax_scale=softmax_scale, workspace=self._ws,
                               error_flag=self.error_flag, k_smooth=self.k_smooth)

    def step(self, k_new: torch.Tensor, v_new: torch.Tensor, q: torch.Tensor,
             softmax_scale=None, out=None, lse=None):
        """append(k_new, v_new) then attend(q) as one library call (zkv_rvq_serve_step: the
        lookup tables are built beside the encode of the evicted token); the same results as
        the two calls.  k_new, v_new fp16 [B, Hkv, d]; q fp16 [B, Hq, d]."""
        self.max_comp_len = min(self.max_comp_len + 1, self.Tcap)
        args = (q, self.k_codes, self.v_codes, self.comp_len, self.Ck, self.Cv, self.win_k,
                self.win_v, self.win_len)
        need = decode_workspace_size(*args, max_comp_len=self.max_comp_len)
        if self._ws is None or self._ws.numel() < need:
            self._ws = torch.empty(need, dtype=torch.uint8, device=q.device)
        return rvq_serve_step(k_new.contiguous(), v_new.contiguous(), q, self.win_k, self.win_v,
                              self.win_len, self.win_head, self.comp_len, self.k_codes,
                              self.v_codes, self.Ck, self.Cv, out=out, lse=lse,
                              max_comp_len=self.max_comp_len, softmax_scale=softmax_scale,
                              workspace=self._ws, error_flag=self.error_flag,
                              k_smooth=self.k_smooth)

    def memory_bytes(self) -> int:
        """Bytes held by codes and window (codebooks are shared across layers' caches)."""
        return sum(t.numel() * t.element_size() for t in
                   (self.k_codes, self.v_codes, self.win_k, self.win_v))


class PQKVCache:
    """Product-VQ (VecInfer-style) compressed KV cache of one attention layer: d/m code bytes
    per token for K and for V (one 256-entry codebook of m-dim sub-vectors per kv head and K or
    V), an fp16 window for the newest tokens.  The same interface as RVQKVCache: prefill(),
    append(), attend(), step(), memory_bytes().  k_smooth: optional float32 [Hkv, d] key
    smoothing factors (the key codebooks must have been trained on smoothed keys)."""

    def __init__(self, k_codebook: torch.Tensor, v_codebook: torch.Tensor, batch: int,
                 capacity: int, window: int, head_dim: int, device="cuda",
                 k_smooth: torch.Tensor | None = None):
        Hkv, _, m = k_codebook.shape
        if head_dim % m:
            raise ValueError("head_dim must be a multiple of the sub-vector size")
        self.Ck, self.Cv = k_codebook.contiguous(), v_codebook.contiguous()
        self.k_smooth = None if k_smooth is None else k_smooth.contiguous()
        self.B, self.Hkv, self.d, self.m = batch, Hkv, head_dim, m
        self.Tcap = (capacity + 15) // 16 * 16
        self.Wcap = window
        dev = torch.device(device)
        nsub = head_dim // m
        self.k_codes = torch.zeros((batch, Hkv, self.Tcap, nsub), dtype=torch.uint8, device=dev)
        self.v_codes = torch.zeros((batch, Hkv, self.Tcap, nsub), dtype=torch.uint8, device=dev)
        self.win_k = torch.zeros((batch, Hkv, window, head_dim), dtype=torch.float16, device=dev)
        self.win_v = torch.zeros((batch, Hkv, window, head_dim), dtype=torch.float16, device=dev)
        self.comp_len = torch.zeros(batch, dtype=torch.int32, device=dev)
        self.win_len = torch.zeros(batch, dtype=torch.int32, device=dev)
        self.win_head = torch.zeros(batch, dtype=torch.int32, device=dev)
        self.error_flag = torch.zeros(1, dtype=torch.int32, device=dev)
        self.max_comp_len = 0
        self._ws = None

    def prefill(self, k: torch.Tensor, v: torch.Tensor):
        """k, v: fp16 [B, Hkv, T, d].  The last min(T, window) tokens go to the window, the
        rest are encoded."""
        T = k.shape[2]
        W = min(T, self.Wcap)
        Tc = T - W
        if Tc > self.Tcap:
            raise ValueError("prompt longer than capacity + window")
        if Tc > 0:
            pq_encode(k[:, :, :Tc].permute(0, 2, 1, 3), self.Ck,
                      codes=self.k_codes[:, :, :Tc].permute(0, 2, 1, 3), smooth=self.k_smooth)
            pq_encode(v[:, :, :Tc].permute(0, 2, 1, 3), self.Cv,
                      codes=self.v_codes[:, :, :Tc].permute(0, 2, 1, 3))
        self.win_k[:, :, :W].copy_(k[:, :, Tc:])
        self.win_v[:, :, :W].copy_(v[:, :, Tc:])
        self.comp_len.fill_(Tc)
        self.win_len.fill_(W)
        self.win_head.zero_()
        self.max_comp_len = Tc

    def append(self, k_new: torch.Tensor, v_new: torch.Tensor):
        """k_new, v_new: fp16 [B, Hkv, d]."""
        pq_append(k_new.contiguous(), v_new.contiguous(), self.win_k, self.win_v, self.win_len,
                  self.win_head, self.comp_len, self.k_codes, self.v_codes, self.Ck, self.Cv,
                  self.error_flag, self.k_smooth)
        self.max_comp_len = min(self.max_comp_len + 1, self.Tcap)

    def attend(self, q: torch.Tensor, softmax_scale=None, out=None, lse=None):
        """q: fp16 [B, Hq, d] -> (out float32 [B, Hq, d], lse float32 [B, Hq])."""
        need = pq_decode_workspace_size(q, self.k_codes, self.Ck, self.win_k,
                                        max_comp_len=self.max_comp_len)
        if self._ws is None or self._ws.numel() < need:
            self._ws = torch.empty(need, dtype=torch.uint8, device=q.device)
        return pq_decode_attn(q, self.k_codes, self.v_codes, self.comp_len, self.Ck, self.Cv,
                              self.win_k, self.win_v, self.win_len, out=out, lse=lse,
                              max_comp_len=self.max_comp_len, softmax_scale=softmax_scale,
                              workspace=self._ws, error_flag=self.error_flag,
                              k_smooth=self.k_smooth)

    def step(self, k_new: torch.Tensor, v_new: torch.Tensor, q: torch.Tensor,
             softmax_scale=None, out=None, lse=None):
        """append(k_new, v_new) then attend(q)."""
        self.append(k_new, v_new)
        return self.attend(q, softmax_scale=softmax_scale, out=out, lse=lse)

    def memory_bytes(self) -> int:
        """Bytes held by codes and window (codebooks are shared across layers' caches)."""
        return sum(t.numel() * t.element_size() for t in
                   (self.k_codes, self.v_codes, self.win_k, self.win_v))
