"""ctypes wrapper of the plain C twin of the oracle (``zkv_oracle_c.c``).

TEST INFRASTRUCTURE, like ``zkv_oracle``: only the test suite, the package smoke check and the
benchmark's CPU baseline arm may use it.  ``build()`` compiles the C source with gcc into
``libzkv_oracle_c.so`` beside it (no value-changing floating-point options); the functions
below take numpy arrays, convert them to the C layouts (float64 inputs, float32 codebooks,
uint8 codes, int64 lengths) and return numpy arrays, with the numpy oracle's signatures.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "zkv_oracle_c.c")
LIB = os.path.join(HERE, "libzkv_oracle_c.so")
CFLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math",
          "-Wall", "-Wextra", "-Werror"]

_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle (when missing or older than its source); returns the path."""
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        tmp = LIB + ".tmp"
        subprocess.run(["gcc", *CFLAGS, "-o", tmp, SRC, "-lm"], check=True)
        os.replace(tmp, LIB)
    return LIB


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        i64, i32, dbl, vp = ctypes.c_int64, ctypes.c_int, ctypes.c_double, ctypes.c_void_p
        L.zo_fwht.argtypes = [i64, i32, dbl, vp, vp]
        L.zo_rvq_encode.argtypes = [i64, i32, i32, i32, vp, vp, i32, vp, vp, vp, vp]
        L.zo_pq_encode.argtypes = [i64, i32, i32, i32, vp, vp, i32, vp, vp]
        L.zo_lse_merge.argtypes = [i32, i32, vp, vp, vp, vp]
        L.zo_decode_attn.argtypes = [i32, i32, i32, i32, i32, i32, i32, i64, i64, dbl,
                                     vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp]
        L.zo_pq_decode_attn.argtypes = [i32, i32, i32, i32, i32, i32, i64, i64, dbl,
                                        vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp]
        for f in ("zo_fwht", "zo_rvq_encode", "zo_pq_encode", "zo_lse_merge", "zo_decode_attn",
                  "zo_pq_decode_attn"):
            getattr(L, f).restype = ctypes.c_int
        _lib = L
    return _lib


def _c(a, dtype):
    return np.ascontiguousarray(np.asarray(a).astype(dtype, copy=False))


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _ok(rc, name):
    if rc != 0:
        raise ValueError(f"{name}: invalid arguments")


def fwht(x, scale: float) -> np.ndarray:
    """scale * H_d x for every row (float64)."""
    x = _c(x, np.float64)
    d = x.shape[-1]
    y = np.empty_like(x)
    _ok(lib().zo_fwht(x.size // d, d, float(scale), _p(x), _p(y)), "zo_fwht")
    return y


def rvq_encode(x, codebooks, rotate: bool = True, smooth=None):
    """Greedy RVQ of rows of x [n][d] against [S][K][d]: (codes, norms, y) as the numpy
    oracle's first three results."""
    x = _c(x, np.float64)
    C = _c(codebooks, np.float32)
    n, d = x.shape
    S, K, _ = C.shape
    lam = None if smooth is None else _c(smooth, np.float32)
    codes = np.empty((n, S), np.uint8)
    norms = np.empty((n, S), np.float32)
    y = np.empty((n, d), np.float32)
    _ok(lib().zo_rvq_encode(n, d, S, K, _p(x), _p(lam), int(bool(rotate)), _p(C), _p(codes),
                            _p(norms), _p(y)), "zo_rvq_encode")
    return codes, norms, y


def pq_encode(x, codebook, smooth=None, rotate: bool = True) -> np.ndarray:
    """Product-VQ codes [n][d/m] of rows of x [n][d] against one codebook [K][m]."""
    x = _c(x, np.float64)
    C = _c(codebook, np.float32)
    n, d = x.shape
    K, m = C.shape
    lam = None if smooth is None else _c(smooth, np.float32)
    codes = np.empty((n, d // m), np.uint8)
    _ok(lib().zo_pq_encode(n, d, m, K, _p(x), _p(lam), int(bool(rotate)), _p(C), _p(codes)),
        "zo_pq_encode")
    return codes


def lse_merge(parts):
    """Combine [(out_i, lse_i)]: (out float64 [d], lse)."""
    outs = _c(np.stack([np.asarray(o, np.float64) for o, _ in parts]), np.float64)
    lses = _c([float(l) for _, l in parts], np.float64)
    out = np.empty(outs.shape[1], np.float64)
    lse = np.empty(1, np.float64)
    _ok(lib().zo_lse_merge(len(parts), outs.shape[1], _p(outs), _p(lses), _p(out), _p(lse)),
        "zo_lse_merge")
    return out, float(lse[0])


def _decode_inputs(q, k_codes, v_codes, comp_len, Ck, Cv, win_k, win_v, win_len, k_smooth):
    return (_c(q, np.float64), _c(k_codes, np.uint8), _c(v_codes, np.uint8),
            _c(comp_len, np.int64), _c(Ck, np.float32), _c(Cv, np.float32),
            _c(win_k, np.float64), _c(win_v, np.float64), _c(win_len, np.int64),
            None if k_smooth is None else _c(k_smooth, np.float32))


def decode_attn(q, k_codes, v_codes, comp_len, Ck, Cv, win_k, win_v, win_len,
                scale: float | None = None, k_smooth=None):
    """RVQ decode attention, direct form: (out float64 [B][Hq][d], lse float64 [B][Hq])."""
    q, kc, vc, cl, Ck, Cv, wk, wv, wl, lam = _decode_inputs(q, k_codes, v_codes, comp_len, Ck,
                                                            Cv, win_k, win_v, win_len, k_smooth)
    B, Hq, d = q.shape
    _, Hkv, Tcap, Sk = kc.shape
    Sv, K = vc.shape[3], Ck.shape[2]
    out = np.empty((B, Hq, d), np.float64)
    lse = np.empty((B, Hq), np.float64)
    _ok(lib().zo_decode_attn(B, Hq, Hkv, d, Sk, Sv, K, Tcap, wk.shape[2],
                             0.0 if scale is None else float(scale), _p(q), _p(kc), _p(vc),
                             _p(cl), _p(Ck), _p(Cv), _p(wk), _p(wv), _p(wl), _p(lam), _p(out),
                             _p(lse)), "zo_decode_attn")
    return out, lse


def pq_decode_attn(q, k_codes, v_codes, comp_len, Ck, Cv, win_k, win_v, win_len,
                   scale: float | None = None, k_smooth=None):
    """Product-VQ decode attention, direct form: (out float64 [B][Hq][d], lse [B][Hq])."""
    q, kc, vc, cl, Ck, Cv, wk, wv, wl, lam = _decode_inputs(q, k_codes, v_codes, comp_len, Ck,
                                                            Cv, win_k, win_v, win_len, k_smooth)
    B, Hq, d = q.shape
    _, Hkv, Tcap, _ = kc.shape
    K, m = Ck.shape[1], Ck.shape[2]
    out = np.empty((B, Hq, d), np.float64)
    lse = np.empty((B, Hq), np.float64)
    _ok(lib().zo_pq_decode_attn(B, Hq, Hkv, d, m, K, Tcap, wk.shape[2],
                                0.0 if scale is None else float(scale), _p(q), _p(kc), _p(vc),
                                _p(cl), _p(Ck), _p(Cv), _p(wk), _p(wv), _p(wl), _p(lam),
                                _p(out), _p(lse)), "zo_pq_decode_attn")
    return out, lse
