"""The C-ABI library loads and exports every function include/zkv.h declares; host-side
argument validation rejects bad calls before any launch.  No GPU needed: every call below
returns during validation, before the CUDA runtime is touched."""
import ctypes
import os
import re

import pytest

from compressed_decode_attention_zkv_b200 import build as B
from compressed_decode_attention_zkv_b200 import zkv

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    B.build()
    return zkv.lib()


def _declared_functions():
    text = open(os.path.join(ROOT, "include", "zkv.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?\w+\*?\s+\*?(zkv_\w+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_boundary():
    names = _declared_functions()
    for n in ("zkv_fwht", "zkv_rvq_encode", "zkv_rvq_decode_attn", "zkv_rvq_reconstruct",
              "zkv_decode_workspace_size", "zkv_rvq_append", "zkv_status_string", "zkv_version"):
        assert n in names


def test_library_exports_every_declared_symbol(L):
    for n in _declared_functions():
        assert hasattr(L, n), f"{n} not exported"


def test_status_strings_and_version(L):
    assert zkv.status_string(0) == "ZKV_OK"
    assert zkv.status_string(3) == "ZKV_ERR_WORKSPACE"
    assert zkv.status_string(99) == "ZKV_ERR_UNKNOWN"
    text = open(os.path.join(ROOT, "include", "zkv.h")).read()
    assert L.zkv_version() == int(re.search(r"#define ZKV_VERSION (\d+)", text).group(1))


def _header_define(name):
    """The value of an integer #define (a literal or a shift of two) or enumerator in
    include/zkv.h."""
    text = open(os.path.join(ROOT, "include", "zkv.h")).read()
    m = (re.search(rf"#define {name}\s+\(?\s*(\w+)\s*(?:<<\s*(\w+))?\s*\)?", text)
         or re.search(rf"\b{name}\s*=\s*(-?\w+)()", text))   # or an enumerator
    assert m, f"{name} not defined"
    lit = lambda t: int(t.rstrip("uUlL"), 0)
    return lit(m.group(1)) << (lit(m.group(2)) if m.group(2) else 0)


def test_binding_constants_match_the_header():
    assert zkv.DECODE_SCRATCH_BYTES == _header_define("ZKV_DECODE_SCRATCH_BYTES")
    for name in dir(zkv):
        if re.fullmatch(r"ZKV_(ERR|DEVERR|DTYPE)_\w+|ZKV_OK", name):
            assert getattr(zkv, name) == _header_define(name), name


def test_fwht_validation(L):
    assert L.zkv_fwht(None, 0, None, -1, 128, 1.0, None) == zkv.ZKV_ERR_INVALID_ARG
    assert L.zkv_fwht(None, 7, None, 4, 128, 1.0, None) == zkv.ZKV_ERR_INVALID_ARG
    assert L.zkv_fwht(None, 0, None, 4, 96, 1.0, None) == zkv.ZKV_ERR_UNSUPPORTED
    assert L.zkv_fwht(None, 0, None, 0, 128, 1.0, None) == zkv.ZKV_OK
    assert L.zkv_fwht(None, 0, None, 4, 128, 1.0, None) == zkv.ZKV_ERR_INVALID_ARG


def test_encode_validation(L):
    p = zkv.EncodeParams(n_batch=1, n_tok=4, n_head=1, d=128, S=4, rotate=1, x_dtype=0)
    assert L.zkv_rvq_encode(ctypes.byref(p), None) == zkv.ZKV_ERR_INVALID_ARG   # null pointers
    p.S = 9
    assert L.zkv_rvq_encode(ctypes.byref(p), None) == zkv.ZKV_ERR_UNSUPPORTED
    p.S, p.d = 4, 100
    assert L.zkv_rvq_encode(ctypes.byref(p), None) == zkv.ZKV_ERR_UNSUPPORTED
    p.d, p.x_dtype = 128, 5
    assert L.zkv_rvq_encode(ctypes.byref(p), None) == zkv.ZKV_ERR_INVALID_ARG
    p.x_dtype, p.n_tok = 0, 0
    assert L.zkv_rvq_encode(ctypes.byref(p), None) == zkv.ZKV_OK               # empty: no-op
    p.n_tok, p.x, p.codebooks, p.codes = 4, 0x1002, 0x1000, 0x1000              # misaligned x
    assert L.zkv_rvq_encode(ctypes.byref(p), None) == zkv.ZKV_ERR_INVALID_ARG
    assert L.zkv_rvq_encode(None, None) == zkv.ZKV_ERR_INVALID_ARG


def _decode_params(**kw):
    base = dict(B=2, Hq=8, Hkv=2, d=128, Sk=4, Sv=4, Tcap=64, Wcap=16, max_comp_len=64,
                softmax_scale=0.0, q=0x1000, k_codes=0x2000, v_codes=0x3000, comp_len=0x4000,
                k_codebooks=0x5000, v_codebooks=0x6000, win_k=0x7000, win_v=0x8000,
                win_len=0x9000, out=0xa000)
    base.update(kw)
    return zkv.DecodeParams(**base)


@pytest.mark.parametrize("kw,status", [
    (dict(Hq=6, Hkv=4), zkv.ZKV_ERR_INVALID_ARG),        # Hq not a multiple of Hkv
    (dict(Hq=32, Hkv=2), zkv.ZKV_ERR_UNSUPPORTED),       # GQA group of 16
    (dict(d=96), zkv.ZKV_ERR_UNSUPPORTED),
    (dict(Sk=0), zkv.ZKV_ERR_UNSUPPORTED),
    (dict(Sv=9), zkv.ZKV_ERR_UNSUPPORTED),
    (dict(Tcap=60, max_comp_len=60), zkv.ZKV_ERR_INVALID_ARG),  # Tcap not a multiple of 16
    (dict(max_comp_len=65), zkv.ZKV_ERR_INVALID_ARG),
    (dict(q=0), zkv.ZKV_ERR_INVALID_ARG),
    (dict(win_k=0), zkv.ZKV_ERR_INVALID_ARG),
    (dict(k_codes=0x2008), zkv.ZKV_ERR_INVALID_ARG),     # misaligned
])
def test_decode_validation(L, kw, status):
    p = _decode_params(**kw)
    assert L.zkv_rvq_decode_attn(ctypes.byref(p), None, 0, None) == status
    shape_error = not any(k in kw for k in ("q", "win_k", "k_codes"))
    assert (L.zkv_decode_workspace_size(ctypes.byref(p)) == 0) == shape_error


def test_decode_workspace_is_required(L):
    p = _decode_params()
    need = L.zkv_decode_workspace_size(ctypes.byref(p))
    assert need > 0
    assert L.zkv_rvq_decode_attn(ctypes.byref(p), None, need, None) == zkv.ZKV_ERR_WORKSPACE
    assert L.zkv_rvq_decode_attn(ctypes.byref(p), 0x10000, need - 1, None) == zkv.ZKV_ERR_WORKSPACE
    assert L.zkv_rvq_decode_attn(ctypes.byref(p), 0x10010, need, None) == zkv.ZKV_ERR_WORKSPACE


def test_append_validation(L):
    p = zkv.AppendParams(B=2, Hkv=2, d=128, Sk=4, Sv=4, Tcap=64, Wcap=0)
    assert L.zkv_rvq_append(ctypes.byref(p), None) == zkv.ZKV_ERR_INVALID_ARG  # no window
    p.Wcap, p.d = 8, 32
    assert L.zkv_rvq_append(ctypes.byref(p), None) == zkv.ZKV_ERR_UNSUPPORTED
    p.d = 128
    assert L.zkv_rvq_append(ctypes.byref(p), None) == zkv.ZKV_ERR_INVALID_ARG  # null pointers


@pytest.mark.parametrize("kw", [
    dict(page_tokens=48, max_pages=4, n_pages=8, Tcap=192, max_comp_len=64),   # not a power of two
    dict(page_tokens=16, max_pages=4, n_pages=8),                             # below 32
    dict(page_tokens=32, max_pages=4, n_pages=8),                             # 4 * 32 != Tcap (64)
    dict(page_tokens=32, max_pages=2, n_pages=0),                             # empty pool
])
def test_paged_layout_validation(L, kw):
    p = _decode_params(block_table=0xf000, **kw)
    assert L.zkv_rvq_decode_attn(ctypes.byref(p), None, 0, None) == zkv.ZKV_ERR_INVALID_ARG
    assert L.zkv_decode_workspace_size(ctypes.byref(p)) == 0
    ok = _decode_params(block_table=0xf000, page_tokens=32, max_pages=2, n_pages=8)
    assert L.zkv_decode_workspace_size(ctypes.byref(ok)) > 0


def _append_params(**kw):
    # the same cache as _decode_params (shapes and shared buffers)
    base = dict(B=2, Hkv=2, d=128, Sk=4, Sv=4, Tcap=64, Wcap=16, new_k=0xb000, new_v=0xc000,
                win_k=0x7000, win_v=0x8000, win_len=0x9000, win_head=0xd000, comp_len=0x4000,
                k_codes=0x2000, v_codes=0x3000, k_codebooks=0x5000, v_codebooks=0x6000)
    base.update(kw)
    return zkv.AppendParams(**base)


@pytest.mark.parametrize("akw,dkw,status", [
    (dict(k_codes=0x2100), {}, zkv.ZKV_ERR_INVALID_ARG),      # another cache's codes
    (dict(comp_len=0x4100), {}, zkv.ZKV_ERR_INVALID_ARG),
    (dict(win_v=0x8100), {}, zkv.ZKV_ERR_INVALID_ARG),
    (dict(Tcap=128), {}, zkv.ZKV_ERR_INVALID_ARG),            # shapes differ
    (dict(B=3), {}, zkv.ZKV_ERR_INVALID_ARG),
    (dict(Sv=3), {}, zkv.ZKV_ERR_INVALID_ARG),
    (dict(new_k=0), {}, zkv.ZKV_ERR_INVALID_ARG),             # the append itself is invalid
    (dict(k_smooth=0xe000), {}, zkv.ZKV_ERR_INVALID_ARG),     # different smoothing factors
    (dict(block_table=0xf000, page_tokens=32, max_pages=2, n_pages=8), {},
     zkv.ZKV_ERR_INVALID_ARG),                                 # paged append, contiguous decode
    (dict(d=96), dict(d=96), zkv.ZKV_ERR_UNSUPPORTED),
    ({}, dict(Hq=6, Hkv=4), zkv.ZKV_ERR_INVALID_ARG),          # the decode itself is invalid
    ({}, {}, zkv.ZKV_ERR_WORKSPACE),                           # consistent, but no workspace
])
def test_serve_step_validation(L, akw, dkw, status):
    """zkv_rvq_serve_step refuses inconsistent or invalid arguments before any launch."""
    ap, dp = _append_params(**akw), _decode_params(**dkw)
    assert L.zkv_rvq_serve_step(ctypes.byref(ap), ctypes.byref(dp), None, 0, None) == status


def test_pq_encode_validation(L):
    def mk(**kw):
        base = dict(n_batch=1, n_tok=4, n_head=1, d=128, m=4, rotate=1, x_dtype=0, x=0x1000,
                    codebook=0x2000, codes=0x3000)
        base.update(kw)
        return zkv.PQEncodeParams(**base)
    for kw, st in ((dict(m=3), zkv.ZKV_ERR_UNSUPPORTED), (dict(m=32), zkv.ZKV_ERR_UNSUPPORTED),
                   (dict(d=96), zkv.ZKV_ERR_UNSUPPORTED), (dict(x_dtype=7), zkv.ZKV_ERR_INVALID_ARG),
                   (dict(x=0), zkv.ZKV_ERR_INVALID_ARG), (dict(codes=0), zkv.ZKV_ERR_INVALID_ARG),
                   (dict(x=0x1002), zkv.ZKV_ERR_INVALID_ARG), (dict(n_tok=-1), zkv.ZKV_ERR_INVALID_ARG),
                   (dict(n_tok=0), zkv.ZKV_OK)):
        assert L.zkv_pq_encode(ctypes.byref(mk(**kw)), None) == st, kw
    assert L.zkv_pq_encode(None, None) == zkv.ZKV_ERR_INVALID_ARG


def test_pq_decode_validation(L):
    def mk(**kw):
        base = dict(B=2, Hq=8, Hkv=2, d=128, m=4, Tcap=64, Wcap=16, max_comp_len=64,
                    softmax_scale=0.0, q=0x1000, k_codes=0x2000, v_codes=0x3000, comp_len=0x4000,
                    k_codebook=0x5000, v_codebook=0x6000, win_k=0x7000, win_v=0x8000,
                    win_len=0x9000, out=0xa000)
        base.update(kw)
        return zkv.PQDecodeParams(**base)
    for kw, st in ((dict(m=16), zkv.ZKV_ERR_UNSUPPORTED),              # d / m must be 32 or 16
                   (dict(m=8, Hq=16), zkv.ZKV_ERR_UNSUPPORTED),        # GQA 8 at (128, 8)
                   (dict(d=256, m=8, Hq=8, Hkv=2), zkv.ZKV_ERR_UNSUPPORTED),   # GQA 4 at d 256
                   (dict(Hq=6, Hkv=4), zkv.ZKV_ERR_INVALID_ARG),
                   (dict(max_comp_len=65), zkv.ZKV_ERR_INVALID_ARG),
                   (dict(q=0), zkv.ZKV_ERR_INVALID_ARG),
                   (dict(q=0x1008), zkv.ZKV_ERR_INVALID_ARG)):
        assert L.zkv_pq_decode_attn(ctypes.byref(mk(**kw)), None, 0, None) == st, kw
    ok = mk()
    assert L.zkv_pq_decode_workspace_size(ctypes.byref(ok)) > 0
    assert L.zkv_pq_decode_attn(ctypes.byref(ok), None, 0, None) == zkv.ZKV_ERR_WORKSPACE
    assert L.zkv_pq_decode_workspace_size(ctypes.byref(mk(m=16))) == 0
    for kw in (dict(m=8), dict(d=64, m=4, Hq=16), dict(d=64, m=2)):   # supported shapes
        assert L.zkv_pq_decode_workspace_size(ctypes.byref(mk(**kw))) > 0, kw


def test_pq_append_validation(L):
    def mk(**kw):
        base = dict(B=2, Hkv=2, d=128, m=4, Tcap=64, Wcap=8, new_k=0x1000, new_v=0x2000,
                    win_k=0x3000, win_v=0x4000, win_len=0x5000, win_head=0x6000,
                    comp_len=0x7000, k_codes=0x8000, v_codes=0x9000, k_codebook=0xa000,
                    v_codebook=0xb000)
        base.update(kw)
        return zkv.PQAppendParams(**base)
    for kw, st in ((dict(d=96), zkv.ZKV_ERR_UNSUPPORTED), (dict(m=3), zkv.ZKV_ERR_UNSUPPORTED),
                   (dict(Wcap=0), zkv.ZKV_ERR_INVALID_ARG), (dict(B=-1), zkv.ZKV_ERR_INVALID_ARG),
                   (dict(Hkv=0), zkv.ZKV_ERR_INVALID_ARG), (dict(win_head=0), zkv.ZKV_ERR_INVALID_ARG),
                   (dict(v_codebook=0), zkv.ZKV_ERR_INVALID_ARG)):
        assert L.zkv_pq_append(ctypes.byref(mk(**kw)), None) == st, kw
    assert L.zkv_pq_append(ctypes.byref(mk(B=0)), None) == zkv.ZKV_OK   # nothing to do
    assert L.zkv_pq_append(None, None) == zkv.ZKV_ERR_INVALID_ARG


def test_pq_decode_workspace_size_binding(L):
    """The binding's size query reads shapes only; the layout is six 256-byte-aligned float32
    arrays: chunk maxima, sums and outputs, then the window's maxima, sums and outputs."""
    import torch
    B, Hq, Hkv, d, m, W = 2, 8, 2, 128, 4, 16
    q = torch.empty((B, Hq, d), device="meta", dtype=torch.float16)
    wk = torch.empty((B, Hkv, W, d), device="meta", dtype=torch.float16)
    Ck = torch.empty((Hkv, 256, m), device="meta")
    for Tcap, chunks in ((64, 1), (2048, 1), (2049, 2), (5000, 3)):
        kc = torch.empty((B, Hkv, Tcap, d // m), device="meta", dtype=torch.uint8)
        pairs, GP = B * Hkv, Hq // Hkv
        a256 = lambda n: (n + 255) // 256 * 256   # noqa: E731
        want = (2 * a256(pairs * chunks * GP * 4) + a256(pairs * chunks * GP * d * 4)
                + 2 * a256(pairs * GP * 4) + a256(pairs * GP * d * 4))
        assert zkv.pq_decode_workspace_size(q, kc, Ck, wk) == want, Tcap


def test_lse_merge_validation(L):
    def mk(**kw):
        base = dict(n_parts=2, rows=4, d=8, part_out=0x1000, out_part_stride=36, out_row_stride=9,
                    part_lse=0x1020, lse_part_stride=36, lse_row_stride=9, out=0x3000, lse=0x4000)
        base.update(kw)
        return zkv.MergeParams(**base)
    for kw in (dict(n_parts=0), dict(d=0), dict(d=5000), dict(rows=-1), dict(part_out=0),
               dict(part_lse=0), dict(out=0)):
        assert L.zkv_lse_merge(ctypes.byref(mk(**kw)), None) == zkv.ZKV_ERR_INVALID_ARG, kw
    assert L.zkv_lse_merge(ctypes.byref(mk(rows=0)), None) == zkv.ZKV_OK   # nothing to do
    assert L.zkv_lse_merge(None, None) == zkv.ZKV_ERR_INVALID_ARG


def test_lse_merge_peers_validation(L):
    def mk(**kw):
        base = dict(n_ranks=2, rank=1, rows=4, d=8, part_out=0x1000, part_lse=0x2000,
                    flags=0x3000, epoch=1, timeout_ns=1000000, out=0x4000, lse=0x5000)
        base.update(kw)
        return zkv.MergePeersParams(**base)
    for kw in (dict(n_ranks=0), dict(n_ranks=65), dict(rank=2), dict(rank=-1), dict(d=0),
               dict(d=5000), dict(rows=-1), dict(epoch=0), dict(timeout_ns=0),
               dict(part_out=0), dict(part_lse=0), dict(flags=0), dict(out=0)):
        assert L.zkv_lse_merge_peers(ctypes.byref(mk(**kw)), None) == zkv.ZKV_ERR_INVALID_ARG, kw
    assert L.zkv_lse_merge_peers(None, None) == zkv.ZKV_ERR_INVALID_ARG


def test_binding_refuses_cpu_tensors():
    import torch
    x = torch.zeros(4, 128, dtype=torch.float16)
    with pytest.raises(ValueError):
        zkv.fwht(x, 1.0)


def test_ctypes_structs_match_the_header_layout(tmp_path):
    """Every parameter struct the binding passes has the C compiler's size and field offsets
    (a field added to the header but not to the binding would shift every later field)."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    pairs = [("zkv_encode_params", zkv.EncodeParams), ("zkv_reconstruct_params", zkv.ReconstructParams),
             ("zkv_decode_params", zkv.DecodeParams), ("zkv_append_params", zkv.AppendParams),
             ("zkv_lse_merge_params", zkv.MergeParams), ("zkv_pq_encode_params", zkv.PQEncodeParams),
             ("zkv_pq_decode_params", zkv.PQDecodeParams),
             ("zkv_pq_append_params", zkv.PQAppendParams),
             ("zkv_lse_merge_peers_params", zkv.MergePeersParams)]
    lines = ['#include <stdio.h>', '#include <stddef.h>', '#include "zkv.h"', "int main(void) {"]
    for cname, cls in pairs:
        lines.append(f'  printf("{cname} size %zu\\n", sizeof({cname}));')
        for f, _ in cls._fields_:
            lines.append(f'  printf("{cname} {f} %zu\\n", offsetof({cname}, {f}));')
    lines += ["  return 0;", "}"]
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines) + "\n")
    exe = tmp_path / "layout"
    subprocess.run([cc, "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)], check=True)
    got = dict()
    for ln in subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split("\n"):
        if ln:
            a, b, v = ln.split()
            got[(a, b)] = int(v)
    for cname, cls in pairs:
        assert got[(cname, "size")] == ctypes.sizeof(cls), cname
        for f, _ in cls._fields_:
            assert got[(cname, f)] == getattr(cls, f).offset, f"{cname}.{f}"
