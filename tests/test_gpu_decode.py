"""GPU parity of compressed decode attention and of the serving step against the CPU oracle
(through the C ABI).  Attention outputs must agree within 2e-3 max-abs; lse within 2e-3 as well.

Decode-only cases draw their code streams from the input generator (skewed or uniform codes);
the end-to-end cases encode on each side with its own encoder."""
import numpy as np
import pytest
import torch

from compressed_decode_attention_zkv_b200 import build as B
from compressed_decode_attention_zkv_b200 import inputs as I
from compressed_decode_attention_zkv_b200 import zkv
from oracle import zkv_oracle as O

pytestmark = pytest.mark.gpu
TOL = 2e-3


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    B.build()
    zkv.lib()


def _cuda(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _run_gpu(case, max_comp_len=None, error_flag=None):
    q, kc, vc, comp, Ck, Cv, wk, wv, win = case
    out, lse = zkv.rvq_decode_attn(_cuda(q), _cuda(kc), _cuda(vc),
                                   _cuda(np.asarray(comp, np.int32)), _cuda(Ck), _cuda(Cv),
                                   _cuda(wk), _cuda(wv), _cuda(np.asarray(win, np.int32)),
                                   max_comp_len=max_comp_len, error_flag=error_flag)
    torch.cuda.synchronize()
    return out.cpu().numpy(), lse.cpu().numpy()


def _compare(case, out, lse, pairs=None):
    want_o, want_l = O.decode_attn(*case, pairs=pairs)
    if pairs is None:
        pairs = [(b, h) for b in range(want_o.shape[0]) for h in range(want_o.shape[1])]
    worst = 0.0
    for b, h in pairs:
        err = np.max(np.abs(out[b, h] - want_o[b, h]))
        worst = max(worst, err)
        assert err <= TOL, f"out ({b},{h}) max-abs {err}"
        if np.isneginf(want_l[b, h]):
            assert np.isneginf(lse[b, h])
        else:
            assert abs(lse[b, h] - want_l[b, h]) <= TOL, f"lse ({b},{h})"
    return worst


def _random_case(seed, B_, Hq, Hkv, d, Sk, Sv, Tcap, comp, Wcap, win, kscale=0.1, vscale=0.3,
                 skewed=True):
    rng = np.random.default_rng(seed)
    wl = I.workload("llama3_8b_32k", B=B_, Hq=Hq, Hkv=Hkv, d=d, Sk=Sk, Sv=Sv)
    kc = I.random_codes(wl, "k", Tcap, seed=seed, skewed=skewed)
    vc = I.random_codes(wl, "v", Tcap, seed=seed + 1, skewed=skewed)
    Ck = (rng.standard_normal((Hkv, Sk, 256, d)) * kscale).astype(np.float32)
    Cv = (rng.standard_normal((Hkv, Sv, 256, d)) * vscale).astype(np.float32)
    Ck[:, :, 0] = 0
    Cv[:, :, 0] = 0
    q = rng.standard_normal((B_, Hq, d)).astype(np.float16)
    wk = rng.standard_normal((B_, Hkv, max(Wcap, 1), d)).astype(np.float16)[:, :, :Wcap]
    wv = rng.standard_normal((B_, Hkv, max(Wcap, 1), d)).astype(np.float16)[:, :, :Wcap]
    if Wcap == 0:
        wk = np.zeros((B_, Hkv, 0, d), np.float16)
        wv = np.zeros((B_, Hkv, 0, d), np.float16)
    return (q, kc, vc, np.asarray(comp), Ck, Cv, np.ascontiguousarray(wk),
            np.ascontiguousarray(wv), np.asarray(win))


CASES = {
    # GQA 4, ragged lengths incl. an empty prefix, several chunks, ragged tail
    "gqa4_ragged": dict(B_=3, Hq=8, Hkv=2, d=128, Sk=4, Sv=4, Tcap=5008, comp=[5001, 0, 2222],
                        Wcap=16, win=[16, 3, 0]),
    # GQA 7 (padded to 8 heads), Sk != Sv
    "gqa7": dict(B_=2, Hq=7, Hkv=1, d=128, Sk=2, Sv=4, Tcap=3008, comp=[3001, 1], Wcap=32,
                 win=[32, 32]),
    # one head per kv head, two stages
    "mha_s2": dict(B_=2, Hq=2, Hkv=2, d=128, Sk=2, Sv=2, Tcap=1040, comp=[1025, 17], Wcap=8,
                   win=[0, 8]),
    # GQA 2, odd stage counts (runtime stage path)
    "gqa2_s3s5": dict(B_=1, Hq=4, Hkv=2, d=128, Sk=3, Sv=5, Tcap=2064, comp=[2050], Wcap=4,
                      win=[4]),
    # 8 stages each
    "s8": dict(B_=1, Hq=4, Hkv=1, d=128, Sk=8, Sv=8, Tcap=1024, comp=[1000], Wcap=8, win=[5]),
    # empty contexts and window-only
    "empty": dict(B_=3, Hq=4, Hkv=1, d=128, Sk=1, Sv=1, Tcap=16, comp=[0, 0, 0], Wcap=4,
                  win=[0, 2, 4]),
    # no window at all
    "nowindow": dict(B_=2, Hq=4, Hkv=1, d=128, Sk=4, Sv=4, Tcap=2048, comp=[2048, 777], Wcap=0,
                     win=[0, 0]),
    # head dims 64 and 256
    "d64": dict(B_=2, Hq=8, Hkv=2, d=64, Sk=4, Sv=4, Tcap=1536, comp=[1500, 1536], Wcap=8,
                win=[8, 1]),
    "d256": dict(B_=1, Hq=4, Hkv=1, d=256, Sk=4, Sv=4, Tcap=1536, comp=[1300], Wcap=8, win=[6]),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_decode_random_codes(name):
    case = _random_case(sum(map(ord, name)) % 1000, **CASES[name])
    out, lse = _run_gpu(case)
    worst = _compare(case, out, lse)
    print(f"{name}: worst max-abs {worst:.2e}")


def test_decode_uniform_codes_peaky_scores():
    # large key codewords make the softmax concentrate on a few tokens
    case = _random_case(11, B_=2, Hq=8, Hkv=2, d=128, Sk=4, Sv=4, Tcap=4096, comp=[4096, 3000],
                        Wcap=16, win=[16, 16], kscale=0.6, skewed=False)
    out, lse = _run_gpu(case)
    _compare(case, out, lse)


@pytest.mark.parametrize("Hq,Sk,Sv", [(4, 4, 4), (1, 2, 2), (7, 2, 4)])
def test_decode_rising_scores_raise_the_reference(Hq, Sk, Sv):
    """Key scores that rise along the prefix (stage-0 codeword c scores c / 255 * 30 nats for the
    first query head, codes rising with the token index) plus one spike near the end: the scan
    keeps meeting scores above its reference, lists those tokens, raises the reference and adds
    them afterwards.  The result must still be the oracle's attention."""
    rng = np.random.default_rng(40 + Hq)
    B_, Hkv, d, Tcap, W = 1, 1, 128, 30000, 8
    q = rng.standard_normal((B_, Hq, d)).astype(np.float16)
    qt = O.fwht(q[0, 0].astype(np.float64), 1.0 / np.sqrt(d))   # rotated query of head 0
    scale = 1.0 / np.sqrt(d)
    Ck = (rng.standard_normal((Hkv, Sk, 256, d)) * 0.02).astype(np.float32)
    sigma = np.arange(256) / 255.0 * 30.0
    Ck[0, 0] = (sigma[:, None] / scale * qt[None, :] / np.dot(qt, qt)).astype(np.float32)
    Ck[:, :, 0] = 0
    Cv = (rng.standard_normal((Hkv, Sv, 256, d)) * 0.3).astype(np.float32)
    Cv[:, :, 0] = 0
    kc = rng.integers(0, 256, (B_, Hkv, Tcap, Sk)).astype(np.uint8)
    kc[0, 0, :, 0] = (np.arange(Tcap) * 250 // Tcap).astype(np.uint8)
    kc[0, 0, 29000, 0] = 255                       # a spike near the end
    vc = rng.integers(0, 256, (B_, Hkv, Tcap, Sv)).astype(np.uint8)
    wk = rng.standard_normal((B_, Hkv, W, d)).astype(np.float16)
    wv = rng.standard_normal((B_, Hkv, W, d)).astype(np.float16)
    case = (q, kc, vc, np.array([Tcap]), Ck, Cv, wk, wv, np.array([W]))
    out, lse = _run_gpu(case)
    worst = _compare(case, out, lse)
    print(f"rising scores Hq {Hq} Sk {Sk} Sv {Sv}: worst max-abs {worst:.2e}")


def test_decode_max_comp_len_bounds_the_read():
    case = _random_case(12, B_=2, Hq=4, Hkv=1, d=128, Sk=4, Sv=4, Tcap=4096, comp=[1000, 2000],
                        Wcap=8, win=[8, 8])
    out, lse = _run_gpu(case, max_comp_len=2000)
    _compare(case, out, lse)


def test_decode_comp_len_beyond_capacity_is_clamped_and_flagged():
    case = list(_random_case(13, B_=1, Hq=4, Hkv=1, d=128, Sk=2, Sv=2, Tcap=512, comp=[512],
                             Wcap=4, win=[4]))
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    case_big = list(case)
    case_big[3] = np.array([9999])
    out, lse = _run_gpu(case_big, error_flag=flag)
    assert int(flag.item()) & zkv.ZKV_DEVERR_COMP_LEN
    _compare(case, out, lse)      # equals the attention over the clamped prefix


# ------------------------------------------------------------------ end to end

def test_tiny_workload_end_to_end():
    """Encode (GPU vs oracle, each its own) then decode, config "tiny"."""
    wl = I.workload("tiny")
    Ck = I.train_codebooks(wl, "k")
    Cv = I.train_codebooks(wl, "v")
    k = I.kv_tokens(wl, "k", 0, 0, wl.T)[None]     # [1][1][T][d]
    v = I.kv_tokens(wl, "v", 0, 0, wl.T)[None]
    q = I.queries(wl)
    Tc = wl.Tc
    cache = zkv.RVQKVCache(_cuda(Ck), _cuda(Cv), batch=1, capacity=Tc, window=wl.W)
    cache.prefill(_cuda(k), _cuda(v))
    out, lse = cache.attend(_cuda(q))
    torch.cuda.synchronize()
    zk, _, _, _ = O.rvq_encode(k[0, 0, :Tc], Ck[0])
    zv, _, _, _ = O.rvq_encode(v[0, 0, :Tc], Cv[0])
    np.testing.assert_array_equal(cache.k_codes[0, 0, :Tc].cpu().numpy(), zk)
    np.testing.assert_array_equal(cache.v_codes[0, 0, :Tc].cpu().numpy(), zv)
    case = (q, zk[None, None], zv[None, None], np.array([Tc]), Ck, Cv,
            k[:, :, Tc:], v[:, :, Tc:], np.array([wl.W]))
    _compare(case, out.cpu().numpy(), lse.cpu().numpy())


def _workload_case(name, seed=0, pairs_per_kvh=1):
    wl = I.workload(name)
    lens = I.ragged_lengths(wl)
    comp = (lens - wl.W).astype(np.int64)
    Tcap = int((comp.max() + 15) // 16 * 16)
    kc = I.random_codes(wl, "k", Tcap, seed=seed)
    vc = I.random_codes(wl, "v", Tcap, seed=seed + 1)
    Ck = I.train_codebooks(wl, "k")
    Cv = I.train_codebooks(wl, "v")
    q = I.queries(wl, seed=seed)
    wk = I.window_tokens(wl, "k", lens, seed=seed)
    wv = I.window_tokens(wl, "v", lens, seed=seed)
    win = np.full(wl.B, wl.W)
    return wl, (q, kc, vc, comp, Ck, Cv, wk, wv, win)


@pytest.mark.parametrize("name", ["llama3_8b_32k", "qwen25_7b_128k", "ragged_serving_64"])
def test_decode_full_size_sampled(name):
    wl, case = _workload_case(name)
    out, lse = _run_gpu(case, max_comp_len=int(np.max(case[3])))
    rng = np.random.default_rng(1)
    pairs = [(int(rng.integers(wl.B)), int(rng.integers(wl.Hq))) for _ in range(6)]
    pairs += [(0, 0), (wl.B - 1, wl.Hq - 1)]
    worst = _compare(case, out, lse, pairs=pairs)
    print(f"{name}: worst max-abs over {len(pairs)} sampled heads {worst:.2e}")
    assert np.all(np.isfinite(out)) and np.all(np.isfinite(lse))


# ------------------------------------------------------------------ serving step

def _state(seed, B_, Hkv, d, S, Tcap, Wcap, win_len, win_head, comp_len, Sv=None):
    rng = np.random.default_rng(seed)
    Sv = S if Sv is None else Sv
    Ck = (rng.standard_normal((Hkv, S, 256, d)) * 0.3).astype(np.float32)
    Cv = (rng.standard_normal((Hkv, Sv, 256, d)) * 0.3).astype(np.float32)
    Ck[:, :, 0] = 0
    Cv[:, :, 0] = 0
    return dict(k_codes=rng.integers(0, 256, (B_, Hkv, Tcap, S)).astype(np.uint8),
                v_codes=rng.integers(0, 256, (B_, Hkv, Tcap, Sv)).astype(np.uint8),
                comp_len=np.array(comp_len), win_len=np.array(win_len),
                win_head=np.array(win_head),
                win_k=rng.standard_normal((B_, Hkv, Wcap, d)).astype(np.float16),
                win_v=rng.standard_normal((B_, Hkv, Wcap, d)).astype(np.float16),
                Ck=Ck, Cv=Cv)


def test_append_steps_match_oracle():
    st = _state(20, B_=5, Hkv=2, d=128, S=3, Tcap=32, Wcap=4, win_len=[0, 2, 4, 4, 4],
                win_head=[0, 0, 1, 3, 0], comp_len=[0, 5, 7, 31, 32])
    g = {k: _cuda(v.astype(np.int32) if k in ("comp_len", "win_len", "win_head") else v)
         for k, v in st.items()}
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    rng = np.random.default_rng(21)
    for step in range(4):
        nk = rng.standard_normal((5, 2, 128)).astype(np.float16)
        nv = rng.standard_normal((5, 2, 128)).astype(np.float16)
        st = O.append_step(st, nk, nv)
        zkv.rvq_append(_cuda(nk), _cuda(nv), g["win_k"], g["win_v"], g["win_len"],
                       g["win_head"], g["comp_len"], g["k_codes"], g["v_codes"], g["Ck"],
                       g["Cv"], error_flag=flag)
        torch.cuda.synchronize()
        for key in ("comp_len", "win_len", "win_head", "k_codes", "v_codes", "win_k", "win_v"):
            np.testing.assert_array_equal(g[key].cpu().numpy(), st[key], err_msg=f"{key} step {step}")
    assert st["error"] and (int(flag.item()) & zkv.ZKV_DEVERR_COMP_LEN)


@pytest.mark.parametrize("B_,Hkv,d,Sk,Sv", [(11, 3, 64, 2, 5), (17, 1, 256, 4, 3),
                                           (9, 2, 128, 8, 1)])
def test_append_row_groups_and_shapes(B_, Hkv, d, Sk, Sv):
    """Several 8-sequence groups per head (the last one ragged), every head dimension, Sk != Sv,
    windows filling and full, one prefix at capacity."""
    Tcap, Wcap = 16, 3
    rng = np.random.default_rng(50 + B_)
    win_len = rng.integers(0, Wcap + 1, B_)
    win_len[: B_ // 2] = Wcap
    comp_len = rng.integers(0, Tcap - 2, B_)
    comp_len[1] = Tcap
    st = _state(60 + B_, B_=B_, Hkv=Hkv, d=d, S=Sk, Sv=Sv, Tcap=Tcap, Wcap=Wcap,
                win_len=win_len, win_head=rng.integers(0, Wcap, B_), comp_len=comp_len)
    g = {k: _cuda(v.astype(np.int32) if k in ("comp_len", "win_len", "win_head") else v)
         for k, v in st.items()}
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    for step in range(3):
        nk = rng.standard_normal((B_, Hkv, d)).astype(np.float16)
        nv = rng.standard_normal((B_, Hkv, d)).astype(np.float16)
        st = O.append_step(st, nk, nv)
        zkv.rvq_append(_cuda(nk), _cuda(nv), g["win_k"], g["win_v"], g["win_len"],
                       g["win_head"], g["comp_len"], g["k_codes"], g["v_codes"], g["Ck"],
                       g["Cv"], error_flag=flag)
        torch.cuda.synchronize()
        for key in ("comp_len", "win_len", "win_head", "k_codes", "v_codes", "win_k", "win_v"):
            np.testing.assert_array_equal(g[key].cpu().numpy(), st[key], err_msg=f"{key} step {step}")
    assert st["error"] and (int(flag.item()) & zkv.ZKV_DEVERR_COMP_LEN)


def test_serving_loop_matches_oracle():
    """prefill -> (append, attend) x 6 through RVQKVCache vs the oracle's step semantics."""
    rng = np.random.default_rng(30)
    Bn, Hq, Hkv, d, S, W = 3, 8, 2, 128, 4, 8
    Ck = (rng.standard_normal((Hkv, S, 256, d)) * 0.15).astype(np.float32)
    Cv = (rng.standard_normal((Hkv, S, 256, d)) * 0.3).astype(np.float32)
    Ck[:, :, 0] = 0
    Cv[:, :, 0] = 0
    T0 = 300
    k = rng.standard_normal((Bn, Hkv, T0, d)).astype(np.float16)
    v = rng.standard_normal((Bn, Hkv, T0, d)).astype(np.float16)
    cache = zkv.RVQKVCache(_cuda(Ck), _cuda(Cv), batch=Bn, capacity=T0 + 16, window=W)
    cache.prefill(_cuda(k), _cuda(v))
    Tc = T0 - W
    Tcap = cache.Tcap
    zk = np.zeros((Bn, Hkv, Tcap, S), np.uint8)
    zv = np.zeros((Bn, Hkv, Tcap, S), np.uint8)
    for b in range(Bn):
        for h in range(Hkv):
            zk[b, h, :Tc] = O.rvq_encode(k[b, h, :Tc], Ck[h])[0]
            zv[b, h, :Tc] = O.rvq_encode(v[b, h, :Tc], Cv[h])[0]
    st = dict(k_codes=zk, v_codes=zv, comp_len=np.full(Bn, Tc), win_len=np.full(Bn, W),
              win_head=np.zeros(Bn, np.int64), win_k=k[:, :, Tc:].copy(),
              win_v=v[:, :, Tc:].copy(), Ck=Ck, Cv=Cv)
    for step in range(6):
        nk = rng.standard_normal((Bn, Hkv, d)).astype(np.float16)
        nv = rng.standard_normal((Bn, Hkv, d)).astype(np.float16)
        q = rng.standard_normal((Bn, Hq, d)).astype(np.float16)
        cache.append(_cuda(nk), _cuda(nv))
        out, lse = cache.attend(_cuda(q))
        st = O.append_step(st, nk, nv)
        case = (q, st["k_codes"], st["v_codes"], st["comp_len"], Ck, Cv, st["win_k"],
                st["win_v"], st["win_len"])
        _compare(case, out.cpu().numpy(), lse.cpu().numpy())
    assert int(cache.error_flag.item()) == 0


def test_cache_step_equals_append_then_attend():
    """RVQKVCache.step (one serving-step call) is bit-identical to append + attend."""
    rng = np.random.default_rng(31)
    Bn, Hq, Hkv, d, S, W = 2, 8, 2, 128, 4, 4
    Ck = (rng.standard_normal((Hkv, S, 256, d)) * 0.15).astype(np.float32)
    Cv = (rng.standard_normal((Hkv, S, 256, d)) * 0.3).astype(np.float32)
    Ck[:, :, 0] = 0
    Cv[:, :, 0] = 0
    k = rng.standard_normal((Bn, Hkv, 100, d)).astype(np.float16)
    v = rng.standard_normal((Bn, Hkv, 100, d)).astype(np.float16)
    caches = [zkv.RVQKVCache(_cuda(Ck), _cuda(Cv), batch=Bn, capacity=112, window=W)
              for _ in range(2)]
    for c in caches:
        c.prefill(_cuda(k), _cuda(v))
    for step in range(5):
        nk = _cuda(rng.standard_normal((Bn, Hkv, d)).astype(np.float16))
        nv = _cuda(rng.standard_normal((Bn, Hkv, d)).astype(np.float16))
        q = _cuda(rng.standard_normal((Bn, Hq, d)).astype(np.float16))
        caches[0].append(nk, nv)
        o0, l0 = caches[0].attend(q)
        o1, l1 = caches[1].step(nk, nv, q)
        assert torch.equal(o0, o1) and torch.equal(l0, l1), step
    for name in ("k_codes", "v_codes", "win_k", "win_v", "comp_len", "win_len", "win_head"):
        assert torch.equal(getattr(caches[0], name), getattr(caches[1], name)), name
    assert int(caches[0].error_flag.item()) == 0 and int(caches[1].error_flag.item()) == 0


def test_prepared_calls_match_the_plain_entry_points():
    """PreparedAppend / PreparedDecode (arguments marshalled once) give bit-identical results
    to rvq_append / rvq_decode_attn over several serving steps."""
    st = _state(80, B_=3, Hkv=2, d=128, S=4, Tcap=64, Wcap=4, win_len=[4, 4, 2],
                win_head=[1, 0, 0], comp_len=[10, 0, 33])
    rng = np.random.default_rng(81)
    sides = []
    for _ in range(2):
        g = {k: _cuda(v.astype(np.int32) if k in ("comp_len", "win_len", "win_head") else v)
             for k, v in st.items()}
        g["err"] = torch.zeros(1, dtype=torch.int32, device="cuda")
        g["new_k"] = torch.zeros((3, 2, 128), dtype=torch.float16, device="cuda")
        g["new_v"] = torch.zeros((3, 2, 128), dtype=torch.float16, device="cuda")
        g["q"] = torch.zeros((3, 8, 128), dtype=torch.float16, device="cuda")
        sides.append(g)
    a, b = sides
    app = zkv.PreparedAppend(b["new_k"], b["new_v"], b["win_k"], b["win_v"], b["win_len"],
                             b["win_head"], b["comp_len"], b["k_codes"], b["v_codes"], b["Ck"],
                             b["Cv"], error_flag=b["err"])
    dec = zkv.PreparedDecode(b["q"], b["k_codes"], b["v_codes"], b["comp_len"], b["Ck"], b["Cv"],
                             b["win_k"], b["win_v"], b["win_len"], max_comp_len=64,
                             error_flag=b["err"])
    for step in range(3):
        nk = _cuda(rng.standard_normal((3, 2, 128)).astype(np.float16))
        nv = _cuda(rng.standard_normal((3, 2, 128)).astype(np.float16))
        q = _cuda(rng.standard_normal((3, 8, 128)).astype(np.float16))
        zkv.rvq_append(nk, nv, a["win_k"], a["win_v"], a["win_len"], a["win_head"],
                       a["comp_len"], a["k_codes"], a["v_codes"], a["Ck"], a["Cv"],
                       error_flag=a["err"])
        o1, l1 = zkv.rvq_decode_attn(q, a["k_codes"], a["v_codes"], a["comp_len"], a["Ck"],
                                     a["Cv"], a["win_k"], a["win_v"], a["win_len"],
                                     max_comp_len=64, error_flag=a["err"])
        b["new_k"].copy_(nk)
        b["new_v"].copy_(nv)
        b["q"].copy_(q)
        app()
        o2, l2 = dec()
        torch.cuda.synchronize()
        assert torch.equal(o1, o2) and torch.equal(l1, l2), f"step {step}"
        for key in ("k_codes", "v_codes", "win_k", "win_v", "comp_len", "win_len", "win_head"):
            assert torch.equal(a[key], b[key]), f"{key} step {step}"


@pytest.mark.parametrize("B_,Hq,Hkv,d,S,Sv,Tcap,Wcap,win_len,win_head,comp_len", [
    (3, 8, 2, 128, 4, 4, 64, 4, [4, 4, 2], [1, 0, 0], [10, 0, 33]),
    (9, 14, 2, 64, 2, 3, 48, 3, [3, 1, 3, 0, 3, 3, 2, 3, 3], [2, 0, 0, 0, 1, 0, 0, 2, 1],
     [47, 5, 0, 0, 20, 48, 3, 8, 16]),
])
def test_serve_step_matches_append_then_decode(B_, Hq, Hkv, d, S, Sv, Tcap, Wcap, win_len,
                                               win_head, comp_len):
    """zkv_rvq_serve_step gives bit-identical outputs and cache state to zkv_rvq_append followed
    by zkv_rvq_decode_attn, step after step (free slots, evictions, a full prefix)."""
    st = _state(90 + B_, B_=B_, Hkv=Hkv, d=d, S=S, Sv=Sv, Tcap=Tcap, Wcap=Wcap, win_len=win_len,
                win_head=win_head, comp_len=comp_len)
    rng = np.random.default_rng(91 + B_)
    sides = []
    for _ in range(2):
        g = {k: _cuda(v.astype(np.int32) if k in ("comp_len", "win_len", "win_head") else v)
             for k, v in st.items()}
        g["err"] = torch.zeros(1, dtype=torch.int32, device="cuda")
        sides.append(g)
    a, b = sides
    for step in range(4):
        nk = _cuda(rng.standard_normal((B_, Hkv, d)).astype(np.float16))
        nv = _cuda(rng.standard_normal((B_, Hkv, d)).astype(np.float16))
        q = _cuda(rng.standard_normal((B_, Hq, d)).astype(np.float16))
        zkv.rvq_append(nk, nv, a["win_k"], a["win_v"], a["win_len"], a["win_head"],
                       a["comp_len"], a["k_codes"], a["v_codes"], a["Ck"], a["Cv"],
                       error_flag=a["err"])
        o1, l1 = zkv.rvq_decode_attn(q, a["k_codes"], a["v_codes"], a["comp_len"], a["Ck"],
                                     a["Cv"], a["win_k"], a["win_v"], a["win_len"],
                                     max_comp_len=Tcap, error_flag=a["err"])
        o2, l2 = zkv.rvq_serve_step(nk, nv, q, b["win_k"], b["win_v"], b["win_len"],
                                    b["win_head"], b["comp_len"], b["k_codes"], b["v_codes"],
                                    b["Ck"], b["Cv"], max_comp_len=Tcap, error_flag=b["err"])
        torch.cuda.synchronize()
        assert torch.equal(o1, o2) and torch.equal(l1, l2), f"step {step}"
        for key in ("k_codes", "v_codes", "win_k", "win_v", "comp_len", "win_len", "win_head",
                    "err"):
            assert torch.equal(a[key], b[key]), f"{key} step {step}"


def test_serve_step_loop_matches_oracle():
    """Prepared serving steps on a trained-codebook cache vs the oracle's append step followed
    by its decode (plain definition)."""
    rng = np.random.default_rng(95)
    wl = I.workload("llama3_8b_32k", B=2, Hq=8, Hkv=2, T=700, W=16, n_cal=2048, kmeans_iters=4)
    Ck, Cv = I.train_codebooks(wl, "k"), I.train_codebooks(wl, "v")
    Tc, Tcap = wl.Tc, (wl.Tc + 32 + 15) // 16 * 16   # capacities are multiples of 16
    zk = np.zeros((wl.B, wl.Hkv, Tcap, wl.Sk), np.uint8)
    zv = np.zeros((wl.B, wl.Hkv, Tcap, wl.Sv), np.uint8)
    wk = np.zeros((wl.B, wl.Hkv, wl.W, wl.d), np.float16)
    wv = np.zeros((wl.B, wl.Hkv, wl.W, wl.d), np.float16)
    for b in range(wl.B):
        xk, xv = I.kv_tokens(wl, "k", b, 0, wl.T), I.kv_tokens(wl, "v", b, 0, wl.T)
        for h in range(wl.Hkv):
            zk[b, h, :Tc] = O.rvq_encode(xk[h, :Tc], Ck[h])[0]
            zv[b, h, :Tc] = O.rvq_encode(xv[h, :Tc], Cv[h])[0]
        wk[b], wv[b] = xk[:, Tc:], xv[:, Tc:]
    st = dict(k_codes=zk, v_codes=zv, comp_len=np.full(wl.B, Tc), win_len=np.full(wl.B, wl.W),
              win_head=np.zeros(wl.B, np.int64), win_k=wk, win_v=wv, Ck=Ck, Cv=Cv)
    g = {k: _cuda(v.astype(np.int32) if k in ("comp_len", "win_len", "win_head") else v)
         for k, v in st.items()}
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    nk_d = torch.zeros((wl.B, wl.Hkv, wl.d), dtype=torch.float16, device="cuda")
    nv_d, q_d = torch.zeros_like(nk_d), torch.zeros((wl.B, wl.Hq, wl.d), dtype=torch.float16,
                                                     device="cuda")
    step_fn = zkv.PreparedServeStep(nk_d, nv_d, q_d, g["win_k"], g["win_v"], g["win_len"],
                                    g["win_head"], g["comp_len"], g["k_codes"], g["v_codes"],
                                    g["Ck"], g["Cv"], max_comp_len=Tcap, error_flag=err)
    for step in range(3):
        nk = rng.standard_normal((wl.B, wl.Hkv, wl.d)).astype(np.float16)
        nv = rng.standard_normal((wl.B, wl.Hkv, wl.d)).astype(np.float16)
        q = rng.standard_normal((wl.B, wl.Hq, wl.d)).astype(np.float16)
        nk_d.copy_(_cuda(nk))
        nv_d.copy_(_cuda(nv))
        q_d.copy_(_cuda(q))
        out, lse = step_fn()
        st = O.append_step(st, nk, nv)
        case = (q, st["k_codes"], st["v_codes"], st["comp_len"], Ck, Cv, st["win_k"],
                st["win_v"], st["win_len"])
        _compare(case, out.cpu().numpy(), lse.cpu().numpy())
        assert np.array_equal(g["k_codes"].cpu().numpy(), st["k_codes"])
        assert np.array_equal(g["v_codes"].cpu().numpy(), st["v_codes"])
    assert int(err.item()) == 0
