"""GPU parity of the Walsh-Hadamard transform, RVQ encode and reconstruction against the
CPU oracle (through the C ABI).

Matching rules: codes bit-exact except counted near-ties (the oracle's distance gap below 1e-5
relative); residual norms within 1e-6 relative; reconstructions within 1e-5 max-abs; the
transform of fp16 input bit-exact (the float64 sums are exact, one rounding at the end)."""
import numpy as np
import pytest
import torch

from compressed_decode_attention_zkv_b200 import build as B
from compressed_decode_attention_zkv_b200 import inputs as I
from compressed_decode_attention_zkv_b200 import zkv
from oracle import zkv_oracle as O

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    B.build()
    zkv.lib()


def _cuda(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


# ------------------------------------------------------------------ FWHT

@pytest.mark.parametrize("d", [64, 128, 256])
def test_fwht_fp16_bit_exact(d):
    rng = np.random.default_rng(d)
    x = (rng.standard_normal((777, d)) * np.exp(rng.uniform(-6, 6, (777, d)))).astype(np.float16)
    for scale in (1.0, 1.0 / np.sqrt(d)):
        got = zkv.fwht(_cuda(x), scale).cpu().numpy()
        want = O.fwht(x, np.float64(np.float32(scale))).astype(np.float32)
        np.testing.assert_array_equal(got, want)


@pytest.mark.parametrize("d", [64, 128, 256])
def test_fwht_fp32_and_in_place(d):
    rng = np.random.default_rng(100 + d)
    x = rng.standard_normal((300, d)).astype(np.float32)
    want = O.fwht(x, 0.5).astype(np.float32)
    got = zkv.fwht(_cuda(x), 0.5).cpu().numpy()
    np.testing.assert_allclose(got, want, rtol=2e-7, atol=1e-7)
    xt = _cuda(x)
    zkv.fwht(xt, 0.5, out=xt)
    np.testing.assert_allclose(xt.cpu().numpy(), want, rtol=2e-7, atol=1e-7)


def test_fwht_involution_on_gpu():
    rng = np.random.default_rng(7)
    x = rng.standard_normal((64, 128)).astype(np.float32)
    s = 1.0 / np.sqrt(128)
    y = zkv.fwht(_cuda(x), s)
    z = zkv.fwht(y, s).cpu().numpy()
    np.testing.assert_allclose(z, x, atol=1e-6)


# ------------------------------------------------------------------ encode

def _check_codes(x_rows, books, codes, norms, label):
    walk = O.rvq_match_walk(x_rows, books, codes)
    assert walk["mismatches"] == 0, f"{label}: {walk['bad']}"
    want_codes, want_norms, _, _ = O.rvq_encode(x_rows, books)
    same = np.all(codes == want_codes, axis=1)
    if norms is not None:
        np.testing.assert_allclose(norms[same], want_norms[same], rtol=1e-6, atol=1e-6)
    return walk


def test_encode_tiny_workload_full():
    """Config "tiny": 1 kv head, d = 128, 1024 tokens, 2 stages, K and V."""
    wl = I.workload("tiny")
    for kind in ("k", "v"):
        books = I.train_codebooks(wl, kind)
        x = I.kv_tokens(wl, kind, 0, 0, wl.T)            # [Hkv][T][d]
        xt = _cuda(x).permute(1, 0, 2)                    # [T, H, d] view
        codes, norms = zkv.rvq_encode(xt, _cuda(books))
        codes = codes[0].cpu().numpy()                    # [T, H, S]
        norms = norms[0].cpu().numpy()
        walk = _check_codes(x[0], books[0], codes[:, 0], norms[:, 0], f"tiny/{kind}")
        print(f"tiny/{kind}: exact {walk['exact']} near-tie exceptions {walk['exceptions']}")


@pytest.mark.parametrize("n_tok", [300, 2213])   # row-group path; tiled path (> 4096 rows)
def test_encode_paths_ragged(n_tok):
    wl = I.workload("llama3_8b_32k", B=1, Hkv=2, Hq=8, T=n_tok, n_cal=2048, kmeans_iters=4)
    books = I.train_codebooks(wl, "k")                    # [2][4][256][128]
    x = I.kv_tokens(wl, "k", 0, 0, n_tok)                 # [2][T][128]
    codes, norms = zkv.rvq_encode(_cuda(x).permute(1, 0, 2), _cuda(books))
    codes = codes[0].cpu().numpy()
    norms = norms[0].cpu().numpy()
    for h in range(2):
        _check_codes(x[h], books[h], codes[:, h], norms[:, h], f"h{h}")


@pytest.mark.parametrize("d,n", [(64, 200), (64, 4500), (256, 100), (256, 4200)])
def test_encode_other_head_dims(d, n):
    rng = np.random.default_rng(d + n)
    S = 3
    books = (rng.standard_normal((1, S, 256, d)) * np.array([1.0, 0.5, 0.25])[None, :, None, None]).astype(np.float32)
    books[:, :, 0] = 0
    x = (rng.standard_normal((n, d)) * 1.5).astype(np.float16)
    codes, norms = zkv.rvq_encode(_cuda(x), _cuda(books))
    _check_codes(x, books[0], codes[0, :, 0].cpu().numpy(), norms[0, :, 0].cpu().numpy(), f"d{d}")


def test_encode_fp32_input_without_rotation():
    rng = np.random.default_rng(3)
    books = rng.standard_normal((1, 2, 256, 128)).astype(np.float32)
    books[:, :, 0] = 0
    y = rng.standard_normal((500, 128)).astype(np.float32)
    codes, norms = zkv.rvq_encode(_cuda(y), _cuda(books), rotate=False)
    walk = O.rvq_match_walk(y, books[0], codes[0, :, 0].cpu().numpy(), rotate=False)
    assert walk["mismatches"] == 0


def test_encode_special_inputs():
    rng = np.random.default_rng(4)
    books = rng.standard_normal((1, 4, 256, 128)).astype(np.float32)
    books[:, :, 0] = 0
    books[0, 0, 77] = books[0, 0, 13]                 # duplicate codeword: lower index wins
    y = np.stack([np.zeros(128, np.float32),          # zero vector -> all codes 0
                  books[0, 0, 200].copy(),            # exact codeword -> 200 then zeros
                  books[0, 0, 13] + 1e-3]).astype(np.float32)
    codes, norms = zkv.rvq_encode(_cuda(y), _cuda(books), rotate=False)
    c = codes[0, :, 0].cpu().numpy()
    n = norms[0, :, 0].cpu().numpy()
    assert list(c[0]) == [0, 0, 0, 0] and np.all(n[0] == 0)
    assert list(c[1]) == [200, 0, 0, 0] and np.all(n[1] == 0)
    assert c[2, 0] == 13


def test_norms_never_increase_on_trained_books():
    wl = I.workload("llama3_8b_32k", B=1, Hkv=1, Hq=4, T=1500, n_cal=2048, kmeans_iters=4)
    books = I.train_codebooks(wl, "v")
    x = I.kv_tokens(wl, "v", 0, 0, 1500)[0]
    codes, norms = zkv.rvq_encode(_cuda(x), _cuda(books))
    n = norms[0, :, 0].cpu().numpy().astype(np.float64)
    y = O.rotate_to_f32(x).astype(np.float64)
    alln = np.concatenate([np.linalg.norm(y, axis=1)[:, None], n], axis=1)
    assert np.all(np.diff(alln, axis=1) <= 1e-5)


# ------------------------------------------------------------------ reconstruction

def test_reconstruct_matches_oracle():
    rng = np.random.default_rng(5)
    books = rng.standard_normal((2, 3, 256, 128)).astype(np.float32)
    codes = rng.integers(0, 256, (4, 37, 2, 3)).astype(np.uint8)    # [B, T, H, S]
    for unrot in (False, True):
        got = zkv.rvq_reconstruct(_cuda(codes), _cuda(books), unrotate=unrot).cpu().numpy()
        for h in range(2):
            want = O.reconstruct(codes[:, :, h], books[h], unrotate=unrot)
            np.testing.assert_allclose(got[:, :, h], want, atol=1e-5, rtol=0)


def test_encode_then_reconstruct_plus_residual_identity():
    rng = np.random.default_rng(6)
    books = (rng.standard_normal((1, 4, 256, 128)) * 0.5).astype(np.float32)
    books[:, :, 0] = 0
    x = rng.standard_normal((400, 128)).astype(np.float16)
    codes, norms = zkv.rvq_encode(_cuda(x), _cuda(books))
    xh = zkv.rvq_reconstruct(codes, _cuda(books)).cpu().numpy()[0, :, 0]
    y = O.rotate_to_f32(x)
    resid = np.linalg.norm(y.astype(np.float64) - xh, axis=1)
    np.testing.assert_allclose(resid, norms[0, :, 0, -1].cpu().numpy(), rtol=1e-5, atol=1e-5)


@pytest.mark.parametrize("kind", ["k", "v"])
def test_encode_full_size_sampled(kind):
    """prefill_encode_64k at full size (65536 tokens x 8 kv heads, d = 128, S = 8), encoded in
    the launch configuration the benchmark times; 256 sampled rows against the oracle, the
    residual norms of every row non-increasing."""
    wl = I.workload("prefill_encode_64k")
    books = I.train_codebooks(wl, kind)                   # [8][8][256][128]
    x = I.kv_tokens(wl, kind, 0, 0, wl.T)                 # [Hkv][T][d] fp16
    codes, norms = zkv.rvq_encode(_cuda(x).permute(1, 0, 2), _cuda(books))
    codes = codes[0].cpu().numpy()                        # [T, H, S]
    norms = norms[0].cpu().numpy()
    rng = np.random.default_rng(7)
    for h in range(wl.Hkv):
        rows = np.sort(rng.choice(wl.T, 32, replace=False))
        rows[0], rows[-1] = 0, wl.T - 1
        _check_codes(x[h, rows], books[h], codes[rows, h], norms[rows, h], f"{kind}/h{h}")
    # every row: the norms after each stage never increase (codeword 0 is zero)
    assert np.all(np.diff(norms.astype(np.float64), axis=2) <= 1e-5 * (1.0 + norms[..., :-1]))
    assert np.all(np.isfinite(norms))
