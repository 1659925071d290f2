"""Seeded synthetic inputs for RVQ KV-cache encode and compressed decode attention.

Both sides of every parity check draw their inputs from here: the CUDA library (through its
Python binding) and the CPU oracle.  This module therefore holds none of the method's own
arithmetic -- no residual quantisation, no lookup tables, no attention.  It only

* draws key / value / query tensors with the shapes and value distributions of the workloads
  (per-channel lognormal scales, outlier channels on keys, rotary position embedding applied to
  keys, fp16 storage),
* trains codebooks by seeded k-means on a separate calibration sample (the VQKV summary,
  section 2.1 "Training", pre-trains its codebooks on text activations that are not available
  here; seeded k-means on synthetic calibration data stands in for that), and
* draws synthetic code streams and ragged sequence lengths for decode-only cases.

The calibration sample is mapped into the Walsh-Hadamard domain with ``scipy.linalg.hadamard``
(a library routine) because codebooks live in the rotated domain; nothing here is shared with
either implementation under test.

Seeds: data 0, calibration 1, k-means 2, ragged lengths 3 (each config may override).
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass

import numpy as np
import scipy.linalg

K_CODEWORDS = 256

SEED_DATA = 0
SEED_CALIB = 1
SEED_KMEANS = 2
SEED_LENGTHS = 3


@dataclass(frozen=True)
class Workload:
    """Shape and distribution recipe of one synthetic workload."""

    name: str
    B: int                      # sequences
    Hq: int                     # query heads
    Hkv: int                    # key/value heads (GQA groups of Hq // Hkv)
    d: int                      # head dimension
    T: int                      # context length per sequence (compressed + window)
    W: int                      # recency-window capacity (fp16 tokens)
    Sk: int                     # RVQ stages for keys
    Sv: int                     # RVQ stages for values
    rope_theta: float | None    # rotary base applied to keys (None: no RoPE)
    k_outliers: int             # outlier channels per key head
    k_outlier_gain: float       # multiplier on those channels
    v_lognormal: bool           # values also get lognormal channel scales
    ragged: tuple[int, int] | None = None   # (lo, hi) inclusive range of per-sequence lengths
    steps: int = 0              # serving steps (ragged serving workload)
    n_cal: int = 8192           # calibration vectors per codebook set
    kmeans_iters: int = 10

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def Tc(self) -> int:
        """Compressed tokens per sequence for the uniform-length workloads."""
        return self.T - self.W


WORKLOADS: dict[str, Workload] = {
    # Tiny single-head case the oracle finishes in seconds.
    "tiny": Workload("tiny", B=1, Hq=1, Hkv=1, d=128, T=1024, W=64, Sk=2, Sv=2,
                     rope_theta=None, k_outliers=4, k_outlier_gain=8.0, v_lognormal=True),
    # Llama-3-8B-shaped single-layer decode, 32K context.
    "llama3_8b_32k": Workload("llama3_8b_32k", B=8, Hq=32, Hkv=8, d=128, T=32768, W=128,
                              Sk=4, Sv=4, rope_theta=500000.0, k_outliers=8,
                              k_outlier_gain=10.0, v_lognormal=False),
    # Qwen2.5-7B-shaped long-context decode, 128K context.
    "qwen25_7b_128k": Workload("qwen25_7b_128k", B=1, Hq=28, Hkv=4, d=128, T=131072, W=256,
                               Sk=2, Sv=4, rope_theta=1000000.0, k_outliers=8,
                               k_outlier_gain=10.0, v_lognormal=False),
    # Prefill encode throughput: 65536 tokens x 8 heads x {K, V}, 8 stages.
    "prefill_encode_64k": Workload("prefill_encode_64k", B=1, Hq=8, Hkv=8, d=128, T=65536,
                                   W=0, Sk=8, Sv=8, rope_theta=500000.0, k_outliers=8,
                                   k_outlier_gain=10.0, v_lognormal=False),
    # Ragged serving batch: 64 sequences, lengths U{1024..16384}.
    "ragged_serving_64": Workload("ragged_serving_64", B=64, Hq=32, Hkv=8, d=128, T=16384,
                                  W=128, Sk=4, Sv=4, rope_theta=500000.0, k_outliers=8,
                                  k_outlier_gain=10.0, v_lognormal=False,
                                  ragged=(1024, 16384), steps=100),
}


def workload(name: str, **overrides) -> Workload:
    """A named workload, optionally with fields replaced (smaller test variants)."""
    return dataclasses.replace(WORKLOADS[name], **overrides)


# --------------------------------------------------------------------------------------------
# Random streams
# --------------------------------------------------------------------------------------------

def _rng(seed: int, *tags: int) -> np.random.Generator:
    """Independent numpy stream for (seed, tags...); tags name the tensor and its batch row."""
    return np.random.default_rng([seed, *tags])


_TAG_KSCALE, _TAG_VSCALE, _TAG_K, _TAG_V, _TAG_Q, _TAG_OUTLIER = 11, 12, 13, 14, 15, 16
_TAG_CODES_K, _TAG_CODES_V, _TAG_CODE_PROBS, _TAG_NEWTOK = 21, 22, 23, 24
_TAG_POS = 31


def channel_scales(wl: Workload, kind: str, seed: int = SEED_DATA) -> np.ndarray:
    """Per (kv head, channel) multipliers, float32 [Hkv][d].

    Lognormal(0, 0.5) for every channel of keys (and of values where the workload says so),
    with ``k_outliers`` channels per key head, picked by a seeded permutation, multiplied by
    ``k_outlier_gain``.  Values of the larger workloads are plain N(0, 1) (all ones here).
    """
    if kind == "k":
        sc = _rng(seed, _TAG_KSCALE).lognormal(0.0, 0.5, size=(wl.Hkv, wl.d))
        orng = _rng(seed, _TAG_OUTLIER)
        for h in range(wl.Hkv):
            idx = orng.permutation(wl.d)[: wl.k_outliers]
            sc[h, idx] *= wl.k_outlier_gain
        return sc.astype(np.float32)
    if kind == "v":
        if wl.v_lognormal:
            return _rng(seed, _TAG_VSCALE).lognormal(0.0, 0.5, size=(wl.Hkv, wl.d)).astype(np.float32)
        return np.ones((wl.Hkv, wl.d), np.float32)
    raise ValueError(kind)


def apply_rope(x: np.ndarray, positions: np.ndarray, theta: float) -> np.ndarray:
    """Rotary position embedding, "rotate-half" pairing (i, i + d/2), in float32.

    x: [..., n, d] float32; positions: [n] integer.  Angle of pair i at position p is
    p * theta**(-2i/d).  This shapes the key distribution like a real post-RoPE cache.
    """
    d = x.shape[-1]
    half = d // 2
    inv_freq = (theta ** (-(np.arange(half, dtype=np.float32) * 2.0) / d)).astype(np.float32)
    ang = positions.astype(np.float32)[:, None] * inv_freq[None, :]
    cos = np.cos(ang).astype(np.float32)
    sin = np.sin(ang).astype(np.float32)
    x1 = x[..., :half]
    x2 = x[..., half:]
    out = np.empty_like(x)
    out[..., :half] = x1 * cos - x2 * sin
    out[..., half:] = x2 * cos + x1 * sin
    return out


def kv_tokens(wl: Workload, kind: str, b: int, t0: int, t1: int,
              seed: int = SEED_DATA) -> np.ndarray:
    """Key or value vectors of sequence ``b`` for positions [t0, t1), fp16 [Hkv][t1-t0][d].

    Each (b, kind) has its own stream, so any slice is reproducible on its own: the stream is
    advanced over [0, t0) in blocks before the requested block is drawn.
    """
    tag = _TAG_K if kind == "k" else _TAG_V
    rng = _rng(seed, tag, b)
    # Draw in position-major blocks so slices are consistent.
    block = 4096
    out = np.empty((wl.Hkv, t1 - t0, wl.d), np.float32)
    scales = channel_scales(wl, kind, seed)
    t = 0
    while t < t1:
        n = min(block, t1 - t) if t >= t0 else min(block, t0 - t)
        z = rng.standard_normal((n, wl.Hkv, wl.d), dtype=np.float32)
        if t >= t0:
            out[:, t - t0:t - t0 + n, :] = np.transpose(z, (1, 0, 2))
        t += n
    out *= scales[:, None, :]
    if kind == "k" and wl.rope_theta is not None:
        pos = np.arange(t0, t1)
        out = apply_rope(out, pos, wl.rope_theta)
    return out.astype(np.float16)


def window_tokens(wl: Workload, kind: str, lengths: np.ndarray,
                  seed: int = SEED_DATA) -> np.ndarray:
    """The W newest tokens of every sequence, fp16 [B][Hkv][W][d], drawn from a stream of
    their own (cheap for long contexts); keys get RoPE at positions len-W .. len-1."""
    tag = 41 if kind == "k" else 42
    out = np.empty((wl.B, wl.Hkv, wl.W, wl.d), np.float16)
    scales = channel_scales(wl, kind, seed)
    for b in range(wl.B):
        z = _rng(seed, tag, b).standard_normal((wl.Hkv, wl.W, wl.d), dtype=np.float32)
        z *= scales[:, None, :]
        if kind == "k" and wl.rope_theta is not None:
            pos = np.arange(int(lengths[b]) - wl.W, int(lengths[b]))
            z = apply_rope(z, pos, wl.rope_theta)
        out[b] = z.astype(np.float16)
    return out


def queries(wl: Workload, seed: int = SEED_DATA, step: int = 0) -> np.ndarray:
    """Decode queries, fp16 N(0, 1), [B][Hq][d]."""
    z = _rng(seed, _TAG_Q, step).standard_normal((wl.B, wl.Hq, wl.d), dtype=np.float32)
    return z.astype(np.float16)


def new_tokens(wl: Workload, step: int, kind: str, positions: np.ndarray,
               seed: int = SEED_DATA) -> np.ndarray:
    """The token each sequence appends at serving step ``step``: fp16 [B][Hkv][d].

    ``positions`` [B] are the tokens' absolute positions (for RoPE on keys).
    """
    tag = 1 if kind == "k" else 2
    z = _rng(seed, _TAG_NEWTOK, step, tag).standard_normal((wl.B, wl.Hkv, wl.d),
                                                           dtype=np.float32)
    z *= channel_scales(wl, kind, seed)[None]
    if kind == "k" and wl.rope_theta is not None:
        out = np.empty_like(z)
        for b in range(wl.B):
            out[b] = apply_rope(z[b][:, None, :], np.array([positions[b]]), wl.rope_theta)[:, 0]
        z = out
    return z.astype(np.float16)


def ragged_lengths(wl: Workload, seed: int = SEED_LENGTHS) -> np.ndarray:
    """Per-sequence context lengths, int64 [B], uniform on the workload's inclusive range."""
    if wl.ragged is None:
        return np.full(wl.B, wl.T, np.int64)
    lo, hi = wl.ragged
    return _rng(seed).integers(lo, hi + 1, size=wl.B).astype(np.int64)


# --------------------------------------------------------------------------------------------
# Codebooks: seeded k-means on a calibration sample (inputs, shared by both sides)
# --------------------------------------------------------------------------------------------

def _calibration_sample(wl: Workload, kind: str, h: int, n: int, seed: int) -> np.ndarray:
    """n calibration vectors of head h, drawn like the data (own seed), float32 [n][d]."""
    rng = _rng(seed, 100 + (0 if kind == "k" else 1), h)
    z = rng.standard_normal((n, wl.d), dtype=np.float32)
    z *= channel_scales(wl, kind, SEED_DATA)[h][None, :]
    if kind == "k" and wl.rope_theta is not None:
        pos = _rng(seed, _TAG_POS, h).integers(0, max(wl.T, 1), size=n)
        z = apply_rope(z[None], pos, wl.rope_theta)[0]
    return z.astype(np.float16).astype(np.float32)


def _kmeans_zero_pinned(X: np.ndarray, K: int, iters: int,
                        rng: np.random.Generator) -> tuple[np.ndarray, np.ndarray]:
    """Lloyd k-means with codeword 0 held at the zero vector.

    Init: K-1 samples chosen by ``rng`` among the distinct nonzero rows of X (residual stages
    contain exact zeros where an earlier centroid was a single sample; seeding from those would
    create duplicate zero codewords).  Empty clusters keep their centroid.
    Returns (centroids float32 [K][d], final assignment int64 [n]).
    """
    n, d = X.shape
    C = np.zeros((K, d), np.float32)
    nz = np.nonzero(np.any(X != 0, axis=1))[0]
    _, first = np.unique(X[nz], axis=0, return_index=True)
    pool = nz[np.sort(first)]
    pick = rng.choice(pool, min(K - 1, len(pool)), replace=False)
    C[1:1 + len(pick)] = X[pick]

    def assign(C):
        score = (C.astype(np.float32) ** 2).sum(1)[None, :] - 2.0 * (X @ C.T)
        return score.argmin(1)

    for _ in range(iters):
        a = assign(C)
        order = np.argsort(a, kind="stable")
        counts = np.bincount(a, minlength=K)
        starts = np.concatenate([[0], np.cumsum(counts)[:-1]])
        nz = np.nonzero(counts)[0]
        sums = np.add.reduceat(X[order].astype(np.float64), starts[nz], axis=0)
        newc = C.astype(np.float64).copy()
        newc[nz] = sums / counts[nz, None]
        newc[0] = 0.0
        C = newc.astype(np.float32)
    return C, assign(C)


def key_smooth_factors(wl: Workload, seed_cal: int = SEED_CALIB) -> np.ndarray:
    """Per-channel key smoothing factors calibrated on the calibration sample, float32
    [Hkv][d]: the square root of each channel's largest magnitude (1 for an all-zero channel).
    Like the codebooks, a pre-calibrated input of the quantiser, shared by both sides."""
    lam = np.ones((wl.Hkv, wl.d), np.float32)
    for h in range(wl.Hkv):
        m = np.abs(_calibration_sample(wl, "k", h, wl.n_cal, seed_cal).astype(np.float64)).max(0)
        lam[h] = np.where(m > 0, np.sqrt(m), 1.0)
    return lam


def train_codebooks(wl: Workload, kind: str, S: int | None = None,
                    seed_cal: int = SEED_CALIB, seed_km: int = SEED_KMEANS,
                    smooth: np.ndarray | None = None) -> np.ndarray:
    """Residual k-means codebooks in the Walsh-Hadamard domain, float32 [Hkv][S][256][d].

    Stage s is trained on the calibration residuals left after stages < s; codeword 0 of every
    stage is the zero vector.  ``smooth`` ([Hkv][d] key smoothing factors): the calibration
    vectors are divided by them before the rotation.
    """
    if S is None:
        S = wl.Sk if kind == "k" else wl.Sv
    Hn = scipy.linalg.hadamard(wl.d).astype(np.float64) / np.sqrt(wl.d)
    books = np.zeros((wl.Hkv, S, K_CODEWORDS, wl.d), np.float32)
    for h in range(wl.Hkv):
        X = _calibration_sample(wl, kind, h, wl.n_cal, seed_cal).astype(np.float64)
        if smooth is not None:
            X = X / np.asarray(smooth[h], np.float64)[None, :]
        R = (X @ Hn.T).astype(np.float32)
        krng = _rng(seed_km, 200 + (0 if kind == "k" else 1), h)
        for s in range(S):
            C, a = _kmeans_zero_pinned(R, K_CODEWORDS, wl.kmeans_iters, krng)
            books[h, s] = C
            R = (R - C[a]).astype(np.float32)
    return books


def train_pq_codebook(wl: Workload, kind: str, m: int, seed_cal: int = SEED_CALIB,
                      seed_km: int = SEED_KMEANS, smooth: np.ndarray | None = None) -> np.ndarray:
    """Product-VQ codebooks, float32 [Hkv][256][m]: seeded k-means over every m-dim sub-vector
    of the rotated calibration vectors of a head (the sub-vectors share one codebook);
    ``smooth`` as in train_codebooks."""
    Hn = scipy.linalg.hadamard(wl.d).astype(np.float64) / np.sqrt(wl.d)
    books = np.zeros((wl.Hkv, K_CODEWORDS, m), np.float32)
    for h in range(wl.Hkv):
        X = _calibration_sample(wl, kind, h, wl.n_cal, seed_cal).astype(np.float64)
        if smooth is not None:
            X = X / np.asarray(smooth[h], np.float64)[None, :]
        R = (X @ Hn.T).astype(np.float32).reshape(-1, m)
        krng = _rng(seed_km, 300 + (0 if kind == "k" else 1), h, m)
        books[h], _ = _kmeans_zero_pinned(R, K_CODEWORDS, wl.kmeans_iters, krng)
    return books


# --------------------------------------------------------------------------------------------
# Synthetic code streams for decode-only cases
# --------------------------------------------------------------------------------------------

def code_probabilities(seed: int = SEED_DATA) -> np.ndarray:
    """A skewed distribution over the 256 codewords (permuted Zipf-like), float64 [256].

    Trained codebooks are used unevenly; a skewed draw makes repeated codes within a tile
    common, which exercises the accumulation paths harder than a uniform draw.
    """
    w = 1.0 / (np.arange(K_CODEWORDS) + 8.0) ** 0.9
    w = w[_rng(seed, _TAG_CODE_PROBS).permutation(K_CODEWORDS)]
    return w / w.sum()


def random_codes(wl: Workload, kind: str, Tcap: int, seed: int = SEED_DATA,
                 skewed: bool = True) -> np.ndarray:
    """Codes drawn i.i.d. per (b, head, token, stage), uint8 [B][Hkv][Tcap][S]."""
    S = wl.Sk if kind == "k" else wl.Sv
    tag = _TAG_CODES_K if kind == "k" else _TAG_CODES_V
    rng = _rng(seed, tag)
    shape = (wl.B, wl.Hkv, Tcap, S)
    if skewed:
        p = code_probabilities(seed)
        return rng.choice(K_CODEWORDS, size=shape, p=p).astype(np.uint8)
    return rng.integers(0, K_CODEWORDS, size=shape, dtype=np.uint8)
