"""CPU oracle for RVQ KV-cache encode and compressed decode attention.

TEST INFRASTRUCTURE.  Only the test suite, the package smoke check and the benchmark's CPU
baseline arm may import or run this module.  The CUDA library and its binding never do, and
this module imports nothing from them: the only code both sides share is the seeded input
generator module, which holds no arithmetic of the method.

Plain and slow on purpose: numpy, float64 wherever the pages do not fix a precision, and no
blocking, fusion or reordering beyond what each definition states.  Sources (web pages):

* "VQKV: High-Fidelity and High-Ratio Cache Compression via Vector-Quantization" (gist.science
  summary of arXiv 2603.16435), section 2.1 "Residual Simple Vector Quantization": greedy
  residual stages ("Process" steps 1-4) and reconstruction x_hat = sum_i Q_i[z_i]; section 2.3
  "Inference Integration": codes stored at prefill, on-demand reconstruction inside attention
  at decode, a local window of recent tokens kept uncompressed.
* "zerokv-neo 4.0.0" (pypi), "Architecture": FWHT energy spreading before quantisation; hot
  tier of recent tokens kept in FP16.
* "VeloxQuant-MLX 0.5.1" (pypi), "VecInfer": Walsh-Hadamard rotation whose inverse is absorbed
  into the query, q_tilde . K_tilde^T == q . K^T; the optional per-channel smooth scaling of the
  keys before the rotation, lambda_i = sqrt(max |K_i|), also absorbed into the query.
* "Differential-KV" (GitHub README), "Decode & Prefill Innovations": flash-style fp32
  log-sum-exp combine of the compressed part with a dense recency window.

Readings where the pages are silent (each is also listed in the design notes):

* Rotation: Sylvester-ordered Hadamard H_d (H[i, j] = (-1)^popcount(i & j)), no random signs,
  scaled by 1/sqrt(d) inside encode/decode (orthonormal and self-inverse).  The rotated vector
  the quantiser works on is float32: the exact product s * (H x) rounded once to float32.
* Greedy stage decision: squared L2 distance evaluated in float64, ties to the lowest index.
  The residual update r <- r - C_s[z_s] is an elementwise float32 subtraction.
* Residual norm n_s = ||r|| after stage s (float64 accumulate, stored float32).
* Product VQ (VecInfer): the rotated (keys: smoothed, then rotated) float32 vector is cut into
  d/m consecutive sub-vectors of m dims; one 256-entry codebook [256][m] per kv head and K or V
  is shared by every sub-vector; each sub-vector takes the nearest codeword (float64 distance,
  lowest index on ties).  Values are rotated, not smoothed.
* Smooth scaling (keys only): the key is multiplied by 1/lambda channel by channel in float64
  (1/lambda itself a float64 division of the float32 factor) before the rotation; the query is
  multiplied by lambda.  A channel that is zero on every calibration token gets lambda = 1.
* Attention: scores = softmax_scale * q . k with softmax_scale defaulting to 1/sqrt(d); the
  first T_c tokens of a sequence are compressed, the window holds the newest ones (order inside
  the window is irrelevant); GQA maps query head h to kv head h // (Hq // Hkv); lse is the
  natural-log log-sum-exp of the scores; an empty part contributes nothing (lse = -inf) and an
  entirely empty context gives out = 0, lse = -inf.
"""
from __future__ import annotations

import numpy as np

F64 = np.float64
F32 = np.float32


# --------------------------------------------------------------------------------------------
# Walsh-Hadamard rotation  (zerokv-neo "Architecture": FWHT; VeloxQuant "VecInfer")
# --------------------------------------------------------------------------------------------

def hadamard(d: int) -> np.ndarray:
    """Sylvester Hadamard matrix of order d (a power of two), entries +-1, float64.

    H[i, j] = (-1)^(number of set bits of i AND j).
    """
    if d < 1 or d & (d - 1):
        raise ValueError("d must be a power of two")
    i = np.arange(d, dtype=np.int64)
    a = np.bitwise_and.outer(i, i)
    parity = np.zeros_like(a)
    while np.any(a):
        parity ^= a & 1
        a >>= 1
    return np.where(parity == 0, 1.0, -1.0).astype(F64)


def fwht(x: np.ndarray, scale: float) -> np.ndarray:
    """y = scale * H_d x for every row of x, float64 (exact products of +-1, then one scale).

    For fp16 inputs every partial sum of H x is exactly representable in float64, so the
    result is the exact transform times ``scale`` rounded once.
    """
    x = np.asarray(x, dtype=F64)
    H = hadamard(x.shape[-1])
    return (x @ H.T) * F64(scale)


def rotate_to_f32(x: np.ndarray) -> np.ndarray:
    """The quantiser's working vector: (1/sqrt(d)) H x rounded once to float32."""
    d = np.asarray(x).shape[-1]
    return fwht(x, 1.0 / np.sqrt(F64(d))).astype(F32)


# --------------------------------------------------------------------------------------------
# Smooth scaling  (VeloxQuant "VecInfer": per-channel lambda_i = sqrt(max |K_i|) before the
# Walsh-Hadamard rotation, inverse absorbed into the query)
# --------------------------------------------------------------------------------------------

def smooth_factors(K: np.ndarray) -> np.ndarray:
    """lambda_i = sqrt(max_t |K[t, i]|) over calibration keys K [n][d] of one kv head, as
    float32; 1 for a channel that is zero on every token."""
    m = np.abs(np.asarray(K, F64)).max(axis=0)
    lam = np.sqrt(m)
    return np.where(m > 0, lam, 1.0).astype(F32)


def smooth_keys(x: np.ndarray, lam: np.ndarray) -> np.ndarray:
    """x / lambda per channel: float64(x) times the float64 reciprocal of the float32 factor."""
    inv = F64(1.0) / np.asarray(lam, F32).astype(F64)
    return np.asarray(x, F64) * inv


# --------------------------------------------------------------------------------------------
# Greedy residual vector quantisation  (VQKV section 2.1, "Process" and "Reconstruction")
# --------------------------------------------------------------------------------------------

def stage_distances(r: np.ndarray, C: np.ndarray, chunk: int = 256) -> np.ndarray:
    """D[n, c] = sum_i (r[n, i] - C[c, i])^2 in float64 for float32 residuals and codewords."""
    r = np.asarray(r, F64)
    C = np.asarray(C, F64)
    D = np.empty((r.shape[0], C.shape[0]), F64)
    for a in range(0, r.shape[0], chunk):
        diff = r[a:a + chunk, None, :] - C[None, :, :]
        D[a:a + chunk] = (diff * diff).sum(axis=2)
    return D


def rvq_encode(x: np.ndarray, codebooks: np.ndarray, rotate: bool = True, smooth=None):
    """Greedy RVQ of rows of x against stage codebooks [S][K][d] (float32, rotated domain).

    Step 1: y = rotate(x) (or x as float32 when ``rotate`` is False); with ``smooth`` (the
    head's lambda [d]) the rows are first divided by lambda channel by channel.
    For each stage s: z_s = argmin_c ||r - C_s[c]||^2 (lowest index on ties),
    r <- r - C_s[z_s] (float32), n_s = ||r||.
    Returns (codes uint8 [n][S], norms float32 [n][S], y float32 [n][d], r_final float32).
    """
    x = np.asarray(x)
    if smooth is not None:
        x = smooth_keys(x, smooth)
    y = rotate_to_f32(x) if rotate else np.asarray(x, F32)
    S = codebooks.shape[0]
    n = y.shape[0]
    codes = np.empty((n, S), np.uint8)
    norms = np.empty((n, S), F32)
    r = y.copy()
    for s in range(S):
        C = np.asarray(codebooks[s], F32)
        D = stage_distances(r, C)
        z = np.argmin(D, axis=1)            # first index of the minimum = lowest on ties
        codes[:, s] = z
        r = (r - C[z]).astype(F32)
        norms[:, s] = np.sqrt((r.astype(F64) ** 2).sum(axis=1)).astype(F32)
    return codes, norms, y, r


def rvq_match_walk(x: np.ndarray, codebooks: np.ndarray, codes: np.ndarray,
                   rel_gap: float = 1e-5, rotate: bool = True, smooth=None) -> dict:
    """Check candidate codes against the greedy rule, stage by stage.

    At each stage the oracle's float64 distances of the current residual are computed.  A
    candidate code equal to the oracle's argmin matches.  A different code whose distance
    exceeds the minimum by less than ``rel_gap`` relative is a counted near-tie exception.
    Anything else is a mismatch.  The walk continues along the candidate's codes, so one
    near-tie does not cascade into later stages.
    Returns counts and the first few mismatches (row, stage, candidate, oracle, rel gap).
    ``smooth``: as in rvq_encode.
    """
    x = np.asarray(x)
    if smooth is not None:
        x = smooth_keys(x, smooth)
    y = rotate_to_f32(x) if rotate else np.asarray(x, F32)
    S = codebooks.shape[0]
    r = y.copy()
    exact = exceptions = mismatches = 0
    bad = []
    rows = np.arange(y.shape[0])
    for s in range(S):
        C = np.asarray(codebooks[s], F32)
        D = stage_distances(r, C)
        best = np.argmin(D, axis=1)
        z = codes[:, s].astype(np.int64)
        dz = D[rows, z]
        db = D[rows, best]
        same = z == best
        near = (~same) & ((dz - db) <= rel_gap * db)
        wrong = (~same) & (~near)
        exact += int(same.sum())
        exceptions += int(near.sum())
        mismatches += int(wrong.sum())
        for i in np.nonzero(wrong)[0][:8]:
            gap = (dz[i] - db[i]) / db[i] if db[i] > 0 else np.inf
            bad.append((int(i), s, int(z[i]), int(best[i]), float(gap)))
        r = (r - C[z]).astype(F32)
    return {"exact": exact, "exceptions": exceptions, "mismatches": mismatches, "bad": bad}


def reconstruct(codes: np.ndarray, codebooks: np.ndarray, unrotate: bool = False) -> np.ndarray:
    """x_hat = sum_s C_s[z_s] (float64) in the rotated domain, or (1/sqrt(d)) H x_hat."""
    codes = np.asarray(codes)
    xh = np.zeros(codes.shape[:-1] + (codebooks.shape[-1],), F64)
    for s in range(codes.shape[-1]):
        xh += np.asarray(codebooks[s], F64)[codes[..., s].astype(np.int64)]
    if unrotate:
        xh = fwht(xh, 1.0 / np.sqrt(F64(codebooks.shape[-1])))
    return xh


def exhaustive_rvq(y: np.ndarray, codebooks: np.ndarray):
    """Brute force over all K^S stage combinations for ONE vector (tiny inputs only).

    Returns (best combination by total distortion ||y - sum_s C_s[z_s]||^2 with ties to the
    lexicographically smallest tuple, its distortion, and the dict of every combination's
    distortion).
    """
    import itertools
    y = np.asarray(y, F64)
    S, K, _ = codebooks.shape
    table = {}
    best, best_d = None, np.inf
    for combo in itertools.product(range(K), repeat=S):
        xh = sum(np.asarray(codebooks[s, combo[s]], F64) for s in range(S))
        dist = float(((y - xh) ** 2).sum())
        table[combo] = dist
        if dist < best_d:
            best, best_d = combo, dist
    return best, best_d, table


# --------------------------------------------------------------------------------------------
# Decode attention  (VQKV section 2.3; Differential-KV "Flash-Style LSE Combine")
# --------------------------------------------------------------------------------------------

def softmax_attention(q: np.ndarray, K: np.ndarray, V: np.ndarray, scale: float):
    """Exact single-query softmax attention in float64.

    Returns (out [d], lse) with lse = log sum_t exp(scale q.k_t); an empty key set gives
    (zeros, -inf).
    """
    q = np.asarray(q, F64)
    K = np.asarray(K, F64)
    V = np.asarray(V, F64)
    if K.shape[0] == 0:
        return np.zeros(V.shape[-1] if V.ndim == 2 else q.shape[-1], F64), -np.inf
    s = F64(scale) * (K @ q)
    m = s.max()
    p = np.exp(s - m)
    l = p.sum()
    return (p @ V) / l, m + np.log(l)


def lse_merge(parts):
    """Combine partial attentions [(out_i, lse_i)] over disjoint key sets.

    lse = M + log sum_i exp(lse_i - M) with M = max_i lse_i; out = sum_i exp(lse_i - lse) out_i.
    Parts with lse = -inf carry no weight; if all are -inf the result is (0, -inf).
    """
    lses = np.array([p[1] for p in parts], F64)
    d = len(parts[0][0])
    if np.all(np.isneginf(lses)):
        return np.zeros(d, F64), -np.inf
    M = lses.max()
    w = np.exp(lses - M)
    lse = M + np.log(w.sum())
    out = np.zeros(d, F64)
    for (o, li) in parts:
        if not np.isneginf(li):
            out += np.exp(li - lse) * np.asarray(o, F64)
    return out, lse


def _check_decode_shapes(q, k_codes, v_codes, Ck, Cv, win_k, win_v):
    B, Hq, d = q.shape
    Hkv = k_codes.shape[1]
    assert Hq % Hkv == 0
    assert Ck.shape[0] == Hkv and Cv.shape[0] == Hkv
    assert win_k.shape[:2] == (B, Hkv) and win_v.shape[:2] == (B, Hkv)
    return B, Hq, Hkv, d


def decode_attn(q, k_codes, v_codes, comp_len, Ck, Cv, win_k, win_v, win_len,
                scale: float | None = None, pairs=None, k_smooth=None):
    """Decode-step attention over a compressed prefix plus an fp16 window (direct form).

    q [B][Hq][d] fp16; k_codes [B][Hkv][Tcap][Sk] / v_codes [B][Hkv][Tcap][Sv] uint8;
    comp_len [B]; Ck [Hkv][Sk][K][d] / Cv [Hkv][Sv][K][d] float32 (rotated domain);
    win_k / win_v [B][Hkv][Wcap][d] fp16 with the first win_len[b] slots valid.

    For every (b, h): the compressed keys and values are reconstructed and rotated back,
    k_t = (1/sqrt(d)) H sum_s Ck_s[zk_{t,s}] (likewise v), joined with the window tokens, and
    exact softmax attention of q over that set is taken in float64.  With ``k_smooth``
    ([Hkv][d] lambda) the compressed keys were smoothed before encoding, so the reconstructed
    key is lambda * k_t (the window keys are raw).
    Returns (out float64 [B][Hq][d], lse float64 [B][Hq]); ``pairs`` restricts to a list of
    (b, h) (other entries are NaN).
    """
    B, Hq, Hkv, d = _check_decode_shapes(q, k_codes, v_codes, Ck, Cv, win_k, win_v)
    G = Hq // Hkv
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    out = np.full((B, Hq, d), np.nan, F64)
    lse = np.full((B, Hq), np.nan, F64)
    if pairs is None:
        pairs = [(b, h) for b in range(B) for h in range(Hq)]
    cache = {}
    for b, h in pairs:
        kvh = h // G
        if (b, kvh) not in cache:
            tc = int(comp_len[b])
            wl = int(win_len[b])
            kh = reconstruct(k_codes[b, kvh, :tc], Ck[kvh], unrotate=True)
            if k_smooth is not None:
                kh = kh * np.asarray(k_smooth[kvh], F32).astype(F64)
            vh = reconstruct(v_codes[b, kvh, :tc], Cv[kvh], unrotate=True)
            Kall = np.concatenate([kh, np.asarray(win_k[b, kvh, :wl], F64)], axis=0)
            Vall = np.concatenate([vh, np.asarray(win_v[b, kvh, :wl], F64)], axis=0)
            cache[(b, kvh)] = (Kall, Vall)
        Kall, Vall = cache[(b, kvh)]
        o, l = softmax_attention(np.asarray(q[b, h], F64), Kall, Vall, scale)
        out[b, h] = o
        lse[b, h] = l
    return out, lse


def decode_attn_lut(q, k_codes, v_codes, comp_len, Ck, Cv, win_k, win_v, win_len,
                    scale: float | None = None, pairs=None, k_smooth=None):
    """The same attention computed the way the method reads codes (second, independent path).

    Compressed part, in the rotated domain: q_tilde = (1/sqrt(d)) H q;
    LUT_s[c] = scale * q_tilde . Ck_s[c]; score_t = sum_s LUT_s[zk_{t,s}];
    o_tilde = sum_t softmax(score)_t sum_s Cv_s[zv_{t,s}], rotated back by (1/sqrt(d)) H.
    Window part: plain attention of q over the fp16 window.  The two parts are joined by the
    log-sum-exp combine.  Equality with ``decode_attn`` pins the rotation absorption
    (q_tilde . k_tilde = q . k) and the combine.  With ``k_smooth`` the query of the
    compressed part is q_tilde = (1/sqrt(d)) H (lambda * q).
    """
    B, Hq, Hkv, d = _check_decode_shapes(q, k_codes, v_codes, Ck, Cv, win_k, win_v)
    G = Hq // Hkv
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    out = np.full((B, Hq, d), np.nan, F64)
    lse = np.full((B, Hq), np.nan, F64)
    if pairs is None:
        pairs = [(b, h) for b in range(B) for h in range(Hq)]
    for b, h in pairs:
        kvh = h // G
        tc = int(comp_len[b])
        wl = int(win_len[b])
        qs = np.asarray(q[b, h], F64)
        if k_smooth is not None:
            qs = qs * np.asarray(k_smooth[kvh], F32).astype(F64)
        qt = fwht(qs, 1.0 / np.sqrt(F64(d)))
        parts = []
        if tc > 0:
            zk = k_codes[b, kvh, :tc].astype(np.int64)
            zv = v_codes[b, kvh, :tc].astype(np.int64)
            score = np.zeros(tc, F64)
            for s in range(zk.shape[1]):
                lut = F64(scale) * (np.asarray(Ck[kvh, s], F64) @ qt)
                score += lut[zk[:, s]]
            m = score.max()
            p = np.exp(score - m)
            vt = np.zeros((tc, d), F64)
            for s in range(zv.shape[1]):
                vt += np.asarray(Cv[kvh, s], F64)[zv[:, s]]
            ot = (p @ vt) / p.sum()
            parts.append((fwht(ot, 1.0 / np.sqrt(F64(d))), m + np.log(p.sum())))
        else:
            parts.append((np.zeros(d, F64), -np.inf))
        parts.append(softmax_attention(np.asarray(q[b, h], F64),
                                       np.asarray(win_k[b, kvh, :wl], F64),
                                       np.asarray(win_v[b, kvh, :wl], F64), scale))
        o, l = lse_merge(parts)
        out[b, h] = o
        lse[b, h] = l
    return out, lse


# --------------------------------------------------------------------------------------------
# Product vector quantisation  (VeloxQuant "VecInfer": smooth scaling + Walsh-Hadamard dual
# transform, then a K-means codebook over sub-vectors; key_sub_dim = 4 gives 2 bits/elem,
# 8 gives 1 bit/elem with 8-bit codes)
# --------------------------------------------------------------------------------------------

def pq_encode(x: np.ndarray, codebook: np.ndarray, smooth=None, rotate: bool = True):
    """Product VQ of rows of x [n][d] against one codebook [K][m] shared by the d/m sub-vectors.

    y = rotate(x / lambda) (or rotate(x); or x as float32 when ``rotate`` is False), cut into
    y_j = y[j m : (j+1) m]; z_j = argmin_c ||y_j - C[c]||^2 (float64, lowest index on ties).
    Returns (codes uint8 [n][d/m], y float32 [n][d]).
    """
    x = np.asarray(x)
    if smooth is not None:
        x = smooth_keys(x, smooth)
    y = rotate_to_f32(x) if rotate else np.asarray(x, F32)
    C = np.asarray(codebook, F32)
    m = C.shape[1]
    n, d = y.shape
    assert d % m == 0
    sub = y.reshape(n * (d // m), m)
    z = np.argmin(stage_distances(sub, C), axis=1)
    return z.reshape(n, d // m).astype(np.uint8), y


def pq_match_walk(x: np.ndarray, codebook: np.ndarray, codes: np.ndarray, rel_gap: float = 1e-5,
                  smooth=None, rotate: bool = True) -> dict:
    """Check candidate product-VQ codes sub-vector by sub-vector: equal to the float64 argmin,
    or a counted near-tie (distance within ``rel_gap`` relative of the minimum), else a
    mismatch.  Returns counts and the first few mismatches (row, sub-vector, code, oracle)."""
    z, y = pq_encode(x, codebook, smooth=smooth, rotate=rotate)
    C = np.asarray(codebook, F32)
    m = C.shape[1]
    sub = y.reshape(-1, m)
    D = stage_distances(sub, C)
    cand = np.asarray(codes).reshape(-1).astype(np.int64)
    rows = np.arange(sub.shape[0])
    dz, db = D[rows, cand], D[rows, z.reshape(-1).astype(np.int64)]
    same = cand == z.reshape(-1)
    near = (~same) & ((dz - db) <= rel_gap * db)
    wrong = (~same) & (~near)
    bad = [(int(i) // (y.shape[1] // m), int(i) % (y.shape[1] // m), int(cand[i]),
            int(z.reshape(-1)[i])) for i in np.nonzero(wrong)[0][:8]]
    return {"exact": int(same.sum()), "exceptions": int(near.sum()),
            "mismatches": int(wrong.sum()), "bad": bad}


def pq_reconstruct(codes: np.ndarray, codebook: np.ndarray, unrotate: bool = False) -> np.ndarray:
    """y_hat = concatenation of C[z_j] over the sub-vectors (float64), or (1/sqrt(d)) H y_hat."""
    C = np.asarray(codebook, F64)
    codes = np.asarray(codes).astype(np.int64)
    y = C[codes].reshape(codes.shape[:-1] + (codes.shape[-1] * C.shape[1],))
    if unrotate:
        y = fwht(y, 1.0 / np.sqrt(F64(y.shape[-1])))
    return y


def pq_decode_attn(q, k_codes, v_codes, comp_len, Ck, Cv, win_k, win_v, win_len,
                   scale: float | None = None, pairs=None, k_smooth=None):
    """decode_attn for product-VQ codes (direct form): k_codes / v_codes [B][Hkv][Tcap][d/m]
    uint8, Ck / Cv [Hkv][K][m].  Keys are reconstructed, rotated back and multiplied by lambda
    (with ``k_smooth``), values reconstructed and rotated back, then exact softmax attention
    over them and the fp16 window in float64."""
    B, Hq, d = q.shape
    Hkv = k_codes.shape[1]
    G = Hq // Hkv
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    out = np.full((B, Hq, d), np.nan, F64)
    lse = np.full((B, Hq), np.nan, F64)
    if pairs is None:
        pairs = [(b, h) for b in range(B) for h in range(Hq)]
    cache = {}
    for b, h in pairs:
        kvh = h // G
        if (b, kvh) not in cache:
            tc, wl = int(comp_len[b]), int(win_len[b])
            kh = pq_reconstruct(k_codes[b, kvh, :tc], Ck[kvh], unrotate=True)
            if k_smooth is not None:
                kh = kh * np.asarray(k_smooth[kvh], F32).astype(F64)
            vh = pq_reconstruct(v_codes[b, kvh, :tc], Cv[kvh], unrotate=True)
            cache[(b, kvh)] = (np.concatenate([kh, np.asarray(win_k[b, kvh, :wl], F64)]),
                               np.concatenate([vh, np.asarray(win_v[b, kvh, :wl], F64)]))
        Kall, Vall = cache[(b, kvh)]
        out[b, h], lse[b, h] = softmax_attention(np.asarray(q[b, h], F64), Kall, Vall, scale)
    return out, lse


def pq_decode_attn_lut(q, k_codes, v_codes, comp_len, Ck, Cv, win_k, win_v, win_len,
                       scale: float | None = None, pairs=None, k_smooth=None):
    """The same attention the way the method reads product-VQ codes: q_tilde = (1/sqrt(d))
    H (lambda q); per sub-vector j a table LUT_j[c] = scale * q_tilde_j . Ck[c]; score_t =
    sum_j LUT_j[zk_{t,j}]; the values as per-sub-vector codeword weights W_j[c] (sum of p over
    tokens with zv_{t,j} = c), o_tilde_j = sum_c W_j[c] Cv[c] / sum p, rotated back; joined with
    the window by the log-sum-exp combine."""
    B, Hq, d = q.shape
    Hkv = k_codes.shape[1]
    G = Hq // Hkv
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    out = np.full((B, Hq, d), np.nan, F64)
    lse = np.full((B, Hq), np.nan, F64)
    if pairs is None:
        pairs = [(b, h) for b in range(B) for h in range(Hq)]
    for b, h in pairs:
        kvh = h // G
        tc, wl = int(comp_len[b]), int(win_len[b])
        CK = np.asarray(Ck[kvh], F64)
        CV = np.asarray(Cv[kvh], F64)
        m = CK.shape[1]
        qs = np.asarray(q[b, h], F64)
        if k_smooth is not None:
            qs = qs * np.asarray(k_smooth[kvh], F32).astype(F64)
        qt = fwht(qs, 1.0 / np.sqrt(F64(d)))
        parts = []
        if tc > 0:
            zk = k_codes[b, kvh, :tc].astype(np.int64)
            zv = v_codes[b, kvh, :tc].astype(np.int64)
            score = np.zeros(tc, F64)
            for j in range(d // m):
                lut = F64(scale) * (CK @ qt[j * m:(j + 1) * m])
                score += lut[zk[:, j]]
            mx = score.max()
            p = np.exp(score - mx)
            ot = np.zeros(d, F64)
            for j in range(d // m):
                W = np.bincount(zv[:, j], weights=p, minlength=CV.shape[0])
                ot[j * m:(j + 1) * m] = W @ CV
            ot /= p.sum()
            parts.append((fwht(ot, 1.0 / np.sqrt(F64(d))), mx + np.log(p.sum())))
        else:
            parts.append((np.zeros(d, F64), -np.inf))
        parts.append(softmax_attention(np.asarray(q[b, h], F64), np.asarray(win_k[b, kvh, :wl], F64),
                                       np.asarray(win_v[b, kvh, :wl], F64), scale))
        out[b, h], lse[b, h] = lse_merge(parts)
    return out, lse


# --------------------------------------------------------------------------------------------
# Serving step  (VQKV section 2.3 "Local Sliding Window"; VeloxQuant append / attend)
# --------------------------------------------------------------------------------------------

def append_step(state: dict, new_k: np.ndarray, new_v: np.ndarray, pq: bool = False) -> dict:
    """One token per sequence enters the window; when the window is full its oldest token
    leaves it and is RVQ-encoded (product-VQ encoded with ``pq``: codes [d/m] per token,
    codebooks [Hkv][K][m]) onto the end of the compressed prefix.

    state: k_codes, v_codes [B][Hkv][Tcap][S] uint8; comp_len [B]; win_k, win_v
    [B][Hkv][Wcap][d] fp16; win_len [B]; win_head [B] (slot of the oldest token once the window
    is full); Ck, Cv codebooks; optional k_smooth [Hkv][d] (evicted keys are smoothed before
    encoding).  new_k / new_v: [B][Hkv][d] fp16.
    While win_len < Wcap the token goes to slot win_len.  Otherwise slot win_head is evicted
    (its key and value are encoded to position comp_len), overwritten, and win_head advances.
    If an eviction is due while comp_len == Tcap, that sequence is left unchanged and the
    returned state's "error" entry is set to True (the prefix has no room).
    Returns a new state dict (inputs are not modified).
    """
    st = {k: (np.array(v, copy=True) if isinstance(v, np.ndarray) else v) for k, v in state.items()}
    st["error"] = bool(state.get("error", False))
    B, Hkv, Wcap, d = st["win_k"].shape
    Tcap = st["k_codes"].shape[2]
    for b in range(B):
        wl = int(st["win_len"][b])
        if wl < Wcap:
            slot = wl
            st["win_len"][b] = wl + 1
        else:
            slot = int(st["win_head"][b])
            pos = int(st["comp_len"][b])
            if pos >= Tcap:
                st["error"] = True
                continue
            for h in range(Hkv):
                ks = st.get("k_smooth")
                lam = None if ks is None else ks[h]
                if pq:
                    zk, _ = pq_encode(st["win_k"][b, h, slot][None], st["Ck"][h], smooth=lam)
                    zv, _ = pq_encode(st["win_v"][b, h, slot][None], st["Cv"][h])
                else:
                    zk, _, _, _ = rvq_encode(st["win_k"][b, h, slot][None], st["Ck"][h],
                                             smooth=lam)
                    zv, _, _, _ = rvq_encode(st["win_v"][b, h, slot][None], st["Cv"][h])
                st["k_codes"][b, h, pos] = zk[0]
                st["v_codes"][b, h, pos] = zv[0]
            st["comp_len"][b] = pos + 1
            st["win_head"][b] = (slot + 1) % Wcap
        st["win_k"][b, :, slot] = new_k[b]
        st["win_v"][b, :, slot] = new_v[b]
    return st
