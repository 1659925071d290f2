"""GPU parity of the product-VQ (VecInfer) encode against the oracle: codes equal to the
float64 argmin of every sub-vector except counted near-ties (distance gap below 1e-5
relative), with and without key smoothing, every head dimension and several sub-vector sizes.
The file name keeps it after every other GPU test in collection order, so that under
``pytest -x`` a failure here cannot hide the results of the established paths."""
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


@pytest.mark.parametrize("d,m,kind,smooth", [(128, 4, "k", True), (128, 8, "k", False),
                                             (64, 4, "v", False), (256, 2, "k", True),
                                             (128, 16, "v", False)])
def test_pq_encode_matches_oracle(d, m, kind, smooth):
    wl = I.workload("llama3_8b_32k", B=1, Hkv=2, Hq=8, d=d, T=333, n_cal=1024, kmeans_iters=3)
    lam = I.key_smooth_factors(wl) if smooth else None
    books = I.train_pq_codebook(wl, kind, m, smooth=lam)           # [2][256][m]
    x = I.kv_tokens(wl, kind, 0, 0, wl.T)                         # [Hkv][T][d]
    codes = zkv.pq_encode(_cuda(x).permute(1, 0, 2), _cuda(books),
                          smooth=None if lam is None else _cuda(lam))
    codes = codes[0].cpu().numpy()                                # [T, H, d/m]
    assert codes.shape == (wl.T, 2, d // m)
    for h in range(2):
        walk = O.pq_match_walk(x[h], books[h], codes[:, h],
                               smooth=None if lam is None else lam[h])
        assert walk["mismatches"] == 0, walk["bad"]
        assert walk["exceptions"] <= 2


def test_pq_encode_strided_batch_views():
    # [B, T, H, d] views of a larger buffer, fp32 input without rotation
    rng = np.random.default_rng(7)
    big = rng.standard_normal((2, 50, 3, 64 + 8)).astype(np.float32)
    x = _cuda(big)[..., :64]
    C = rng.standard_normal((3, 256, 4)).astype(np.float32)
    codes = zkv.pq_encode(x, _cuda(C), rotate=False).cpu().numpy()
    for b in range(2):
        for h in range(3):
            want, _ = O.pq_encode(big[b, :, h, :64], C[h], rotate=False)
            np.testing.assert_array_equal(codes[b, :, h], want)
