"""The size limits (needs a B200), checked against closed forms because the
fp64 oracle cannot run at these sizes in reasonable time.

* min(rows, cols) = DMUON_MAX_M = 32768: a Hadamard matrix H (entries +-1)
  has all singular values equal, so Newton-Schulz maps it to
  f^k(s0) H / sqrt(m) with s0 = sqrt(m) / (m + 1e-7) (the scalar map of the
  equal singular values; f(s) = 1.5 s - 0.5 s^3).
* max(rows, cols) = DMUON_MAX_N = 2^24, a tall 2^24 x 64 matrix of 2^30
  elements through a whole Muon step.  Each block of 64 rows is a 64 x 64
  Hadamard matrix times its own scale a_b, so the 64 columns are orthogonal
  with equal norm sigma = sqrt(64 sum a_b^2) and the orthogonalised update is
  f^k(1/8) G / sigma in real arithmetic; with zero weights and buffers the
  new weights are -lr f^k(1/8) G / sigma and the new buffers are G, bit for
  bit.  (The block scales vary the 2^24 products that the Gram diagonal sums
  in one fp32 accumulator: with identical products that sum rounds the same
  way nearly every time and drifts by about 2 %, a property of the fp32
  accumulator at this length, not of the method.)
"""
import math

import pytest
import torch

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _cubic(s, k):
    for _ in range(k):
        s = 1.5 * s - 0.5 * s ** 3
    return s


def _hadamard_sign(rows, cols, dtype):
    """(-1)^popcount(i & j) on the GPU."""
    i = torch.arange(rows, device=DEV, dtype=torch.int32)[:, None]
    j = torch.arange(cols, device=DEV, dtype=torch.int32)[None, :]
    x = i & j
    for sh in (16, 8, 4, 2, 1):
        x = x ^ (x >> sh)
    return (1 - 2 * (x & 1)).to(dtype)


def test_max_min_side_hadamard(cuda_lib):
    dm = cuda_lib
    m = 32768
    H = _hadamard_sign(m, m, torch.bfloat16)
    X = H.clone()
    dm.dmuon_ns_orthogonalize(X, 5)
    torch.cuda.synchronize()
    assert dm.dmuon_device_status() == 0
    s0 = math.sqrt(m) / (m + 1e-7)
    c = _cubic(s0, 5) / math.sqrt(m)
    # relative Frobenius error against c * H, computed on the GPU in fp64 by row blocks
    num = den = 0.0
    for r in range(0, m, 4096):
        Xb = X[r:r + 4096].double()
        Yb = c * H[r:r + 4096].double()
        num += float(((Xb - Yb) ** 2).sum())
        den += float((Yb ** 2).sum())
    rel = math.sqrt(num / den)
    assert rel <= 2e-2, rel
    del H, X
    torch.cuda.empty_cache()


def test_max_long_side_tall_step(cuda_lib):
    dm = cuda_lib
    rows, cols = 1 << 24, 64
    H64 = _hadamard_sign(cols, cols, torch.float32)
    blocks = rows // cols
    b = torch.arange(blocks, device=DEV, dtype=torch.int64)
    a = (0.5 + ((b * 2654435761) % 256).float() / 256.0)             # exact in bf16: 8-bit mantissas
    G = (H64.repeat(blocks, 1) * a.repeat_interleave(cols)[:, None]).to(torch.bfloat16)
    sigma = math.sqrt(cols * float((a.double() ** 2).sum()))
    W = torch.zeros(rows, cols, dtype=torch.bfloat16, device=DEV)
    B = torch.zeros(rows, cols, dtype=torch.float32, device=DEV)
    lr = 1.0
    dm.dmuon_muon_step_batched([W], [G], [B], lr=lr, momentum=0.95, nesterov=True, weight_decay=0.0,
                               ns_steps=5)
    torch.cuda.synchronize()
    assert dm.dmuon_device_status() == 0
    assert torch.equal(B, G.float())                      # buf = 0.95 * 0 + g, bit for bit
    c = -lr * _cubic(1.0 / 8.0, 5) / sigma
    num = den = 0.0
    for r in range(0, rows, 1 << 21):
        Wb = W[r:r + (1 << 21)].double()
        Yb = c * G[r:r + (1 << 21)].double()
        num += float(((Wb - Yb) ** 2).sum())
        den += float((Yb ** 2).sum())
    rel = math.sqrt(num / den)
    assert rel <= 2e-2, rel
    # blocks with the same scale carry the same values
    same = int(torch.nonzero(a[1:] == a[0])[0]) + 1
    assert torch.equal(W[:64], W[64 * same:64 * same + 64])
    del G, W, B
    torch.cuda.empty_cache()
