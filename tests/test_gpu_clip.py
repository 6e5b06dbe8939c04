"""Per-segment gradient clipping against the oracle (needs a B200).

dmuon_clip_grad_norm_buckets clips several gradient groups in one pass, each
with its own norm and coefficient (the training guide's fused regular / Muon /
AdamW clipping, "梯度裁剪").  The scaled gradients must equal the oracle's
bit for bit (fl32(g * c) rounded to the storage type), the coefficients too,
and the norms to fp32 rounding of the fp64 norm.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from tests.gpu_helpers import host

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _rand(shape, dtype, seed, std):
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    return (torch.randn(shape, generator=g, device=DEV) * std).to(dtype)


def _check(dm, segments, max_norms):
    before = [[(host(g), g.dtype == torch.bfloat16) for g in seg if g is not None] for seg in segments]
    norms, coefs = dm.dmuon_clip_grad_norm_buckets(segments, max_norms)
    torch.cuda.synchronize()
    assert dm.dmuon_device_status() == 0
    want, wnorms, wcoefs = oracle.clip_grad_norm_buckets(before, max_norms)
    norms, coefs = norms.cpu().numpy(), coefs.cpu().numpy()
    for s, seg in enumerate(segments):
        got = [g for g in seg if g is not None]
        assert coefs[s] == wcoefs[s], (s, coefs[s], wcoefs[s])
        if math.isfinite(wnorms[s]):
            assert abs(float(norms[s]) - wnorms[s]) <= 1e-6 * max(wnorms[s], 1e-30), (s, norms[s], wnorms[s])
        else:
            assert not math.isfinite(float(norms[s]))
        for k, (g, w) in enumerate(zip(got, want[s])):
            h = host(g).reshape(w.shape)
            assert np.array_equal(h.view(np.uint32), w.view(np.uint32)) or \
                np.array_equal(h, w, equal_nan=True), (s, k, g.shape, g.dtype)
    return norms, coefs


def test_three_segments_mixed_dtypes(cuda_lib):
    dm = cuda_lib
    regular = [_rand((127, 513), torch.bfloat16, 1, 1e-2), _rand((4096,), torch.float32, 2, 1e-2),
               _rand((1000003,), torch.bfloat16, 3, 1e-3)]
    muon = [_rand((1024, 4096), torch.bfloat16, 4, 1e-3), _rand((4096, 1024), torch.bfloat16, 5, 1e-3),
            _rand((300, 77), torch.float32, 6, 1e-1)]
    adamw = [_rand((32000, 256), torch.bfloat16, 7, 1e-4), _rand((17,), torch.float32, 8, 1e-4)]
    # regular and Muon are clipped, AdamW is below its bound and stays as it is
    adamw0 = [a.clone() for a in adamw]
    norms, coefs = _check(dm, [regular, muon, adamw], [0.5, 1.0, 10.0])
    assert coefs[0] < 1.0 and coefs[1] < 1.0 and coefs[2] == 1.0
    for a, b in zip(adamw, adamw0):
        assert torch.equal(a, b)


def test_unaligned_views_and_skipped_tensors(cuda_lib):
    dm = cuda_lib
    base_b = _rand((70001,), torch.bfloat16, 11, 1.0)
    base_f = _rand((50003,), torch.float32, 12, 1.0)
    seg0 = [base_b[1:], None, base_f[3:]]          # 2- and 4-byte aligned starts: scalar path
    seg1 = [_rand((8, 8), torch.bfloat16, 13, 3.0)]
    _check(dm, [seg0, seg1], [7.5, 2.0])


def test_many_tensors_span_several_launches(cuda_lib):
    dm = cuda_lib
    segs = [[], [], []]
    for i in range(700):                           # more than 512 tensors per launch
        shape = (int(37 + 13 * (i % 29)),) if i % 3 else (int(5 + i % 7), 129)
        dt = torch.bfloat16 if i % 2 else torch.float32
        segs[i % 3].append(_rand(shape, dt, 100 + i, 1e-2 * (1 + i % 5)))
    _check(dm, segs, [0.1, 0.2, 1e3])


def test_infinite_bound_empty_segment_and_nan(cuda_lib):
    dm = cuda_lib
    a = _rand((4096, 33), torch.bfloat16, 21, 1.0)
    b = _rand((513,), torch.float32, 22, 1.0)
    b[7] = float("nan")
    c = _rand((999,), torch.bfloat16, 23, 1.0)
    a0, b0 = a.clone(), b.clone()
    norms, coefs = _check(dm, [[a], [b], [], [c]], [math.inf, 1.0, 1.0, 0.25])
    assert torch.equal(a, a0) and math.isfinite(float(norms[0])) and coefs[0] == 1.0
    assert math.isnan(float(norms[1])) and coefs[1] == 1.0 and torch.equal(b[:7], b0[:7])
    assert norms[2] == 0.0 and coefs[2] == 1.0
    assert coefs[3] < 1.0


def test_deterministic(cuda_lib):
    dm = cuda_lib
    x1 = [_rand((2048, 2048), torch.bfloat16, 31, 1.0), _rand((12345,), torch.float32, 32, 1.0)]
    x2 = [t.clone() for t in x1]
    n1, c1 = dm.dmuon_clip_grad_norm_buckets([x1], [3.0])
    n2, c2 = dm.dmuon_clip_grad_norm_buckets([x2], [3.0])
    torch.cuda.synchronize()
    assert torch.equal(n1, n2) and torch.equal(c1, c2)
    for a, b in zip(x1, x2):
        assert torch.equal(a, b)


def test_caller_workspace(cuda_lib):
    dm = cuda_lib
    seg = [_rand((3000, 700), torch.bfloat16, 41, 1.0)]
    need = dm.dmuon_clip_workspace_bytes([seg])
    ws = torch.full((need,), 0xAB, dtype=torch.uint8, device=DEV)
    ref = [seg[0].clone()]
    dm.dmuon_clip_grad_norm_buckets([ref], [5.0])
    dm.dmuon_clip_grad_norm_buckets([seg], [5.0], workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(seg[0], ref[0])
    with pytest.raises(dm.DmuonError):
        dm.dmuon_clip_grad_norm_buckets([seg], [5.0], workspace=ws[: need - 256])
