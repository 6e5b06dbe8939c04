"""The bf16 prologue's input paths against the fp64 oracle (needs a B200).

Whole, 16-byte aligned work items reach the prologue through shared memory:
bulk copies for wide matrices, 2-D tensor loads through per-matrix tensor
maps for tall ones.  Items at a ragged edge, and every item of a matrix whose
gradient or momentum rows are not 16-byte aligned, are read from global
memory directly.  These tests drive each path, and the tensor maps' addresses
as the caller's tensors move between calls (aligned -> unaligned -> aligned),
and check the momentum buffers bit for bit and the weights within one bf16 ulp.
"""
import numpy as np
import pytest
import torch

from tests.gpu_helpers import check_bf16_weights, host, oracle_step

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
# tall (transposed items: whole, ragged bottom, ragged right, cols % 8 != 0) and wide shapes
SHAPES = [(1000, 256), (600, 136), (328, 200), (520, 100), (136, 600), (256, 1000)]
HP = dict(lr=0.02, momentum=0.95, nesterov=True, weight_decay=0.01, ns_steps=3)


def _rand(shape, dtype, seed, std):
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    return (torch.randn(shape, generator=g, device=DEV) * std).to(dtype)


def _offset_copy(t, offset):
    """A copy of `t` whose data starts `offset` elements into a larger buffer
    (so, for offset 1, 2 or 4 bytes past a 16-byte boundary)."""
    base = torch.empty(t.numel() + 16, dtype=t.dtype, device=DEV)
    v = base[offset:offset + t.numel()].view(t.shape)
    v.copy_(t)
    return v


def _check(dm, Ws, Gs, Bs, what):
    W0 = [w.clone() for w in Ws]
    B0 = [b.clone() for b in Bs]
    dm.dmuon_muon_step_batched(Ws, Gs, Bs, **HP)
    torch.cuda.synchronize()
    assert dm.dmuon_device_status() == 0
    for i in range(len(Ws)):
        buf_ref, X_ref, W_ref = oracle_step(W0[i], Gs[i], B0[i], **HP)
        assert np.array_equal(host(Bs[i]).view(np.uint32), buf_ref.view(np.uint32)), (what, i)
        check_bf16_weights(host(Ws[i]), W_ref, X_ref, HP["lr"], f"{what} W[{i}] {tuple(Ws[i].shape)}")


@pytest.mark.parametrize("gdt", [torch.bfloat16, torch.float32], ids=["g_bf16", "g_f32"])
def test_aligned_inputs(cuda_lib, gdt):
    Ws = [_rand(s, torch.bfloat16, 10 + i, 0.02) for i, s in enumerate(SHAPES)]
    Gs = [_rand(s, gdt, 20 + i, 1e-3) for i, s in enumerate(SHAPES)]
    Bs = [_rand(s, torch.float32, 30 + i, 1e-3) for i, s in enumerate(SHAPES)]
    _check(cuda_lib, Ws, Gs, Bs, f"aligned {gdt}")


def test_unaligned_gradient_and_buffer_rows(cuda_lib):
    """Gradients and buffers one element past a 16-byte boundary: no item is
    staged, every one is read from global memory."""
    Ws = [_rand(s, torch.bfloat16, 40 + i, 0.02) for i, s in enumerate(SHAPES)]
    Gs = [_offset_copy(_rand(s, torch.bfloat16, 50 + i, 1e-3), 1) for i, s in enumerate(SHAPES)]
    Bs = [_offset_copy(_rand(s, torch.float32, 60 + i, 1e-3), 1) for i, s in enumerate(SHAPES)]
    assert all(g.data_ptr() % 16 != 0 for g in Gs)
    _check(cuda_lib, Ws, Gs, Bs, "unaligned")


def test_alignment_changes_between_calls(cuda_lib):
    """One set of shapes (one launch plan), three calls: aligned tensors,
    then unaligned copies of the state, then aligned copies at new addresses.
    Each call patches the plan, including the prologue's tensor maps."""
    dm = cuda_lib
    builds0 = None
    Ws = [_rand(s, torch.bfloat16, 70 + i, 0.02) for i, s in enumerate(SHAPES)]
    Bs = [_rand(s, torch.float32, 80 + i, 1e-3) for i, s in enumerate(SHAPES)]
    for call, offset in enumerate([0, 1, 0]):
        Gs = [_rand(s, torch.bfloat16, 100 * call + i, 1e-3) for i, s in enumerate(SHAPES)]
        if offset:
            Gs = [_offset_copy(g, offset) for g in Gs]
            Bs = [_offset_copy(b, offset) for b in Bs]
        elif call:
            Bs = [b.clone() for b in Bs]
        _check(dm, Ws, Gs, Bs, f"call {call}")
        if builds0 is None:
            builds0 = dm.dmuon_plan_builds()
    assert dm.dmuon_plan_builds() == builds0, "a call with moved tensors built a plan"
