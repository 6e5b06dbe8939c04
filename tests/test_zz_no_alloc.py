"""The allocation-free entry point, dmuon_ns_orthogonalize_noalloc (needs a GPU).

It exists for callers that may not allocate device memory (a host framework
that owns all of it, a sandbox without cudaMalloc, a path that must not block
on an allocation).  Its scratch is a fixed array inside the library, shared by
every call.  These tests check it against the regular entry point,
dmuon_ns_orthogonalize, and against the fp64 oracle, on calls in a row, so
each call runs on the scratch the one before it left behind (different shapes
back to back, so the launch description and tensor maps in the shared array
change between calls).  They also check that oversized matrices are refused
and that a call takes no device memory.

The file is named to be collected last: if it fails, a run that stops at the
first failure has already run every other test.
"""
import pytest
import torch

import oracle
from tests.gpu_helpers import TOL_BF16, check_rel, host

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _rand(shape, seed):
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    return torch.randn(shape, generator=g, device=DEV).to(torch.bfloat16)


def test_noalloc_matches_regular_entry_on_two_calls_in_a_row(cuda_lib):
    dm = cuda_lib
    cases = [((1024, 2048), 5, 11), ((1500, 520), 3, 12), ((96, 3000), 0, 13)]
    for shape, steps, seed in cases:
        G = _rand(shape, seed)
        want = G.clone()
        dm.dmuon_ns_orthogonalize(want, steps)
        got = G.clone()
        dm.dmuon_ns_orthogonalize_noalloc(got, steps)
        torch.cuda.synchronize()
        assert dm.dmuon_device_status() == 0
        check_rel(host(got), host(want), TOL_BF16, f"noalloc {shape} k={steps}")
        X_ref = oracle.newton_schulz(host(G), steps)
        check_rel(host(got), X_ref, TOL_BF16, f"noalloc vs oracle {shape} k={steps}")


def test_noalloc_takes_no_device_memory(cuda_lib):
    dm = cuda_lib
    X = _rand((2048, 2048), 21)
    dm.dmuon_ns_orthogonalize_noalloc(X, 5)          # first call on the device: set-up
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for seed in (22, 23):
        Y = _rand((2048, 2048), seed)
        torch.cuda.synchronize()
        free0, _ = torch.cuda.mem_get_info()
        dm.dmuon_ns_orthogonalize_noalloc(Y, 5)
        torch.cuda.synchronize()
        free1, _ = torch.cuda.mem_get_info()
        # its 24 MiB of scratch would show up here if it were allocated per call
        assert free0 - free1 < (2 << 20), (free0, free1)
    assert dm.dmuon_device_status() == 0


def test_noalloc_refuses_matrices_beyond_its_scratch(cuda_lib):
    dm = cuda_lib
    X = _rand((4096, 4096), 31)
    X0 = X.clone()
    with pytest.raises(dm.DmuonError) as e:
        dm.dmuon_ns_orthogonalize_noalloc(X, 5)
    assert e.value.code == -2
    assert "static scratch" in str(e.value)
    torch.cuda.synchronize()
    assert torch.equal(X, X0)
