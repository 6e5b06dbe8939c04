"""The C-ABI library without a GPU: it loads, exports every symbol declared in
include/dmuon.h, and rejects bad arguments on the host before any CUDA call."""
import ctypes
import os
import re

import pytest

import newton_schulz_09_b200 as dm
from newton_schulz_09_b200 import build as dmbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dmuon.h")


@pytest.fixture(scope="module")
def lib():
    dmbuild.build()
    return dm.load_library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(dmuon_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for must in ("dmuon_ns_orthogonalize", "dmuon_muon_step_batched",
                 "dmuon_muon_step_batched_ex", "dmuon_workspace_bytes", "dmuon_last_error",
                 "dmuon_backend_string"):
        assert must in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_library_is_built_for_sm100a_only():
    assert "arch=compute_100a,code=sm_100a" in " ".join(dmbuild.NVCC_FLAGS)


def _shapes(*dims, pdt=dm.DMUON_BF16, gdt=dm.DMUON_BF16):
    S = (dm.DmuonShape * len(dims))()
    for i, (r, c) in enumerate(dims):
        S[i] = dm.DmuonShape(r, c, pdt, gdt)
    return S


def _ptrs(*vals):
    return (ctypes.c_void_p * len(vals))(*vals)


def _call(lib, S, n, P=None, G=None, B=None, steps=5):
    P = P or _ptrs(*([0x10000] * n))
    G = G or _ptrs(*([0x20000] * n))
    B = B or _ptrs(*([0x30000] * n))
    return lib.dmuon_muon_step_batched(P, G, B, S, n, 0.02, 0.95, 1, 0.0, steps, None)


def test_count_zero_is_a_noop(lib):
    assert _call(lib, _shapes((4, 4)), 0) == 0


def test_invalid_arguments_are_rejected_on_the_host(lib):
    assert _call(lib, _shapes((4, 4)), -1) == -1
    assert _call(lib, _shapes((4, 4)), 1, steps=-1) == -1
    assert _call(lib, _shapes((0, 4)), 1) == -1
    assert "rows and cols" in dm.dmuon_last_error()
    assert _call(lib, _shapes((4, 4)), 1, P=_ptrs(None)) == -1
    assert _call(lib, _shapes((4, 4)), 1, B=_ptrs(None)) == -1
    assert _call(lib, _shapes((4, 4)), 1, P=_ptrs(0x10001)) == -1      # odd bf16 address
    assert "aligned" in dm.dmuon_last_error()
    assert _call(lib, _shapes((4, 4), pdt=7), 1) == -2
    assert _call(lib, _shapes((40000, 40000)), 1) == -2                # min side too large
    assert lib.dmuon_ns_orthogonalize(None, 4, 4, 5, None) == -1
    assert lib.dmuon_ns_orthogonalize(ctypes.c_void_p(0x1000), 4, 4, -3, None) == -1


def test_null_gradient_is_skipped_before_any_device_work(lib):
    # Every matrix without a gradient: nothing to do, no CUDA call, success.
    assert _call(lib, _shapes((4, 4), (8, 8)), 2, G=_ptrs(None, None)) == 0


def test_workspace_bytes(lib):
    # One 256x512 bf16 matrix, 5 steps: X0 and X1 (256 x 512), A (256 x 256),
    # then 1 KiB regions: norm partials, scales, gradient-norm partials and the
    # clip scalars (every region rounded up to 1 KiB).
    small = 4 * 1024
    assert lib.dmuon_workspace_bytes(_shapes((256, 512)), 1, 5) == 2 * 262144 + 131072 + small
    # Tall matrix: same m x n view.
    assert lib.dmuon_workspace_bytes(_shapes((512, 256)), 1, 5) == 2 * 262144 + 131072 + small
    # No second iterate and no Gram for steps == 0.
    assert lib.dmuon_workspace_bytes(_shapes((256, 512)), 1, 0) == 262144 + small
    # Ragged shape: rows padded to 16 bytes (8 bf16 / 4 fp32).
    assert lib.dmuon_workspace_bytes(_shapes((3, 5)), 1, 1) == 1024 + 1024 + small
    assert lib.dmuon_workspace_bytes(_shapes((0, 5)), 1, 1) == 0
    assert lib.dmuon_ns_workspace_bytes(256, 512, dm.DMUON_F32) == 4 * 524288 + 262144 + small
    # Two dtype groups: per-group regions, one clip region.
    S = (dm.DmuonShape * 2)(dm.DmuonShape(256, 512, dm.DMUON_BF16, dm.DMUON_BF16),
                            dm.DmuonShape(256, 512, dm.DMUON_F32, dm.DMUON_F32))
    assert lib.dmuon_workspace_bytes(S, 2, 5) == (2 * 262144 + 131072) + (4 * 524288 + 262144) + 7 * 1024


def test_step_options_defaults_and_checks(lib):
    o = dm.DmuonStepOptions()
    lib.dmuon_step_options_default(ctypes.byref(o))
    assert o.struct_size == ctypes.sizeof(dm.DmuonStepOptions)
    assert abs(o.lr - 0.02) < 1e-9 and abs(o.momentum - 0.95) < 1e-7 and o.nesterov == 1
    assert o.ns_steps == 5 and o.ns_a == 1.5 and o.ns_b == -0.5
    assert o.lr_scale == dm.DMUON_LR_PLAIN and o.max_grad_norm == 0.0
    P, G, B = _ptrs(0x10000), _ptrs(0x20000), _ptrs(0x30000)
    S = _shapes((4, 4))
    bad = dm.DmuonStepOptions(); lib.dmuon_step_options_default(ctypes.byref(bad)); bad.struct_size = 8
    assert lib.dmuon_muon_step_batched_opts(P, G, B, S, 1, ctypes.byref(bad), None, 0, None) == -1
    assert "struct_size" in dm.dmuon_last_error()
    for field, value in (("max_grad_norm", -1.0), ("lr_scale", 7), ("ns_a", float("nan"))):
        x = dm.DmuonStepOptions(); lib.dmuon_step_options_default(ctypes.byref(x))
        setattr(x, field, value)
        assert lib.dmuon_muon_step_batched_opts(P, G, B, S, 1, ctypes.byref(x), None, 0, None) == -1
    assert lib.dmuon_muon_step_batched_opts(P, G, B, S, 1, None, None, 0, None) == -1


def test_backend_string(lib):
    s = dm.dmuon_backend_string()
    assert "tcgen05" in s and "sm_100a" in s


def test_no_cpu_fallback_without_device():
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    with pytest.raises(ValueError):
        dm.dmuon_ns_orthogonalize(torch.zeros(4, 4, dtype=torch.bfloat16))


def test_host_buffer_step_rejects_bad_arguments_on_the_host(lib):
    o = dm.DmuonStepOptions()
    lib.dmuon_step_options_default(ctypes.byref(o))
    P, G, B = _ptrs(0x10000), _ptrs(0x20000), _ptrs(0x30000)
    HG, HP = _ptrs(0x40000), _ptrs(0x50000)
    S = _shapes((4, 4))
    call = lambda opts, chunks=0, hg=HG, n=1: lib.dmuon_muon_step_batched_host(
        P, G, B, hg, HP, S, n, opts, chunks, None, 0, None)
    assert call(ctypes.byref(o), n=0) == 0
    assert call(None) == -1
    assert call(ctypes.byref(o), chunks=dm.DMUON_MAX_CHUNKS + 1) == -1
    clip = dm.DmuonStepOptions(); lib.dmuon_step_options_default(ctypes.byref(clip))
    clip.max_grad_norm = 1.0
    assert call(ctypes.byref(clip)) == -2
    assert "clipping" in dm.dmuon_last_error()
    # no host gradient at all: nothing to do, no CUDA call
    assert call(ctypes.byref(o), hg=_ptrs(None)) == 0
    # pointers that are not page-locked host memory are refused
    assert call(ctypes.byref(o)) == -2
    assert "page-locked" in dm.dmuon_last_error()


def _partition(lib, dims, which):
    S = _shapes(*dims)
    cap = len(dims) + 1
    B = (ctypes.c_int * cap)()
    n = lib.dmuon_debug_partition(S, len(dims), which, B, cap)
    assert n > 0, dm.dmuon_last_error()
    b = list(B[:n + 1])
    assert b[0] == 0 and b[-1] == len(dims) and all(x < y for x, y in zip(b, b[1:]))
    return b


def _llama_dims():
    from newton_schulz_09_b200 import synthetic
    return [(s.rows, s.cols) for s in synthetic.workload("llama8b").specs]


def test_device_call_groups(lib):
    """Consecutive groups of at most 2^28 elements, each as full as the next
    matrix allows, at most 32."""
    dims = _llama_dims()
    b = _partition(lib, dims, 0)
    elems = [r * c for r, c in dims]
    for lo, hi in zip(b, b[1:]):
        assert sum(elems[lo:hi]) <= 2 ** 28 or hi - lo == 1
        if hi < len(dims):
            assert sum(elems[lo:hi + 1]) > 2 ** 28
    assert len(b) - 1 == 32
    assert _partition(lib, [(256, 512), (512, 256)], 0) == [0, 2]
    big = [(16384, 16384)] * 64                       # 1.7e10 elements: the cap of 32 groups
    assert len(_partition(lib, big, 0)) - 1 <= 32


def test_host_step_groups_ramp(lib):
    """The host-buffer step's automatic groups start and end small and grow
    by at most 1.5x (plus one matrix) from one group to the next."""
    dims = _llama_dims()
    b = _partition(lib, dims, 1)
    nbytes = [r * c * 2 for r, c in dims]
    sizes = [sum(nbytes[lo:hi]) for lo, hi in zip(b, b[1:])]
    total, biggest = sum(nbytes), max(nbytes)
    assert 8 <= len(sizes) <= 32
    assert sizes[0] <= total / 32 and sizes[-1] <= total / 32
    assert max(sizes) <= (1 << 30) + biggest
    first = 64 << 20
    for k, sz in enumerate(sizes[:-1]):
        assert sz < first * 1.5 ** k + biggest
    assert _partition(lib, [(256, 512)] * 3, 1) == [0, 3]     # small totals: one group


def test_partition_rejects_bad_arguments(lib):
    B = (ctypes.c_int * 4)()
    assert lib.dmuon_debug_partition(_shapes((4, 4)), 1, 2, B, 4) == -1
    assert lib.dmuon_debug_partition(_shapes((0, 4)), 1, 0, B, 4) == -1
    assert lib.dmuon_debug_partition(_shapes((4, 4)), 1, 0, B, 1) == -1


def test_reduce_step_rejects_bad_arguments_on_the_host(lib):
    o = dm.DmuonStepOptions()
    lib.dmuon_step_options_default(ctypes.byref(o))
    P, B = _ptrs(0x10000), _ptrs(0x30000)
    S = _shapes((4, 4))
    call = lambda grads, world, n=1, opts=ctypes.byref(o): lib.dmuon_muon_step_batched_reduce(
        P, grads, B, S, n, world, opts, None, 0, None)
    assert call(_ptrs(0x20000), 1, n=0) == 0                       # nothing to do
    assert call(_ptrs(0x20000), 0) == -1 and "world" in dm.dmuon_last_error()
    assert call(_ptrs(*([0x20000] * 65)), 65) == -1
    assert call(_ptrs(0x20000), 1, opts=None) == -1
    assert call(_ptrs(0x20000, None), 2) == -1 and "rank 1" in dm.dmuon_last_error()
    assert call(_ptrs(None, 0x20000), 2) == -1
    assert call(_ptrs(0x20000, 0x20001), 2) == -1 and "misaligned" in dm.dmuon_last_error()
    assert call(_ptrs(None, None), 2) == 0                         # no gradient on any rank: skipped


def test_caller_workspace_must_be_device_memory_of_the_matrices_device():
    """A host tensor as scratch would hand the kernels a host address: the
    binding refuses it, and counts a workspace's size in bytes, not elements."""
    import torch
    cuda0 = torch.device("cuda", 0)
    assert dm._workspace(None, cuda0) == (None, 0)
    with pytest.raises(ValueError, match="workspace"):
        dm._workspace(torch.empty(4096, dtype=torch.uint8), cuda0)
    with pytest.raises(ValueError, match="workspace"):
        dm._workspace("not a tensor", cuda0)


def test_header_serves_a_plain_c99_program(lib):
    """include/dmuon.h is plain C: a C99 program compiled with -pedantic
    -Werror against it links to the library and gets the documented host-side
    answers (tests/c_consumer.c)."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    out_dir = os.path.join(ROOT, "_build", "c_consumer")
    os.makedirs(out_dir, exist_ok=True)
    exe = os.path.join(out_dir, "c_consumer")
    libdir = os.path.dirname(dm.library_path())
    subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror",
                    "-I", os.path.join(ROOT, "include"), os.path.join(ROOT, "tests", "c_consumer.c"),
                    "-o", exe, "-L", libdir, "-ldmuon", f"-Wl,-rpath,{libdir}"], check=True,
                   env=dict(os.environ, TMPDIR=out_dir))
    r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == "ok"


def test_missing_library_fails_loudly(monkeypatch):
    """Without the built library every entry point raises: there is no
    Python or CPU path to fall back to."""
    import torch
    monkeypatch.setattr(dm, "_lib", None)
    monkeypatch.setattr(dm, "_LIB_PATH", os.path.join(ROOT, "_build", "no_such_library.so"))
    with pytest.raises(RuntimeError, match="missing"):
        dm.load_library()
    with pytest.raises(RuntimeError, match="missing"):
        dm.dmuon_backend_string()
    with pytest.raises(RuntimeError, match="missing"):
        dm.dmuon_muon_step_batched([], [], [])
    with pytest.raises(RuntimeError, match="missing"):
        dm.dmuon_ns_orthogonalize(torch.zeros(4, 4, dtype=torch.bfloat16))


def test_clip_buckets_argument_checks(lib):
    D = (dm.DmuonGradDesc * 3)(dm.DmuonGradDesc(10000, dm.DMUON_BF16, 0),
                               dm.DmuonGradDesc(5, dm.DMUON_F32, 2),
                               dm.DmuonGradDesc(8192, dm.DMUON_BF16, 1))
    # 32 KB work items: 10000 bf16 -> 1, 5 fp32 -> 1, 8192 bf16 -> 1: three fp64
    # partials (256 bytes) and three coefficients (256 bytes)
    assert lib.dmuon_clip_workspace_bytes(D, 3, 3) == 512
    assert lib.dmuon_clip_workspace_bytes(D, 3, 2) == 0          # segment 2 out of range
    G = (ctypes.c_void_p * 3)(0x10000, 0x20000, 0x30000)
    M = (ctypes.c_float * 3)(1.0, 1.0, 1.0)

    def call(G=G, D=D, n=3, M=M, nseg=3):
        return lib.dmuon_clip_grad_norm_buckets(G, D, n, M, nseg, None, None, None, 0, None)

    assert call(nseg=0) == -1
    assert call(nseg=dm.DMUON_MAX_SEGMENTS + 1) == -1
    assert call(n=-1) == -1
    assert call(nseg=2) == -1 and "segment 2" in dm.dmuon_last_error()
    assert call(M=(ctypes.c_float * 3)(1.0, 0.0, 1.0)) == -1 and "max_norms[1]" in dm.dmuon_last_error()
    assert call(M=(ctypes.c_float * 3)(1.0, float("nan"), 1.0)) == -1
    bad = (dm.DmuonGradDesc * 1)(dm.DmuonGradDesc(0, dm.DMUON_BF16, 0))
    assert call(D=bad, n=1, nseg=1) == -1
    bad = (dm.DmuonGradDesc * 1)(dm.DmuonGradDesc(4, 9, 0))
    assert call(D=bad, n=1, nseg=1) == -2
    odd = (ctypes.c_void_p * 3)(0x10001, 0x20000, 0x30000)   # odd bf16 address
    assert call(G=odd) == -1 and "aligned" in dm.dmuon_last_error()


def test_options_struct_sizes_and_quintic_workspace(lib):
    o = dm.DmuonStepOptions()
    lib.dmuon_step_options_default(ctypes.byref(o))
    assert o.ns_c == 0.0
    P, G, B = _ptrs(0x10000), _ptrs(None), _ptrs(0x30000)
    S = _shapes((4, 4))
    # a caller built before ns_c existed passes the shorter size: accepted
    o.struct_size = dm.DmuonStepOptions.ns_c.offset
    assert lib.dmuon_muon_step_batched_opts(P, G, B, S, 1, ctypes.byref(o), None, 0, None) == 0
    o.struct_size = ctypes.sizeof(dm.DmuonStepOptions) + 4
    assert lib.dmuon_muon_step_batched_opts(P, G, B, S, 1, ctypes.byref(o), None, 0, None) == -1
    lib.dmuon_step_options_default(ctypes.byref(o))
    o.ns_c = float("inf")
    assert lib.dmuon_muon_step_batched_opts(P, G, B, S, 1, ctypes.byref(o), None, 0, None) == -1
    # workspace: cubic as dmuon_workspace_bytes; quintic adds P (m x lda) per matrix
    S2 = _shapes((256, 512), (512, 256))
    lib.dmuon_step_options_default(ctypes.byref(o))
    cubic = lib.dmuon_workspace_bytes_opts(S2, 2, ctypes.byref(o))
    assert cubic == lib.dmuon_workspace_bytes(S2, 2, 5)
    o.ns_c = 2.0315
    assert lib.dmuon_workspace_bytes_opts(S2, 2, ctypes.byref(o)) == cubic + 2 * 256 * 256 * 2
    o.ns_steps = 0
    assert lib.dmuon_workspace_bytes_opts(S2, 2, ctypes.byref(o)) == lib.dmuon_workspace_bytes(S2, 2, 0)


def test_last_plan_query_without_plans(lib):
    # host only: no plan exists in a process that made no device call
    assert lib.dmuon_debug_last_plan(None, 0) == 0
    assert dm.dmuon_debug_last_plan() == []
