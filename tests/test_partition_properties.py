"""Properties of the library's two grouping rules over random shape lists
(host logic, no GPU), read through ``dmuon_debug_partition``:

* device groups (a call above 2^28 elements runs as consecutive groups):
  at most 32 groups; a call of at most 2^28 elements is one group; a group
  is closed only when the next matrix would take it past a target of at
  least 2^28 elements;
* host-buffer groups (the ramp of the host-buffer step): at most 32 groups;
  every group but the last holds at least 64 MiB of
  gradient bytes, so a small call is one group.
"""
import ctypes

from hypothesis import HealthCheck, given, settings, strategies as st

import newton_schulz_09_b200 as dm
from newton_schulz_09_b200 import build as dmbuild

SIDES = [1, 7, 64, 128, 136, 1000, 1024, 4096, 8191, 14336, 32768]
dims_strategy = st.lists(st.tuples(st.sampled_from(SIDES), st.sampled_from(SIDES)), min_size=1,
                         max_size=80)
SETTINGS = settings(max_examples=300, deadline=None,
                    suppress_health_check=[HealthCheck.too_slow])

_lib = None


def lib():
    global _lib
    if _lib is None:
        dmbuild.build()
        _lib = dm.load_library()
    return _lib


def partition(dims, which):
    n = len(dims)
    S = (dm.DmuonShape * n)(*[dm.DmuonShape(r, c, dm.DMUON_BF16, dm.DMUON_BF16) for r, c in dims])
    B = (ctypes.c_int * (n + 1))()
    g = lib().dmuon_debug_partition(S, n, which, B, n + 1)
    assert g > 0, dm.dmuon_last_error()
    b = list(B[:g + 1])
    assert b[0] == 0 and b[-1] == n and all(x < y for x, y in zip(b, b[1:]))
    return b


@SETTINGS
@given(dims_strategy)
def test_device_groups(dims):
    b = partition(dims, 0)
    elems = [r * c for r, c in dims]
    total = sum(elems)
    assert len(b) - 1 <= 32
    if total <= 2 ** 28:
        assert b == [0, len(dims)]
    for lo, hi in zip(b[:-1], b[1:-1]):
        # closed only because the next matrix would overflow the target (>= 2^28)
        assert sum(elems[lo:hi + 1]) > 2 ** 28


@SETTINGS
@given(dims_strategy)
def test_host_buffer_groups(dims):
    b = partition(dims, 1)
    nbytes = [2 * r * c for r, c in dims]
    total = sum(nbytes)
    first = 64 << 20
    assert len(b) - 1 <= 32
    for lo, hi in zip(b[:-2], b[1:-1]):
        assert sum(nbytes[lo:hi]) >= first
    if total < first:
        assert b == [0, len(dims)]
