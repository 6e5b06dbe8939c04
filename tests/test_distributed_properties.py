"""Properties of the owner partition (host logic, no GPU or process group).

* ``lpt_partition``: every item gets one owner in [0, world); the largest
  load is at most the list-scheduling bound total/world + max item, and on
  small cases within Graham's bound (4/3 - 1/(3 world)) of the optimum found
  by brute force over every assignment.
* ``owner_chunks``: each owner's items, in index order, cut into at most
  ``chunks_per_owner`` non-empty consecutive chunks.
* ``global_schedule``: every (owner, chunk) pair exactly once, ordered by
  chunk index, then owner.
"""
import itertools

from hypothesis import given, settings, strategies as st

from newton_schulz_09_b200 import distributed as dmd

costs_strategy = st.lists(st.integers(min_value=0, max_value=10 ** 6).map(float), min_size=0,
                          max_size=60)


def loads(costs, owner, world):
    out = [0.0] * world
    for c, r in zip(costs, owner):
        out[r] += c
    return out


@settings(max_examples=300, deadline=None)
@given(costs_strategy, st.integers(min_value=1, max_value=9))
def test_lpt_owner_range_and_list_scheduling_bound(costs, world):
    owner = dmd.lpt_partition(costs, world)
    assert len(owner) == len(costs) and all(0 <= r < world for r in owner)
    assert owner == dmd.lpt_partition(costs, world)              # the same on every rank
    if costs:
        assert max(loads(costs, owner, world)) <= sum(costs) / world + max(costs) + 1e-6


@settings(max_examples=150, deadline=None)
@given(st.lists(st.integers(min_value=1, max_value=100).map(float), min_size=1, max_size=7),
       st.integers(min_value=2, max_value=3))
def test_lpt_within_grahams_bound_of_the_optimum(costs, world):
    owner = dmd.lpt_partition(costs, world)
    lpt = max(loads(costs, owner, world))
    opt = min(max(loads(costs, a, world)) for a in itertools.product(range(world), repeat=len(costs)))
    assert lpt <= (4.0 / 3.0 - 1.0 / (3.0 * world)) * opt + 1e-9


@settings(max_examples=300, deadline=None)
@given(st.lists(st.tuples(st.integers(0, 5), st.integers(1, 10 ** 7)), min_size=0, max_size=50),
       st.integers(min_value=1, max_value=6))
def test_owner_chunks_and_schedule(items, chunks_per_owner):
    world = 6
    owner = [o for o, _ in items]
    numel = [n for _, n in items]
    ch = dmd.owner_chunks(owner, numel, world, chunks_per_owner)
    assert len(ch) == world
    for r in range(world):
        assert sum(ch[r], []) == [i for i, o in enumerate(owner) if o == r]
        assert len(ch[r]) <= chunks_per_owner and all(ch[r])
    sched = dmd.global_schedule(ch)
    assert sorted(sched) == sorted((r, c) for r in range(world) for c in range(len(ch[r])))
    assert sched == sorted(sched, key=lambda rc: (rc[1], rc[0]))
