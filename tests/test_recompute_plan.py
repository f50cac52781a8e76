"""Host-only checks of the depth-stack recompute plan (reportify.cn mHC summary,
[21] recompute, [22] the memory-optimal recompute block).

* mhc_recompute_plan (C ABI) against a replay of the schedule that DepthStack
  executes: the replay counts, step by step, the activations the stack holds per
  token (units of C elements: n for a kept or rebuilt stream x_l, 1 each for a
  rebuilt h_in_l and f_out_l); the plan's block must be the smallest block with
  the lowest replayed peak, and its resident figure that peak.
* the schedule itself: every layer runs forward once in order, is rebuilt once,
  runs backward once from the last layer down, is rebuilt from an input that is
  held at that point, and every kept input is released.
* the closed forms: one block per layer and one block for the whole stack give
  n (L - 1) + n + 2 and (n + 2) L, and the plan's cost lies between the
  real-valued minimum 2 sqrt(n (n + 2) L) - n and that minimum plus 2n + 2.
No test here launches a kernel.
"""
import math

import pytest

from manifold_constrained_hyper_token_b200 import build
from manifold_constrained_hyper_token_b200.depth import recompute_blocks, schedule


@pytest.fixture(scope="module")
def plan():
    build.build()
    from manifold_constrained_hyper_token_b200 import mhc_recompute_plan
    return mhc_recompute_plan


def _replay(L, n, block):
    """Peak of the activations held per token (units of C) over the schedule, and a
    check that the schedule is a valid training-order recompute."""
    fwd, bwd = schedule(L, block)
    starts = {l0 for l0, _ in recompute_blocks(L, block)}
    held, peak = 0, 0
    kept, rebuilt_x, rebuilt = set(), set(), set()
    assert [s[1] for s in fwd] == list(range(L))
    for _, l, keep in fwd:
        assert keep == (l in starts)
        if keep:
            kept.add(l)
            held += n
        peak = max(peak, held)
    order = []
    for step in bwd:
        kind, l = step[0], step[1]
        if kind == "recompute":
            assert l in kept or l in rebuilt_x, ("rebuilt from a stream not held", l)
            assert l not in rebuilt
            rebuilt.add(l)
            held += 2
            if step[2]:
                assert l + 1 not in starts
                rebuilt_x.add(l + 1)
                held += n
        elif kind == "backward":
            assert l in rebuilt
            order.append(l)
            held -= 2
            if l in rebuilt_x:
                rebuilt_x.remove(l)
                held -= n
        else:
            assert kind == "release" and l in kept
            kept.remove(l)
            held -= n
        peak = max(peak, held)
    assert order == list(reversed(range(L)))
    assert rebuilt == set(range(L))
    assert held == 0 and not kept and not rebuilt_x
    return peak


@pytest.mark.parametrize("n", [1, 2, 4, 8, 16])
def test_plan_is_the_replayed_minimum(plan, n):
    for L in range(1, 65):
        peaks = {B: _replay(L, n, B) for B in range(1, L + 1)}
        best = min(peaks.values())
        B, res = plan(n, L)
        assert B == min(b for b, p in peaks.items() if p == best), (n, L)
        assert res == best, (n, L)


@pytest.mark.parametrize("n", [1, 4, 8])
def test_closed_forms(n):
    for L in (1, 2, 7, 24, 61):
        assert _replay(L, n, 1) == n * (L - 1) + n + 2
        assert _replay(L, n, L) == (n + 2) * L


@pytest.mark.parametrize("n", [1, 2, 4, 8, 16])
def test_plan_within_real_bounds(plan, n):
    # Over real B, n (L/B - 1) + (n + 2) B >= 2 sqrt(n (n + 2) L) - n, and it lower-bounds
    # the cost since ceil(L/B) >= L/B.  B = ceil(sqrt(n L / (n + 2))) costs at most
    # 2 sqrt(n (n + 2) L) + n + 2, since ceil(L/B) - 1 < L/B.
    for L in list(range(1, 130)) + [200, 512, 1000]:
        _, res = plan(n, L)
        root = 2.0 * math.sqrt(n * (n + 2) * L)
        assert root - n - 1e-9 <= res <= root + n + 2 + 1e-9, (n, L, res)


def test_depth_stack_shape(plan):
    # the 24-layer, n = 4 stack: blocks of 4, 44 C per token against 144 C kept
    assert plan(4, 24) == (4, 44)
    assert recompute_blocks(24, 4) == [(l, l + 4) for l in range(0, 24, 4)]
    assert recompute_blocks(10, 4) == [(0, 2), (2, 6), (6, 10)]


def test_rejects_bad_arguments(plan):
    from manifold_constrained_hyper_token_b200 import MhcError
    for n, L in ((0, 4), (4, 0), (-1, 3)):
        with pytest.raises(MhcError):
            plan(n, L)
    with pytest.raises(ValueError):
        recompute_blocks(0, 1)
