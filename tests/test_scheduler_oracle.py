"""Pins of the dynamic-batching scheduler oracle (CPU): brute force over every cut of the
sorted queue, closed forms, invariants, the waiting-time boost and FIFO by hand.

The oracle module is loaded from its file so that a planted-mistake copy can stand in for
it (SCHED_ORACLE_OVERRIDE), as the C oracle's mutants do."""
import importlib.util
import itertools
import os
import random

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _load():
    path = os.environ.get("SCHED_ORACLE_OVERRIDE", os.path.join(ROOT, "oracle", "scheduler.py"))
    spec = importlib.util.spec_from_file_location("sched_oracle_under_test", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


S = _load()


def random_table(rng, max_b, max_s, kind):
    if kind == "linear":
        c0, c1 = rng.uniform(0.5, 5.0), rng.uniform(0.001, 0.02)
        return [[c0 + c1 * b * s for s in range(1, max_s + 1)] for b in range(1, max_b + 1)]
    # arbitrary positive table (not even monotone): the DP must still be exact
    return [[rng.uniform(0.1, 10.0) for _ in range(max_s)] for _ in range(max_b)]


def all_cuts(n, max_b):
    """Every split of range(n) into consecutive groups of size <= max_b."""
    for mask in range(1 << max(0, n - 1)):
        bounds = [0] + [k + 1 for k in range(n - 1) if mask >> k & 1] + [n]
        groups = list(zip(bounds[:-1], bounds[1:]))
        if all(b - a <= max_b for a, b in groups):
            yield groups


def total(groups, sl, table):
    return sum(table[b - a - 1][sl[b - 1] - 1] for a, b in groups)


@pytest.mark.parametrize("seed", range(40))
def test_dp_is_the_brute_force_optimum(seed):
    rng = random.Random(seed)
    n, max_b, max_s = rng.randint(1, 9), rng.randint(1, 4), 12
    table = random_table(rng, max_b, max_s, "linear" if seed % 2 else "any")
    sl = sorted(rng.randint(1, max_s) for _ in range(n))
    groups = S.dp_groups(sl, max_b, lambda b, s: table[b - 1][s - 1])
    best = min(total(g, sl, table) for g in all_cuts(n, max_b))
    assert abs(total(groups, sl, table) - best) <= 1e-12 * max(1.0, best)
    assert groups[0][0] == 0 and groups[-1][1] == n
    assert all(a < b and b - a <= max_b for a, b in groups)
    assert all(groups[k][1] == groups[k + 1][0] for k in range(len(groups) - 1))


def test_closed_forms():
    # cost = padded tokens only: batching never pays, so with distinct lengths and ties broken
    # toward the larger last group the minimum is reached with no padding at all
    table = [[b * s for s in range(1, 9)] for b in range(1, 5)]
    sl = [1, 2, 3, 5, 8]
    g = S.dp_groups(sl, 4, lambda b, s: table[b - 1][s - 1])
    assert total(g, sl, table) == sum(sl)
    # equal lengths and a fixed cost per batch: full batches of max_batch
    table = [[10.0 + b * s for s in range(1, 9)] for b in range(1, 5)]
    g = S.dp_groups([4] * 10, 4, lambda b, s: table[b - 1][s - 1])
    assert sorted(b - a for a, b in g) == [2, 4, 4]
    # max_batch 1: every request alone
    assert S.dp_groups([3, 3, 7], 1, lambda b, s: 1.0) == [(0, 1), (1, 2), (2, 3)]


def test_hand_example():
    # lengths 2, 9, 3, 8 (indices 0..3), cost(b, s) = 1 + b * s, max_batch 2.  Sorted: 2 (0),
    # 3 (2), 8 (3), 9 (1).  Worked by hand: best[1] = 3; best[2] = min(0 + 7, 3 + 4) = 7 at the
    # pair (first minimum); best[3] = min(3 + 17, 7 + 9) = 16; best[4] = min(7 + 19, 16 + 10)
    # = 26 at the pair {8, 9}.  Groups {2, 3} and {8, 9}.
    table = [[1.0 + b * s for s in range(1, 10)] for b in range(1, 3)]
    group_of, order = S.plan([2, 9, 3, 8], [0.0, 0.0, 0.0, 0.0], 0.0, 2, table, 1.0)
    assert group_of == [0, 1, 0, 1]
    # priorities: group 0: 5 tokens / 7, group 1: 17 tokens / 19 -> group 1 first
    assert order == [1, 0]


def test_waiting_time_raises_priority_and_prevents_starvation():
    table = [[1.0 + b * s for s in range(1, 17)] for b in range(1, 3)]
    lengths = [1, 16, 16]
    # the short request alone is the least efficient group ...
    g, order = S.plan(lengths, [0.0, 0.0, 0.0], 0.0, 2, table, 1.0)
    assert g[0] != g[1] and order[-1] == g[0]
    # ... but once it has waited long enough it goes first
    g, order = S.plan(lengths, [0.0, 50.0, 50.0], 50.0, 2, table, 1.0)
    assert order[0] == g[0]
    # the order flips exactly where the boost makes up the efficiency gap: 0.5 (1 + w) = 32/33
    g, order = S.plan(lengths, [0.0, 0.9, 0.9], 0.9, 2, table, 1.0)       # 0.95 < 0.9697
    assert order[0] == g[1]
    g, order = S.plan(lengths, [0.0, 1.0, 1.0], 1.0, 2, table, 1.0)       # 1.0 > 0.9697
    assert order[0] == g[0]


@pytest.mark.parametrize("seed", range(10))
def test_plan_invariants(seed):
    rng = random.Random(100 + seed)
    n, max_b = rng.randint(1, 60), rng.randint(1, 16)
    lengths = [rng.randint(1, 32) for _ in range(n)]
    arrivals = [rng.uniform(0, 10) for _ in range(n)]
    table = random_table(rng, max_b, 32, "linear")
    group_of, order = S.plan(lengths, arrivals, 10.0, max_b, table, 3.0)
    ng = max(group_of) + 1
    assert sorted(order) == list(range(ng))
    sizes = [group_of.count(g) for g in range(ng)]
    assert all(1 <= s <= max_b for s in sizes)
    for g in range(ng - 1):                                  # groups follow length order
        assert max(l for l, q in zip(lengths, group_of) if q == g) <= \
            min(l for l, q in zip(lengths, group_of) if q == g + 1)


def test_fifo_by_hand():
    assert S.fifo([3.0, 1.0, 2.0, 1.0, 0.5], 2) == [2, 0, 1, 1, 0]
    assert S.fifo([], 4) == []
