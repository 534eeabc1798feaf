"""The C++ dynamic-batching scheduler (host runtime, CPU only) against its oracle: the same
groups and the same priority order on seeded request queues, FIFO packing, and the
host-side argument checks."""
import importlib.util
import os
import random

import pytest
from hypothesis import given, settings, strategies as hs

from padding_free_varlen_b200 import capi, synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
_spec = importlib.util.spec_from_file_location("sched_oracle", os.path.join(ROOT, "oracle", "scheduler.py"))
oracle_sched = importlib.util.module_from_spec(_spec)
_spec.loader.exec_module(oracle_sched)


@pytest.fixture(scope="module", autouse=True)
def lib():
    from padding_free_varlen_b200 import build
    build.build()
    return capi.load()


def linear_table(max_b, max_s, c0, c1):
    return [[c0 + c1 * b * s for s in range(1, max_s + 1)] for b in range(1, max_b + 1)]


@pytest.mark.parametrize("seed", range(30))
def test_plan_matches_oracle(seed):
    rng = random.Random(seed)
    n = rng.choice([1, 2, 7, 33, 128, 300])
    max_b, max_s = rng.choice([1, 4, 16, 64]), 256
    # lengths U[1, 256] from the seeded generator (the dynamic-batch workload's draw)
    lengths = [int(v) for v in synth.uniform_int(n, 1, max_s, 20260005 + seed, synth.TID_LENGTHS)]
    arrivals = [round(rng.uniform(0.0, 5.0), rng.choice([0, 3, 9])) for _ in range(n)]   # with ties
    if seed % 3 == 0:
        table = [[rng.uniform(0.1, 10.0) for _ in range(max_s)] for _ in range(max_b)]
    else:
        table = linear_table(max_b, max_s, rng.uniform(1e-3, 5e-2), rng.uniform(1e-6, 1e-5))
    now = 6.0
    got = capi.energon_sched_plan(lengths, arrivals, now, max_b, table, 0.5)
    ref = oracle_sched.plan(lengths, arrivals, now, max_b, table, 0.5)
    assert got == (list(ref[0]), list(ref[1]))


def test_plan_empty_queue_and_fifo():
    assert capi.energon_sched_plan([], [], 0.0, 4, [[1.0]], 1.0) == ([], [])
    arrivals = [3.0, 1.0, 2.0, 1.0, 0.5]
    assert capi.energon_sched_fifo(arrivals, 2) == oracle_sched.fifo(arrivals, 2) == [2, 0, 1, 1, 0]
    rng = random.Random(7)
    arr = [rng.uniform(0, 1) for _ in range(500)]
    assert capi.energon_sched_fifo(arr, 64) == oracle_sched.fifo(arr, 64)


def test_plan_rejects_bad_arguments():
    table = linear_table(2, 8, 1.0, 1.0)
    for args in (([9], [0.0], 0.0, 2, table, 1.0),                      # length beyond the table
                 ([0], [0.0], 0.0, 2, table, 1.0),                      # empty request
                 ([3], [float("nan")], 0.0, 2, table, 1.0),             # time not finite
                 ([3], [0.0], 0.0, 0, table, 1.0),                      # max_batch 0
                 ([3], [0.0], 0.0, 2, table, 0.0),                      # age scale 0
                 ([3, 4], [0.0, 0.0], 0.0, 2, [[1.0] * 8, [-1.0] * 8], 1.0)):   # bad cost
        with pytest.raises(capi.EnergonError) as e:
            capi.energon_sched_plan(*args)
        assert e.value.code == capi.ENERGON_ERR_INVALID_ARGUMENT
    with pytest.raises(capi.EnergonError):
        capi.energon_sched_fifo([0.0, 1.0], 0)


@settings(max_examples=150, deadline=None)
@given(data=hs.data())
def test_plan_matches_oracle_on_arbitrary_queues(data):
    """Random queues (ties in length and arrival included) and random positive cost tables,
    monotone or not: the C++ runtime and the oracle take the same decisions."""
    n = data.draw(hs.integers(0, 40))
    max_b = data.draw(hs.integers(1, 8))
    max_s = data.draw(hs.integers(1, 12))
    lengths = data.draw(hs.lists(hs.integers(1, max_s), min_size=n, max_size=n))
    arrivals = data.draw(hs.lists(hs.sampled_from([0.0, 0.25, 0.5, 1.0, 2.0]), min_size=n, max_size=n))
    table = data.draw(hs.lists(hs.lists(hs.floats(0.01, 100.0), min_size=max_s, max_size=max_s),
                               min_size=max_b, max_size=max_b))
    now = data.draw(hs.sampled_from([2.0, 3.5, 10.0]))
    age = data.draw(hs.sampled_from([0.1, 1.0, 7.0]))
    got = capi.energon_sched_plan(lengths, arrivals, now, max_b, table, age)
    ref = oracle_sched.plan(lengths, arrivals, now, max_b, table, age)
    assert got == (list(ref[0]), list(ref[1]))
    assert capi.energon_sched_fifo(arrivals, max_b) == oracle_sched.fifo(arrivals, max_b)
