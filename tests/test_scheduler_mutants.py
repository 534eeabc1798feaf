"""Mutation check of the scheduler oracle's pins (CPU only): each case plants one plausible
mistake in a copy of ``oracle/scheduler.py`` and runs ``test_scheduler_oracle.py`` against
it; every mutant must fail a pin."""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "scheduler.py")

MUTANTS = [  # (name, text, replacement)
    ("dp_group_too_large", "range(max(0, j - max_batch), j)", "range(max(0, j - max_batch - 1), j)"),
    ("dp_ties_last_minimum", "if best[j] is None or c < best[j]:", "if best[j] is None or c <= best[j]:"),
    ("dp_cost_at_first_length", "cost(j - i, sorted_lengths[j - 1])", "cost(j - i, sorted_lengths[i])"),
    ("sort_by_arrival", "key=lambda i: (lengths[i], arrivals[i], i))", "key=lambda i: (arrivals[i], i))"),
    ("priority_no_wait_boost", "(1.0 + wait / age_scale)", "(1.0 + 0.0 * wait / age_scale)"),
    ("priority_padded_to_shortest", "tokens / cost(b - a, sl[b - 1])", "tokens / cost(b - a, sl[a])"),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_scheduler_pins_catch_mutant(tmp_path, name, old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not found once"
    mutant = tmp_path / "scheduler_mutant.py"
    mutant.write_text(src.replace(old, new))
    env = dict(os.environ, SCHED_ORACLE_OVERRIDE=str(mutant))
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_scheduler_oracle.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode != 0, f"mutant {name} passed every pin:\n{r.stdout[-2000:]}"
