"""ORACLE - test infrastructure only.  A plain Python statement of the dynamic-batching
scheduler that the C++ runtime implements (only the tests and the bench's CPU legs use it).

Sources (pages on Energon-AI):
  [A] QbitAI article, section "Serving": requests in the queue are packed into batches as
      the machine's performance suits best, and the batch of highest priority is run first,
      priority coming from the waiting time, the batch size and the batch's expansion
      possibility (its length after padding); this keeps the GPU busy while avoiding
      starvation.  Section "性能测试": compared with FIFO packing, GPT-3, lengths random
      up to 256, every batch padded to its longest sequence.
  [B] EnergonAI README, section "Batching": the same rule, inspired by TurboTransformer's
      dynamic-programming batch scheduler; FIFO batching is the comparison.

The pages give no formula.  Readings taken here (each one stated where it is used):
  * Packing (the DP): requests sorted by length (ties by arrival, then index) are cut into
    consecutive groups of at most max_batch; the cut minimises the summed cost of the groups,
    cost(B, S) from a table measured on the machine (B sequences padded to S tokens).
  * Priority of a group g: useful tokens per unit cost, raised by the waiting time of its
    oldest request:  prio(g) = (sum of lengths in g) / cost(|g|, max length in g)
                               * (1 + wait(g) / age_scale).
    The batch size and the padded length enter through the cost (a larger batch amortises the
    fixed cost; a longer padded length means more wasted work per useful token), and the
    waiting time keeps old requests from starving.
  * Ties: the DP keeps the first minimum found scanning the group start upward (the larger
    last group); the priority order is by descending priority, ties by ascending group index.
"""
from __future__ import annotations


def sort_order(lengths, arrivals):
    """Request indices by (length, arrival, index)."""
    return sorted(range(len(lengths)), key=lambda i: (lengths[i], arrivals[i], i))


def dp_groups(sorted_lengths, max_batch, cost):
    """Cut lengths (ascending) into consecutive groups of <= max_batch minimising
    sum(cost(size, last length)).  Returns the list of (start, end) half-open ranges."""
    n = len(sorted_lengths)
    best = [0.0] + [None] * n
    cut = [0] * (n + 1)
    for j in range(1, n + 1):                       # groups ending at request j-1
        for i in range(max(0, j - max_batch), j):   # group = [i, j)
            c = best[i] + cost(j - i, sorted_lengths[j - 1])
            if best[j] is None or c < best[j]:
                best[j] = c
                cut[j] = i
    groups = []
    j = n
    while j > 0:
        groups.append((cut[j], j))
        j = cut[j]
    return groups[::-1]


def plan(lengths, arrivals, now, max_batch, cost_table, age_scale):
    """The scheduler's decision for a queue snapshot.

    cost_table[b - 1][s - 1] = cost of b sequences padded to s tokens.  Returns
    (group_of, order): group_of[i] = group index of request i (groups numbered in ascending
    length order), order = group indices by descending priority."""
    n = len(lengths)
    if n == 0:
        return [], []

    def cost(b, s):
        return cost_table[b - 1][s - 1]

    idx = sort_order(lengths, arrivals)
    sl = [lengths[i] for i in idx]
    groups = dp_groups(sl, max_batch, cost)
    group_of = [0] * n
    prio = []
    for g, (a, b) in enumerate(groups):
        members = idx[a:b]
        for i in members:
            group_of[i] = g
        tokens = 0
        for i in members:
            tokens += lengths[i]
        oldest = min(arrivals[i] for i in members)
        wait = now - oldest
        prio.append(tokens / cost(b - a, sl[b - 1]) * (1.0 + wait / age_scale))
    order = sorted(range(len(groups)), key=lambda g: (-prio[g], g))
    return group_of, order


def fifo(arrivals, max_batch):
    """FIFO packing (the pages' baseline): arrival order (ties by index), consecutive groups
    of max_batch.  Returns group_of."""
    idx = sorted(range(len(arrivals)), key=lambda i: (arrivals[i], i))
    group_of = [0] * len(arrivals)
    for k, i in enumerate(idx):
        group_of[i] = k // max_batch
    return group_of
