"""Dynamic-programming batch scheduler, and exhaustive search (TEST INFRASTRUCTURE ONLY).

"TurboTransformers: An Efficient GPU Serving System For Transformer Models"
(abstract; proposed-method section) describes a serving framework whose batch
scheduler uses dynamic programming to reach the optimal throughput on
variable-length requests, grouping them with minimal padding after ordering
requests by length.  The page gives no recurrence; the plainest reading,
used here:

  1. stable-sort the queued requests by (length, arrival index):
     l_1 <= l_2 <= ... <= l_n;
  2. a batch of b requests whose longest has length L costs the integer
     T(b, L) -- by default c0 + c1*b*L (a fixed per-batch cost plus the
     padded-token work of a batch padded to its longest member), or a
     supplied table that is non-decreasing in L;
  3. dp[0] = 0,  dp[i] = min over j in [max(0, i - Bmax), i - 1] of
     dp[j] + T(i - j, l_i); ties go to the smallest j (the largest last batch);
  4. walk the choices back from n; batches are numbered 0..nb-1 in execution
     order, i.e. ascending longest length.

Total time is minimised, which maximises throughput over the queue.  For any
T non-decreasing in L some partition that is contiguous in sorted order is
optimal, so the DP's optimum equals the exhaustive search over all set
partitions (``brute_force_cost``), which is what pins it.

Latency-aware variants.  The same review's main results report the DP
scheduler's mean latency at its serving rate, and note that long sequences
wait somewhat longer.  Two knobs, each the plainest reading of serving to a
latency target rather than to throughput alone:

  * objective LATENCY: minimise the sum of the queued requests' completion
    times instead of the total time.  The batches still run in ascending
    longest length, back to back from time 0, so batch k (sorted positions
    s_k .. e_k - 1) delays every request from s_k on by its cost:
    sum of completions = sum_k T(b_k, L_k) * (n - s_k), and the recurrence
    becomes dp[i] = min_j dp[j] + T(i - j, l_i) * (n - j).  Among batchings
    of the sorted queue run in that order, this is exact
    (``brute_force_sorted``); other execution orders are not considered.
  * max_cost C > 0: no batch of two or more requests may cost more than C
    (a single request is always allowed, so a schedule always exists).  It
    bounds how long any request can sit behind one batch.  With the
    throughput objective the sorted refill argument still holds under the
    cap (refilling never raises a batch's cost), so the DP still equals the
    exhaustive search over all set partitions that respect the cap.
"""
from __future__ import annotations

from typing import Callable, Iterator, List, Optional, Tuple

import numpy as np

CostFn = Callable[[int, int], int]


def linear_cost(c0: int, c1: int) -> CostFn:
    """T(b, L) = c0 + c1*b*L."""
    return lambda b, L: int(c0) + int(c1) * int(b) * int(L)


def table_cost(table: np.ndarray) -> CostFn:
    """T(b, L) = table[b-1][L-1] for an integer table indexed by size and length."""
    t = np.asarray(table, dtype=np.int64)
    return lambda b, L: int(t[b - 1, L - 1])


def sorted_order(lengths: np.ndarray) -> np.ndarray:
    """Indices ordered by (length, original index)."""
    lengths = np.asarray(lengths)
    return np.array(sorted(range(len(lengths)), key=lambda i: (int(lengths[i]), i)), dtype=np.int64)


THROUGHPUT, LATENCY = 0, 1


def allowed(b: int, t: int, max_cost: int) -> bool:
    """A batch of b requests costing t respects the cap (0 = no cap)."""
    return max_cost <= 0 or b == 1 or t <= max_cost


def schedule_dp(lengths: np.ndarray, bmax: int, cost: CostFn, objective: int = THROUGHPUT,
                max_cost: int = 0) -> Tuple[np.ndarray, int]:
    """Return (batch id per request, optimal objective value)."""
    lengths = np.asarray(lengths)
    n = len(lengths)
    order = sorted_order(lengths)
    ls = [int(lengths[i]) for i in order]
    INF = None
    dp: List[Optional[int]] = [0] + [INF] * n
    choice = [0] * (n + 1)
    for i in range(1, n + 1):
        for j in range(max(0, i - bmax), i):
            t = cost(i - j, ls[i - 1])
            if not allowed(i - j, t, max_cost):
                continue
            c = dp[j] + (t if objective == THROUGHPUT else t * (n - j))
            if dp[i] is INF or c < dp[i]:
                dp[i] = c
                choice[i] = j
    # walk back: segments (j, i] in sorted order
    segs = []
    i = n
    while i > 0:
        segs.append((choice[i], i))
        i = choice[i]
    segs.reverse()
    batch = np.empty(n, dtype=np.int32)
    for b, (j, i) in enumerate(segs):
        for t in range(j, i):
            batch[order[t]] = b
    return batch, (dp[n] if n else 0)


def schedule_cost(lengths: np.ndarray, batch: np.ndarray, cost: CostFn) -> int:
    """Total cost of an arbitrary assignment of requests to batches."""
    lengths = np.asarray(lengths)
    total = 0
    for b in np.unique(batch):
        members = lengths[batch == b]
        total += cost(len(members), int(members.max()))
    return total


def latency_cost(lengths: np.ndarray, batch: np.ndarray, cost: CostFn) -> int:
    """Sum of completion times when the batches run back to back in id order."""
    lengths = np.asarray(lengths)
    batch = np.asarray(batch)
    t, total = 0, 0
    for b in sorted(np.unique(batch)):
        members = lengths[batch == b]
        t += cost(len(members), int(members.max()))
        total += t * len(members)
    return total


def compositions(n: int) -> Iterator[List[int]]:
    """Every way to cut 0..n-1 into consecutive runs, as run sizes."""
    if n == 0:
        yield []
        return
    for first in range(1, n + 1):
        for rest in compositions(n - first):
            yield [first] + rest


def brute_force_sorted(lengths: np.ndarray, bmax: int, cost: CostFn, objective: int,
                       max_cost: int = 0) -> int:
    """Best objective over every batching of the sorted queue into consecutive
    runs (run in that order), by enumeration."""
    ls = [int(lengths[i]) for i in sorted_order(lengths)]
    n = len(ls)
    best = None
    for sizes in compositions(n):
        if max(sizes, default=0) > bmax:
            continue
        start, clock, total, ok = 0, 0, 0, True
        for b in sizes:
            t = cost(b, ls[start + b - 1])
            if not allowed(b, t, max_cost):
                ok = False
                break
            clock += t
            total += t if objective == THROUGHPUT else clock * b
            start += b
        if ok and (best is None or total < best):
            best = total
    return best if best is not None else 0


def set_partitions(n: int) -> Iterator[List[int]]:
    """Every set partition of 0..n-1 as a restricted growth string a[0..n-1]
    (a[0] = 0, a[i] <= 1 + max(a[:i]))."""
    if n == 0:
        yield []
        return
    a = [0] * n

    def rec(i: int, m: int):
        if i == n:
            yield list(a)
            return
        for v in range(m + 2):
            a[i] = v
            yield from rec(i + 1, max(m, v))

    a[0] = 0
    yield from rec(1, 0)


def brute_force_cost(lengths: np.ndarray, bmax: int, cost: CostFn, max_cost: int = 0) -> int:
    """Minimum total cost over all set partitions with blocks of size <= bmax
    (and, with a cap, blocks that respect it)."""
    lengths = [int(x) for x in lengths]
    n = len(lengths)
    best = None
    for a in set_partitions(n):
        size = {}
        lmax = {}
        for i, b in enumerate(a):
            size[b] = size.get(b, 0) + 1
            lmax[b] = max(lmax.get(b, 0), lengths[i])
        if max(size.values(), default=0) > bmax:
            continue
        if not all(allowed(size[b], cost(size[b], lmax[b]), max_cost) for b in size):
            continue
        c = sum(cost(size[b], lmax[b]) for b in size)
        if best is None or c < best:
            best = c
    return best if best is not None else 0
