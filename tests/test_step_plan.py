"""The step kernel's split of a launch over CTAs (`tern_step_plan`, host
only): every tile is streamed by exactly one CTA, in order, and the largest
CTA cost (1024-k units plus the staging of every product a CTA starts) is
the smallest any cut into at most `grid` ranges can reach, checked against
an exhaustive search on small cases.  The cost of staging one product
mirrors the kernel's own model (piece_cost in tern_gemv_step.cu): it is
scheduling, not the method's arithmetic."""
import random

import pytest

from ternary_weight_only_b200 import tern as T

ROWS = 16  # rows per tile


def piece_cost(K, M):
    B = K // 1024
    if M == 1:
        return 5 + (12 * B) // 5
    if M == 2:
        return 6 + (5 * B) // 2
    if M <= 4:
        return 10 + (13 * B) // 5
    return 20 + 3 * B


def tiles_of(shapes):
    out, t = [], 0
    for N, K in shapes:
        n = (N + ROWS - 1) // ROWS
        out.append((t, n, K))
        t += n
    return out, t


def range_cost(spans, M, a, b):
    """Units plus piece costs of the flat tiles [a, b)."""
    cost = 0
    for t0, n, K in spans:
        lo, hi = max(a, t0), min(b, t0 + n)
        if lo < hi:
            cost += piece_cost(K, M) + (hi - lo) * (K // 1024)
    return cost


def best_bottleneck(spans, total, M, grid):
    """Smallest possible largest range cost over cuts into <= grid ranges
    (exhaustive dynamic programme over cut positions)."""
    inf = float("inf")
    cost = [[0] * (total + 1) for _ in range(total + 1)]
    for a in range(total):
        for b in range(a + 1, total + 1):
            cost[a][b] = range_cost(spans, M, a, b)
    best = [inf] * (total + 1)  # best[b]: first b tiles in the ranges so far
    best[0] = 0
    result = inf
    for _ in range(grid):
        nxt = best[:]  # a range may stay empty
        for b in range(1, total + 1):
            for a in range(b):
                if best[a] < inf:
                    v = max(best[a], cost[a][b])
                    if v < nxt[b]:
                        nxt[b] = v
        best = nxt
        result = min(result, best[total])
    return result


def check_structure(first, total, grid):
    assert len(first) == grid + 1
    assert first[0] == 0 and first[-1] == total
    assert all(first[c] <= first[c + 1] for c in range(grid))


def plan_max_cost(first, spans, M):
    return max(range_cost(spans, M, first[c], first[c + 1]) for c in range(len(first) - 1)
               if first[c] < first[c + 1])


@pytest.mark.parametrize("seed", range(16))
def test_small_cases_reach_the_best_bottleneck(seed):
    rng = random.Random(seed)
    count = rng.randint(1, 5)
    shapes = [(rng.choice([16, 40, 96, 160, 320]), rng.choice([1024, 2048, 5120, 17408])) for _ in range(count)]
    M = rng.choice([1, 2, 3, 4, 6, 8])
    spans, total = tiles_of(shapes)
    for grid in (1, 2, 3, 5, 8):
        first = T.tern_step_plan(shapes, M, grid)
        check_structure(first, total, grid)
        got = plan_max_cost(first, spans, M)
        assert got == best_bottleneck(spans, total, M, grid), (shapes, M, grid, first)


LAYER = [(6144, 5120), (1024, 5120), (1024, 5120), (5120, 6144), (17408, 5120), (17408, 5120), (5120, 17408)]


def greedy_bound(spans, M, grid):
    """Smallest C whose fill-as-much-as-possible cut needs <= grid ranges."""
    def ranges_needed(C):
        n, acc, open_ = 0, 0, False
        for _, ntile, K in spans:
            B, pc, left = K // 1024, piece_cost(K, M), ntile
            while left:
                if open_ and acc + pc + B > C:
                    n, acc = n + 1, 0
                open_ = True
                acc += pc
                take = min(left, max(1, (C - acc) // B))
                acc += take * B
                left -= take
                if left:
                    n, acc, open_ = n + 1, 0, False
        return n + (1 if open_ else 0)
    # (no range costs less than one tile and its product's staging)
    lo = max(K // 1024 + piece_cost(K, M) for _, _, K in spans)
    hi = max(lo, sum(n * (K // 1024 + piece_cost(K, M)) for _, n, K in spans))
    while lo < hi:
        mid = (lo + hi) // 2
        if ranges_needed(mid) <= grid:
            hi = mid
        else:
            lo = mid + 1
    return lo


@pytest.mark.parametrize("M", [1, 2, 4, 8])
@pytest.mark.parametrize("name,shapes", [
    ("layer", LAYER),
    ("gate_up", [(17408, 5120)] * 2),
    ("qkv", LAYER[:3]),
    ("head", [(151936, 5120)]),
    ("k", [(1024, 5120)]),
    ("launch_of_96", (LAYER * 14)[:96]),
])
def test_decode_launches_are_balanced(name, shapes, M):
    spans, total = tiles_of(shapes)
    grid = 148
    first = T.tern_step_plan(shapes, M, grid)
    check_structure(first, total, grid)
    bound = greedy_bound(spans, M, min(grid, total))
    assert plan_max_cost(first, spans, M) <= bound
    used = sum(1 for c in range(grid) if first[c] < first[c + 1])
    assert used == min(grid, total) or used >= grid - 4, (name, M, used)
    if len(shapes) == 1:
        # one product: the tiles are shared as evenly as whole tiles allow
        sizes = [first[c + 1] - first[c] for c in range(grid) if first[c] < first[c + 1]]
        assert max(sizes) - min(sizes) <= 1


def test_rejects_bad_arguments():
    with pytest.raises(T.TernError):
        T.tern_step_plan([(1024, 1000)], 1, 148)  # K not a multiple of 1024
    with pytest.raises(T.TernError):
        T.tern_step_plan([(1024, 5120)], 9, 148)
    with pytest.raises(T.TernError):
        T.tern_step_plan([(1024, 5120)], 1, 0)
    with pytest.raises(T.TernError):
        T.tern_step_plan([(1024, 5120)] * 97, 1, 148)
