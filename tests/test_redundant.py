"""Redundant experts (618zxw.cn news article on DeepSeek-V3: the most loaded
experts are duplicated for inference load balance).  CPU pins of the
oracle's reading (copies minimise the largest rows per copy; an expert's
rows cut into near-equal consecutive pieces) by brute force, and the
library's host planner against the oracle (it runs on the host: no GPU)."""
import itertools

import numpy as np
import pytest

import oracle


def _best_max_load(counts, n_extra):
    """Brute force: the smallest achievable max_e ceil(c_e / r_e)."""
    N = len(counts)
    best = None
    for extra in itertools.product(range(n_extra + 1), repeat=N):
        if sum(extra) != n_extra:
            continue
        m = max(-(-c // (1 + x)) for c, x in zip(counts, extra))
        best = m if best is None else min(best, m)
    return best


@pytest.mark.parametrize("seed", range(40))
def test_plan_reaches_the_brute_force_optimum(seed):
    rng = np.random.default_rng(seed)
    N = int(rng.integers(1, 5))
    R = int(rng.integers(0, 6))
    counts = rng.integers(0, 40, N).tolist()
    rep, slots = oracle.redundant_plan(counts, R)
    assert rep.sum() == N + R and np.all(rep >= 1)
    assert np.array_equal(slots, np.repeat(np.arange(N), rep))
    assert max(-(-c // r) for c, r in zip(counts, rep)) == _best_max_load(counts, R)


def test_split_pieces_cover_each_expert_in_order():
    off = np.array([0, 10, 10, 17, 40, 50], np.int32)  # 4 experts + shared rows
    rep = np.array([3, 2, 1, 4], np.int32)
    so, sw = oracle.split_groups(off, rep)
    # counts 10, 0, 7, 23 with 3, 2, 1, 4 copies; shared rows [40, 50)
    assert so.tolist() == [0, 4, 7, 10, 10, 10, 17, 23, 29, 35, 40, 50]
    assert sw.tolist() == [0, 0, 0, 1, 1, 2, 3, 3, 3, 3, 4]
    sizes = np.diff(so)
    assert sizes.tolist() == [4, 3, 3, 0, 0, 7, 6, 6, 6, 5, 10]


def test_library_planner_matches_the_oracle():
    import fp8_block_scaled_affinity_b200 as moe
    rng = np.random.default_rng(9)
    for _ in range(50):
        N = int(rng.integers(1, 300))
        R = int(rng.integers(0, 64))
        counts = (rng.zipf(1.3, N) * rng.integers(1, 50)).clip(0, 2 ** 20).tolist()
        rep, slots = moe.moe_plan_redundant_experts(counts, R)
        rep_o, slots_o = oracle.redundant_plan(counts, R)
        assert np.array_equal(rep, rep_o) and np.array_equal(slots, slots_o)


def test_skewed_batch_load_is_spread():
    """The motivating case: on the skewed batch one expert serves every
    token; 64 extra copies bring the largest rows per copy from 16384 down
    to the brute-force-free bound ceil(total / slots) or the next-hottest
    expert's share."""
    counts = [0] * 256
    counts[0], counts[1], counts[2] = 16384, 12000, 4000
    rep, _ = oracle.redundant_plan(counts, 64)
    worst = max(-(-c // r) for c, r in zip(counts, rep))
    assert worst <= 16384 // 32
