"""Draft-tree sizing on a verify-cost staircase (nvfp4_weight_gemm_b200.staircut), on the host.

Pins: the geometric closed form of a chain's expected tokens, brute force over every subtree of
small random trees, and what the pages' own staircase implies (a pass of 16 rows costs less than
one of 8, so 15 nodes always beat 7 when the tree has them)."""

import itertools
import json
import random

import pytest

from nvfp4_weight_gemm_b200 import staircut as sc

# the post's GB10 staircase at 1k context: verify ms by rows
GB10 = sc.Staircase({8: 75.5, 16: 74.4, 24: 83.1, 32: 87.8})


def random_tree(rng, n, lo=0.0, hi=1.0):
    parents = [-1] + [rng.randrange(-1, i) for i in range(1, n)]
    accept = [rng.uniform(lo, hi) for _ in range(n)]
    return parents, accept


def test_chain_expected_tokens_closed_form():
    # a chain of n nodes, each accepted with p given its parent: 1 + p (1 - p^n) / (1 - p)
    for p in (0.1, 0.5, 0.9):
        for n in (1, 7, 15, 31):
            parents = [-1] + list(range(n - 1))
            got = sc.expected_tokens(parents, [p] * n, range(n))
            assert got == pytest.approx(1.0 + p * (1.0 - p ** n) / (1.0 - p), rel=1e-12)


def _subtrees(parents, n):
    # every set of n nodes that holds each member's parent
    for combo in itertools.combinations(range(len(parents)), n):
        s = set(combo)
        if all(parents[i] < 0 or parents[i] in s for i in combo):
            yield combo


def test_cut_is_the_best_subtree_brute_force():
    rng = random.Random(5)
    for _ in range(60):
        size = rng.randrange(1, 10)
        parents, accept = random_tree(rng, size)
        pp = sc.path_probs(parents, accept)
        for n in range(1, size + 1):
            cut = sc.cut_tree(parents, accept, n)
            assert len(cut) == n
            assert all(parents[i] < 0 or parents[i] in cut for i in cut), "cut is not a subtree"
            best = max(sum(pp[i] for i in s) for s in _subtrees(parents, n))
            assert sum(pp[i] for i in cut) == pytest.approx(best, rel=1e-12, abs=1e-15)


def test_ties_keep_parents_first():
    # acceptance 1 gives a child its parent's path probability: the parent (lower index) is kept
    parents = [-1, 0, 1, -1]
    accept = [0.5, 1.0, 1.0, 0.5]
    cut = sc.cut_tree(parents, accept, 2)
    assert cut == [0, 1]


def test_pages_staircase_prefers_15_over_7():
    rng = random.Random(7)
    for _ in range(200):
        parents, accept = random_tree(rng, rng.randrange(15, 60))
        c = sc.choose(parents, accept, GB10)
        assert c.size != 7, "16 rows cost less than 8 on the pages' staircase"
        assert c.rows == c.size + 1 and c.size in sc.SNAP_NODES


def test_flat_price_takes_the_largest_tree_and_steep_price_the_smallest():
    parents = [-1] + list(range(39))
    flat = sc.Staircase({8: 10.0, 16: 10.0, 24: 10.0, 32: 10.0})
    assert sc.choose(parents, [0.9] * 40, flat).size == 31
    steep = sc.Staircase({8: 10.0, 16: 40.0, 24: 160.0, 32: 640.0})
    assert sc.choose(parents, [0.3] * 40, steep).size == 7


def test_overhead_and_small_trees():
    parents, accept = [-1, 0, 0], [0.8, 0.5, 0.4]
    c = sc.choose(parents, accept, GB10, overhead_ms=2.0)
    assert c.size == 3 and c.rows == 4 and c.ms == pytest.approx(75.5 + 2.0)
    assert c.tokens == pytest.approx(1.0 + 0.8 + 0.4 + 0.32)
    with pytest.raises(ValueError):
        sc.choose(parents, accept, GB10, overhead_ms=-1.0)


def test_staircase_pricing_and_bench_line():
    st = sc.Staircase({1: 1.8, 8: 1.9, 16: 2.0, 32: 2.1})
    assert st.cost_ms(1) == 1.8 and st.cost_ms(2) == 1.9 and st.cost_ms(9) == 2.0 and st.cost_ms(17) == 2.1
    with pytest.raises(ValueError):
        st.cost_ms(33)
    with pytest.raises(ValueError):
        st.cost_ms(0)
    line = json.dumps({"metric": "m", "staircase": {"1": {"us": 1800.0}, "32": {"us": 2100.0}}})
    assert sc.Staircase.from_bench_line(line).ms == {1: 1.8, 32: 2.1}


def test_invalid_trees_are_refused():
    with pytest.raises(ValueError):
        sc.path_probs([-1, 1], [0.5, 0.5])          # parent not before the node
    with pytest.raises(ValueError):
        sc.path_probs([-1], [1.5])                   # acceptance outside [0, 1]
    with pytest.raises(ValueError):
        sc.path_probs([-1, 0], [0.5])                # lengths differ


def test_report_on_a_staircase():
    flat = sc.Staircase({m: 2.0 for m in range(1, 33)})
    r = sc.report(flat)
    assert set(r) == {"p=0.3", "p=0.5", "p=0.7", "p=0.9"}
    assert all(v["nodes"] == 31 and v["rows"] == 32 for v in r.values())   # flat price: the largest tree
    r2 = sc.report(GB10)
    assert all(v["nodes"] in sc.SNAP_NODES and v["nodes"] != 7 for v in r2.values())
