"""Draft-tree size on a measured verify-cost staircase (host side).

StairCut (the author's "Research" page, the entry "StairCut: sizing speculative draft trees on
a measured verification-cost staircase", "What it says"; and the author's post announcing the
engine and the paper) prices each speculative round on the measured cost of a verify pass as a
function of its row count, a staircase rather than a line, and cuts the round's candidate tree
to the node count that gives the most expected committed tokens per millisecond, choosing among
7, 15, 23 and 31 nodes. A tree of n nodes is verified together with the current token, so it
costs one pass of n + 1 rows (8, 16, 24 or 32: the staircase's steps in the post).

What the pages leave open, and the reading taken here:
- The acceptance model. Each node carries the probability that the target model accepts it
  given that its parent was accepted (from the drafters' confidences, or any other estimate);
  a node's path probability is the product along its path from the root. The expected number
  of committed tokens of a cut tree is 1 (the token the verify pass always yields) plus the sum
  of its nodes' path probabilities.
- The cut. For a given node count the best subtree keeps the nodes with the largest path
  probabilities: a node's path probability never exceeds its parent's, so those nodes always
  form a subtree (ties go to the lower index; nodes are numbered parents first).
- The price. A round costs the verify pass of n + 1 rows from the measured staircase plus a
  fixed per-round overhead (drafting, sampling) that the caller supplies; the staircase itself
  comes from the verify GEMM's own measurements (``bench.py``'s ``staircase``).
- A tree with fewer nodes than a size is offered at its own node count, priced at its own rows.
"""

from __future__ import annotations

import json
from dataclasses import dataclass
from typing import Dict, List, Optional, Sequence, Tuple

SNAP_NODES: Tuple[int, ...] = (7, 15, 23, 31)


@dataclass(frozen=True)
class Staircase:
    """Measured time of one verify pass (ms) by row count M. A row count that was not measured
    is priced at the next measured one above it (a pass of M rows costs at least what the
    kernel's tile for M costs); above the largest measured M there is no price."""

    ms: Dict[int, float]

    def cost_ms(self, rows: int) -> float:
        if rows < 1:
            raise ValueError("a verify pass has at least one row")
        for m in sorted(self.ms):
            if m >= rows:
                return self.ms[m]
        raise ValueError(f"no measured verify cost for {rows} rows (largest measured: {max(self.ms)})")

    @staticmethod
    def from_bench_line(line: str) -> "Staircase":
        """From one JSON line of ``bench.py``: its ``staircase`` (median µs per stack pass by M)."""
        d = json.loads(line)
        return Staircase({int(m): float(v["us"]) / 1000.0 for m, v in d["staircase"].items()})


def path_probs(parents: Sequence[int], accept: Sequence[float]) -> List[float]:
    """Path probability of every node: accept[i] times its parent's (parents[i] = -1 for a child
    of the root). Nodes must be numbered parents first (parents[i] < i)."""
    if len(parents) != len(accept):
        raise ValueError("parents and accept differ in length")
    out: List[float] = []
    for i, (p, a) in enumerate(zip(parents, accept)):
        if not (0.0 <= a <= 1.0):
            raise ValueError(f"node {i}: acceptance {a} outside [0, 1]")
        if p >= i or p < -1:
            raise ValueError(f"node {i}: parent {p} must be -1 or a lower index")
        out.append(a if p < 0 else a * out[p])
    return out


def cut_tree(parents: Sequence[int], accept: Sequence[float], n: int) -> List[int]:
    """The n nodes (or all, if fewer) with the largest path probabilities, ties to the lower
    index, in increasing order: a subtree that contains every kept node's parent."""
    pp = path_probs(parents, accept)
    order = sorted(range(len(pp)), key=lambda i: (-pp[i], i))
    return sorted(order[:max(0, n)])


def expected_tokens(parents: Sequence[int], accept: Sequence[float], nodes: Sequence[int]) -> float:
    """Expected committed tokens of a round that verifies `nodes`: 1 + their path probabilities."""
    pp = path_probs(parents, accept)
    return 1.0 + sum(pp[i] for i in nodes)


@dataclass(frozen=True)
class Choice:
    nodes: List[int]          # the kept nodes
    size: int                 # their count
    rows: int                 # verify rows (size + 1)
    tokens: float             # expected committed tokens
    ms: float                 # price of the round
    tokens_per_ms: float


def choose(parents: Sequence[int], accept: Sequence[float], stair: Staircase, overhead_ms: float = 0.0,
           sizes: Sequence[int] = SNAP_NODES) -> Choice:
    """The cut of the candidate tree with the most expected committed tokens per millisecond
    among the allowed sizes (ties to the smaller size)."""
    if overhead_ms < 0.0:
        raise ValueError("overhead_ms must be >= 0")
    n_nodes = len(parents)
    best: Optional[Choice] = None
    for size in sorted(set(min(s, n_nodes) for s in sizes)):
        nodes = cut_tree(parents, accept, size)
        tok = expected_tokens(parents, accept, nodes)
        ms = stair.cost_ms(len(nodes) + 1) + overhead_ms
        c = Choice(nodes, len(nodes), len(nodes) + 1, tok, ms, tok / ms)
        if best is None or c.tokens_per_ms > best.tokens_per_ms:
            best = c
    assert best is not None
    return best


def report(stair: Staircase, overhead_ms: float = 0.0, accept: Sequence[float] = (0.3, 0.5, 0.7, 0.9),
           n_nodes: int = 40) -> Dict[str, Dict[str, float]]:
    """The cut chosen on `stair` for chains of `n_nodes` drafts each accepted with probability p
    given its parent, for each p: a summary of what the staircase implies for the tree size."""
    out: Dict[str, Dict[str, float]] = {}
    parents = [-1] + list(range(n_nodes - 1))
    for p in accept:
        c = choose(parents, [p] * n_nodes, stair, overhead_ms)
        out[f"p={p:g}"] = {"nodes": c.size, "rows": c.rows, "tokens": round(c.tokens, 4),
                           "ms": round(c.ms, 4), "tokens_per_ms": round(c.tokens_per_ms, 4)}
    return out
