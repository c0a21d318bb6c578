"""Host-side choice of a fixed candidate tree.

"Medusa heads versus separate draft model" (section "Acceptance", tree
paragraph) combines the top few candidates of each head into a tree but does
not say which combinations a fixed N-node tree keeps. This module keeps the N
rank tuples (r_1, ..., r_k) with the largest ``prod_i a_i / (r_i + 1)`` (a_i
the expected acceptance at depth i), ties broken by depth, then by the tuple.
A child never outscores its parent and a rank never outscores a lower rank of
the same parent, so a best-first expansion from the root visits tuples in
exactly that order; scores are exact rationals.
"""
from __future__ import annotations

import heapq
from fractions import Fraction


def select_tree(k_per_head, accept, n_nodes: int):
    """Rank tuples of the n_nodes candidates, in node order (root excluded)."""
    K = len(k_per_head)
    a = [Fraction(str(x)) for x in accept]

    def key(score, tup):
        return (-score, len(tup), tup)

    heap = [key(a[0], (0,))]
    seen = {(0,)}
    picked = []
    while heap and len(picked) < n_nodes:
        negs, _, tup = heapq.heappop(heap)
        score = -negs
        picked.append(tup)
        d = len(tup)
        # next sibling: same parent, next rank
        if tup[-1] + 1 < k_per_head[d - 1]:
            sib = tup[:-1] + (tup[-1] + 1,)
            if sib not in seen:
                seen.add(sib)
                heapq.heappush(heap, key(score * (tup[-1] + 1) / (tup[-1] + 2), sib))
        # first child: rank 0 of the next head
        if d < K:
            ch = tup + (0,)
            if ch not in seen:
                seen.add(ch)
                heapq.heappush(heap, key(score * a[d], ch))
    if len(picked) < n_nodes:
        raise ValueError("tree larger than all rank combinations")
    return sorted(picked, key=lambda t: (len(t), t))


def tree_arrays(tuples):
    """parent and head_rank lists (root first) for the C ABI."""
    index = {(): 0}
    for j, t in enumerate(tuples, start=1):
        index[tuple(t)] = j
    parent = [-1] + [index[tuple(t)[:-1]] for t in tuples]
    rank = [0] + [t[-1] for t in tuples]
    return parent, rank
