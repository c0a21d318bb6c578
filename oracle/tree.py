"""Oracle: the candidate tree (test infrastructure).

Definition followed ("Medusa heads versus separate draft model", section
"Acceptance", tree paragraph): each head offers its best-scoring candidates and
their combinations make up the tree; head k guesses independently of heads
1..k-1 ("What each one is"), so a node at depth k is a tuple of ranks
(r_1, ..., r_k), and its token is the rank-r_k candidate of head k.

Readings where the pages are silent:

* Which combinations make up a fixed N-node tree is not stated. The oracle
  keeps the N rank tuples with the largest ``prod_i a_i / (r_i + 1)`` (a_i is
  the per-depth acceptance of the workload), ties broken by depth and then by
  the tuple in lexicographic order; scores are exact rationals. A child's
  score never exceeds its parent's, so the kept set is closed under parents.
* Node order: the root, then the kept tuples by (depth, tuple).
* N counts candidates; the root is an extra node, so T = N + 1 tokens.
* Position ids are prefix length + depth (the root sits at the prefix length).
"""
from __future__ import annotations

import itertools
from fractions import Fraction

import numpy as np


def _score(tup, accept):
    s = Fraction(1)
    for depth, r in enumerate(tup):
        s *= Fraction(str(accept[depth])) / (r + 1)
    return s


def select_tree(k_per_head, accept, n_nodes: int):
    """The n_nodes rank tuples of the tree, in node order (root excluded).

    Brute force: every tuple of every depth is scored and sorted.
    """
    K = len(k_per_head)
    allt = []
    for depth in range(1, K + 1):
        for tup in itertools.product(*[range(k) for k in k_per_head[:depth]]):
            allt.append(tup)
    if n_nodes > len(allt):
        raise ValueError("tree larger than all rank combinations")
    allt.sort(key=lambda t: (-_score(t, accept), len(t), t))
    kept = allt[:n_nodes]
    keep = set(kept)
    for t in kept:
        if len(t) > 1 and t[:-1] not in keep:
            raise AssertionError("selected set is not closed under parents")
    return sorted(kept, key=lambda t: (len(t), t))


def spec_from_tuples(tuples):
    """parent, head_rank and depth arrays (length T, node 0 = root)."""
    index = {(): 0}
    for j, t in enumerate(tuples, start=1):
        index[tuple(t)] = j
    T = len(tuples) + 1
    parent = np.full(T, -1, dtype=np.int32)
    rank = np.zeros(T, dtype=np.int32)
    depth = np.zeros(T, dtype=np.int32)
    for t, j in index.items():
        if j == 0:
            continue
        parent[j] = index[t[:-1]]
        rank[j] = t[-1]
        depth[j] = len(t)
    return parent, rank, depth


def ancestors(parent):
    """anc[j] = the set of j and every node on the path from the root to j."""
    T = len(parent)
    out = []
    for j in range(T):
        s = set()
        n = j
        while n != -1:
            s.add(n)
            n = int(parent[n])
        out.append(s)
    return out


def depths(parent):
    return np.array([len(a) - 1 for a in ancestors(parent)], dtype=np.int32)


def ancestor_words(parent) -> np.ndarray:
    """Ancestor mask as bitsets: bit j%32 of word j//32 of row i is set iff
    j is an ancestor of i or i itself. uint32 [T, ceil(T/32)]."""
    T = len(parent)
    W = (T + 31) // 32
    out = np.zeros((T, W), dtype=np.uint32)
    for i, a in enumerate(ancestors(parent)):
        for j in a:
            out[i, j // 32] |= np.uint32(1 << (j % 32))
    return out


def tree_build(parent, head_rank, topk_ids, root_token, prefix_len, head_row=None):
    """tokens [B, T], parent [T], ancestor words [T, W], positions [B, T].

    tokens[b, 0] is the request's root token; a node at depth d with rank r
    takes ``topk_ids[row_b, d - 1, r]``; row_b is ``head_row[b]`` or b.
    """
    parent = np.asarray(parent)
    B = len(root_token)
    T = len(parent)
    dep = depths(parent)
    tokens = np.zeros((B, T), dtype=np.int32)
    pos = np.zeros((B, T), dtype=np.int32)
    for b in range(B):
        row = b if head_row is None else int(head_row[b])
        for j in range(T):
            if j == 0:
                tokens[b, j] = root_token[b]
            else:
                tokens[b, j] = topk_ids[row, dep[j] - 1, head_rank[j]]
            pos[b, j] = prefix_len[b] + dep[j]
    return tokens, parent.astype(np.int32), ancestor_words(parent), pos
