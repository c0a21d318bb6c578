"""Pins for the oracle's candidate tree (CPU only)."""
import itertools

import numpy as np
import pytest

from oracle import tree as ot
from seeded_inputs.workloads import TREE_ACCEPT


def test_chain_tree_is_top1_per_depth():
    tups = ot.select_tree((1, 1, 1, 1), TREE_ACCEPT, 4)
    assert tups == [(0,), (0, 0), (0, 0, 0), (0, 0, 0, 0)]
    parent, rank, depth = ot.spec_from_tuples(tups)
    assert list(parent) == [-1, 0, 1, 2, 3] and list(depth) == [0, 1, 2, 3, 4]


def test_64_node_tree_shape():
    """Depth profile of the 64-candidate tree from top-10 heads.

    Independent derivation: with a = (.80, .65, .50, .40) the kept depth-1
    ranks are 0..9 (all of them), and the counts per depth are 10/31/18/5.
    """
    tups = ot.select_tree((10, 10, 10, 10), TREE_ACCEPT, 64)
    counts = [sum(1 for t in tups if len(t) == d) for d in range(1, 5)]
    assert counts == [10, 31, 18, 5]
    assert max(t[0] for t in tups if len(t) == 1) == 9


def _score_float(t, a):
    s = 1.0
    for i, r in enumerate(t):
        s *= a[i] / (r + 1)
    return s


@pytest.mark.parametrize("kph,n", [((4, 3, 2, 2), 16), ((10, 10, 10, 10), 64),
                                   ((10, 10, 10, 10), 16), ((3, 3, 3), 20)])
def test_selected_set_is_a_best_prefix(kph, n):
    """Every kept tuple scores at least as high as every dropped one, and the
    set is closed under parents; node order is (depth, tuple)."""
    a = TREE_ACCEPT
    tups = ot.select_tree(kph, a, n)
    assert len(tups) == n and len(set(tups)) == n
    kept = set(tups)
    allt = [t for d in range(1, len(kph) + 1) for t in itertools.product(*[range(k) for k in kph[:d]])]
    lo = min(_score_float(t, a) for t in tups)
    hi = max(_score_float(t, a) for t in allt if t not in kept)
    assert lo >= hi - 1e-12
    for t in tups:
        assert len(t) == 1 or t[:-1] in kept
    assert tups == sorted(tups, key=lambda t: (len(t), t))
    parent, rank, depth = ot.spec_from_tuples(tups)
    for j in range(1, n + 1):
        assert parent[j] < j


def test_ancestor_sets_follow_the_parent_recursion():
    rng = np.random.default_rng(3)
    for _ in range(50):
        T = int(rng.integers(1, 130))
        parent = [-1] + [int(rng.integers(0, j)) for j in range(1, T)]
        anc = ot.ancestors(parent)
        words = ot.ancestor_words(parent)
        dep = ot.depths(parent)
        assert words.shape == (T, (T + 31) // 32)
        for j in range(T):
            want = {j} if j == 0 else anc[parent[j]] | {j}
            assert anc[j] == want
            bits = {w * 32 + b for w in range(words.shape[1]) for b in range(32) if (int(words[j, w]) >> b) & 1}
            assert bits == anc[j]
            assert len(bits) == dep[j] + 1


def test_tree_build_tokens_decode_to_head_and_rank():
    """topk_ids encodes (row, head, rank); each token must decode to the
    row of its request, head = depth - 1 and the node's own rank."""
    tups = ot.select_tree((4, 3, 2, 2), TREE_ACCEPT, 16)
    parent, rank, depth = ot.spec_from_tuples(tups)
    M, K, kmax = 5, 4, 4
    ids = np.array([[[1000 * m + 100 * k + r for r in range(kmax)] for k in range(K)] for m in range(M)])
    head_row = np.array([3, 0, 4])
    root = np.array([7, 8, 9])
    P = np.array([10, 0, 33])
    tokens, par, anc, pos = ot.tree_build(parent, rank, ids, root, P, head_row=head_row)
    for b in range(3):
        assert tokens[b, 0] == root[b]
        for j in range(1, len(parent)):
            t = int(tokens[b, j])
            assert t // 1000 == head_row[b]
            assert (t % 1000) // 100 == len(tups[j - 1]) - 1
            assert t % 100 == tups[j - 1][-1]
        assert list(pos[b] - P[b]) == list(depth)
    assert list(par) == list(parent)
