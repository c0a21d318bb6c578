"""Pins for the oracle's acceptance rules (CPU only).

* The page's expected-length formula E = 1 + a1 + a1 a2 + a1 a2 a3 + a1 a2 a3 a4
  and its table values, reproduced by Monte-Carlo on planted top-1 chains.
* The same expectation on trees, against a closed-form recursion.
* Brute-force path enumeration against the parent-recursion form.
* Typical acceptance: limiting cases and closed-form entropies.
"""
import json
import math
import os

import numpy as np
import pytest

from oracle import accept as oacc
from oracle import tree as ot
from seeded_inputs import synth
from seeded_inputs.workloads import TREE_ACCEPT


def _parent_recursion(match, parent):
    """acc[j] = acc[parent j] and match[j]; L = deepest accepted depth; ties
    to the smallest node index."""
    T = len(parent)
    acc = [True] + [False] * (T - 1)
    depth = [0] * T
    for j in range(1, T):
        depth[j] = depth[parent[j]] + 1
        acc[j] = acc[parent[j]] and match[j]
    L = max(depth[j] for j in range(T) if acc[j])
    node = min(j for j in range(T) if acc[j] and depth[j] == L)
    return L, node


def test_path_enumeration_equals_parent_recursion():
    rng = np.random.default_rng(5)
    for _ in range(400):
        T = int(rng.integers(1, 40))
        parent = [-1] + [int(rng.integers(max(0, j - 6), j)) for j in range(1, T)]
        match = [False] + list(rng.random(T - 1) < 0.6)
        K = int(ot.depths(parent).max())
        L, path = oacc._walk_paths(match, parent, K)
        L2, node = _parent_recursion(match, parent)
        assert (L, path[-1]) == (L2, node)
        assert len(path) == L + 1 and path[0] == 0
        for a, b in zip(path[:-1], path[1:]):
            assert parent[b] == a


def test_chain_counts_leading_matches():
    """On a chain, greedy verification accepts the drafts up to the first
    mismatch (textbook speculative decoding)."""
    rng = np.random.default_rng(6)
    parent = [-1, 0, 1, 2, 3]
    V = 20
    for _ in range(200):
        logits = rng.standard_normal((1, 5, V)).astype(np.float32)
        amax = logits[0].argmax(axis=1)
        tokens = rng.integers(0, V, (1, 5))
        flip = rng.random(5) < 0.7
        tokens[0, 1:] = np.where(flip[1:], amax[:-1], tokens[0, 1:])
        L, path, bonus, _ = oacc.greedy_accept(logits, tokens, parent, 4)
        want = 0
        for j in range(1, 5):
            if tokens[0, j] != amax[j - 1]:
                break
            want += 1
        assert L[0] == want
        assert list(path[0, :want + 1]) == list(range(want + 1))
        assert bonus[0] == amax[want]


def test_argmax_ties_go_to_lowest_id():
    row = np.array([1.0, 3.0, -2.0, 3.0, 3.0], dtype=np.float32)
    assert oacc.argmax_lowest_id(row) == 1


def _mc_expected_length(parent, accept, n, seed, V=32):
    tokens = synth.synthetic_tree_tokens(seed, n, parent, V)
    logits = synth.planted_logits(seed, parent, tokens, V, accept)
    K = int(ot.depths(parent).max())
    L, _, _, _ = oacc.greedy_accept(logits, tokens, parent, K)
    x = L.astype(np.float64) + 1
    return x.mean(), x.std() / math.sqrt(n)


def _page_rows(golden_dir):
    with open(os.path.join(golden_dir, "paper_figures.json")) as f:
        return json.load(f)["acceptance_table"]["rows"]


@pytest.mark.parametrize("row", [0, 1, 2])
def test_expected_length_matches_page_table(golden_dir, row):
    r = _page_rows(golden_dir)[row]
    a = r["accept"]
    exact = 1 + a[0] + a[0] * a[1] + a[0] * a[1] * a[2] + a[0] * a[1] * a[2] * a[3]
    assert round(exact, 2) == r["E"]
    mean, se = _mc_expected_length([-1, 0, 1, 2, 3], a, 20000, seed=100 + row)
    assert abs(mean - exact) <= 4 * se, (mean, exact, se)
    # and the page's speedup column is E / cost
    assert round(r["E"] / r["cost"], 2) == pytest.approx(r["speedup"], abs=0.011)


def _closed_form_tree_E(parent, accept):
    T = len(parent)
    ch = [[] for _ in range(T)]
    for j in range(1, T):
        ch[parent[j]].append(j)
    dep = ot.depths(parent)

    def f(p):
        if not ch[p]:
            return 0.0
        return accept[dep[p]] * (1 + sum(f(c) for c in ch[p]) / len(ch[p]))

    return 1 + f(0)


def test_expected_length_on_tiny_tree():
    tups = ot.select_tree((4, 3, 2, 2), TREE_ACCEPT, 16)
    parent, _, _ = ot.spec_from_tuples(tups)
    exact = _closed_form_tree_E(list(parent), TREE_ACCEPT)
    assert abs(exact - 2.4002) < 1e-4       # value derived independently for this tree rule
    mean, se = _mc_expected_length(list(parent), TREE_ACCEPT, 12000, seed=7)
    assert abs(mean - exact) <= 4 * se


def test_typical_limits():
    tups = ot.select_tree((4, 3, 2, 2), TREE_ACCEPT, 16)
    parent, _, _ = ot.spec_from_tuples(tups)
    T = len(parent)
    V = 64
    rng = np.random.default_rng(8)
    logits = (3 * rng.standard_normal((3, T, V))).astype(np.float32)
    tokens = synth.synthetic_tree_tokens(9, 3, parent, V)
    depth = int(ot.depths(parent).max())
    L, path, bonus, _ = oacc.typical_accept(logits, tokens, parent, 4, 0.7, 0.0, 0.3)
    assert list(L) == [depth] * 3                       # threshold 0: every child passes
    L, path, bonus, _ = oacc.typical_accept(logits, tokens, parent, 4, 0.7, 1.0, 1e30)
    assert list(L) == [0] * 3                           # threshold 1: nothing passes
    for b in range(3):
        assert bonus[b] == oacc.argmax_lowest_id(logits[b, 0])


def test_typical_on_uniform_rows():
    """All-equal logits: p = 1/V and H = ln V, so the threshold is
    min(eps, alpha / V)."""
    V = 50
    parent = [-1, 0]
    logits = np.zeros((1, 2, V), dtype=np.float32)
    tokens = np.array([[3, 4]])
    p, H = oacc.typical_stats(logits[0, 0], 0.7)
    assert abs(H - math.log(V)) < 1e-12 and abs(p[4] - 1 / V) < 1e-15
    L, _, _, m = oacc.typical_accept(logits, tokens, parent, 1, 0.7, 0.09, 0.3)   # thr 0.006 < 0.02
    assert L[0] == 1 and abs(m[0, 1] - (0.02 - 0.006) / 0.006) < 1e-9
    L, _, _, _ = oacc.typical_accept(logits, tokens, parent, 1, 0.7, 0.09, 1.5)   # thr 0.03 > 0.02
    assert L[0] == 0
    L, _, _, _ = oacc.typical_accept(logits, tokens, parent, 1, 0.7, 0.01, 1.5)   # thr eps 0.01
    assert L[0] == 1


def test_typical_stats_two_level_row():
    V, top, tau = 10, 2.0, 0.5
    row = np.zeros(V, dtype=np.float32)
    row[6] = top
    p, H = oacc.typical_stats(row, tau)
    e = math.exp(top / tau)
    p1 = e / (e + V - 1)
    q = 1 / (e + V - 1)
    assert abs(p[6] - p1) < 1e-15 and abs(p[0] - q) < 1e-15
    assert abs(H - (-p1 * math.log(p1) - (V - 1) * q * math.log(q))) < 1e-13


# ------------------------- sampled (lossless) acceptance -------------------------

def test_inverse_cdf_on_exact_rows():
    """Rows whose probabilities are exact binary fractions: the draw is the
    smallest id whose CDF exceeds u, ids with zero probability are never drawn
    and a draw of u exactly on a boundary goes to the next id."""
    row = np.zeros(4)                                   # p = 1/4 each, CDF .25 .5 .75 1
    for u, v in [(0.0, 0), (0.2499, 0), (0.25, 1), (0.5, 2), (0.7499, 2), (0.75, 3), (0.99999, 3)]:
        assert oacc.inverse_cdf_sample(row, 1.0, u)[0] == v, u
    row = np.array([0.0, -np.inf, 0.0, 0.0])            # p = 1/3, 0, 1/3, 1/3
    assert [oacc.inverse_cdf_sample(row, 1.0, u)[0] for u in (0.1, 0.34, 0.7)] == [0, 2, 3]
    # temperature divides the logits: logits (0, 2 ln 3) at temperature 2 give p = (1/4, 3/4)
    row = np.array([0.0, 2 * math.log(3.0)])
    assert oacc.inverse_cdf_sample(row, 2.0, 0.249)[0] == 0
    assert oacc.inverse_cdf_sample(row, 2.0, 0.251)[0] == 1


def test_sampled_acceptance_reproduces_the_target_distribution():
    """Rejection sampling must leave the target's sampling distribution intact:
    over many uniform draws, the first emitted token (the accepted child's
    token, else the bonus) follows the root row's softmax, and the token after
    an accepted child follows that child's row."""
    V = 5
    parent = np.array([-1, 0, 0, 1])                    # root -> {1, 2}; 1 -> {3}
    tokens = np.array([[0, 1, 3, 2]])
    rng = np.random.default_rng(7)
    logits = rng.normal(0.0, 1.0, (1, 4, V))
    tau = 0.8
    N = 20000
    u = rng.random((N, 4))
    first, second_after_1 = [], []
    for i in range(N):
        L, path, bonus, y, _ = oacc.sampled_accept(logits, tokens, parent, 2, tau, u[i][None, :])
        emitted = [int(tokens[0, j]) for j in path[0, 1:L[0] + 1]] + [int(bonus[0])]
        first.append(emitted[0])
        if emitted[0] == 1:
            second_after_1.append(emitted[1])
    for counts, row in ((np.bincount(first, minlength=V), logits[0, 0]),
                        (np.bincount(second_after_1, minlength=V), logits[0, 1])):
        p, _ = oacc.typical_stats(row, tau)
        n = counts.sum()
        sigma = np.sqrt(n * p * (1 - p))
        assert np.all(np.abs(counts - n * p) <= 5 * sigma + 1), (counts, n * p)


def test_sampled_acceptance_tends_to_greedy_at_low_temperature():
    """With well-separated logits and a temperature near zero every draw is the
    argmax, so the sampled rule accepts exactly what the greedy rule accepts."""
    kph, n = (4, 3, 2, 2), 16
    parent, _, _ = ot.spec_from_tuples(ot.select_tree(kph, TREE_ACCEPT, n))
    tokens = synth.synthetic_tree_tokens(3, 4, parent, 64)
    logits = synth.planted_logits(3, parent, tokens, 64, TREE_ACCEPT, bump=4.0)
    g = oacc.greedy_accept(logits, tokens, parent, 4)
    u = np.random.default_rng(1).random((4, len(parent)))
    s = oacc.sampled_accept(logits, tokens, parent, 4, 1e-3, u)
    for i in range(3):
        assert np.array_equal(g[i], s[i])
