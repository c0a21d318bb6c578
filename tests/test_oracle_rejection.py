"""Pins of oracle/rejection.py (sampled drafts, lossless acceptance).

What pins it, independently of its own arithmetic:

* The draws: Gumbel-top-k must be sampling without replacement. The first
  candidate's frequency must match q(a) and the ordered pair's frequency
  q(a) q(b) / (1 - q(a)) (closed forms), within 4 sigma over 60k draws.
* Losslessness (the point of rejection sampling, "Medusa heads versus
  separate draft model", section "Training"): over many runs with random
  drafts and random acceptance uniforms, the first emitted token must follow
  the root's target row p, and, given that an accepted child emitted token a,
  the next token must follow that child's target row. A wrong ratio direction,
  a missing renormalisation of q after a rejected sibling, or a wrong residual
  each fails these.
* Limiting cases: a head equal to the target accepts its first draft always;
  a target concentrated on a token no head drafts rejects every child and
  emits that token.
"""
import numpy as np
import pytest

from oracle import rejection as orj


def _freq_ok(counts, probs, n):
    sigma = np.sqrt(probs * (1 - probs) / n)
    return np.all(np.abs(counts / n - probs) <= 4 * sigma + 1e-12), (counts / n, probs)


def test_gumbel_top2_is_sampling_without_replacement():
    rng = np.random.default_rng(0)
    V, N, tau = 5, 60000, 0.8
    x = rng.normal(0, 1, V)
    q = np.exp(x / tau) / np.exp(x / tau).sum()
    u = rng.random((N, 1, V))
    ids, keys = orj.sampled_drafts(np.broadcast_to(x, (N, 1, V)), (2,), 2, tau, u)
    assert np.all(np.diff(keys[:, 0, :], axis=1) <= 0)
    first = np.bincount(ids[:, 0, 0], minlength=V)
    ok, info = _freq_ok(first, q, N)
    assert ok, info
    pair = np.zeros((V, V))
    np.add.at(pair, (ids[:, 0, 0], ids[:, 0, 1]), 1)
    expect = np.array([[q[a] * q[b] / (1 - q[a]) if a != b else 0.0 for b in range(V)] for a in range(V)])
    ok, info = _freq_ok(pair.ravel(), expect.ravel(), N)
    assert ok, info
    assert np.all(np.diag(pair) == 0)              # never the same token twice


def _tiny_tree():
    # root -> 3 children (ranks 0, 1, 2); child rank 0 -> 2 children; child rank 1 -> 1 child
    parent = [-1, 0, 0, 0, 1, 1, 2]
    rank = [0, 0, 1, 2, 0, 1, 0]
    return parent, rank


def _simulate(N, V, seed, p_root, p_next, q_heads, tau=1.0, tau_q=1.0):
    """N independent runs of drafting + acceptance on the tiny tree. Target
    row of node j is p_root at the root, else p_next[token of j] (the target
    depends on the emitted token only). Returns acc_len, path, bonus, tokens."""
    rng = np.random.default_rng(seed)
    parent, rank = _tiny_tree()
    T, K = len(parent), 2
    depth = [0, 1, 1, 1, 2, 2, 2]
    hl = np.broadcast_to(np.log(q_heads), (N, K, V)).astype(np.float64)
    ids, _ = orj.sampled_drafts(hl, (3, 2), 3, tau_q, rng.random((N, K, V)))
    tokens = np.zeros((N, T), dtype=np.int64)
    for j in range(1, T):
        tokens[:, j] = ids[:, depth[j] - 1, rank[j]]
    tl = np.empty((N, T, V))
    tl[:, 0] = np.log(p_root) * tau
    for j in range(1, T):
        tl[:, j] = np.log(p_next[tokens[:, j]]) * tau
    acc, path, bonus, _ = orj.rejection_accept(tl, tokens, parent, rank, K, tau, hl, np.arange(N), tau_q,
                                                rng.random((N, T)), rng.random((N, T)))
    return acc, path, bonus, tokens


def test_acceptance_keeps_the_target_distribution():
    rng = np.random.default_rng(3)
    V, N = 6, 40000
    p_root = rng.dirichlet(np.ones(V))
    p_next = rng.dirichlet(np.ones(V), size=V)          # target after emitting token a
    q_heads = rng.dirichlet(np.ones(V), size=2)         # unrelated draft heads
    acc, path, bonus, tokens = _simulate(N, V, 11, p_root, p_next, q_heads)
    first = np.where(acc >= 1, tokens[np.arange(N), np.maximum(path[:, 1], 0)], bonus)
    ok, info = _freq_ok(np.bincount(first, minlength=V), p_root, N)
    assert ok, info
    # second emitted token, given that an accepted depth-1 child emitted a
    second = np.where(acc >= 2, tokens[np.arange(N), np.maximum(path[:, 2], 0)], bonus)
    tested = 0
    for a in range(V):
        sel = (acc >= 1) & (first == a)
        n = int(sel.sum())
        if n < 2000:
            continue
        ok, info = _freq_ok(np.bincount(second[sel], minlength=V), p_next[a], n)
        assert ok, (a, info)
        tested += 1
    assert tested >= 2
    assert 0.05 < np.mean(acc >= 1) < 0.95          # both outcomes exercised


def test_temperatures_apply_to_their_own_rows():
    """Target at temperature 0.6, heads at 1.3: the first emitted token follows
    softmax(target logits / 0.6)."""
    rng = np.random.default_rng(5)
    V, N, tau, tau_q = 5, 40000, 0.6, 1.3
    z = rng.normal(0, 1, V)
    p_root = np.exp(z / tau) / np.exp(z / tau).sum()
    p_next = rng.dirichlet(np.ones(V), size=V)
    q_heads = rng.dirichlet(np.ones(V), size=2)
    acc, path, bonus, tokens = _simulate(N, V, 12, p_root, p_next, q_heads, tau=tau, tau_q=tau_q)
    first = np.where(acc >= 1, tokens[np.arange(N), np.maximum(path[:, 1], 0)], bonus)
    ok, info = _freq_ok(np.bincount(first, minlength=V), p_root, N)
    assert ok, info


def test_head_equal_to_target_accepts_its_first_draft():
    rng = np.random.default_rng(7)
    V, N = 7, 300
    p = rng.dirichlet(np.ones(V))
    acc, path, bonus, tokens = _simulate(N, V, 13, p, np.broadcast_to(p, (V, V)), np.stack([p, p]))
    assert np.all(acc == 2)                       # both depths accept
    assert np.all(path[:, 1] == 1) and np.all(np.isin(path[:, 2], [4]))   # always rank 0


def test_target_on_an_undrafted_token_rejects_everything():
    V, N = 6, 200
    q_heads = np.array([[0.25, 0.25, 0.25, 0.25, 0.0, 0.0]] * 2) + 1e-300
    p_root = np.full(V, 1e-30)
    p_root[5] = 1.0
    p_root /= p_root.sum()
    acc, path, bonus, tokens = _simulate(N, V, 14, p_root, np.full((V, V), 1.0 / V), q_heads)
    assert np.all(acc == 0) and np.all(bonus == 5)
    assert np.all(tokens[:, 1:4] <= 3)


def test_rejects_children_that_skip_a_rank():
    with pytest.raises(ValueError):
        orj.rejection_accept(np.zeros((1, 3, 4)), np.zeros((1, 3), dtype=int), [-1, 0, 0], [0, 0, 2], 1, 1.0,
                             np.zeros((1, 1, 4)), [0], 1.0, np.zeros((1, 3)), np.zeros((1, 3)))
