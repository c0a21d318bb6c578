"""Oracle: acceptance of the longest matching branch (test infrastructure).

Definition followed ("Medusa heads versus separate draft model", section
"Acceptance", tree paragraph): the target checks the whole tree in a single
pass, and decoding continues along a branch that matches. Row t of the target logits is the
target's distribution for the token after node t, so a non-root node j matches
when its token is what the target emits after its parent.

Greedy rule: j matches iff ``tokens[j] == argmax(logits[parent(j)])``, argmax
taking the lowest id among equal maxima (the comparison is on the given fp32
values, which is exact). Every root-to-leaf path is enumerated; along a path
the accepted length is the number of leading matching nodes below the root.
L is the largest such count; the accepted path ends at the depth-L node with
the smallest node index. The bonus token is the argmax of the last accepted
node's row (the root's row when L = 0).

Typical rule (same page, section "Training": typical acceptance trades the
target distribution for more accepted drafts; the page gives no formula). Reading: with ``p = softmax(logits / temperature)`` of the parent's
row and its entropy ``H = -sum p ln p``, child j matches iff
``p(tokens[j]) > min(eps, alpha * exp(-H))`` (strict, natural log). Same path
rule; the bonus token is still the greedy argmax. This rule is parity
unpinned against the pages: only its limiting cases are fixed.

Sampled (lossless) rule (same section: the page recommends rejection sampling
when the target distribution must be kept exactly, and gives no algorithm for a
tree of deterministic candidates). Reading: rejection sampling of a candidate chosen with certainty
(a point-mass draft q = delta_c) accepts it with probability p(c) and, on
rejection, samples from p with c removed; over the candidate children of a node
in turn this is the same as drawing one token y from p = softmax(logits /
temperature) of the node's row and accepting the child whose token is y. So
each row t gets one draw ``y_t = min{v : sum_{w <= v} p(w) > u_t}`` (inverse
CDF in id order) from a supplied uniform u_t in [0, 1); node j matches iff
``tokens[j] == y[parent(j)]``; same path rule; the bonus token is y of the last
accepted node. The emitted tokens then follow the target's own sampling
distribution exactly (pinned by simulation in the tests).
"""
from __future__ import annotations

import numpy as np

from .tree import depths


def argmax_lowest_id(row) -> int:
    row = np.asarray(row)
    return int(np.flatnonzero(row == row.max())[0])


def root_to_leaf_paths(parent):
    """Every path from the root to a node without children, as node lists."""
    T = len(parent)
    children = [[] for _ in range(T)]
    for j in range(1, T):
        children[int(parent[j])].append(j)
    paths = []

    def walk(n, prefix):
        prefix = prefix + [n]
        if not children[n]:
            paths.append(prefix)
        for c in children[n]:
            walk(c, prefix)

    walk(0, [])
    return paths


def _walk_paths(match, parent, K):
    """Longest accepted prefix over all root-to-leaf paths.

    match[j] says whether non-root node j passes its test against its parent.
    Returns (L, path node list).
    """
    best_len, best_node, best_path = -1, None, None
    for path in root_to_leaf_paths(parent):
        L = 0
        for j in path[1:]:
            if not match[j]:
                break
            L += 1
        node = path[L]
        if L > best_len or (L == best_len and node < best_node):
            best_len, best_node, best_path = L, node, path[:L + 1]
    return best_len, best_path


def greedy_accept(logits, tokens, parent, K: int):
    """accept_len [B], path [B, K+1] (-1 padded), bonus [B], amax [B, T]."""
    B, T, _ = logits.shape
    amax = np.array([[argmax_lowest_id(logits[b, t]) for t in range(T)] for b in range(B)])
    acc_len = np.zeros(B, dtype=np.int32)
    path = np.full((B, K + 1), -1, dtype=np.int32)
    bonus = np.zeros(B, dtype=np.int32)
    for b in range(B):
        match = [False] + [int(tokens[b, j]) == int(amax[b, parent[j]]) for j in range(1, T)]
        L, p = _walk_paths(match, parent, K)
        acc_len[b] = L
        path[b, :L + 1] = p
        bonus[b] = amax[b, p[-1]]
    return acc_len, path, bonus, amax


def typical_stats(row, temperature):
    """p = softmax(row / temperature) and its entropy H (fp64)."""
    x = np.asarray(row, dtype=np.float64) / temperature
    e = np.exp(x - x.max())
    p = e / e.sum()
    nz = p > 0
    H = -np.sum(p[nz] * np.log(p[nz]))
    return p, H


def typical_accept(logits, tokens, parent, K: int, temperature: float, eps: float, alpha: float):
    """Like greedy_accept, plus the per-node relative margin (p - thr) / thr
    (NaN at the root), so a caller can see decisions that sit near the
    threshold. Returns (accept_len, path, bonus, margin)."""
    B, T, _ = logits.shape
    acc_len = np.zeros(B, dtype=np.int32)
    path = np.full((B, K + 1), -1, dtype=np.int32)
    bonus = np.zeros(B, dtype=np.int32)
    margin = np.full((B, T), np.nan)
    for b in range(B):
        stats = [typical_stats(logits[b, t], temperature) for t in range(T)]
        match = [False]
        for j in range(1, T):
            p, H = stats[int(parent[j])]
            thr = min(eps, alpha * np.exp(-H))
            pj = p[int(tokens[b, j])]
            with np.errstate(divide="ignore"):
                margin[b, j] = (pj - thr) / thr if thr > 0 else np.inf
            match.append(bool(pj > thr))
        L, pth = _walk_paths(match, parent, K)
        acc_len[b] = L
        path[b, :L + 1] = pth
        bonus[b] = argmax_lowest_id(logits[b, pth[-1]])
    return acc_len, path, bonus, margin


def tree_depth(parent) -> int:
    return int(depths(parent).max())


def inverse_cdf_sample(row, temperature: float, u: float):
    """One draw from p = softmax(row / temperature) (fp64): the smallest id v
    with sum_{w <= v} p(w) > u; if rounding leaves u at or above the total, the
    last id with p > 0. Returns (v, margin), margin = the distance from u to
    the nearer end of v's CDF interval (how far the decision is from a tie)."""
    p, _ = typical_stats(row, temperature)
    cdf = np.cumsum(p)
    v = int(np.searchsorted(cdf, u, side="right"))
    if v >= len(p):
        v = int(np.flatnonzero(p > 0)[-1])
    lo = cdf[v - 1] if v > 0 else 0.0
    return v, float(min(u - lo, cdf[v] - u))


def sampled_accept(logits, tokens, parent, K: int, temperature: float, uniforms):
    """Sampled acceptance. Returns (accept_len [B], path [B, K+1], bonus [B],
    y [B, T] (each row's draw), margin [B, T])."""
    B, T, _ = logits.shape
    y = np.zeros((B, T), dtype=np.int64)
    margin = np.zeros((B, T))
    acc_len = np.zeros(B, dtype=np.int32)
    path = np.full((B, K + 1), -1, dtype=np.int32)
    bonus = np.zeros(B, dtype=np.int32)
    for b in range(B):
        for t in range(T):
            y[b, t], margin[b, t] = inverse_cdf_sample(logits[b, t], temperature, float(uniforms[b, t]))
        match = [False] + [int(tokens[b, j]) == int(y[b, parent[j]]) for j in range(1, T)]
        L, pth = _walk_paths(match, parent, K)
        acc_len[b] = L
        path[b, :L + 1] = pth
        bonus[b] = y[b, pth[-1]]
    return acc_len, path, bonus, y, margin
