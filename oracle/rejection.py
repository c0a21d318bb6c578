"""Oracle: drafts sampled from the heads' own distributions, and lossless
acceptance of the tree by rejection sampling (test infrastructure).

Source: "Medusa heads versus separate draft model", section "Training": when
the output must follow the target's distribution exactly, standard rejection
sampling is used instead of typical acceptance. The page gives no algorithm
for a tree of drafts; this module takes the following readings.

Drafts. Head d (0-based; it drafts depth d + 1 of the tree) has the
distribution q_d = softmax(x_d / tau_q) over its logits x_d. Its k_d
candidates are k_d draws from q_d without replacement, in draw order. They are
made with the Gumbel-top-k construction (Gumbel-max, extended to several
draws): with one uniform u[v] in (0, 1) per token, supplied by the caller,

    key[v] = x_d[v] / tau_q - ln(-ln u[v]),

and the candidates are the k_d tokens of largest key, by key descending (ties
to the lower id). The i-th candidate is then distributed as q_d restricted to
the tokens not drawn before it, renormalised. A node of depth d + 1 and rank r
takes candidate r of head d, as in the Medusa tree.

Acceptance, at a tree node t whose children c_1 .. c_m carry the ranks
0 .. m - 1 of the next head (their tokens y_1 .. y_m are that head's first m
draws). With p = softmax(z_t / tau) the target's row for t:

    r_1 = p
    for i = 1 .. m:
        q_i = q restricted to the tokens other than y_1 .. y_{i-1}, renormalised
        child c_i is accepted iff  u_acc[c_i] < r_i(y_i) / q_i(y_i)
            (probability min(1, r_i / q_i): rejection sampling of r_i by q_i)
        otherwise  r_{i+1} = max(0, r_i - q_i) / sum(max(0, r_i - q_i))

If c_i is accepted its token is emitted and the walk continues at c_i. If no
child is accepted, or t has no children, one token is drawn from r_{m+1} (from
p at a leaf) by inverse CDF in id order with the uniform u_res[t], emitted as
the bonus token, and the walk stops. Each round is one step of standard
rejection sampling with target r_i and proposal q_i, so the token emitted
after t follows p exactly (the reading is pinned by simulation in the tests).
L counts the accepted nodes; the path lists the root and the accepted nodes.

All arithmetic is fp64; logits arrive as fp32 values.
"""
from __future__ import annotations

import numpy as np


def softmax(row, temperature: float) -> np.ndarray:
    x = np.asarray(row, dtype=np.float64) / temperature
    e = np.exp(x - x.max())
    return e / e.sum()


def gumbel_keys(logits_row, temperature: float, uniforms_row) -> np.ndarray:
    """key[v] = x[v] / tau - ln(-ln u[v]) (fp64)."""
    x = np.asarray(logits_row, dtype=np.float64)
    u = np.asarray(uniforms_row, dtype=np.float64)
    return x / temperature - np.log(-np.log(u))


def sampled_drafts(head_logits, k_per_head, kmax: int, temperature: float, uniforms):
    """Candidates of every (row, head): head_logits and uniforms [M, K, V].

    Returns ids int32 [M, K, kmax] (-1 padded) and keys [M, K, kmax] (-inf
    padded), each head's k candidates by key descending, ties to the lower id.
    """
    M, K, V = head_logits.shape
    ids = np.full((M, K, kmax), -1, dtype=np.int32)
    keys = np.full((M, K, kmax), -np.inf)
    for m in range(M):
        for k in range(K):
            key = gumbel_keys(head_logits[m, k], temperature, uniforms[m, k])
            order = np.lexsort((np.arange(V), -key))[:k_per_head[k]]
            ids[m, k, :len(order)] = order
            keys[m, k, :len(order)] = key[order]
    return ids, keys


def children_by_rank(parent, rank):
    """Children of every node ordered by head rank."""
    T = len(parent)
    ch = [[] for _ in range(T)]
    for j in range(1, T):
        ch[int(parent[j])].append(j)
    return [sorted(c, key=lambda j: int(rank[j])) for c in ch]


def inverse_cdf(weights, u: float):
    """The smallest id v with sum_{w <= v} weights[w] > u * sum(weights), and
    the distance (in units of the total) from u to the nearer end of v's
    interval."""
    w = np.asarray(weights, dtype=np.float64)
    total = w.sum()
    cdf = np.cumsum(w) / total
    v = int(np.searchsorted(cdf, u, side="right"))
    if v >= len(w):
        v = int(np.flatnonzero(w > 0)[-1])
    lo = cdf[v - 1] if v > 0 else 0.0
    return v, float(min(u - lo, cdf[v] - u))


def rejection_accept(target_logits, tokens, parent, rank, K: int, temperature: float, head_logits, head_row,
                     temperature_q: float, u_acc, u_res):
    """Lossless acceptance of sampled drafts.

    target_logits [B, T, V] (row t: the target after node t), tokens [B, T],
    head_logits [M, K, V] with head_row [B] (the row whose drafts built request
    b's tree), u_acc / u_res [B, T] uniforms in [0, 1).

    Returns accept_len [B], path [B, K+1] (-1 padded), bonus [B], and per
    request a list of the decisions taken, each (node, ratio, u) for an
    acceptance test or (node, margin) for the bonus draw, so a caller can see
    how far each decision was from its threshold.
    """
    B, T, V = target_logits.shape
    ch = children_by_rank(parent, rank)
    for c in ch:
        if [int(rank[j]) for j in c] != list(range(len(c))):
            raise ValueError("every node's children must carry the ranks 0 .. m-1")
    acc_len = np.zeros(B, dtype=np.int32)
    path = np.full((B, K + 1), -1, dtype=np.int32)
    bonus = np.zeros(B, dtype=np.int32)
    decisions = []
    for b in range(B):
        node, depth, steps, log = 0, 0, [0], []
        while True:
            p = softmax(target_logits[b, node], temperature)
            r = p.copy()
            accepted = None
            if ch[node]:
                q = softmax(head_logits[int(head_row[b]), depth], temperature_q)
                removed = np.zeros(V, dtype=bool)
                for c in ch[node]:
                    y = int(tokens[b, c])
                    qi = np.where(removed, 0.0, q)
                    qi = qi / qi.sum()
                    ratio = r[y] / qi[y]
                    log.append((c, float(ratio), float(u_acc[b, c])))
                    if u_acc[b, c] < ratio:
                        accepted = c
                        break
                    res = np.maximum(r - qi, 0.0)
                    r = res / res.sum()
                    removed[y] = True
            if accepted is None:
                y, margin = inverse_cdf(r, float(u_res[b, node]))
                log.append((node, margin))
                bonus[b] = y
                break
            steps.append(accepted)
            node, depth = accepted, depth + 1
        acc_len[b] = len(steps) - 1
        path[b, :len(steps)] = steps
        decisions.append(log)
    return acc_len, path, bonus, decisions
