"""Oracle: the K Medusa draft heads and the per-head top-k (test infrastructure).

Definition followed ("Medusa heads versus separate draft model", sections
"What each one is" and "Cost per step"): head k applies a residual block
to the target's last hidden state h and then a d x V vocabulary projection of
its own.
The block is read as ``z_k = h + SiLU(h W1_k + b1_k)`` (a d x d layer plus a
bias: 67.1M parameters at d = 8,192); the projection has no bias (1,050.7M =
d x V exactly). Head k drafts the token k places ahead, and every head reads the
same h in a single parallel pass.

Readings where the pages are silent:

* W1 is stored input-major: ``u_o = b1_o + sum_i h_i W1[k, i, o]``; Wv is
  ``Wv[k, i, v]`` (also input-major).
* z is rounded to bf16 (round to nearest even) before the projection; the
  logits are kept in full precision (fp64 here).
* Top-k orders by value descending, then token id ascending (ties go to the
  lower id). Inputs are finite.

All arithmetic is fp64; weights and activations arrive as bf16 bit patterns
(uint16) and are widened exactly.
"""
from __future__ import annotations

import numpy as np


def bf16_to_f64(bits) -> np.ndarray:
    """Exact value of bf16 bit patterns."""
    u32 = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u32.view(np.float32).astype(np.float64)


def f64_to_bf16(x) -> np.ndarray:
    """Round fp64 values directly to bf16 (nearest, ties to even).

    Works on the fp64 bit pattern: the 52-bit fraction is rounded to bf16's 7
    bits, after which the value is exactly an fp32 whose top half is the bf16
    pattern. Values below bf16's normal range (other than zero) do not occur
    in these workloads and are rejected rather than rounded.
    """
    x = np.ascontiguousarray(x, dtype=np.float64)
    tiny = (x != 0) & (np.abs(x) < 2.0 ** -126)
    if np.any(tiny):
        raise ValueError("f64_to_bf16: subnormal bf16 result")
    b = x.view(np.uint64)
    keep = np.uint64(45)
    lsb = (b >> keep) & np.uint64(1)
    r = (b + (np.uint64(1) << np.uint64(44)) - np.uint64(1) + lsb) & ~((np.uint64(1) << keep) - np.uint64(1))
    y = r.view(np.float64).astype(np.float32)           # exact: at most 8 significant bits
    return (y.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def silu(u: np.ndarray) -> np.ndarray:
    """SiLU(u) = u * sigmoid(u) = u / (1 + e^-u)."""
    with np.errstate(over="ignore"):
        return u / (1.0 + np.exp(-u))


def residual_block(h_bits, W1_bits, b1_bits, cols=None) -> np.ndarray:
    """z[m, k, :] = bf16(h[m] + SiLU(h[m] W1[k] + b1[k])) as bf16 bits [M, K, d].

    ``cols`` optionally restricts the output to those hidden units (the
    result is then [M, K, len(cols)]).
    """
    d = h_bits.shape[1]
    cols = np.arange(d) if cols is None else np.asarray(cols)
    return residual_block_columns(h_bits, W1_bits[:, :, cols], b1_bits[:, cols], cols)


def residual_block_columns(h_bits, W1c_bits, b1c_bits, cols) -> np.ndarray:
    """The residual block for the hidden units ``cols`` only, given their
    weight columns ``W1c[k] = W1[k][:, cols]`` and biases ``b1c[k] = b1[k][cols]``.
    Returns z bits [M, K, len(cols)]."""
    h = bf16_to_f64(h_bits)                                   # [M, d]
    K = W1c_bits.shape[0]
    M = h.shape[0]
    cols = np.asarray(cols)
    z = np.empty((M, K, len(cols)), dtype=np.uint16)
    for k in range(K):
        u = h @ bf16_to_f64(W1c_bits[k]) + bf16_to_f64(b1c_bits[k])[None, :]
        z[:, k, :] = f64_to_bf16(h[:, cols] + silu(u))
    return z


def vocab_logits(z_bits, Wv_bits, cols=None, col_chunk: int = 16384) -> np.ndarray:
    """logits[m, k, v] = sum_i z[m, k, i] Wv[k, i, v] in fp64, [M, K, V].

    ``cols`` optionally restricts the output to a list of vocabulary ids (the
    result is then [M, K, len(cols)]).
    """
    M, K, d = z_bits.shape
    V = Wv_bits.shape[2]
    z = bf16_to_f64(z_bits)
    if cols is not None:
        cols = np.asarray(cols)
        out = np.empty((M, K, len(cols)))
        for k in range(K):
            out[:, k, :] = z[:, k, :] @ bf16_to_f64(Wv_bits[k][:, cols])
        return out
    out = np.empty((M, K, V))
    for k in range(K):
        for lo in range(0, V, col_chunk):
            hi = min(V, lo + col_chunk)
            out[:, k, lo:hi] = z[:, k, :] @ bf16_to_f64(Wv_bits[k, :, lo:hi])
    return out


def topk(values, k: int):
    """The k largest entries of a 1-D array: ids and values, ordered by
    (value descending, id ascending)."""
    values = np.asarray(values)
    ids = np.arange(values.shape[0])
    order = np.lexsort((ids, -values))[:k]
    return order.astype(np.int64), values[order]


def heads_topk(logits, k_per_head, kmax: int):
    """Per-head top-k of logits [M, K, V] -> ids int32 [M, K, kmax] (unused
    slots -1) and values [M, K, kmax] (unused slots -inf)."""
    M, K, _ = logits.shape
    ids = np.full((M, K, kmax), -1, dtype=np.int32)
    vals = np.full((M, K, kmax), -np.inf)
    for m in range(M):
        for k in range(K):
            i, v = topk(logits[m, k], k_per_head[k])
            ids[m, k, :len(i)] = i
            vals[m, k, :len(v)] = v
    return ids, vals


def medusa_heads(h_bits, W1_bits, b1_bits, Wv_bits, k_per_head, kmax=None):
    """The whole draft stage: residual blocks, projections and top-k.

    Returns (topk_ids, topk_vals, logits, z_bits).
    """
    kmax = max(k_per_head) if kmax is None else kmax
    z = residual_block(h_bits, W1_bits, b1_bits)
    logits = vocab_logits(z, Wv_bits)
    ids, vals = heads_topk(logits, k_per_head, kmax)
    return ids, vals, logits, z


def medusa_heads_shared(h_bits, W1_bits, b1_bits, Wv_bits, k_per_head, kmax=None):
    """The draft stage with one vocabulary projection shared by every head.

    Source: "Medusa heads versus separate draft model", section "What
    interviewers probe next": each head normally has its own projection;
    sharing one saves (K - 1) d V parameters at some cost to acceptance. The
    residual blocks stay per head; Wv_bits is [d, V].
    Returns (topk_ids, topk_vals, logits, z_bits).
    """
    kmax = max(k_per_head) if kmax is None else kmax
    z = residual_block(h_bits, W1_bits, b1_bits)
    K = z.shape[1]
    logits = vocab_logits(z, np.broadcast_to(Wv_bits, (K,) + Wv_bits.shape))
    ids, vals = heads_topk(logits, k_per_head, kmax)
    return ids, vals, logits, z


def head_parameter_counts(d: int, V: int, K: int):
    """Parameter counts of the heads as this oracle shapes them.

    Returns (residual block, vocabulary projection, one head, all K heads).
    The shapes are W1 [d, d], b1 [d], Wv [d, V]; no projection bias.
    """
    block = d * d + d
    proj = d * V
    return block, proj, block + proj, K * (block + proj)
