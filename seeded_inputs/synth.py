"""Synthetic stand-ins for what the target model would produce.

There is no target model, no trained head and no dataset here, so the target's
logits are drawn from the seeded generator and the acceptance profile is
*planted* into them. Nothing in this file computes a step of the Medusa method;
it only decides where the target's argmax lies before either side runs.

Planting rule, for each request ``b`` and each tree node ``p`` that has
children (``depth(p) = d``):

* draw ``u`` uniform in [0, 1) (stream ``plant``, index ``b*T + p``);
* if ``u < accept[d]`` one child ``c`` of ``p`` is picked uniformly
  (stream ``plant_pick``) and ``logits[b, p, tokens[b, c]]`` is set to
  ``rowmax + bump`` (fp32 add), so the target's greedy token after ``p`` is
  that child's token;
* otherwise a token that is *not* the token of any child of ``p`` is picked
  uniformly and raised the same way, so no child of ``p`` matches.

Rows of nodes without children keep their drawn values. With this rule the
expected accepted length along a top-1 chain is exactly
``1 + a1 + a1 a2 + a1 a2 a3 + a1 a2 a3 a4``.
"""
from __future__ import annotations

import numpy as np

from .gen import (normal_f32, stream_key, uniform_int_at, uniform_unit_at)


def node_depths(parent) -> np.ndarray:
    parent = np.asarray(parent)
    depth = np.zeros(len(parent), dtype=np.int64)
    for j in range(1, len(parent)):
        depth[j] = depth[parent[j]] + 1
    return depth


def children_lists(parent):
    ch = [[] for _ in range(len(parent))]
    for j in range(1, len(parent)):
        ch[int(parent[j])].append(j)
    return ch


def synthetic_tree_tokens(seed: int, B: int, parent, V: int, root_tokens=None) -> np.ndarray:
    """Token ids for every tree node, distinct among siblings, int32 [B, T]."""
    T = len(parent)
    key = stream_key(seed, "tokens")
    ch = children_lists(parent)
    out = np.zeros((B, T), dtype=np.int64)
    for b in range(B):
        if root_tokens is None:
            out[b, 0] = uniform_int_at(key, np.array([b * T * 16]), V)[0]
        else:
            out[b, 0] = root_tokens[b]
        for p in range(T):
            used = set()
            for c in ch[p]:
                attempt = 0
                while True:
                    t = int(uniform_int_at(key, np.array([(b * T + c) * 16 + 1 + attempt]), V)[0])
                    attempt += 1
                    if t not in used:
                        break
                used.add(t)
                out[b, c] = t
    return out.astype(np.int32)


def plant_choices(seed: int, parent, tokens, V: int, accept):
    """The planting decisions: (b, p, x) = raise token x of row (b, p)."""
    tokens = np.asarray(tokens)
    B, T = tokens.shape
    depth = node_depths(parent)
    ch = children_lists(parent)
    kp = stream_key(seed, "plant")
    kq = stream_key(seed, "plant_pick")
    out = []
    for b in range(B):
        for p in range(T):
            if not ch[p]:
                continue
            idx = np.array([b * T + p])
            u = float(uniform_unit_at(kp, idx)[0])
            child_tokens = sorted({int(tokens[b, c]) for c in ch[p]})
            if u < accept[int(depth[p])]:
                c = ch[p][int(uniform_int_at(kq, idx, len(ch[p]))[0])]
                x = int(tokens[b, c])
            else:
                j = int(uniform_int_at(kq, idx, V - len(child_tokens))[0])
                for t in child_tokens:  # j-th token id that is not a child token
                    if t <= j:
                        j += 1
                x = j
            out.append((b, p, x))
    return out


def planted_logits(seed: int, parent, tokens, V: int, accept, sigma: float = 1.0,
                   bump: float = 1.0, logits: np.ndarray | None = None) -> np.ndarray:
    """Target logits fp32 [B, T, V] with the acceptance profile planted.

    ``accept[d]`` is the probability that the target's greedy token after a
    node of depth ``d`` is the token of one of its children.
    """
    tokens = np.asarray(tokens)
    B, T = tokens.shape
    if logits is None:
        logits = normal_f32(seed, "logits", (B, T, V), sigma)
    bump32 = np.float32(bump)
    for b, p, x in plant_choices(seed, parent, tokens, V, accept):
        row = logits[b, p]
        row[x] = np.float32(np.float32(row.max()) + bump32)
    return logits


def planted_logits_device(seed: int, parent, tokens, V: int, accept, sigma: float = 1.0,
                          bump: float = 1.0, device="cuda"):
    """The same tensor as planted_logits, drawn and planted on the GPU (torch
    float32 tensor): the draws come from the device twin of the generator and
    each planted value is the same fp32 sum row max + bump."""
    import torch

    from .device import fill_normal
    tokens = np.asarray(tokens)
    B, T = tokens.shape
    logits = fill_normal(torch.empty((B, T, V), dtype=torch.float32, device=device), seed, "logits", sigma)
    ch = plant_choices(seed, parent, tokens, V, accept)
    if ch:
        b = torch.tensor([c[0] for c in ch], device=device)
        p = torch.tensor([c[1] for c in ch], device=device)
        x = torch.tensor([c[2] for c in ch], device=device)
        top = logits[b, p].amax(dim=-1)
        logits[b, p, x] = top + torch.tensor(bump, dtype=torch.float32, device=device)
    return logits


def prefix_lengths(seed: int, B: int, lo: int, hi: int) -> np.ndarray:
    """Per-request KV prefix lengths uniform in [lo, hi], int32 [B]."""
    from .gen import uniform_int
    if lo == hi:
        return np.full(B, lo, dtype=np.int32)
    return uniform_int(seed, "prefix_len", (B,), lo, hi).astype(np.int32)


def root_tokens(seed: int, B: int, V: int) -> np.ndarray:
    from .gen import uniform_int
    return uniform_int(seed, "root_token", (B,), 0, V - 1).astype(np.int32)
