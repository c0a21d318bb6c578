"""Oracle: sequentially dependent (Hydra) drafting of the candidate tree
(test infrastructure).

Sources:

* "Medusa heads versus separate draft model", section "Acceptance": a Medusa
  head drafts its token without seeing what the earlier heads drafted, which
  is why its acceptance drops faster with depth than a draft model's.
* "Hydra: Sequentially-Dependent Draft Heads for Medusa Decoding" (abstract):
  Hydra heads are a drop-in replacement for the draft heads in which each
  head's guess is conditioned on the tokens before it in the candidate
  continuation.

Readings (the pages give no Hydra architecture):

* A Hydra head keeps the Medusa head's shape (the d x d residual block with
  its bias, then a d x V projection of its own), so that it is a drop-in
  replacement; what changes is its input. The head that drafts the children
  of tree node p reads ``x_p = bf16(h + E[token_p])``: the request's hidden
  state plus the target's input embedding of p's token (E is [V, d]). The sum
  is formed exactly and rounded once to bf16 (nearest even).
* Only the token directly before the drafted one enters (the parent's token;
  for depth 1 that is the root token). Earlier tokens reach a head only
  through the tree: the drafts differ from branch to branch.
* Node j at depth d with rank r takes the rank-r candidate of head d applied
  to x_parent(j). Ties order as in the Medusa heads: value descending, then
  id ascending.

So the drafting runs depth by depth: the heads of depth d+1 need the tokens
of depth d. Everything is fp64 except the bf16 roundings named above.
"""
from __future__ import annotations

import numpy as np

from . import heads as oh
from . import tree as ot


def head_input(h_row_bits, E_bits, token: int) -> np.ndarray:
    """x = bf16(h + E[token]) as bf16 bits [d]."""
    return oh.f64_to_bf16(oh.bf16_to_f64(h_row_bits) + oh.bf16_to_f64(E_bits[token]))


def head_logits(x_bits, W1_bits, b1_bits, Wv_bits, head: int) -> np.ndarray:
    """Logits [V] of head ``head`` (0-based) on the input row x."""
    z = oh.residual_block(x_bits[None, :], W1_bits[head:head + 1], b1_bits[head:head + 1])   # [1, 1, d]
    return oh.vocab_logits(z, Wv_bits[head:head + 1])[0, 0]


def hydra_draft(parent, head_rank, h_bits, E_bits, W1_bits, b1_bits, Wv_bits, root_token, prefix_len,
                head_row=None):
    """Tokens of every tree node, drafted depth by depth.

    Node order is the tree's (parents before children), so a parent's token is
    known when its children are drafted. The logits of each parent are
    computed once and shared by its children.

    Returns (tokens [B, T] int32, parent [T], ancestor words [T, W] uint32,
    pos [B, T] int32, logits) where ``logits[(b, p)]`` is the fp64 logit row
    of the head that drafted p's children, for every node p with children.
    """
    parent = np.asarray(parent)
    B = len(root_token)
    T = len(parent)
    dep = ot.depths(parent)
    tokens = np.zeros((B, T), dtype=np.int32)
    pos = np.zeros((B, T), dtype=np.int32)
    logits = {}
    for b in range(B):
        row = b if head_row is None else int(head_row[b])
        for j in range(T):
            pos[b, j] = prefix_len[b] + dep[j]
            if j == 0:
                tokens[b, j] = root_token[b]
                continue
            p = int(parent[j])
            if (b, p) not in logits:
                x = head_input(h_bits[row], E_bits, int(tokens[b, p]))
                logits[(b, p)] = head_logits(x, W1_bits, b1_bits, Wv_bits, int(dep[j]) - 1)
            ids, _ = oh.topk(logits[(b, p)], int(head_rank[j]) + 1)
            tokens[b, j] = ids[int(head_rank[j])]
    return tokens, parent.astype(np.int32), ot.ancestor_words(parent), pos, logits
