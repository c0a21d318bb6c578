"""Oracle: tree-masked attention over the KV prefix plus the tree (test infrastructure).

Definition followed ("Medusa heads versus separate draft model", section
"Acceptance", tree paragraph): all branches are verified in one pass of the
target with a tree attention mask. A tree token sees the whole KV prefix and,
inside the tree, exactly its ancestors and itself.

Readings where the pages are silent:

* K/V of the tree tokens sit in the cache right after the prefix: node j of
  request b at slot ``prefix_len[b] + j``.
* Grouped-query attention: query head h reads KV head ``h // (Hq / Hkv)``.
* Softmax scale 1/sqrt(dh) unless given; rotary embedding is applied by the
  caller (Q and K arrive rotated).

Per (request, node, query head): scores in fp64, max-subtracted softmax,
weighted sum of V.
"""
from __future__ import annotations

import math

import numpy as np

from .heads import bf16_to_f64
from .tree import ancestors


def tree_attention(q_bits, k_bits, v_bits, prefix_len, parent, scale=None, rows=None):
    """out[b, t, h, :] in fp64, [B, T, Hq, dh].

    q_bits [B, T, Hq, dh]; k_bits, v_bits [B, Hkv, S_max, dh] (bf16 bits).
    ``rows`` optionally lists (b, t, h) triples to compute (others stay NaN).
    """
    B, T, Hq, dh = q_bits.shape
    Hkv = k_bits.shape[1]
    group = Hq // Hkv
    scale = 1.0 / math.sqrt(dh) if not scale else float(scale)
    anc = ancestors(parent)
    out = np.full((B, T, Hq, dh), np.nan)
    want = None if rows is None else {tuple(int(x) for x in r) for r in rows}
    for b in range(B):
        P = int(prefix_len[b])
        for hk in range(Hkv):
            heads = range(hk * group, (hk + 1) * group)
            if want is not None and not any((b, t, h) in want for t in range(T) for h in heads):
                continue
            Kf = bf16_to_f64(k_bits[b, hk, :P + T])
            Vf = bf16_to_f64(v_bits[b, hk, :P + T])
            for t in range(T):
                keys = list(range(P)) + [P + a for a in sorted(anc[t])]
                for h in heads:
                    if want is not None and (b, t, h) not in want:
                        continue
                    qv = bf16_to_f64(q_bits[b, t, h])
                    s = (Kf[keys] @ qv) * scale
                    w = np.exp(s - s.max())
                    out[b, t, h] = (w @ Vf[keys]) / w.sum()
    return out
