"""Oracle: advancing along the accepted branch (test infrastructure).

Definition followed ("Medusa heads versus separate draft model", section
"Acceptance", tree paragraph): decoding continues along the branch that
matches. Reading: the tokens of the accepted path (root, then the L accepted
nodes) join the sequence, so their keys and values must sit contiguously
after the prefix; the bonus token becomes the next step's root; the next
heads read the hidden state of the last accepted node.

For request b with prefix length P and accepted path path[0..L]:

* K/V slot P + i receives the K/V of slot P + path[i], for i = 0..L (the
  root, path[0] = 0, stays where it is); every other slot is unchanged;
* the new prefix length is P + L + 1;
* next_root = bonus;
* next_head_row = b * T + path[L] (the row of that node when the heads ran on
  every tree node, B * T rows).
"""
from __future__ import annotations

import numpy as np


def tree_commit(k_cache, v_cache, prefix_len, accept_len, path, bonus, T: int):
    """Returns (k_cache', v_cache', new_prefix_len, next_root, next_head_row);
    the inputs are not modified."""
    k = np.array(k_cache, copy=True)
    v = np.array(v_cache, copy=True)
    B = k.shape[0]
    new_p = np.zeros(B, dtype=np.int32)
    next_root = np.zeros(B, dtype=np.int32)
    next_row = np.zeros(B, dtype=np.int32)
    for b in range(B):
        P = int(prefix_len[b])
        L = int(accept_len[b])
        src = [P + int(path[b, i]) for i in range(L + 1)]
        k[b, :, P:P + L + 1] = k_cache[b][:, src]
        v[b, :, P:P + L + 1] = v_cache[b][:, src]
        new_p[b] = P + L + 1
        next_root[b] = bonus[b]
        next_row[b] = b * T + int(path[b, L])
    return k, v, new_p, next_root, next_row
