"""Pins for the oracle's KV compaction (CPU only)."""
import math

import numpy as np
import torch
import torch.nn.functional as F

from oracle import attention as oa
from oracle import commit as oc
from oracle import tree as ot
from seeded_inputs import gen
from seeded_inputs.workloads import TREE_ACCEPT


def _caches(seed, B, Hkv, S, dh):
    k = gen.normal_bf16(seed, "k_cache", (B, Hkv, S, dh), 1.0)
    v = gen.normal_bf16(seed, "v_cache", (B, Hkv, S, dh), 1.0)
    return k, v


def _f64(bits):
    return torch.from_numpy(gen.bf16_bits_to_f32(bits).astype(np.float64))


def test_chain_commit_is_identity_on_the_cache():
    k, v = _caches(1, 2, 2, 40, 64)
    P = np.array([10, 20])
    path = np.array([[0, 1, 2, -1, -1], [0, -1, -1, -1, -1]])
    L = np.array([2, 0])
    k2, v2, newp, root, row = oc.tree_commit(k, v, P, L, path, np.array([7, 8]), T=5)
    assert np.array_equal(k2, k) and np.array_equal(v2, v)
    assert list(newp) == [13, 21] and list(root) == [7, 8] and list(row) == [2, 5]


def test_overlapping_moves_read_the_original_slots():
    """path 0, 2, 5: slot P+2 is both a source (for i = 1) and a destination."""
    k, v = _caches(2, 1, 1, 16, 64)
    P = np.array([4])
    k2, v2, newp, _, row = oc.tree_commit(k, v, P, np.array([2]), np.array([[0, 2, 5]]), np.array([1]), T=6)
    assert np.array_equal(k2[0, 0, 5], k[0, 0, 6])      # P + 1 <- P + 2
    assert np.array_equal(k2[0, 0, 6], k[0, 0, 9])      # P + 2 <- P + 5
    assert np.array_equal(k2[0, 0, :5], k[0, 0, :5]) and np.array_equal(k2[0, 0, 7:], k[0, 0, 7:])
    assert newp[0] == 7 and row[0] == 5


def test_committed_cache_gives_the_tree_attention_of_the_last_node():
    """After advancing, the accepted tokens are an ordinary causal sequence:
    plain attention of the last accepted node's query over slots [0, P+L+1)
    of the compacted cache equals the tree-masked attention of that node over
    the original cache."""
    tups = ot.select_tree((4, 3, 2, 2), TREE_ACCEPT, 16)
    parent, _, depth = ot.spec_from_tuples(tups)
    T, B, Hq, Hkv, dh, S = len(parent), 2, 4, 2, 64, 80
    q = gen.normal_bf16(3, "q", (B, T, Hq, dh), 1.0)
    k, v = _caches(3, B, Hkv, S, dh)
    P = np.array([30, 55])
    ref = oa.tree_attention(q, k, v, P, parent)
    for node in range(T):
        pth, n = [], node
        while n != -1:
            pth.append(n)
            n = int(parent[n])
        pth = pth[::-1]
        L = len(pth) - 1
        path = np.full((B, 5), -1)
        path[:, :L + 1] = pth
        k2, v2, newp, _, _ = oc.tree_commit(k, v, P, np.array([L, L]), path, np.array([0, 0]), T)
        for b in range(B):
            n_keys = newp[b]
            for h in range(Hq):
                hk = h // (Hq // Hkv)
                out = F.scaled_dot_product_attention(_f64(q[b, node, h])[None, None], _f64(k2[b, hk, :n_keys])[None],
                                                     _f64(v2[b, hk, :n_keys])[None], scale=1 / math.sqrt(dh))[0, 0]
                assert np.max(np.abs(out.numpy() - ref[b, node, h])) < 1e-12
