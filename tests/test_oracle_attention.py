"""Pins for the oracle's tree attention (CPU only).

The oracle builds each query's key set from the ancestor sets. These checks
reach the same numbers by other routes: torch's scaled_dot_product_attention
in fp64 with a plain or causal mask, and brute-force gathering of the
sequence [prefix, root .. t].
"""
import math

import numpy as np
import torch
import torch.nn.functional as F

from oracle import attention as oa
from oracle import tree as ot
from seeded_inputs import gen
from seeded_inputs.workloads import TREE_ACCEPT


def _inputs(seed, B, T, Hq, Hkv, dh, S):
    q = gen.normal_bf16(seed, "q", (B, T, Hq, dh), 1.0)
    k = gen.normal_bf16(seed, "k_cache", (B, Hkv, S, dh), 1.0)
    v = gen.normal_bf16(seed, "v_cache", (B, Hkv, S, dh), 1.0)
    return q, k, v


def _f64(bits):
    return torch.from_numpy(gen.bf16_bits_to_f32(bits).astype(np.float64))


def test_root_only_tree_is_decode_attention():
    B, Hq, Hkv, dh, S = 2, 4, 2, 64, 80
    q, k, v = _inputs(11, B, 1, Hq, Hkv, dh, S)
    P = np.array([37, 79])
    out = oa.tree_attention(q, k, v, P, [-1])
    for b in range(B):
        n = P[b] + 1
        qq = _f64(q[b, 0])[:, None, :]                           # [Hq, 1, dh]
        kk = _f64(k[b, :, :n]).repeat_interleave(Hq // Hkv, 0)   # [Hq, n, dh]
        vv = _f64(v[b, :, :n]).repeat_interleave(Hq // Hkv, 0)
        ref = F.scaled_dot_product_attention(qq, kk, vv)[:, 0, :].numpy()
        assert np.max(np.abs(out[b, 0] - ref)) < 1e-12


def test_chain_tree_is_causal_attention():
    B, Hq, Hkv, dh, S = 1, 4, 2, 64, 64
    parent = [-1, 0, 1, 2, 3]
    T = len(parent)
    q, k, v = _inputs(12, B, T, Hq, Hkv, dh, S)
    P = np.array([50])
    out = oa.tree_attention(q, k, v, P, parent)
    n = P[0] + T
    qq = _f64(q[0]).permute(1, 0, 2)                               # [Hq, T, dh]
    kk = _f64(k[0, :, :n]).repeat_interleave(Hq // Hkv, 0)
    vv = _f64(v[0, :, :n]).repeat_interleave(Hq // Hkv, 0)
    mask = torch.ones(T, n, dtype=torch.bool).tril(diagonal=int(P[0]))
    ref = F.scaled_dot_product_attention(qq, kk, vv, attn_mask=mask).permute(1, 0, 2).numpy()
    assert np.max(np.abs(out[0] - ref)) < 1e-12


def test_any_node_equals_attention_over_its_own_path():
    """Node t sees exactly [prefix, root, ..., t]: gather that sequence and
    attend with the last position's query, no mask."""
    tups = ot.select_tree((4, 3, 2, 2), TREE_ACCEPT, 16)
    parent, _, _ = ot.spec_from_tuples(tups)
    T = len(parent)
    B, Hq, Hkv, dh = 2, 4, 2, 64
    P = np.array([20, 41])
    S = 64
    q, k, v = _inputs(13, B, T, Hq, Hkv, dh, S)
    out = oa.tree_attention(q, k, v, P, parent, scale=0.1)
    for b in range(B):
        for t in range(T):
            path = []
            n = t
            while n != -1:
                path.append(n)
                n = int(parent[n])
            slots = list(range(P[b])) + [P[b] + j for j in reversed(path)]
            for h in range(Hq):
                hk = h // (Hq // Hkv)
                kk = _f64(k[b, hk, slots])
                vv = _f64(v[b, hk, slots])
                qq = _f64(q[b, t, h])
                ref = F.scaled_dot_product_attention(qq[None, None], kk[None], vv[None], scale=0.1)[0, 0].numpy()
                assert np.max(np.abs(out[b, t, h] - ref)) < 1e-12


def test_default_scale_and_row_selection():
    B, T, Hq, Hkv, dh, S = 1, 3, 2, 1, 64, 16
    q, k, v = _inputs(14, B, T, Hq, Hkv, dh, S)
    parent = [-1, 0, 0]
    P = np.array([5])
    full = oa.tree_attention(q, k, v, P, parent)
    explicit = oa.tree_attention(q, k, v, P, parent, scale=1 / math.sqrt(dh))
    assert np.array_equal(full, explicit)
    part = oa.tree_attention(q, k, v, P, parent, rows=[(0, 2, 1)])
    assert np.array_equal(part[0, 2, 1], full[0, 2, 1])
    assert np.isnan(part[0, 0, 0]).all()
