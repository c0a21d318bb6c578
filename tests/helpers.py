"""Shared test helpers: seeded inputs for a workload, device upload, and the
comparison rules of the parity tests."""
from __future__ import annotations

import numpy as np

from seeded_inputs import gen, synth

# Tolerances (normwise relative error per row: max|gpu - ref| / max|ref|).
HEADS_RTOL = 1e-2
ATTN_RTOL = 2e-3


def bf16_tensor(bits, device="cuda"):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)


def to_bits(t):
    import torch
    return t.detach().cpu().view(torch.int16).numpy().view(np.uint16)


def i32(a, device="cuda"):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(device)


def f32(a, device="cuda"):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device)


def normwise(g, r, axis=-1):
    g = np.asarray(g, dtype=np.float64)
    r = np.asarray(r, dtype=np.float64)
    return np.max(np.abs(g - r), axis=axis) / np.max(np.abs(r), axis=axis)


def head_weights(seed, d, V, K, M, w_sigma=0.02):
    h = gen.normal_bf16(seed, "h", (M, d), 1.0)
    W1 = gen.normal_bf16(seed, "W1", (K, d, d), w_sigma)
    b1 = gen.normal_bf16(seed, "b1", (K, d), w_sigma)
    Wv = gen.normal_bf16(seed, "Wv", (K, d, V), w_sigma)
    return h, W1, b1, Wv


def kv_inputs(seed, B, T, Hq, Hkv, dh, S_max):
    q = gen.normal_bf16(seed, "q", (B, T, Hq, dh), 1.0)
    k = gen.normal_bf16(seed, "k_cache", (B, Hkv, S_max, dh), 1.0)
    v = gen.normal_bf16(seed, "v_cache", (B, Hkv, S_max, dh), 1.0)
    return q, k, v


def check_topk_row(gpu_ids, gpu_vals, ref_row, k):
    """Compare one row's GPU top-k with the oracle's full-precision logits.

    Unique parts must agree exactly: the id at every rank whose oracle value
    is separated from its neighbours by more than twice the row's observed
    logit error. Everything else must be valid: each GPU value equals the
    oracle logit at that id within the error, and no id left out beats the
    weakest pick by more than the error. Returns the number of ranks that
    were only checked for validity.
    """
    ref_row = np.asarray(ref_row, dtype=np.float64)
    gpu_ids = np.asarray(gpu_ids[:k])
    gpu_vals = np.asarray(gpu_vals[:k], dtype=np.float64)
    order = np.lexsort((np.arange(ref_row.size), -ref_row))
    ref_ids = order[:k + 1]
    err = np.max(np.abs(gpu_vals - ref_row[gpu_ids]))
    # the GPU's values must themselves meet the logit tolerance before their
    # error may widen the tie window used below
    assert err <= HEADS_RTOL * np.max(np.abs(ref_row)), (err, np.max(np.abs(ref_row)))
    tol = 2 * err + 1e-7 * np.max(np.abs(ref_row))
    assert len(set(gpu_ids.tolist())) == k
    assert np.all(np.diff(gpu_vals) <= 0)
    weakest = ref_row[gpu_ids].min()
    mask = np.ones(ref_row.size, dtype=bool)
    mask[gpu_ids] = False
    assert ref_row[mask].max() <= weakest + tol
    fuzzy = 0
    vals = ref_row[order[:k + 1]]
    for r in range(k):
        lo_gap = vals[r] - vals[r + 1]
        hi_gap = vals[r - 1] - vals[r] if r > 0 else np.inf
        if lo_gap > tol and hi_gap > tol:
            assert gpu_ids[r] == ref_ids[r], (r, gpu_ids, ref_ids)
        else:
            fuzzy += 1
    return fuzzy


def planted_for_tokens(seed, parent, tokens, V, accept, sigma=1.0, bump=1.0):
    return synth.planted_logits(seed, parent, tokens, V, accept, sigma=sigma, bump=bump)
