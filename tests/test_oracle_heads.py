"""Pins for the oracle's draft heads and top-k (CPU only).

Each check fixes the oracle against something other than itself: numbers the
page prints, closed forms, identities of SiLU, exactly rounded sums and a
brute-force sort.
"""
import json
import math
import os

import numpy as np
import pytest

from oracle import heads as oh
from seeded_inputs import gen


def _golden(golden_dir):
    with open(os.path.join(golden_dir, "paper_figures.json")) as f:
        return json.load(f)


def test_parameter_counts_match_page(golden_dir):
    g = _golden(golden_dir)
    d, V, K = g["head_shapes"]["d"], g["head_shapes"]["V"], g["head_shapes"]["K"]
    block, proj, head, allk = oh.head_parameter_counts(d, V, K)
    assert round(block / 1e6, 1) == g["residual_block_params_M"]["value"]
    assert round(proj / 1e6, 1) == g["vocab_projection_params_M"]["value"]
    assert round(head / 1e6, 1) == g["per_head_params_M"]["value"]
    assert round(allk / 1e9, 2) == g["four_heads_params_B"]["value"]
    assert round(2 * allk / 1e9, 2) == g["four_heads_GB_bf16"]["value"]
    share = 100 * round(2 * allk / 1e9, 2) / g["target_step_GB"]["value"]
    assert round(share, 1) == g["heads_share_of_step_pct"]["value"]
    assert round(100 * proj / head) == g["vocab_share_of_head_params_pct"]["value"]
    assert round((K - 1) * proj / 1e9, 2) == g["shared_projection_saving_B"]["value"]
    # the projection count is d * V exactly: a bias of V would show at this precision
    assert round((proj + V) / 1e6, 1) != g["vocab_projection_params_M"]["value"]


def test_oracle_accepts_exactly_the_counted_shapes():
    d, V, K, M = 64, 96, 3, 2
    h = gen.normal_bf16(1, "h", (M, d), 1.0)
    W1 = gen.normal_bf16(1, "W1", (K, d, d), 0.02)
    b1 = gen.normal_bf16(1, "b1", (K, d), 0.02)
    Wv = gen.normal_bf16(1, "Wv", (K, d, V), 0.02)
    ids, vals, logits, z = oh.medusa_heads(h, W1, b1, Wv, (3, 2, 1))
    assert z.shape == (M, K, d) and logits.shape == (M, K, V) and ids.shape == (M, K, 3)
    block, proj, _, allk = oh.head_parameter_counts(d, V, K)
    assert W1[0].size + b1[0].size == block and Wv[0].size == proj
    assert W1.size + b1.size + Wv.size == allk


def _bf16_neighbours(x):
    """Brute force: the two bf16 values bracketing fp64 x, by walking the grid."""
    f = np.float32(x)
    b = np.array([f], dtype=np.float32).view(np.uint32)[0] >> 16
    cands = []
    for dv in (-2, -1, 0, 1, 2):
        bits = np.uint16((int(b) + dv) & 0xFFFF)
        v = float(oh.bf16_to_f64(np.array([bits]))[0])
        if math.isfinite(v):
            cands.append((bits, v))
    return cands


def test_f64_to_bf16_is_nearest_even():
    rng = np.random.default_rng(0)
    xs = np.concatenate([rng.standard_normal(3000) * 10.0 ** rng.integers(-20, 20, 3000),
                         # exact halfway cases between bf16 neighbours
                         np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -(1.0 + 2.0 ** -8),
                                   2.0 ** 10 * (1 + 2.0 ** -8), 0.0])])
    got = oh.f64_to_bf16(xs)
    for x, gb in zip(xs, got):
        cands = _bf16_neighbours(x)
        best = min(abs(v - x) for _, v in cands)
        near = [(bits, v) for bits, v in cands if abs(v - x) == best]
        if len(near) == 2:  # tie: even mantissa wins
            near = [c for c in near if int(c[0]) % 2 == 0]
        assert int(gb) == int(near[0][0]), (x, gb, near)


def test_silu_closed_forms():
    ln3 = math.log(3.0)
    s = oh.silu(np.array([0.0, ln3, -ln3, 50.0, -50.0, 2.5, -2.5]))
    assert s[0] == 0.0
    assert abs(s[1] - 0.75 * ln3) < 1e-15
    assert abs(s[2] + 0.25 * ln3) < 1e-15
    assert abs(s[3] - 50.0) < 1e-12 and abs(s[4]) < 1e-18
    # odd part identity: SiLU(u) - SiLU(-u) = u
    assert abs((s[5] - s[6]) - 2.5) < 1e-15


def test_residual_block_zero_weights_is_identity():
    d, K, M = 128, 3, 2
    h = gen.normal_bf16(3, "h", (M, d), 1.0)
    W1 = np.zeros((K, d, d), dtype=np.uint16)
    b1 = np.zeros((K, d), dtype=np.uint16)
    z = oh.residual_block(h, W1, b1)
    for k in range(K):
        assert np.array_equal(z[:, k, :], h)


def test_residual_block_orientation_and_bias():
    """W1[k, i, perm[i]] = c routes h_i into output perm[i]: input-major."""
    d, K = 64, 2
    rng = np.random.default_rng(1)
    h = gen.normal_bf16(4, "h", (1, d), 1.0)
    hv = oh.bf16_to_f64(h)[0]
    c = 0.5
    cb = int(np.array([c], dtype=np.float32).view(np.uint32)[0] >> 16)
    W1 = np.zeros((K, d, d), dtype=np.uint16)
    perms = [rng.permutation(d) for _ in range(K)]
    for k in range(K):
        W1[k, np.arange(d), perms[k]] = cb
    b1 = np.zeros((K, d), dtype=np.uint16)
    b1[1, :] = cb                                  # head 1 also adds bias c
    z = oh.residual_block(h, W1, b1)
    for k in range(K):
        u = np.empty(d)
        u[perms[k]] = c * hv                       # output perm[i] receives c * h_i
        u += c if k == 1 else 0.0
        want = hv + u / (1 + np.exp(-u))
        zf = oh.bf16_to_f64(z[0, k])
        assert np.all(np.abs(zf - want) <= np.abs(want) * 2.0 ** -8 + 1e-30)


def test_vocab_logits_against_exactly_rounded_sums():
    d, V, K, M = 96, 50, 2, 2
    z = gen.normal_bf16(5, "h", (M, K, d), 1.0)
    Wv = gen.normal_bf16(5, "Wv", (K, d, V), 0.02)
    got = oh.vocab_logits(z, Wv)
    zf = oh.bf16_to_f64(z)
    wf = oh.bf16_to_f64(Wv)
    for m in range(M):
        for k in range(K):
            for v in range(0, V, 7):
                exact = math.fsum(zf[m, k, i] * wf[k, i, v] for i in range(d))
                assert abs(got[m, k, v] - exact) <= 1e-13
    # the restricted-column form agrees with the full one
    cols = [0, 3, 49, 17]
    assert np.array_equal(oh.vocab_logits(z, Wv, cols=cols), got[:, :, cols])


def test_topk_matches_brute_force_sort_with_ties():
    rng = np.random.default_rng(7)
    for trial in range(200):
        n = int(rng.integers(1, 300))
        vals = rng.integers(-4, 5, n).astype(np.float64)   # many exact ties
        k = int(rng.integers(1, 17))
        ids, v = oh.topk(vals, k)
        brute = sorted(range(n), key=lambda i: (-vals[i], i))[:k]
        assert list(ids) == brute
        assert list(v) == [vals[i] for i in brute]


def test_heads_topk_pads_unused_slots():
    logits = np.arange(2 * 3 * 10, dtype=np.float64).reshape(2, 3, 10)
    ids, vals = oh.heads_topk(logits, (3, 1, 2), 4)
    assert ids.shape == (2, 3, 4)
    assert list(ids[0, 0]) == [9, 8, 7, -1]
    assert list(ids[1, 1]) == [9, -1, -1, -1]
    assert np.isneginf(vals[0, 1, 1])


@pytest.mark.parametrize("w_scale", [0.02])
def test_zero_block_reduces_to_plain_projection(w_scale):
    """W1 = 0, b1 = 0 gives z = h, so logits = h Wv: checked per entry with
    exactly rounded sums."""
    d, V, K = 64, 40, 2
    h = gen.normal_bf16(9, "h", (1, d), 1.0)
    W1 = np.zeros((K, d, d), dtype=np.uint16)
    b1 = np.zeros((K, d), dtype=np.uint16)
    Wv = gen.normal_bf16(9, "Wv", (K, d, V), w_scale)
    ids, vals, logits, z = oh.medusa_heads(h, W1, b1, Wv, (5, 5))
    hf = oh.bf16_to_f64(h)[0]
    wf = oh.bf16_to_f64(Wv)
    for k in range(K):
        exact = np.array([math.fsum(hf * wf[k, :, v]) for v in range(V)])
        assert np.max(np.abs(logits[0, k] - exact)) <= 1e-14
        brute = sorted(range(V), key=lambda v: (-exact[v], v))[:5]
        assert list(ids[0, k]) == brute


def test_residual_block_column_subset_agrees():
    d, K = 128, 2
    h, W1, b1, _ = (gen.normal_bf16(2, "h", (2, d), 1.0), gen.normal_bf16(2, "W1", (K, d, d), 0.02),
                    gen.normal_bf16(2, "b1", (K, d), 0.02), None)
    full = oh.residual_block(h, W1, b1)
    cols = [5, 0, 127, 64]
    assert np.array_equal(oh.residual_block(h, W1, b1, cols=cols), full[:, :, cols])


def test_shared_projection_equals_per_head_projections_that_agree():
    """A shared projection is the per-head form with every Wv_k equal to it."""
    d, V, K, M = 64, 300, 3, 2
    h, W1, b1 = (gen.normal_bf16(6, "h", (M, d), 1.0), gen.normal_bf16(6, "W1", (K, d, d), 0.02),
                 gen.normal_bf16(6, "b1", (K, d), 0.02))
    Wv = gen.normal_bf16(6, "Wv", (d, V), 0.02)
    a = oh.medusa_heads_shared(h, W1, b1, Wv, (5, 4, 3))
    b = oh.medusa_heads(h, W1, b1, np.stack([Wv] * K), (5, 4, 3))
    for x, y in zip(a, b):
        assert np.array_equal(x, y)
    # and the saving the page prints: (K - 1) projections of d x V
    assert (4 - 1) * 8192 * 128256 == 3 * oh.head_parameter_counts(8192, 128256, 4)[1]
