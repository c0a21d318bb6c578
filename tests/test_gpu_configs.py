"""GPU parity at every workload's own shapes, in the launch configurations the
benchmark times: the batched 70B step (8 requests, 64 q / 8 kv heads, prefix
lengths uniform in [1024, 8192], heads over all 520 tree tokens) and the 8B
sweep's extremes (32k prefix; 32 requests on the single-CTA tensor-core heads;
the 2080 = 32 x 65 tree-token rows on the CTA-pair heads). The oracle computes
the sampled rows one by one; every sample is chosen so that each kernel tile of
the launch (request x query tile x KV head for attention, each CTA of each pair
for the heads) contributes at least one row."""
import numpy as np
import pytest

import medusa_draft_heads_b200 as md
from oracle import attention as oa
from oracle import heads as oh
from oracle import tree as ot
from seeded_inputs import device, synth
from seeded_inputs.workloads import BATCHED70B, sweep_8b

from .helpers import ATTN_RTOL, HEADS_RTOL, check_topk_row, i32, normwise, to_bits

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def _dev_normal(shape, seed, stream, sigma, dtype=None):
    t = torch.empty(shape, dtype=dtype or torch.bfloat16, device="cuda")
    return device.fill_normal(t, seed, stream, sigma)


def _tile_rows(B, T, Hq, Hkv, per_tile=2, seed=0):
    """(b, t, h) rows covering every (request, 128-row query tile, KV head) of
    the tensor-core attention launch: the first and last live row of each tile
    plus `per_tile - 2` random ones. A tile's rows are (token, head of the GQA
    group) pairs, token-major."""
    G = Hq // Hkv
    R = T * G
    rng = np.random.default_rng(seed)
    rows = []
    for b in range(B):
        for hk in range(Hkv):
            for r0 in range(0, R, 128):
                r1 = min(R, r0 + 128) - 1
                picks = {r0, r1} | {int(x) for x in rng.integers(r0, r1 + 1, max(0, per_tile - 2))}
                for r in sorted(picks):
                    rows.append((b, r // G, hk * G + r % G))
    return rows


def _attention_at(w_B, Hq, Hkv, dh, T, P, S_max, spec, seed):
    parent, rank = spec
    tree = md.Tree(parent, rank, [16] * 4)
    q = _dev_normal((w_B, T, Hq, dh), seed, "q", 1.0)
    k = _dev_normal((w_B, Hkv, S_max, dh), seed, "k_cache", 1.0)
    v = _dev_normal((w_B, Hkv, S_max, dh), seed, "v_cache", 1.0)
    out = torch.full((w_B, T, Hq, dh), np.nan, dtype=torch.float32, device="cuda")
    ws = md.workspace(md.attention_workspace_bytes(w_B, T, Hq, Hkv, dh, S_max))
    md.tree_attention(q, k, v, i32(P), tree, out, ws)
    torch.cuda.synchronize()
    assert md.device_status() == 0
    return out.cpu().numpy(), to_bits(q), to_bits(k), to_bits(v)


def _tree(kph, accept, n):
    parent, rank, _ = ot.spec_from_tuples(ot.select_tree(kph, accept, n))
    return parent, rank


def test_batched_70b_attention_every_tile():
    """Batched 70B layer: 8 requests with the workload's own prefix lengths
    (uniform in [1024, 8192]), 64 q / 8 kv heads, dh 128, 65 tree tokens: five
    128-row tiles per KV head, the fifth holding the last token's 8 heads."""
    w = BATCHED70B
    spec = _tree(w.k_per_head, w.accept, w.n_nodes)
    parent = spec[0]
    P = synth.prefix_lengths(w.seed, w.B, *w.prefix)
    assert P.min() >= 1024 and P.max() <= 8192 and len(set(P.tolist())) > 1
    out, q, k, v = _attention_at(w.B, w.Hq, w.Hkv, w.dh, w.T, P, w.S_max, spec, w.seed)
    rows = _tile_rows(w.B, w.T, w.Hq, w.Hkv, per_tile=3, seed=1)
    assert len(rows) >= w.B * w.Hkv * 5 * 2
    ref = oa.tree_attention(q, k, v, P, parent, rows=rows)
    errs = [normwise(out[b, t, h], ref[b, t, h]) for b, t, h in rows]
    assert max(errs) <= ATTN_RTOL, max(errs)
    assert np.all(np.isfinite(out))


def test_sweep_32k_prefix_attention():
    """8B sweep corner: 4 requests with a 32768-token prefix, 32 q / 8 kv heads,
    64-node tree (three 128-row tiles per KV head, the last with 4 rows)."""
    w = sweep_8b(4, "64", 32768)
    spec = _tree(w.k_per_head, w.accept, w.n_nodes)
    parent = spec[0]
    P = np.full(w.B, 32768, dtype=np.int32)
    out, q, k, v = _attention_at(w.B, w.Hq, w.Hkv, w.dh, w.T, P, w.S_max, spec, w.seed + 7)
    rows = _tile_rows(w.B, w.T, w.Hq, w.Hkv, per_tile=2, seed=2)
    ref = oa.tree_attention(q, k, v, P, parent, rows=rows)
    errs = [normwise(out[b, t, h], ref[b, t, h]) for b, t, h in rows]
    assert max(errs) <= ATTN_RTOL, max(errs)
    assert np.all(np.isfinite(out))


def _device_heads(d, V, K, seed, sigma=0.02):
    W1 = _dev_normal((K, d, d), seed, "W1", sigma)
    b1 = _dev_normal((K, d), seed, "b1", sigma)
    Wv = _dev_normal((K, d, V), seed, "Wv", sigma)
    return W1, b1, Wv


def _run_heads(h, W1, b1, Wv, kph, kmax):
    M = h.shape[0]
    K, d, V = Wv.shape
    ids = torch.full((M, K, kmax), -7, dtype=torch.int32, device="cuda")
    vals = torch.full((M, K, kmax), np.nan, dtype=torch.float32, device="cuda")
    ws = md.workspace(md.heads_workspace_bytes(M, d, V, K, kmax))
    md.medusa_heads(h, W1, b1, Wv, kph, ids, vals, ws)
    fused = (ids.cpu().numpy().copy(), vals.cpu().numpy().copy())
    logits = torch.empty((M, K, V), dtype=torch.float32, device="cuda")
    md.medusa_heads(h, W1, b1, Wv, kph, ids, vals, ws, logits_dbg=logits)
    torch.cuda.synchronize()
    assert md.device_status() == 0
    # writing the logits changes nothing else
    assert np.array_equal(fused[0], ids.cpu().numpy())
    assert np.array_equal(fused[1], vals.cpu().numpy())
    return fused, logits


def _check_heads_rows(runs, W1, b1, Wv, kph):
    """runs: list of (h, rows, (ids, vals), logits). Every logit of the listed
    rows against the oracle, and each head's top-k."""
    K = Wv.shape[0]
    W1b, b1b = to_bits(W1), to_bits(b1)
    zs = [oh.residual_block(to_bits(h)[rows], W1b, b1b) for h, rows, _, _ in runs]
    del W1b
    gs = [logits[torch.from_numpy(rows).cuda()].cpu().numpy() for _, rows, _, logits in runs]
    fuzzy = 0
    for k in range(K):
        Wk = to_bits(Wv[k:k + 1])
        for (h, rows, (ids, vals), _), z, g in zip(runs, zs, gs):
            ref = oh.vocab_logits(z[:, k:k + 1], Wk)[:, 0]
            for i, m in enumerate(rows):
                assert normwise(g[i, k], ref[i]) <= HEADS_RTOL, (m, k)
                fuzzy += check_topk_row(ids[m, k], vals[m, k], ref[i], kph[k])
        del Wk
    return fuzzy


def test_batched_70b_heads_whole_request_and_every_cta():
    """Batched 70B heads on 520 rows (CTA-pair tcgen05 GEMM): every row of
    request 0 (65 tree tokens) and one row in each CTA of each pair (rows
    0-127 / 128-255 / 256-383 / 384-511 / 512-519)."""
    w = BATCHED70B
    W1, b1, Wv = _device_heads(w.d, w.V, w.K, w.seed)
    h = _dev_normal((w.M, w.d), w.seed, "h", 1.0)
    fused, logits = _run_heads(h, W1, b1, Wv, w.k_per_head, w.kmax)
    rows = np.array(list(range(65)) + [130, 300, 400, 511, 519])
    fuzzy = _check_heads_rows([(h, rows, fused, logits)], W1, b1, Wv, w.k_per_head)
    # ranks checked only for validity (oracle neighbours closer than twice the
    # observed logit error): at most 10 % of the ranks
    assert fuzzy * 10 <= len(rows) * sum(w.k_per_head), fuzzy


def test_sweep_8b_heads_b32_single_cta_and_pair_gemm():
    """8B sweep heads at B = 32: the sweep's one hidden row per request
    (M = 32, tcgen05 with the weights as the MMA's M), every row checked; and all 32 x 65 tree
    tokens (M = 2080, CTA-pair GEMM, 17 row tiles in 9 pairs), one row in each
    128-row tile plus the last row."""
    w = sweep_8b(32, "64", 1024)
    W1, b1, Wv = _device_heads(w.d, w.V, w.K, w.seed)
    h32 = _dev_normal((32, w.d), w.seed + 32, "h", 1.0)
    h2080 = _dev_normal((32 * w.T, w.d), w.seed + 2080, "h", 1.0)
    f32_, l32 = _run_heads(h32, W1, b1, Wv, w.k_per_head, w.kmax)
    f2080, l2080 = _run_heads(h2080, W1, b1, Wv, w.k_per_head, w.kmax)
    rows32 = np.arange(32)
    rows2080 = np.array(sorted({i * 128 + (37 * i) % 128 for i in range(17)} | {2079}))
    rows2080 = rows2080[rows2080 < 2080]
    fuzzy = _check_heads_rows([(h32, rows32, f32_, l32), (h2080, rows2080, f2080, l2080)], W1, b1, Wv,
                              w.k_per_head)
    assert fuzzy * 10 <= (len(rows32) + len(rows2080)) * sum(w.k_per_head), fuzzy
