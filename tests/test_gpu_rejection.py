"""GPU parity of sampled drafting (md_medusa_heads_sampled) and lossless
acceptance of sampled drafts (md_tree_accept_rejection) against
oracle/rejection.py, plus a statistical check of the GPU walk itself.

Decisions that floating point takes near a threshold are compared only where
the oracle's own margin is clear of the fp32 evaluation error: an acceptance
test u < r(y)/q(y) whose sides differ by more than 1e-3 relative, a bonus draw
whose uniform lies more than 1e-5 (of the total mass) from its CDF boundary:
fp32 prefix sums over up to 128k weights carry ~1e-6 relative error. Requests with any
decision inside those bands are counted and must be few; every other request
must agree bit for bit (accepted length, path, bonus token)."""
import numpy as np
import pytest

import medusa_draft_heads_b200 as md
from oracle import heads as oh
from oracle import rejection as orj
from oracle import tree as ot
from seeded_inputs.workloads import TREE_ACCEPT

from .helpers import bf16_tensor, check_topk_row, f32, head_weights, i32

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def _uniforms(rng, shape):
    # open interval (0, 1), fp32
    return np.clip(rng.random(shape), 1e-7, 1 - 1e-7).astype(np.float32)


@pytest.mark.parametrize("M,d,V,kph,tau", [(1, 256, 1024, (4, 3, 2, 2), 0.7), (3, 320, 2056, (10, 10, 10, 10), 1.0),
                                           (20, 256, 4096, (10, 10, 10, 10), 0.7),
                                           (160, 192, 1288, (16, 8, 4, 2), 1.3)])
def test_sampled_drafts_match_oracle(M, d, V, kph, tau):
    """Streaming (M = 1), weights-as-M and CTA-pair tensor-core paths: the
    logits equal md_medusa_heads' exactly, and the candidates are the Gumbel
    top-k of the oracle's keys (ids exact where the oracle's neighbouring keys
    are clear of the observed key error)."""
    K = len(kph)
    kmax = max(kph)
    h, W1, b1, Wv = head_weights(40 + M, d, V, K, M)
    rng = np.random.default_rng(M)
    u = _uniforms(rng, (M, K, V))
    th = [bf16_tensor(x) for x in (h, W1, b1, Wv)]
    ids = torch.full((M, K, kmax), -7, dtype=torch.int32, device="cuda")
    keys = torch.zeros((M, K, kmax), dtype=torch.float32, device="cuda")
    logits = torch.zeros((M, K, V), dtype=torch.float32, device="cuda")
    ws = md.workspace(md.heads_workspace_bytes(M, d, V, K, kmax))
    md.medusa_heads_sampled(*th, kph, f32(u), ids, keys, logits, ws, temperature=tau)
    ref_logits = torch.zeros_like(logits)
    gids = torch.empty_like(ids)
    gvals = torch.empty_like(keys)
    md.medusa_heads(*th, kph, gids, gvals, ws, logits_dbg=ref_logits)
    torch.cuda.synchronize()
    assert md.device_status() == 0
    assert torch.equal(logits, ref_logits)
    rid, _, rlog, _ = oh.medusa_heads(h, W1, b1, Wv, kph, kmax)
    ids_, keys_ = ids.cpu().numpy(), keys.cpu().numpy()
    fuzzy = 0
    for m in range(M):
        for k, kk in enumerate(kph):
            ref_keys = orj.gumbel_keys(rlog[m, k], tau, u[m, k])
            fuzzy += check_topk_row(ids_[m, k], keys_[m, k], ref_keys, kk)
            assert np.all(ids_[m, k, kk:] == -1)
    assert fuzzy * 10 <= M * sum(kph)
    # the draws are not the greedy top-k
    assert not np.array_equal(ids_, gids.cpu().numpy())


def _case(seed, kph, n, B, V, M_rows, corr, tau, tau_q):
    """Random head logits, drafts from the oracle's Gumbel top-k, the tree's
    tokens, and target logits: request b's rows follow its heads' logits with
    probability `corr` (so deep paths are accepted), else independent noise."""
    rng = np.random.default_rng(seed)
    parent, rank, _ = ot.spec_from_tuples(ot.select_tree(kph, TREE_ACCEPT, n))
    T, K = len(parent), len(kph)
    depth = ot.depths(parent)
    hl = (rng.normal(0, 2.0, (M_rows, K, V))).astype(np.float32)
    head_row = rng.permutation(M_rows)[:B].astype(np.int32)
    ids, _ = orj.sampled_drafts(hl, kph, max(kph), tau_q, _uniforms(rng, (M_rows, K, V)))
    tokens = np.zeros((B, T), dtype=np.int32)
    for b in range(B):
        tokens[b, 0] = rng.integers(0, V)
        for j in range(1, T):
            tokens[b, j] = ids[head_row[b], depth[j] - 1, rank[j]]
    tl = rng.normal(0, 2.0, (B, T, V)).astype(np.float32)
    for b in range(B):
        if rng.random() < corr:
            for t in range(T):
                if depth[t] < K:
                    tl[b, t] = (hl[head_row[b], depth[t]] * (tau / tau_q) +
                                rng.normal(0, 0.3, V)).astype(np.float32)
    return parent, rank, tokens, tl, hl, head_row, _uniforms(rng, (B, T)), _uniforms(rng, (B, T))


def _run_gpu(parent, rank, tokens, tl, hl, head_row, ua, ur, tau, tau_q, K=4):
    B, T, V = tl.shape
    tree = md.Tree(parent, rank, [16] * K)
    acc = torch.full((B,), -9, dtype=torch.int32, device="cuda")
    path = torch.full((B, K + 1), -9, dtype=torch.int32, device="cuda")
    bonus = torch.full((B,), -9, dtype=torch.int32, device="cuda")
    md.tree_accept_rejection(f32(tl), i32(tokens), tree, f32(hl), f32(ua), f32(ur), acc, path, bonus,
                             temperature=tau, temperature_q=tau_q, head_row=i32(head_row))
    torch.cuda.synchronize()
    assert md.device_status() == 0
    return acc.cpu().numpy(), path.cpu().numpy(), bonus.cpu().numpy()


def _clear(decisions):
    for d in decisions:
        if len(d) == 3:
            _, ratio, u = d
            if abs(ratio - u) <= 1e-3 * max(1.0, abs(ratio)):
                return False
        elif d[1] <= 1e-5:
            return False
    return True


@pytest.mark.parametrize("kph,n,B,V,tau,tau_q", [((4, 3, 2, 2), 16, 32, 1024, 0.7, 0.7),
                                                  ((10, 10, 10, 10), 64, 16, 128256, 0.7, 1.0),
                                                  ((1, 1, 1, 1), 4, 16, 32000, 1.0, 0.8),
                                                  # a vocabulary that splits unevenly over the 8 CTAs
                                                  ((4, 3, 2, 2), 16, 24, 1030, 0.9, 0.7)])
def test_rejection_acceptance_matches_oracle(kph, n, B, V, tau, tau_q):
    case = _case(n + B, kph, n, B, V, B + 3, 0.6, tau, tau_q)
    parent, rank, tokens, tl, hl, head_row, ua, ur = case
    acc, path, bonus = _run_gpu(*case, tau, tau_q)
    racc, rpath, rbonus, dec = orj.rejection_accept(tl, tokens, parent, rank, 4, tau, hl, head_row, tau_q, ua, ur)
    compared = 0
    for b in range(B):
        if not _clear(dec[b]):
            continue
        compared += 1
        assert acc[b] == racc[b], (b, acc[b], racc[b])
        assert np.array_equal(path[b], rpath[b]), (b, path[b], rpath[b])
        assert bonus[b] == rbonus[b], (b, bonus[b], rbonus[b])
    assert compared >= B - max(2, B // 4), compared
    assert racc.max() >= 2 and racc.min() == 0         # deep accepts and full rejections both exercised


def test_gpu_walk_keeps_the_target_distribution():
    """4096 requests on a tiny tree (V = 8): the first token the GPU emits
    must follow the root's target row, within 4 sigma per token."""
    B, V, tau = 4096, 8, 1.0
    rng = np.random.default_rng(9)
    kph = (3, 2)
    parent, rank, _ = ot.spec_from_tuples(ot.select_tree(kph, TREE_ACCEPT[:2], 9))
    T = len(parent)
    depth = ot.depths(parent)
    q = rng.dirichlet(np.ones(V), size=2)
    hl = np.broadcast_to(np.log(q), (B, 2, V)).astype(np.float32).copy()
    ids, _ = orj.sampled_drafts(hl, kph, 3, tau, _uniforms(rng, (B, 2, V)))
    p_root = rng.dirichlet(np.ones(V))
    tokens = np.zeros((B, T), dtype=np.int32)
    for j in range(1, T):
        tokens[:, j] = ids[:, depth[j] - 1, rank[j]]
    tl = np.broadcast_to(np.log(p_root), (B, T, V)).astype(np.float32).copy()
    acc, path, bonus = _run_gpu(parent, rank, tokens, tl, hl, np.arange(B, dtype=np.int32),
                                _uniforms(rng, (B, T)), _uniforms(rng, (B, T)), tau, tau, K=2)
    first = np.where(acc >= 1, tokens[np.arange(B), np.maximum(path[:, 1], 0)], bonus)
    freq = np.bincount(first, minlength=V) / B
    sigma = np.sqrt(p_root * (1 - p_root) / B)
    assert np.all(np.abs(freq - p_root) <= 4 * sigma + 1e-9), (freq, p_root)
    assert 0.1 < np.mean(acc >= 1) < 0.95


def test_rejection_refuses_children_that_skip_a_rank():
    tree = md.Tree([-1, 0, 0], [0, 0, 2], [4])
    z = torch.zeros((1, 3, 64), dtype=torch.float32, device="cuda")
    t = torch.zeros((1, 3), dtype=torch.int32, device="cuda")
    u = torch.full((1, 3), 0.5, dtype=torch.float32, device="cuda")
    o = torch.zeros((1,), dtype=torch.int32, device="cuda")
    p = torch.zeros((1, 2), dtype=torch.int32, device="cuda")
    with pytest.raises(md.MedusaError, match="unsupported"):
        md.tree_accept_rejection(z, t, tree, torch.zeros((1, 1, 64), device="cuda"), u, u, o, p, o)
