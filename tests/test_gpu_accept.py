"""GPU parity of md_tree_accept against the oracle (identical fp32 logits)."""
import numpy as np
import pytest

import medusa_draft_heads_b200 as md
from oracle import accept as oacc
from oracle import tree as ot
from seeded_inputs import synth
from seeded_inputs.workloads import CHAIN_ACCEPT, TREE_ACCEPT

from .helpers import f32, i32

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def _run(logits, tokens, parent, rank, K, mode="greedy", temperature=0.7, eps=0.09, alpha=0.3):
    B, T, V = logits.shape
    tree = md.Tree(parent, rank, [16] * K)
    acc = torch.full((B,), -9, dtype=torch.int32, device="cuda")
    path = torch.full((B, K + 1), -9, dtype=torch.int32, device="cuda")
    bonus = torch.full((B,), -9, dtype=torch.int32, device="cuda")
    ws = md.workspace(md.accept_workspace_bytes(B, T, V))
    md.tree_accept(f32(logits), i32(tokens), tree, acc, path, bonus, ws, mode=mode, temperature=temperature,
                   eps=eps, alpha=alpha)
    torch.cuda.synchronize()
    return acc.cpu().numpy(), path.cpu().numpy(), bonus.cpu().numpy()


@pytest.mark.parametrize("name,kph,n,accept,B,V,sigma,bump", [
    ("tiny", (4, 3, 2, 2), 16, TREE_ACCEPT, 6, 1024, 1.0, 1.0),
    ("chain", (1, 1, 1, 1), 4, CHAIN_ACCEPT, 16, 4096, 1.0, 1.0),
    ("64node-b8-70b-vocab", (10, 10, 10, 10), 64, TREE_ACCEPT, 8, 128256, 1.0, 1.0),
    ("16node-sweep", (10, 10, 10, 10), 16, TREE_ACCEPT, 32, 8192, 3.0, 3.0),
])
def test_greedy_bit_exact(name, kph, n, accept, B, V, sigma, bump):
    tups = ot.select_tree(kph, accept, n)
    parent, rank, _ = ot.spec_from_tuples(tups)
    seed = len(name) * 3
    tokens = synth.synthetic_tree_tokens(seed, B, parent, V)
    logits = synth.planted_logits(seed, parent, tokens, V, accept, sigma=sigma, bump=bump)
    acc, path, bonus = _run(logits, tokens, parent, rank, 4)
    racc, rpath, rbonus, _ = oacc.greedy_accept(logits, tokens, parent, 4)
    assert np.array_equal(acc, racc)
    assert np.array_equal(path, rpath)
    assert np.array_equal(bonus, rbonus)
    assert md.device_status() == 0
    assert racc.max() > 0          # the planted profile really accepted something


def test_greedy_argmax_ties_and_duplicate_maxima():
    """Rows with exact ties at the maximum: the lowest id is the argmax, on
    both the match test and the bonus token."""
    parent, rank = [-1, 0, 0, 1], [0, 0, 1, 0]
    V = 2048
    rng = np.random.default_rng(1)
    logits = rng.standard_normal((3, 4, V)).astype(np.float32)
    for b in range(3):
        for t in range(4):
            ids = rng.choice(V, 3, replace=False)
            logits[b, t, ids] = 9.0
    tokens = np.zeros((3, 4), dtype=np.int32)
    for b in range(3):
        amin = [int(np.flatnonzero(logits[b, t] == 9.0).min()) for t in range(4)]
        amax_other = [int(np.flatnonzero(logits[b, t] == 9.0).max()) for t in range(4)]
        tokens[b] = [7, amin[0], amax_other[0] if b == 1 else 3, amin[1] if b != 2 else amax_other[1]]
    acc, path, bonus = _run(logits, tokens, parent, rank, 2)
    racc, rpath, rbonus, _ = oacc.greedy_accept(logits, tokens, parent, 2)
    assert np.array_equal(acc, racc) and np.array_equal(path, rpath) and np.array_equal(bonus, rbonus)


def test_root_only_tree():
    V = 512
    logits = np.random.default_rng(2).standard_normal((2, 1, V)).astype(np.float32)
    tokens = np.array([[3], [4]], dtype=np.int32)
    acc, path, bonus = _run(logits, tokens, [-1], [0], 1)
    assert list(acc) == [0, 0]
    assert list(path[:, 0]) == [0, 0] and np.all(path[:, 1] == -1)
    assert list(bonus) == [int(np.argmax(logits[0, 0])), int(np.argmax(logits[1, 0]))]


@pytest.mark.parametrize("kph,n,B,V", [((10, 10, 10, 10), 64, 4, 128256), ((10, 10, 10, 10), 16, 16, 32768),
                                       ((1, 1, 1, 1), 4, 32, 8192)])
def test_typical_matches_oracle_away_from_threshold(kph, n, B, V):
    """Typical acceptance (tau 0.7, eps 0.09, alpha 0.3) on N(0,1)*3 logits
    with a planted mode. Requests whose decision on any node sits within
    1e-3 (relative) of the threshold are only checked for validity."""
    tups = ot.select_tree(kph, TREE_ACCEPT, n)
    parent, rank, _ = ot.spec_from_tuples(tups)
    tokens = synth.synthetic_tree_tokens(17, B, parent, V)
    logits = synth.planted_logits(17, parent, tokens, V, TREE_ACCEPT, sigma=3.0, bump=3.0)
    acc, path, bonus = _run(logits, tokens, parent, rank, 4, mode="typical")
    racc, rpath, rbonus, margin = oacc.typical_accept(logits, tokens, parent, 4, 0.7, 0.09, 0.3)
    near = np.nanmin(np.abs(margin), axis=1) < 1e-3
    assert near.sum() <= max(1, B // 8)
    ok = ~near
    assert np.array_equal(acc[ok], racc[ok])
    assert np.array_equal(path[ok], rpath[ok])
    assert np.array_equal(bonus[ok], rbonus[ok])
    assert racc.max() > 0


def test_typical_limits_on_gpu():
    tups = ot.select_tree((4, 3, 2, 2), TREE_ACCEPT, 16)
    parent, rank, _ = ot.spec_from_tuples(tups)
    V = 1024
    tokens = synth.synthetic_tree_tokens(5, 3, parent, V)
    logits = synth.planted_logits(5, parent, tokens, V, TREE_ACCEPT, sigma=3.0)
    acc, _, _ = _run(logits, tokens, parent, rank, 4, mode="typical", eps=0.0, alpha=0.3)
    assert list(acc) == [4, 4, 4]
    acc, _, bonus = _run(logits, tokens, parent, rank, 4, mode="typical", eps=1.0, alpha=1e30)
    assert list(acc) == [0, 0, 0]
    assert list(bonus) == [oacc.argmax_lowest_id(logits[b, 0]) for b in range(3)]


def test_bad_token_sets_status():
    parent, rank = [-1, 0], [0, 0]
    logits = np.zeros((1, 2, 256), dtype=np.float32)
    tokens = np.array([[1, 999]], dtype=np.int32)
    md.device_status(clear=True)
    acc, _, _ = _run(logits, tokens, parent, rank, 1, mode="typical")
    assert md.device_status(clear=True) == md.binding.DEV_BAD_TOKEN
    assert acc[0] == 0


# ------------------------- sampled (lossless) acceptance -------------------------

def _run_sampled(logits, tokens, parent, rank, K, u, temperature):
    """Returns the outputs and the per-row draws (the library keeps them at the
    front of the workspace, one int32 per tree row)."""
    B, T, V = logits.shape
    tree = md.Tree(parent, rank, [16] * K)
    acc = torch.full((B,), -9, dtype=torch.int32, device="cuda")
    path = torch.full((B, K + 1), -9, dtype=torch.int32, device="cuda")
    bonus = torch.full((B,), -9, dtype=torch.int32, device="cuda")
    ws = md.workspace(md.accept_workspace_bytes(B, T, V))
    md.tree_accept_sampled(f32(logits), i32(tokens), tree, f32(u), acc, path, bonus, ws, temperature=temperature)
    torch.cuda.synchronize()
    y = ws[:B * T * 4].view(torch.int32).cpu().numpy().reshape(B, T)
    return acc.cpu().numpy(), path.cpu().numpy(), bonus.cpu().numpy(), y


@pytest.mark.parametrize("name,kph,n,B,V,sigma,bump,tau", [
    ("tiny", (4, 3, 2, 2), 16, 4, 1024, 1.0, 2.0, 0.7),
    ("70b-vocab", (10, 10, 10, 10), 64, 3, 128256, 3.0, 6.0, 0.7),
    ("ragged-vocab", (10, 10, 10, 10), 16, 3, 5000, 3.0, 3.0, 1.0),
])
def test_sampled_matches_oracle(name, kph, n, B, V, sigma, bump, tau):
    """Each row's draw equals the oracle's exact inverse-CDF draw wherever the
    uniform is more than 1e-4 from a CDF boundary (elsewhere it must be one of
    the ids whose interval is within 1e-4 of u); the walk over the GPU's draws
    reproduces accept_len, path and bonus bit for bit."""
    tups = ot.select_tree(kph, TREE_ACCEPT, n)
    parent, rank, _ = ot.spec_from_tuples(tups)
    seed = len(name) * 5
    tokens = synth.synthetic_tree_tokens(seed, B, parent, V)
    logits = synth.planted_logits(seed, parent, tokens, V, TREE_ACCEPT, sigma=sigma, bump=bump)
    u = np.random.default_rng(seed).random((B, len(parent))).astype(np.float32)
    acc, path, bonus, y = _run_sampled(logits, tokens, parent, rank, 4, u, tau)
    racc, rpath, rbonus, ry, rmargin = oacc.sampled_accept(logits, tokens, parent, 4, tau, u.astype(np.float64))
    assert md.device_status() == 0
    near = rmargin <= 1e-4
    assert np.array_equal(y[~near], ry[~near])
    for b, t in zip(*np.nonzero(near)):
        p, _ = oacc.typical_stats(logits[b, t], tau)
        cdf = np.cumsum(p)
        v = int(y[b, t])
        lo = cdf[v - 1] if v > 0 else 0.0
        assert p[v] > 0 and lo - 1e-4 <= u[b, t] < cdf[v] + 1e-4
    # the walk over the GPU's own draws
    for b in range(B):
        match = [False] + [int(tokens[b, j]) == int(y[b, parent[j]]) for j in range(1, len(parent))]
        L, pth = oacc._walk_paths(match, parent, 4)
        assert acc[b] == L and list(path[b, :L + 1]) == pth and np.all(path[b, L + 1:] == -1)
        assert bonus[b] == y[b, pth[-1]]
    if not near.any():
        assert np.array_equal(acc, racc) and np.array_equal(path, rpath) and np.array_equal(bonus, rbonus)
    assert acc.max() > 0


def test_sampled_low_temperature_is_greedy_on_gpu():
    tups = ot.select_tree((4, 3, 2, 2), TREE_ACCEPT, 16)
    parent, rank, _ = ot.spec_from_tuples(tups)
    V = 4096
    tokens = synth.synthetic_tree_tokens(9, 5, parent, V)
    logits = synth.planted_logits(9, parent, tokens, V, TREE_ACCEPT, bump=4.0)
    u = np.random.default_rng(2).random((5, len(parent))).astype(np.float32)
    acc, path, bonus, _ = _run_sampled(logits, tokens, parent, rank, 4, u, 1e-3)
    racc, rpath, rbonus, _ = oacc.greedy_accept(logits, tokens, parent, 4)
    assert np.array_equal(acc, racc) and np.array_equal(path, rpath) and np.array_equal(bonus, rbonus)


def test_sampled_rejects_bad_temperature():
    parent, rank = [-1, 0], [0, 0]
    logits = np.zeros((1, 2, 256), dtype=np.float32)
    tokens = np.array([[1, 2]], dtype=np.int32)
    u = np.full((1, 2), 0.5, dtype=np.float32)
    with pytest.raises(md.MedusaError):
        _run_sampled(logits, tokens, parent, rank, 1, u, 0.0)
