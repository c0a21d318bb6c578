"""Hydra drafting (md_hydra_draft) through the C ABI against the oracle.

Small cases compare every head row's logits and every token; the tokens are
compared exactly where the oracle's candidates are separated by far more than
the logit error (checked on the oracle side first). A closed-form shift
construction pins the level indexing on the GPU with exact arithmetic. At the
70B shapes, the rank-0 path is followed level by level with the oracle (each
level's input token is the oracle's own), on the launch configuration the
benchmark times.
"""
import numpy as np
import pytest

import medusa_draft_heads_b200 as md
from oracle import heads as oh
from oracle import hydra as ohy
from oracle import tree as ot
from seeded_inputs import device, gen, synth
from seeded_inputs.workloads import LLAMA70B, TREE_ACCEPT

from .helpers import HEADS_RTOL, bf16_tensor, i32, normwise, to_bits
from .test_oracle_hydra import _shift_expected, _shift_weights

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def _outputs(B, T):
    i32d = dict(dtype=torch.int32, device="cuda")
    return (torch.full((B, T), -7, **i32d), torch.full((T,), -7, **i32d),
            torch.zeros((T, (T + 31) // 32), **i32d), torch.full((B, T), -7, **i32d))


def _min_gap(logits, depth, kph):
    """Smallest gap between consecutive top-(k+1) oracle logits of any head
    row, relative to the row's largest magnitude."""
    worst = np.inf
    for (_, p), row in logits.items():
        s = np.sort(row)[::-1][:kph[depth[p]] + 1]
        worst = min(worst, np.min(-np.diff(s)) / np.max(np.abs(row)))
    return worst


@pytest.mark.parametrize("case", ["tiny-b3-rows", "64node-b2"])
def test_small_hydra_matches_oracle(case):
    if case == "tiny-b3-rows":
        seed, B, M, d, V, kph, n = 3, 3, 5, 256, 2048, (4, 3, 2, 2), 16
        head_row = np.array([4, 0, 2], dtype=np.int32)       # levels of 3, 12, 9, 3 rows
    else:
        seed, B, M, d, V, kph, n = 12, 2, 2, 128, 1024, (10, 10, 10, 10), 64
        head_row = None                                       # levels of 2, 20, 20, 8 rows
    K = len(kph)
    tups = md.select_tree(kph, TREE_ACCEPT, n)
    parent, rank, depth = ot.spec_from_tuples(ot.select_tree(kph, TREE_ACCEPT, n))
    h = gen.normal_bf16(seed, "h", (M, d), 1.0)
    E = gen.normal_bf16(seed, "E", (V, d), 1.0)
    W1 = gen.normal_bf16(seed, "W1", (K, d, d), 0.02)
    b1 = gen.normal_bf16(seed, "b1", (K, d), 0.02)
    Wv = gen.normal_bf16(seed, "Wv", (K, d, V), 0.02)
    root = synth.root_tokens(seed, B, V)
    P = np.array([9, 300, 17][:B], dtype=np.int32)
    rtok, rpar, ranc, rpos, rlog = ohy.hydra_draft(parent, rank, h, E, W1, b1, Wv, root, P, head_row=head_row)
    # exact token comparison is meaningful: every decision the tree reads is
    # separated by far more than the GPU's logit error (~1e-7 of the row max)
    assert _min_gap(rlog, depth, kph) > 2e-5

    tree = md.Tree(*md.tree_arrays(tups), kph)
    rows, nrows = md.hydra_logit_rows(tree, B)
    tok, par, anc, pos = _outputs(B, tree.T)
    logits = torch.empty((nrows, V), dtype=torch.float32, device="cuda")
    ws = md.workspace(md.hydra_workspace_bytes(tree, B, d, V, max(kph)))
    md.hydra_draft(tree, bf16_tensor(h), bf16_tensor(E), bf16_tensor(W1), bf16_tensor(b1), bf16_tensor(Wv), i32(root),
                   i32(P), tok, par, anc, pos, ws, head_row=None if head_row is None else i32(head_row),
                   logits_dbg=logits)
    torch.cuda.synchronize()
    assert md.device_status() == 0
    g = logits.cpu().numpy()
    for (b, p), ref in rlog.items():
        assert normwise(g[rows[(b, p)]], ref) <= HEADS_RTOL, (b, p)
    assert np.array_equal(tok.cpu().numpy(), rtok)
    assert np.array_equal(par.cpu().numpy(), rpar)
    assert np.array_equal(anc.cpu().numpy().view(np.uint32), ranc)
    assert np.array_equal(pos.cpu().numpy(), rpos)


@pytest.mark.parametrize("kph,n", [((10, 10, 10, 10), 64), ((4, 3, 2, 2), 16), ((1, 1, 1, 1), 4)])
def test_shift_construction_exact_on_gpu(kph, n):
    """h = 0, W1 = 0, b1 = 0, one-hot embeddings and per-head shift
    permutations: every logit is exactly 0 or 1, so the tokens follow the
    closed form exactly (ties among the zeros go to the lower id)."""
    V = 256
    B = 2
    h, E, W1, b1, Wv = _shift_weights(V, 4)
    h = np.zeros((B, V), dtype=np.uint16)
    roots = np.array([5, 250], dtype=np.int32)
    parent, rank, depth = ot.spec_from_tuples(ot.select_tree(kph, TREE_ACCEPT, n))
    tree = md.Tree(*md.tree_arrays(md.select_tree(kph, TREE_ACCEPT, n)), kph)
    tok, par, anc, pos = _outputs(B, tree.T)
    ws = md.workspace(md.hydra_workspace_bytes(tree, B, V, V, max(kph)))
    md.hydra_draft(tree, bf16_tensor(h), bf16_tensor(E), bf16_tensor(W1), bf16_tensor(b1), bf16_tensor(Wv),
                   i32(roots), i32(np.zeros(B)), tok, par, anc, pos, ws)
    torch.cuda.synchronize()
    assert md.device_status() == 0
    got = tok.cpu().numpy()
    for b in range(B):
        assert np.array_equal(got[b], _shift_expected(parent, rank, depth, int(roots[b]), V)), b


def test_root_only_tree_and_bad_head_row():
    V, d, B = 512, 128, 2
    tree = md.Tree([-1], [0], (3,))
    h = bf16_tensor(gen.normal_bf16(5, "h", (B, d), 1.0))
    E = bf16_tensor(gen.normal_bf16(5, "E", (V, d), 1.0))
    W1 = bf16_tensor(gen.normal_bf16(5, "W1", (1, d, d), 0.02))
    b1 = bf16_tensor(gen.normal_bf16(5, "b1", (1, d), 0.02))
    Wv = bf16_tensor(gen.normal_bf16(5, "Wv", (1, d, V), 0.02))
    tok, par, anc, pos = _outputs(B, 1)
    ws = md.workspace(md.hydra_workspace_bytes(tree, B, d, V, 3))
    md.hydra_draft(tree, h, E, W1, b1, Wv, i32([7, 9]), i32([100, 0]), tok, par, anc, pos, ws)
    torch.cuda.synchronize()
    assert md.device_status() == 0
    assert tok.cpu().tolist() == [[7], [9]] and pos.cpu().tolist() == [[100], [0]]
    assert par.cpu().tolist() == [-1] and anc.cpu().tolist() == [[1]]

    # a head row outside [0, M): status bit, defined outputs, no fault
    tree2 = md.Tree([-1, 0, 0], [0, 0, 1], (2,))
    tok, par, anc, pos = _outputs(B, 3)
    ws = md.workspace(md.hydra_workspace_bytes(tree2, B, d, V, 2))
    md.hydra_draft(tree2, h, E, W1, b1, Wv, i32([7, 9]), i32([0, 0]), tok, par, anc, pos, ws, head_row=i32([1, 5]))
    torch.cuda.synchronize()
    assert md.device_status(clear=True) == md.binding.DEV_BAD_ROW
    t = tok.cpu().numpy()
    assert t[:, 0].tolist() == [7, 9] and np.all((t[:, 1:] >= 0) & (t[:, 1:] < V))


def test_hydra_rejects_bad_arguments():
    V, d, B = 512, 128, 1
    tree = md.Tree([-1, 0], [0, 0], (2, 2))
    z = lambda *s: torch.zeros(s, dtype=torch.bfloat16, device="cuda")    # noqa: E731
    tok, par, anc, pos = _outputs(B, 2)
    ws = md.workspace(md.hydra_workspace_bytes(tree, B, d, V, 2))
    with pytest.raises(ValueError):          # three heads for a two-head tree
        md.hydra_draft(tree, z(B, d), z(V, d), z(3, d, d), z(3, d), z(3, d, V), i32([1]), i32([0]), tok, par, anc,
                       pos, ws)
    with pytest.raises(md.MedusaError, match="workspace"):
        md.hydra_draft(tree, z(B, d), z(V, d), z(2, d, d), z(2, d), z(2, d, V), i32([1]), i32([0]), tok, par, anc,
                       pos, md.workspace(256))
    assert md.device_status() == 0


def test_70b_hydra_rank0_path_matches_oracle():
    """70B shapes, B = 1, the 64-node tree: level by level along the rank-0
    path, the head row's logits against the oracle and the children's tokens
    against the oracle's top-k (exact where the candidates are separated by
    more than the observed logit error, valid otherwise); the path continues
    with the oracle's own rank-0 token."""
    w = LLAMA70B
    d, V, K = w.d, w.V, w.K
    cuda = dict(dtype=torch.bfloat16, device="cuda")
    W1 = device.fill_normal(torch.empty((K, d, d), **cuda), w.seed, "W1", w.w_sigma)
    b1 = device.fill_normal(torch.empty((K, d), **cuda), w.seed, "b1", w.w_sigma)
    Wv = device.fill_normal(torch.empty((K, d, V), **cuda), w.seed, "Wv", w.w_sigma)
    h = device.fill_normal(torch.empty((1, d), **cuda), w.seed, "h", 1.0)
    E = device.fill_normal(torch.empty((V, d), **cuda), w.seed, "E", 1.0)
    tups = md.select_tree(w.k_per_head, w.accept, w.n_nodes)
    parent, rank, depth = ot.spec_from_tuples(ot.select_tree(w.k_per_head, w.accept, w.n_nodes))
    tree = md.Tree(*md.tree_arrays(tups), w.k_per_head)
    rows, nrows = md.hydra_logit_rows(tree, 1)
    tok, par, anc, pos = _outputs(1, tree.T)
    logits = torch.empty((nrows, V), dtype=torch.float32, device="cuda")
    root = synth.root_tokens(w.seed, 1, V)
    P = np.array([w.prefix[0]], dtype=np.int32)
    ws = md.workspace(md.hydra_workspace_bytes(tree, 1, d, V, w.kmax))
    md.hydra_draft(tree, h, E, W1, b1, Wv, i32(root), i32(P), tok, par, anc, pos, ws)     # fused: no logits
    tok_fused = tok.cpu().numpy().copy()
    md.hydra_draft(tree, h, E, W1, b1, Wv, i32(root), i32(P), tok, par, anc, pos, ws, logits_dbg=logits)
    torch.cuda.synchronize()
    assert md.device_status() == 0
    gtok = tok.cpu().numpy()[0]
    assert np.array_equal(tok_fused[0], gtok)
    g = logits.cpu().numpy()
    del logits
    hb = to_bits(h)[0]
    kids = {}
    for j in range(1, len(parent)):
        kids.setdefault(int(parent[j]), []).append(j)
    node, node_tok, checked = 0, int(root[0]), 0
    while node in kids:
        lvl = int(depth[node])
        x = ohy.head_input(hb, {node_tok: to_bits(E[node_tok])}, node_tok)
        ref = ohy.head_logits(x, to_bits(W1[lvl:lvl + 1]), to_bits(b1[lvl:lvl + 1]), to_bits(Wv[lvl:lvl + 1]), 0)
        gr = g[rows[(0, node)]]
        assert normwise(gr, ref) <= HEADS_RTOL
        err = np.max(np.abs(gr - ref))
        tol = 2 * err + 1e-7 * np.max(np.abs(ref))
        order = np.lexsort((np.arange(V), -ref))
        nxt = None
        for j in kids[node]:
            r = int(rank[j])
            lo = ref[order[r]] - ref[order[r + 1]]
            hi = ref[order[r - 1]] - ref[order[r]] if r > 0 else np.inf
            if lo > tol and hi > tol:
                assert gtok[j] == order[r], (node, j)
                checked += 1
            else:
                assert abs(ref[gtok[j]] - ref[order[r]]) <= tol
            if r == 0 and lo > tol:
                nxt = (j, int(order[0]))
        if nxt is None:
            break
        node, node_tok = nxt
    assert checked >= 10
