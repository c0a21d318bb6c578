"""GPU parity of md_tree_build and md_tree_attention against the oracle."""
import numpy as np
import pytest

import medusa_draft_heads_b200 as md
from oracle import attention as oa
from oracle import tree as ot
from seeded_inputs.workloads import TREE_ACCEPT

from .helpers import ATTN_RTOL, bf16_tensor, i32, kv_inputs, normwise

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def _random_tree(rng, T, K, kmax):
    """A random valid tree spec: parent < j, depth <= K, distinct sibling ranks."""
    assert T - 1 <= sum(kmax ** d for d in range(1, K + 1)), "no tree of that size exists"
    parent, rank, depth = [-1], [0], [0]
    used = {}
    for j in range(1, T):
        while True:
            p = int(rng.integers(0, j))
            if depth[p] < K and len(used.get(p, ())) < kmax:
                break
        r = int(rng.choice([x for x in range(kmax) if x not in used.get(p, set())]))
        used.setdefault(p, set()).add(r)
        parent.append(p)
        rank.append(r)
        depth.append(depth[p] + 1)
    return parent, rank


@pytest.mark.parametrize("T,B,K", [(17, 1, 4), (65, 3, 4), (128, 5, 8), (1, 2, 4), (17, 2, 1)])
def test_tree_build_bit_exact(T, B, K):
    rng = np.random.default_rng(T * 10 + B)
    kmax = 16
    parent, rank = _random_tree(rng, T, K, kmax)
    tree = md.Tree(parent, rank, [kmax] * K)
    M = B + 2
    topk = rng.integers(0, 128256, (M, K, kmax)).astype(np.int32)
    head_row = rng.integers(0, M, B).astype(np.int32)
    root = rng.integers(0, 128256, B).astype(np.int32)
    P = rng.integers(0, 5000, B).astype(np.int32)
    W = (T + 31) // 32
    tokens = torch.zeros((B, T), dtype=torch.int32, device="cuda")
    par = torch.zeros((T,), dtype=torch.int32, device="cuda")
    anc = torch.zeros((T, W), dtype=torch.int32, device="cuda")
    pos = torch.zeros((B, T), dtype=torch.int32, device="cuda")
    md.tree_build(tree, i32(topk), i32(root), i32(P), tokens, par, anc, pos, head_row=i32(head_row))
    torch.cuda.synchronize()
    rt, rp, ra, rpos = ot.tree_build(parent, rank, topk, root, P, head_row=head_row)
    assert np.array_equal(tokens.cpu().numpy(), rt)
    assert np.array_equal(par.cpu().numpy(), rp)
    assert np.array_equal(anc.cpu().numpy().view(np.uint32), ra)
    assert np.array_equal(pos.cpu().numpy(), rpos)
    assert md.device_status() == 0


def test_tree_build_flags_bad_row():
    parent, rank, _ = ot.spec_from_tuples(ot.select_tree((4, 3, 2, 2), TREE_ACCEPT, 16))
    tree = md.Tree(parent, rank, (4, 3, 2, 2))
    topk = np.arange(2 * 4 * 4, dtype=np.int32).reshape(2, 4, 4)
    tokens = torch.zeros((2, 17), dtype=torch.int32, device="cuda")
    par = torch.zeros((17,), dtype=torch.int32, device="cuda")
    anc = torch.zeros((17, 1), dtype=torch.int32, device="cuda")
    pos = torch.zeros((2, 17), dtype=torch.int32, device="cuda")
    md.device_status(clear=True)
    md.tree_build(tree, i32(topk), i32([5, 6]), i32([0, 0]), tokens, par, anc, pos, head_row=i32([1, 9]))
    assert md.device_status(clear=True) == md.binding.DEV_BAD_ROW
    t = tokens.cpu().numpy()
    assert t[1, 0] == 6 and np.all(t[1, 1:] == -1) and np.all(t[0, 1:] >= 0)


def _attention_case(seed, tups, B, Hq, Hkv, dh, P, S_max, scale=0.0):
    parent, rank, _ = ot.spec_from_tuples(tups)
    T = len(parent)
    tree = md.Tree(parent, rank, [16] * 4)
    q, k, v = kv_inputs(seed, B, T, Hq, Hkv, dh, S_max)
    out = torch.full((B, T, Hq, dh), np.nan, dtype=torch.float32, device="cuda")
    ws = md.workspace(md.attention_workspace_bytes(B, T, Hq, Hkv, dh, S_max))
    md.tree_attention(bf16_tensor(q), bf16_tensor(k), bf16_tensor(v), i32(P), tree, out, ws, scale=scale)
    torch.cuda.synchronize()
    return out.cpu().numpy(), (q, k, v, parent)


@pytest.mark.parametrize("name,tree,B,Hq,Hkv,dh,P", [
    ("tiny", ((4, 3, 2, 2), 16), 1, 4, 2, 64, [128]),
    ("ragged", ((10, 10, 10, 10), 16), 3, 8, 2, 128, [0, 37, 300]),
    ("8b", ((10, 10, 10, 10), 64), 1, 32, 8, 128, [2048]),
    ("70b-chain", ((1, 1, 1, 1), 4), 1, 64, 8, 128, [4096]),
    ("gqa16", ((10, 10, 10, 10), 16), 2, 16, 1, 64, [129, 255]),
    # GQA groups that do not divide 128 rows take the CUDA-core kernel
    ("g3-cuda-core", ((4, 3, 2, 2), 16), 2, 6, 2, 128, [77, 300]),
    ("g12-cuda-core", ((10, 10, 10, 10), 64), 1, 12, 1, 64, [1000]),
    # long prefix: many key chunks per split, B = 4 with ragged lengths
    ("long-ragged", ((10, 10, 10, 10), 64), 4, 32, 8, 128, [1024, 8191, 333, 5000]),
    # 9 row tiles per KV head (more than a portable cluster): one CTA per tile, no multicast
    ("g16-9tiles", ((10, 10, 10, 10), 64), 2, 16, 1, 64, [700, 2100]),
    # more (request, KV head, row tile) tiles than one wave holds (160 and 768):
    # 64-key chunks, two CTAs per SM
    ("many-tiles-dh64", ((4, 3, 2, 2), 16), 40, 16, 4, 64, [int(x) for x in np.arange(40) * 37 % 400 + 60]),
    ("many-tiles-dh128", ((10, 10, 10, 10), 64), 32, 32, 8, 128, [int(x) for x in np.arange(32) * 113 % 700 + 40]),
])
def test_tree_attention_matches_oracle(name, tree, B, Hq, Hkv, dh, P):
    kph, n = tree
    tups = ot.select_tree(kph, TREE_ACCEPT, n)
    T = n + 1
    S_max = (max(P) + T + 63) // 64 * 64
    out, (q, k, v, parent) = _attention_case(len(name), tups, B, Hq, Hkv, dh, np.array(P), S_max)
    ref = oa.tree_attention(q, k, v, np.array(P), parent)
    err = normwise(out, ref)
    assert err.max() <= ATTN_RTOL, err.max()
    assert md.device_status() == 0


def test_tree_attention_70b_sampled_rows():
    """70B-shaped layer (64 q / 8 kv heads, dh 128, prefix 4096, 65 tree
    tokens) at full size, checked on a sample of rows."""
    tups = ot.select_tree((10, 10, 10, 10), TREE_ACCEPT, 64)
    P = np.array([4096])
    out, (q, k, v, parent) = _attention_case(70, tups, 1, 64, 8, 128, P, 4224)
    rng = np.random.default_rng(0)
    rows = [(0, int(t), int(h)) for t, h in zip(rng.integers(0, 65, 96), rng.integers(0, 64, 96))]
    rows += [(0, 0, 0), (0, 64, 63)]
    ref = oa.tree_attention(q, k, v, P, parent, rows=rows)
    for b, t, h in rows:
        assert normwise(out[b, t, h], ref[b, t, h]) <= ATTN_RTOL


@pytest.mark.parametrize("S_max", [128, 1024])
def test_tree_attention_bad_prefix_sets_status_and_zeros(S_max):
    """A prefix that leaves no room for the tree zeroes that request only: it
    owns no work units, and the merge kernel writes its rows as zeros. With
    S_max = 1024 the valid first case spreads each tile's chunks over several
    CTAs, whose partials the merge kernel combines."""
    tups = ot.select_tree((4, 3, 2, 2), TREE_ACCEPT, 16)
    md.device_status(clear=True)
    out, _ = _attention_case(3, tups, 2, 4, 2, 64, np.array([S_max - 28, 60]), S_max)   # P + 17 <= S_max: valid
    assert md.device_status(clear=True) == 0
    out, (q, k, v, parent) = _attention_case(3, tups, 2, 4, 2, 64, np.array([S_max - 8, 60]), S_max)  # P + 17 > S_max
    assert md.device_status(clear=True) == md.binding.DEV_BAD_PREFIX
    assert np.all(out[0] == 0) and np.all(np.isfinite(out[1])) and np.any(out[1] != 0)
    ref = oa.tree_attention(q[1:], k[1:], v[1:], np.array([60]), parent)
    assert normwise(out[1:], ref).max() <= ATTN_RTOL


def test_tree_attention_explicit_scale_and_determinism():
    tups = ot.select_tree((4, 3, 2, 2), TREE_ACCEPT, 16)
    P = np.array([90])
    a, (q, k, v, parent) = _attention_case(4, tups, 1, 4, 2, 64, P, 128, scale=0.05)
    b, _ = _attention_case(4, tups, 1, 4, 2, 64, P, 128, scale=0.05)
    assert np.array_equal(a, b)
    ref = oa.tree_attention(q, k, v, P, parent, scale=0.05)
    assert normwise(a, ref).max() <= ATTN_RTOL
