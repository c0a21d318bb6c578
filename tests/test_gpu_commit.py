"""GPU parity of md_tree_commit against the oracle (bit-exact moves)."""
import numpy as np
import pytest

import medusa_draft_heads_b200 as md
from oracle import accept as oacc
from oracle import commit as oc
from oracle import tree as ot
from seeded_inputs import gen, synth
from seeded_inputs.workloads import TREE_ACCEPT

from .helpers import bf16_tensor, i32, to_bits

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("kph,n,B,Hkv,dh,V", [((4, 3, 2, 2), 16, 6, 2, 64, 1024), ((10, 10, 10, 10), 64, 8, 8, 128, 4096),
                                             ((1, 1, 1, 1), 4, 5, 8, 128, 1000)])
def test_commit_matches_oracle(kph, n, B, Hkv, dh, V):
    tups = ot.select_tree(kph, TREE_ACCEPT, n)
    parent, rank, _ = ot.spec_from_tuples(tups)
    T = len(parent)
    seed = n + B
    tokens = synth.synthetic_tree_tokens(seed, B, parent, V)
    logits = synth.planted_logits(seed, parent, tokens, V, TREE_ACCEPT)
    L, path, bonus, _ = oacc.greedy_accept(logits, tokens, parent, 4)     # inputs from the oracle
    P = gen.uniform_int(seed, "prefix_len", (B,), 0, 300).astype(np.int32)
    S = 300 + T + 5
    k = gen.normal_bf16(seed, "k_cache", (B, Hkv, S, dh), 1.0)
    v = gen.normal_bf16(seed, "v_cache", (B, Hkv, S, dh), 1.0)
    rk, rv, rp, rroot, rrow = oc.tree_commit(k, v, P, L, path, bonus, T)

    tree = md.Tree(parent, rank, [16] * 4)
    kc, vc = bf16_tensor(k), bf16_tensor(v)
    newp = torch.zeros(B, dtype=torch.int32, device="cuda")
    root = torch.zeros(B, dtype=torch.int32, device="cuda")
    row = torch.zeros(B, dtype=torch.int32, device="cuda")
    md.device_status(clear=True)
    md.tree_commit(kc, vc, tree, i32(P), i32(L), i32(path), i32(bonus), newp, root, row)
    torch.cuda.synchronize()
    assert md.device_status() == 0
    assert np.array_equal(to_bits(kc), rk) and np.array_equal(to_bits(vc), rv)
    assert np.array_equal(newp.cpu().numpy(), rp)
    assert np.array_equal(root.cpu().numpy(), rroot)
    assert np.array_equal(row.cpu().numpy(), rrow)
    assert L.max() > 0


def test_commit_rejects_a_path_that_is_not_in_the_tree():
    parent, rank = [-1, 0, 0, 1], [0, 0, 1, 0]
    tree = md.Tree(parent, rank, [2, 1])
    k = gen.normal_bf16(1, "k_cache", (2, 1, 16, 64), 1.0)
    kc, vc = bf16_tensor(k), bf16_tensor(k)
    path = np.array([[0, 2, 3], [0, 1, 3]])        # request 0: node 3's parent is 1, not 2
    newp = torch.zeros(2, dtype=torch.int32, device="cuda")
    root = torch.zeros(2, dtype=torch.int32, device="cuda")
    row = torch.zeros(2, dtype=torch.int32, device="cuda")
    md.device_status(clear=True)
    md.tree_commit(kc, vc, tree, i32([5, 5]), i32([2, 2]), i32(path), i32([9, 9]), newp, root, row)
    assert md.device_status(clear=True) == md.binding.DEV_BAD_PATH
    got = to_bits(kc)
    assert np.array_equal(got[0], k[0])             # request 0 untouched
    assert newp.cpu().tolist() == [5, 8] and row.cpu().tolist() == [-1, 4 + 3]
