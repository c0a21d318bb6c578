"""Several draft-and-verify steps in a row through the C ABI, against the
oracle running the same loop.

Each step: heads on every tree node's hidden state of the previous step
(M = B * T rows; the row that feeds this step's tree comes from the previous
commit), tree build, the tree tokens' K/V written into slots P .. P + T - 1
(what the target's verification pass would do), tree attention, acceptance on
planted target logits, and commit (KV compaction, next root, next prefix
length, next head row). Hidden states, Q and the tree K/V of each step are
fresh seeded draws; the planted logits follow the oracle's tokens.
"""
import numpy as np
import pytest

import medusa_draft_heads_b200 as md
from medusa_draft_heads_b200.step import MedusaStep
from oracle import accept as oacc
from oracle import attention as oa
from oracle import commit as oc
from oracle import heads as oh
from oracle import tree as ot
from seeded_inputs import gen, synth
from seeded_inputs.workloads import TREE_ACCEPT

from .helpers import ATTN_RTOL, HEADS_RTOL, bf16_tensor, check_topk_row, f32, i32, normwise, to_bits

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def test_three_step_decode_loop_matches_oracle():
    B, d, V, K, kph, n = 3, 256, 2048, 4, (4, 3, 2, 2), 16
    Hq, Hkv, dh = 4, 2, 64
    T = n + 1
    S_max = 128 + 4 * T
    tups = ot.select_tree(kph, TREE_ACCEPT, n)
    parent, rank, _ = ot.spec_from_tuples(tups)
    W1 = gen.normal_bf16(0, "W1", (K, d, d), 0.02)
    b1 = gen.normal_bf16(0, "b1", (K, d), 0.02)
    Wv = gen.normal_bf16(0, "Wv", (K, d, V), 0.02)
    kc = gen.normal_bf16(0, "k_cache", (B, Hkv, S_max, dh), 1.0)
    vc = gen.normal_bf16(0, "v_cache", (B, Hkv, S_max, dh), 1.0)
    P = np.array([17, 40, 128], dtype=np.int32)
    root = synth.root_tokens(0, B, V)
    head_row = np.arange(B, dtype=np.int32) * T          # first step: each request's root row

    step = MedusaStep(B=B, M=B * T, d=d, V=V, K=K, k_per_head=kph, tree_tuples=md.select_tree(kph, TREE_ACCEPT, n),
                      Hq=Hq, Hkv=Hkv, dh=dh, S_max=S_max, keep_logits=True)
    gW1, gb1, gWv = bf16_tensor(W1), bf16_tensor(b1), bf16_tensor(Wv)
    gk, gv = bf16_tensor(kc), bf16_tensor(vc)
    gP, groot, grow = i32(P), i32(root), i32(head_row)
    accepted = 0
    for s in range(3):
        seed = 100 + s
        h = gen.normal_bf16(seed, "h", (B * T, d), 1.0)
        q = gen.normal_bf16(seed, "q", (B, T, Hq, dh), 1.0)
        newk = gen.normal_bf16(seed, "k_cache", (B, Hkv, T, dh), 1.0)
        newv = gen.normal_bf16(seed, "v_cache", (B, Hkv, T, dh), 1.0)

        # ---- oracle step ----
        rid, _, rlog, _ = oh.medusa_heads(h, W1, b1, Wv, kph)
        rtok, _, _, rpos = ot.tree_build(parent, rank, rid, root, P, head_row=head_row)
        for b in range(B):
            kc[b, :, P[b]:P[b] + T] = newk[b]
            vc[b, :, P[b]:P[b] + T] = newv[b]
        rout = oa.tree_attention(q, kc, vc, P, parent)
        logits = synth.planted_logits(seed, parent, rtok, V, TREE_ACCEPT)
        racc, rpath, rbonus, _ = oacc.greedy_accept(logits, rtok, parent, K)
        kc, vc, P2, root2, row2 = oc.tree_commit(kc, vc, P, racc, rpath, rbonus, T)

        # ---- the same step on the GPU ----
        step.heads(bf16_tensor(h), gW1, gb1, gWv)
        step.build(groot, gP, head_row=grow)
        for b in range(B):
            gk[b, :, P[b]:P[b] + T] = bf16_tensor(newk[b])
            gv[b, :, P[b]:P[b] + T] = bf16_tensor(newv[b])
        step.attention(bf16_tensor(q), gk, gv, gP)
        step.accept(f32(logits))
        step.commit(gk, gv, gP)
        torch.cuda.synchronize()
        assert md.device_status() == 0

        assert normwise(step.logits_dbg.cpu().numpy(), rlog).max() <= HEADS_RTOL
        gids, gvals = step.topk_ids.cpu().numpy(), step.topk_vals.cpu().numpy()
        for r in head_row:            # the rows this step's tree reads must have unique top-k ranks
            for k_ in range(K):
                assert check_topk_row(gids[r, k_], gvals[r, k_], rlog[r, k_], kph[k_]) == 0
        assert np.array_equal(step.tokens.cpu().numpy(), rtok), s
        assert np.array_equal(step.pos.cpu().numpy(), rpos)
        assert normwise(step.attn_out.cpu().numpy(), rout).max() <= ATTN_RTOL
        assert np.array_equal(step.accept_len.cpu().numpy(), racc)
        assert np.array_equal(step.path.cpu().numpy(), rpath)
        assert np.array_equal(step.bonus.cpu().numpy(), rbonus)
        assert np.array_equal(to_bits(gk), kc) and np.array_equal(to_bits(gv), vc)
        assert np.array_equal(step.new_prefix_len.cpu().numpy(), P2)
        assert np.array_equal(step.next_root.cpu().numpy(), root2)
        assert np.array_equal(step.next_head_row.cpu().numpy(), row2)
        accepted += int(racc.sum())

        P, root, head_row = P2, root2, row2
        gP = step.new_prefix_len.clone()
        groot = step.next_root.clone()
        grow = step.next_head_row.clone()
    assert accepted > 0
