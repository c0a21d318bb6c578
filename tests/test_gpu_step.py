"""The whole step through the C ABI against the oracle's own chain, and the
heads at full 70B / 8B shapes (the launch configuration the benchmark times)."""
import numpy as np
import pytest

import medusa_draft_heads_b200 as md
from medusa_draft_heads_b200.step import MedusaStep
from oracle import accept as oacc
from oracle import attention as oa
from oracle import heads as oh
from oracle import tree as ot
from seeded_inputs import device, gen, synth
from seeded_inputs.workloads import LLAMA8B, LLAMA70B, TINY

from .helpers import (ATTN_RTOL, HEADS_RTOL, bf16_tensor, check_topk_row, head_weights, i32, f32, kv_inputs,
                      normwise, to_bits)

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def test_tiny_step_matches_oracle_chain():
    w = TINY
    tups = md.select_tree(w.k_per_head, w.accept, w.n_nodes)
    h, W1, b1, Wv = head_weights(w.seed, w.d, w.V, w.K, w.M)
    root = synth.root_tokens(w.seed, w.B, w.V)
    P = synth.prefix_lengths(w.seed, w.B, *w.prefix)
    q, k, v = kv_inputs(w.seed, w.B, w.T, w.Hq, w.Hkv, w.dh, w.S_max)

    # oracle chain
    rid, rval, rlog, _ = oh.medusa_heads(h, W1, b1, Wv, w.k_per_head)
    parent, rank, _ = ot.spec_from_tuples(ot.select_tree(w.k_per_head, w.accept, w.n_nodes))
    rtok, rpar, ranc, rpos = ot.tree_build(parent, rank, rid, root, P)
    rout = oa.tree_attention(q, k, v, P, parent)
    logits = synth.planted_logits(w.seed, parent, rtok, w.V, w.accept)      # planted on the oracle's tokens
    racc, rpath, rbonus, _ = oacc.greedy_accept(logits, rtok, parent, w.K)

    step = MedusaStep(B=w.B, M=w.M, d=w.d, V=w.V, K=w.K, k_per_head=w.k_per_head, tree_tuples=tups, Hq=w.Hq,
                      Hkv=w.Hkv, dh=w.dh, S_max=w.S_max, keep_logits=True)
    step.run(bf16_tensor(h), bf16_tensor(W1), bf16_tensor(b1), bf16_tensor(Wv), i32(root), i32(P),
             bf16_tensor(q), bf16_tensor(k), bf16_tensor(v), f32(logits))
    torch.cuda.synchronize()
    assert md.device_status() == 0
    assert normwise(step.logits_dbg.cpu().numpy(), rlog).max() <= HEADS_RTOL
    ids = step.topk_ids.cpu().numpy()
    for k_ in range(w.K):
        assert check_topk_row(ids[0, k_], step.topk_vals.cpu().numpy()[0, k_], rlog[0, k_], w.k_per_head[k_]) == 0
    assert np.array_equal(step.tokens.cpu().numpy(), rtok)
    assert np.array_equal(step.parent.cpu().numpy(), rpar)
    assert np.array_equal(step.anc.cpu().numpy().view(np.uint32), ranc)
    assert np.array_equal(step.pos.cpu().numpy(), rpos)
    assert normwise(step.attn_out.cpu().numpy(), rout).max() <= ATTN_RTOL
    assert np.array_equal(step.accept_len.cpu().numpy(), racc)
    assert np.array_equal(step.path.cpu().numpy(), rpath)
    assert np.array_equal(step.bonus.cpu().numpy(), rbonus)


def _device_weights(w):
    """Head weights drawn on the device by the generator twin (bit-identical
    to the host draws, see test_gpu_generator)."""
    W1 = device.fill_normal(torch.empty((w.K, w.d, w.d), dtype=torch.bfloat16, device="cuda"), w.seed, "W1",
                            w.w_sigma)
    b1 = device.fill_normal(torch.empty((w.K, w.d), dtype=torch.bfloat16, device="cuda"), w.seed, "b1", w.w_sigma)
    Wv = device.fill_normal(torch.empty((w.K, w.d, w.V), dtype=torch.bfloat16, device="cuda"), w.seed, "Wv",
                            w.w_sigma)
    h = device.fill_normal(torch.empty((w.M, w.d), dtype=torch.bfloat16, device="cuda"), w.seed, "h", 1.0)
    return h, W1, b1, Wv


@pytest.mark.parametrize("w", [LLAMA8B, LLAMA70B], ids=["8b", "70b"])
def test_full_size_heads_match_oracle(w):
    """Full-size heads at B = 1 in the benchmark's launch configuration: every
    logit of every head against the oracle, and each head's top-10."""
    h, W1, b1, Wv = _device_weights(w)
    kmax = w.kmax
    ids = torch.empty((1, w.K, kmax), dtype=torch.int32, device="cuda")
    vals = torch.empty((1, w.K, kmax), dtype=torch.float32, device="cuda")
    logits = torch.empty((1, w.K, w.V), dtype=torch.float32, device="cuda")
    ws = md.workspace(md.heads_workspace_bytes(1, w.d, w.V, w.K, kmax))
    md.medusa_heads(h, W1, b1, Wv, w.k_per_head, ids, vals, ws)          # fused path: no logits written
    ids_fused = ids.cpu().numpy().copy()
    vals_fused = vals.cpu().numpy().copy()
    md.medusa_heads(h, W1, b1, Wv, w.k_per_head, ids, vals, ws, logits_dbg=logits)
    torch.cuda.synchronize()
    assert md.device_status() == 0
    assert np.array_equal(ids_fused, ids.cpu().numpy())
    assert np.array_equal(vals_fused, vals.cpu().numpy())
    hb, W1b, b1b = to_bits(h), to_bits(W1), to_bits(b1)
    z = oh.residual_block(hb, W1b, b1b)
    del W1b
    g = logits.cpu().numpy()
    for k in range(w.K):
        Wk = to_bits(Wv[k:k + 1])
        ref = oh.vocab_logits(z[:, k:k + 1], Wk)[0, 0]
        del Wk
        assert normwise(g[0, k], ref) <= HEADS_RTOL
        check_topk_row(ids_fused[0, k], vals_fused[0, k], ref, w.k_per_head[k])
