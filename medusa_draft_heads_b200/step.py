"""One Medusa draft-and-verify step through the C ABI.

Owns the output buffers and workspaces of the four calls and issues them in
order on one stream: heads + top-k -> tree build -> tree attention (one layer
of the verification pass) -> acceptance. No arithmetic happens here.
"""
from __future__ import annotations

import torch

from .binding import (Tree, accept_workspace_bytes, attention_workspace_bytes, heads_shared_workspace_bytes,
                      heads_workspace_bytes, medusa_heads, medusa_heads_sampled, medusa_heads_shared, tree_accept,
                      tree_accept_rejection, tree_accept_sampled, tree_attention, tree_build, tree_commit, workspace)
from .tree_spec import tree_arrays


class MedusaStep:
    def __init__(self, *, B, M, d, V, K, k_per_head, tree_tuples, Hq, Hkv, dh, S_max, mode="greedy",
                 temperature=0.7, eps=0.09, alpha=0.3, device="cuda", keep_logits=False, shared_vocab=False):
        parent, rank = tree_arrays(tree_tuples)
        self.tree = Tree(parent, rank, k_per_head)
        self.B, self.M, self.d, self.V, self.K = B, M, d, V, K
        self.k_per_head = list(k_per_head)
        self.kmax = max(k_per_head)
        self.T = self.tree.T
        self.Hq, self.Hkv, self.dh, self.S_max = Hq, Hkv, dh, S_max
        self.mode, self.temperature, self.eps, self.alpha = mode, temperature, eps, alpha
        dev = torch.device(device)
        i32 = dict(dtype=torch.int32, device=dev)
        f32 = dict(dtype=torch.float32, device=dev)
        self.topk_ids = torch.empty((M, K, self.kmax), **i32)
        self.topk_vals = torch.empty((M, K, self.kmax), **f32)
        # mode "rejection": candidates drawn from the heads' distributions, whose
        # logits the lossless acceptance reads, so they are always kept
        keep_logits = keep_logits or mode == "rejection"
        self.logits_dbg = torch.empty((M, K, V), **f32) if keep_logits else None
        self.tokens = torch.empty((B, self.T), **i32)
        self.parent = torch.empty((self.T,), **i32)
        self.anc = torch.empty((self.T, (self.T + 31) // 32), **i32)
        self.pos = torch.empty((B, self.T), **i32)
        self.attn_out = torch.empty((B, self.T, Hq, dh), **f32)
        # the step's result in one buffer (accept_len [B], path [B, K+1],
        # bonus [B]), so a caller reads it back with one copy
        self.result = torch.empty((B * (K + 3),), **i32)
        self.accept_len = self.result[:B]
        self.path = self.result[B:B * (K + 2)].view(B, K + 1)
        self.bonus = self.result[B * (K + 2):]
        self.new_prefix_len = torch.empty((B,), **i32)
        self.next_root = torch.empty((B,), **i32)
        self.next_head_row = torch.empty((B,), **i32)
        self.shared_vocab = shared_vocab
        # mode "sample": one uniform in [0, 1) per tree row, supplied by the caller
        self.uniforms = torch.full((B, self.T), 0.5, **f32) if mode == "sample" else None
        # mode "rejection": uniforms for the draws [M, K, V] and for the tests
        # and bonus draws [B, T] each; the caller refills them every step
        self.u_draft = torch.full((M, K, V), 0.5, **f32) if mode == "rejection" else None
        self.u_accept = torch.full((B, self.T), 0.5, **f32) if mode == "rejection" else None
        self.u_residual = torch.full((B, self.T), 0.5, **f32) if mode == "rejection" else None
        self.head_row = None
        ws_fn = heads_shared_workspace_bytes if shared_vocab else heads_workspace_bytes
        self.ws_heads = workspace(ws_fn(M, d, V, K, self.kmax), dev)
        self.ws_attn = workspace(attention_workspace_bytes(B, self.T, Hq, Hkv, dh, S_max), dev)
        self.ws_acc = workspace(accept_workspace_bytes(B, self.T, V), dev)

    def heads(self, h, W1, b1, Wv, stream=None):
        if self.mode == "rejection":
            medusa_heads_sampled(h, W1, b1, Wv, self.k_per_head, self.u_draft, self.topk_ids, self.topk_vals,
                                 self.logits_dbg, self.ws_heads, temperature=self.temperature, stream=stream)
            return
        fn = medusa_heads_shared if self.shared_vocab else medusa_heads
        fn(h, W1, b1, Wv, self.k_per_head, self.topk_ids, self.topk_vals, self.ws_heads,
           logits_dbg=self.logits_dbg, stream=stream)

    def build(self, root_token, prefix_len, head_row=None, stream=None):
        self.head_row = head_row
        tree_build(self.tree, self.topk_ids, root_token, prefix_len, self.tokens, self.parent, self.anc,
                   self.pos, head_row=head_row, stream=stream)

    def attention(self, q, k_cache, v_cache, prefix_len, stream=None):
        tree_attention(q, k_cache, v_cache, prefix_len, self.tree, self.attn_out, self.ws_attn, stream=stream)

    def accept(self, logits, stream=None, uniforms=None):
        """Greedy / typical acceptance, (mode "sample") the lossless sampled
        rule with one uniform per tree row ([B, T] fp32: `uniforms`, else the
        step's own `self.uniforms`, which the caller refills each step), or
        (mode "rejection") lossless acceptance of drafts sampled from the heads."""
        if self.mode == "rejection":
            tree_accept_rejection(logits, self.tokens, self.tree, self.logits_dbg, self.u_accept, self.u_residual,
                                  self.accept_len, self.path, self.bonus, temperature=self.temperature,
                                  temperature_q=self.temperature, head_row=self.head_row, stream=stream)
            return
        if self.mode == "sample":
            u = self.uniforms if uniforms is None else uniforms
            tree_accept_sampled(logits, self.tokens, self.tree, u, self.accept_len, self.path, self.bonus,
                                self.ws_acc, temperature=self.temperature, stream=stream)
            return
        tree_accept(logits, self.tokens, self.tree, self.accept_len, self.path, self.bonus, self.ws_acc,
                    mode=self.mode, temperature=self.temperature, eps=self.eps, alpha=self.alpha, stream=stream)

    def commit(self, k_cache, v_cache, prefix_len, stream=None):
        tree_commit(k_cache, v_cache, self.tree, prefix_len, self.accept_len, self.path, self.bonus,
                    self.new_prefix_len, self.next_root, self.next_head_row, stream=stream)

    def run(self, h, W1, b1, Wv, root_token, prefix_len, q, k_cache, v_cache, logits, head_row=None,
            stream=None):
        self.heads(h, W1, b1, Wv, stream)
        self.build(root_token, prefix_len, head_row, stream)
        self.attention(q, k_cache, v_cache, prefix_len, stream)
        self.accept(logits, stream)
