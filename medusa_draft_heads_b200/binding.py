"""ctypes binding of libmedusa (include/medusa.h): argument marshalling only.

Every function takes torch tensors, checks dtype / device / contiguity,
derives the sizes the C call wants from their shapes, and passes raw
pointers plus the current CUDA stream. All computation happens in the CUDA
kernels behind the C ABI; there is no CPU path. If ``libmedusa.so`` is not
built, the first call raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libmedusa.so")

MD_ACCEPT_GREEDY = 0
MD_ACCEPT_TYPICAL = 1
DEV_BAD_PREFIX, DEV_BAD_ROW, DEV_BAD_TOKEN, DEV_TIMEOUT, DEV_BAD_PATH = 1, 2, 4, 8, 16

_lib = None
_P = ctypes.c_void_p
_I = ctypes.c_int32
_F = ctypes.c_float
_SZ = ctypes.c_size_t

_SIGNATURES = {
    "md_tree_create": [_P, _P, _I, _I, _P, ctypes.POINTER(_P)],
    "md_tree_destroy": [_P],
    "md_tree_info": [_P, ctypes.POINTER(_I), ctypes.POINTER(_I)],
    "md_heads_workspace": [_I, _I, _I, _I, _I, ctypes.POINTER(_SZ)],
    "md_medusa_heads": [_P, _P, _P, _P, _I, _I, _I, _I, _P, _I, _P, _P, _P, _P, _SZ, _P],
    "md_medusa_heads_sampled": [_P, _P, _P, _P, _I, _I, _I, _I, _P, _I, _F, _P, _P, _P, _P, _P, _SZ, _P],
    "md_heads_shared_workspace": [_I, _I, _I, _I, _I, ctypes.POINTER(_SZ)],
    "md_medusa_heads_shared": [_P, _P, _P, _P, _I, _I, _I, _I, _P, _I, _P, _P, _P, _P, _SZ, _P],
    "md_tree_build": [_P, _P, _I, _I, _P, _P, _P, _I, _P, _P, _P, _P, _P],
    "md_hydra_workspace": [_P, _I, _I, _I, _I, ctypes.POINTER(_SZ)],
    "md_hydra_draft": [_P, _P, _I, _P, _P, _P, _P, _P, _I, _I, _I, _I, _P, _P, _I, _P, _P, _P, _P, _P, _P, _SZ,
                       _P],
    "md_attention_workspace": [_I, _I, _I, _I, _I, _I, ctypes.POINTER(_SZ)],
    "md_tree_attention": [_P, _P, _P, _P, _I, _P, _I, _I, _I, _I, _F, _P, _P, _SZ, _P],
    "md_accept_workspace": [_I, _I, _I, ctypes.POINTER(_SZ)],
    "md_tree_accept": [_P, _I, _P, _P, _I, _I, _I, _F, _F, _F, _P, _P, _P, _P, _SZ, _P],
    "md_tree_accept_sampled": [_P, _I, _P, _P, _I, _I, _F, _P, _P, _P, _P, _P, _SZ, _P],
    "md_tree_accept_rejection": [_P, _I, _P, _P, _I, _I, _F, _P, _I, _I, _P, _F, _P, _P, _P, _P, _P, _P],
    "md_tree_commit": [_P, _P, _I, _I, _I, _P, _I, _P, _P, _P, _I, _P, _P, _P, _P, _P],
    "md_get_device_status": [_P, ctypes.POINTER(_I), _I],
    "md_set_wait_limit": [ctypes.c_uint64],
    "md_stream_read": [ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p, ctypes.c_void_p],
    "md_test_withhold_attention_chunk": [_I],
    "md_status_string": [_I],
    "md_version": [],
}


class MedusaError(RuntimeError):
    pass


def lib():
    """The loaded libmedusa (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise MedusaError(f"{LIB_PATH} is missing: build it with `python -m medusa_draft_heads_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, args in _SIGNATURES.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = ctypes.c_char_p if name == "md_status_string" else ctypes.c_int32
        _lib = L
    return _lib


def status_string(rc: int) -> str:
    return lib().md_status_string(rc).decode()


def _check(rc: int, what: str):
    if rc != 0:
        raise MedusaError(f"{what}: {status_string(rc)} ({rc})")


def _ptr(t, dtype, name, ndim=None):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name}: expected a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name}: must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name}: expected {ndim} dims, got {t.dim()}")
    return t.data_ptr()


def _same(what, **pairs):
    for name, (got, want) in pairs.items():
        if got != want:
            raise ValueError(f"{what}: {name} has shape {got}, expected {want}")


def _host_i32(values):
    arr = (ctypes.c_int32 * len(values))(*[int(v) for v in values])
    return arr


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


class Tree:
    """Host-side tree spec (md_tree): parent and head-rank arrays, root first."""

    def __init__(self, parent, head_rank, k_per_head):
        self.parent = [int(p) for p in parent]
        self.head_rank = [int(r) for r in head_rank]
        self.k_per_head = [int(k) for k in k_per_head]
        h = _P()
        rc = lib().md_tree_create(_host_i32(self.parent), _host_i32(self.head_rank), len(self.parent),
                                  len(self.k_per_head), _host_i32(self.k_per_head), ctypes.byref(h))
        _check(rc, "md_tree_create")
        self._h = h
        T, md = _I(), _I()
        _check(lib().md_tree_info(self._h, ctypes.byref(T), ctypes.byref(md)), "md_tree_info")
        self.T, self.max_depth, self.K = T.value, md.value, len(self.k_per_head)

    @property
    def handle(self):
        return self._h

    def __del__(self):
        h = getattr(self, "_h", None)
        if h is not None and _lib is not None:
            _lib.md_tree_destroy(h)
            self._h = None


def heads_workspace_bytes(M, d, V, K, kmax) -> int:
    n = _SZ()
    _check(lib().md_heads_workspace(M, d, V, K, kmax, ctypes.byref(n)), "md_heads_workspace")
    return n.value


def heads_shared_workspace_bytes(M, d, V, K, kmax) -> int:
    n = _SZ()
    _check(lib().md_heads_shared_workspace(M, d, V, K, kmax, ctypes.byref(n)), "md_heads_shared_workspace")
    return n.value


def attention_workspace_bytes(B, T, Hq, Hkv, dh, S_max) -> int:
    n = _SZ()
    _check(lib().md_attention_workspace(B, T, Hq, Hkv, dh, S_max, ctypes.byref(n)), "md_attention_workspace")
    return n.value


def accept_workspace_bytes(B, T, V) -> int:
    n = _SZ()
    _check(lib().md_accept_workspace(B, T, V, ctypes.byref(n)), "md_accept_workspace")
    return n.value


def workspace(nbytes: int, device=None) -> torch.Tensor:
    """A caller-owned workspace buffer (256-byte aligned by the allocator)."""
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device or "cuda")


def medusa_heads(h, W1, b1, Wv, k_per_head, topk_ids, topk_vals, ws, logits_dbg=None, stream=None):
    """md_medusa_heads: h [M,d], W1 [K,d,d], b1 [K,d], Wv [K,d,V] bf16 ->
    topk_ids [M,K,kmax] int32, topk_vals [M,K,kmax] fp32."""
    M, d = h.shape
    K, _, V = Wv.shape
    kmax = topk_ids.shape[2]
    _same("medusa_heads", W1=(tuple(W1.shape), (K, d, d)), b1=(tuple(b1.shape), (K, d)),
          Wv=(tuple(Wv.shape), (K, d, V)), topk_ids=(tuple(topk_ids.shape), (M, K, kmax)),
          topk_vals=(tuple(topk_vals.shape), (M, K, kmax)), k_per_head=(len(k_per_head), K))
    if logits_dbg is not None:
        _same("medusa_heads", logits_dbg=(tuple(logits_dbg.shape), (M, K, V)))
    rc = lib().md_medusa_heads(
        _ptr(h, torch.bfloat16, "h", 2), _ptr(W1, torch.bfloat16, "W1", 3), _ptr(b1, torch.bfloat16, "b1", 2),
        _ptr(Wv, torch.bfloat16, "Wv", 3), M, d, V, K, _host_i32(k_per_head), kmax,
        _ptr(topk_ids, torch.int32, "topk_ids", 3), _ptr(topk_vals, torch.float32, "topk_vals", 3),
        _ptr(logits_dbg, torch.float32, "logits_dbg", 3), _ptr(ws, torch.uint8, "ws"), ws.numel(), _stream(stream))
    _check(rc, "md_medusa_heads")


def medusa_heads_sampled(h, W1, b1, Wv, k_per_head, uniforms, topk_ids, topk_keys, logits, ws, temperature=1.0,
                         stream=None):
    """md_medusa_heads_sampled: the heads with candidates drawn from softmax(logits / temperature)
    without replacement (Gumbel-top-k over uniforms [M,K,V] fp32) -> topk_ids [M,K,kmax] int32
    (draw order), topk_keys [M,K,kmax] fp32, logits [M,K,V] fp32."""
    M, d = h.shape
    K, _, V = Wv.shape
    kmax = topk_ids.shape[2]
    _same("medusa_heads_sampled", W1=(tuple(W1.shape), (K, d, d)), b1=(tuple(b1.shape), (K, d)),
          Wv=(tuple(Wv.shape), (K, d, V)), topk_ids=(tuple(topk_ids.shape), (M, K, kmax)),
          topk_keys=(tuple(topk_keys.shape), (M, K, kmax)), k_per_head=(len(k_per_head), K),
          uniforms=(tuple(uniforms.shape), (M, K, V)), logits=(tuple(logits.shape), (M, K, V)))
    rc = lib().md_medusa_heads_sampled(
        _ptr(h, torch.bfloat16, "h", 2), _ptr(W1, torch.bfloat16, "W1", 3), _ptr(b1, torch.bfloat16, "b1", 2),
        _ptr(Wv, torch.bfloat16, "Wv", 3), M, d, V, K, _host_i32(k_per_head), kmax, float(temperature),
        _ptr(uniforms, torch.float32, "uniforms", 3), _ptr(topk_ids, torch.int32, "topk_ids", 3),
        _ptr(topk_keys, torch.float32, "topk_keys", 3), _ptr(logits, torch.float32, "logits", 3),
        _ptr(ws, torch.uint8, "ws"), ws.numel(), _stream(stream))
    _check(rc, "md_medusa_heads_sampled")


def medusa_heads_shared(h, W1, b1, Wv, k_per_head, topk_ids, topk_vals, ws, logits_dbg=None, stream=None):
    """md_medusa_heads_shared: h [M,d], W1 [K,d,d], b1 [K,d], ONE Wv [d,V] bf16 ->
    topk_ids [M,K,kmax] int32, topk_vals [M,K,kmax] fp32."""
    M, d = h.shape
    K = W1.shape[0]
    V = Wv.shape[1]
    kmax = topk_ids.shape[2]
    _same("medusa_heads_shared", W1=(tuple(W1.shape), (K, d, d)), b1=(tuple(b1.shape), (K, d)),
          Wv=(tuple(Wv.shape), (d, V)), topk_ids=(tuple(topk_ids.shape), (M, K, kmax)),
          topk_vals=(tuple(topk_vals.shape), (M, K, kmax)), k_per_head=(len(k_per_head), K))
    if logits_dbg is not None:
        _same("medusa_heads_shared", logits_dbg=(tuple(logits_dbg.shape), (M, K, V)))
    rc = lib().md_medusa_heads_shared(
        _ptr(h, torch.bfloat16, "h", 2), _ptr(W1, torch.bfloat16, "W1", 3), _ptr(b1, torch.bfloat16, "b1", 2),
        _ptr(Wv, torch.bfloat16, "Wv", 2), M, d, V, K, _host_i32(k_per_head), kmax,
        _ptr(topk_ids, torch.int32, "topk_ids", 3), _ptr(topk_vals, torch.float32, "topk_vals", 3),
        _ptr(logits_dbg, torch.float32, "logits_dbg", 3), _ptr(ws, torch.uint8, "ws"), ws.numel(), _stream(stream))
    _check(rc, "md_medusa_heads_shared")


def tree_build(tree: Tree, topk_ids, root_token, prefix_len, tokens, parent, anc, pos, head_row=None,
               stream=None):
    """md_tree_build: tokens [B,T], parent [T], anc [T,W] (int32 view of uint32), pos [B,T]."""
    M, Kt, kmax = topk_ids.shape
    B = root_token.shape[0]
    T, W = tree.T, (tree.T + 31) // 32
    _same("tree_build", topk_ids_heads=(Kt, tree.K), prefix_len=(tuple(prefix_len.shape), (B,)),
          tokens=(tuple(tokens.shape), (B, T)), parent=(tuple(parent.shape), (T,)), anc=(tuple(anc.shape), (T, W)),
          pos=(tuple(pos.shape), (B, T)))
    if head_row is not None:
        _same("tree_build", head_row=(tuple(head_row.shape), (B,)))
    rc = lib().md_tree_build(
        tree.handle, _ptr(topk_ids, torch.int32, "topk_ids", 3), M, kmax, _ptr(head_row, torch.int32, "head_row"),
        _ptr(root_token, torch.int32, "root_token"), _ptr(prefix_len, torch.int32, "prefix_len"), B,
        _ptr(tokens, torch.int32, "tokens"), _ptr(parent, torch.int32, "parent"), _ptr(anc, torch.int32, "anc"),
        _ptr(pos, torch.int32, "pos"), _stream(stream))
    _check(rc, "md_tree_build")


def hydra_workspace_bytes(tree: Tree, B, d, V, kmax) -> int:
    n = _SZ()
    _check(lib().md_hydra_workspace(tree.handle, B, d, V, kmax, ctypes.byref(n)), "md_hydra_workspace")
    return n.value


def hydra_logit_rows(tree: Tree, B):
    """Row of each (request b, node p with children) in md_hydra_draft's debug
    logits: level by level, then request by request, then the level's nodes
    with children in node order. Returns ({(b, p): row}, rows)."""
    parents = sorted(set(tree.parent[1:]))
    depth = [0] * tree.T
    for j in range(1, tree.T):
        depth[j] = depth[tree.parent[j]] + 1
    rows, r = {}, 0
    for lvl in range(tree.max_depth):
        nodes = [p for p in parents if depth[p] == lvl]
        for b in range(B):
            for p in nodes:
                rows[(b, p)] = r
                r += 1
    return rows, r


def hydra_draft(tree: Tree, h, E, W1, b1, Wv, root_token, prefix_len, tokens, parent, anc, pos, ws, kmax=None,
                head_row=None, logits_dbg=None, stream=None):
    """md_hydra_draft: sequentially dependent heads on h [M,d] with the input
    embedding E [V,d] and W1 [K,d,d], b1 [K,d], Wv [K,d,V] (bf16) -> tokens
    [B,T], parent [T], anc [T,W] (int32 view of uint32), pos [B,T]."""
    M, d = h.shape
    K, _, V = Wv.shape
    kmax = max(tree.k_per_head) if kmax is None else int(kmax)
    B = root_token.shape[0]
    T, W = tree.T, (tree.T + 31) // 32
    _same("hydra_draft", heads=(K, tree.K), E=(tuple(E.shape), (V, d)), W1=(tuple(W1.shape), (K, d, d)),
          b1=(tuple(b1.shape), (K, d)), prefix_len=(tuple(prefix_len.shape), (B,)),
          tokens=(tuple(tokens.shape), (B, T)), parent=(tuple(parent.shape), (T,)), anc=(tuple(anc.shape), (T, W)),
          pos=(tuple(pos.shape), (B, T)))
    if head_row is not None:
        _same("hydra_draft", head_row=(tuple(head_row.shape), (B,)))
    if logits_dbg is not None:
        _same("hydra_draft", logits_dbg=(tuple(logits_dbg.shape), (hydra_logit_rows(tree, B)[1], V)))
    rc = lib().md_hydra_draft(
        tree.handle, _ptr(h, torch.bfloat16, "h", 2), M, _ptr(head_row, torch.int32, "head_row"),
        _ptr(E, torch.bfloat16, "E", 2), _ptr(W1, torch.bfloat16, "W1", 3), _ptr(b1, torch.bfloat16, "b1", 2),
        _ptr(Wv, torch.bfloat16, "Wv", 3), d, V, K, kmax, _ptr(root_token, torch.int32, "root_token"),
        _ptr(prefix_len, torch.int32, "prefix_len"), B, _ptr(tokens, torch.int32, "tokens"),
        _ptr(parent, torch.int32, "parent"), _ptr(anc, torch.int32, "anc"), _ptr(pos, torch.int32, "pos"),
        _ptr(logits_dbg, torch.float32, "logits_dbg", 2), _ptr(ws, torch.uint8, "ws"), ws.numel(), _stream(stream))
    _check(rc, "md_hydra_draft")


def tree_attention(q, k_cache, v_cache, prefix_len, tree: Tree, out, ws, scale=0.0, stream=None):
    """md_tree_attention: q [B,T,Hq,dh], k/v cache [B,Hkv,S_max,dh] bf16 -> out fp32 [B,T,Hq,dh]."""
    B, T, Hq, dh = q.shape
    _, Hkv, S_max, _ = k_cache.shape
    _same("tree_attention", T=(T, tree.T), k_cache=(tuple(k_cache.shape), (B, Hkv, S_max, dh)),
          v_cache=(tuple(v_cache.shape), (B, Hkv, S_max, dh)), prefix_len=(tuple(prefix_len.shape), (B,)),
          out=(tuple(out.shape), (B, T, Hq, dh)))
    rc = lib().md_tree_attention(
        _ptr(q, torch.bfloat16, "q", 4), _ptr(k_cache, torch.bfloat16, "k_cache", 4),
        _ptr(v_cache, torch.bfloat16, "v_cache", 4), _ptr(prefix_len, torch.int32, "prefix_len"), S_max,
        tree.handle, B, Hq, Hkv, dh, float(scale), _ptr(out, torch.float32, "out", 4), _ptr(ws, torch.uint8, "ws"),
        ws.numel(), _stream(stream))
    _check(rc, "md_tree_attention")


def tree_accept(logits, tokens, tree: Tree, accept_len, path, bonus, ws, mode="greedy", temperature=1.0,
                eps=0.09, alpha=0.3, stream=None):
    """md_tree_accept: logits [B,T,V] fp32, tokens [B,T] -> accept_len [B], path [B,K+1], bonus [B]."""
    B, T, V = logits.shape
    K = path.shape[1] - 1
    _same("tree_accept", T=(T, tree.T), tokens=(tuple(tokens.shape), (B, T)),
          accept_len=(tuple(accept_len.shape), (B,)), bonus=(tuple(bonus.shape), (B,)), path_rows=(path.shape[0], B))
    m = {"greedy": MD_ACCEPT_GREEDY, "typical": MD_ACCEPT_TYPICAL}[mode]
    rc = lib().md_tree_accept(
        _ptr(logits, torch.float32, "logits", 3), V, _ptr(tokens, torch.int32, "tokens", 2), tree.handle, B, K, m,
        float(temperature), float(eps), float(alpha), _ptr(accept_len, torch.int32, "accept_len"),
        _ptr(path, torch.int32, "path", 2), _ptr(bonus, torch.int32, "bonus"), _ptr(ws, torch.uint8, "ws"),
        ws.numel(), _stream(stream))
    _check(rc, "md_tree_accept")


def tree_accept_sampled(logits, tokens, tree: Tree, uniforms, accept_len, path, bonus, ws, temperature=1.0,
                        stream=None):
    """md_tree_accept_sampled: logits [B,T,V] fp32, tokens [B,T], uniforms [B,T] fp32 in [0, 1)
    -> accept_len [B], path [B,K+1], bonus [B] (lossless sampled acceptance)."""
    B, T, V = logits.shape
    K = path.shape[1] - 1
    _same("tree_accept_sampled", T=(T, tree.T), tokens=(tuple(tokens.shape), (B, T)),
          uniforms=(tuple(uniforms.shape), (B, T)), accept_len=(tuple(accept_len.shape), (B,)),
          bonus=(tuple(bonus.shape), (B,)), path_rows=(path.shape[0], B))
    rc = lib().md_tree_accept_sampled(
        _ptr(logits, torch.float32, "logits", 3), V, _ptr(tokens, torch.int32, "tokens", 2), tree.handle, B, K,
        float(temperature), _ptr(uniforms, torch.float32, "uniforms", 2), _ptr(accept_len, torch.int32, "accept_len"),
        _ptr(path, torch.int32, "path", 2), _ptr(bonus, torch.int32, "bonus"), _ptr(ws, torch.uint8, "ws"),
        ws.numel(), _stream(stream))
    _check(rc, "md_tree_accept_sampled")


def tree_accept_rejection(logits, tokens, tree: Tree, head_logits, u_accept, u_residual, accept_len, path, bonus,
                          temperature=1.0, temperature_q=1.0, head_row=None, stream=None):
    """md_tree_accept_rejection: lossless acceptance of sampled drafts. logits [B,T,V] fp32,
    tokens [B,T], head_logits [M,Kh,V] fp32, u_accept / u_residual [B,T] fp32 in [0, 1)
    -> accept_len [B], path [B,K+1], bonus [B]."""
    B, T, V = logits.shape
    M, Kh, Vh = head_logits.shape
    K = path.shape[1] - 1
    _same("tree_accept_rejection", T=(T, tree.T), tokens=(tuple(tokens.shape), (B, T)), head_V=(Vh, V),
          u_accept=(tuple(u_accept.shape), (B, T)), u_residual=(tuple(u_residual.shape), (B, T)),
          accept_len=(tuple(accept_len.shape), (B,)), bonus=(tuple(bonus.shape), (B,)), path_rows=(path.shape[0], B))
    if head_row is not None:
        _same("tree_accept_rejection", head_row=(tuple(head_row.shape), (B,)))
    rc = lib().md_tree_accept_rejection(
        _ptr(logits, torch.float32, "logits", 3), V, _ptr(tokens, torch.int32, "tokens", 2), tree.handle, B, K,
        float(temperature), _ptr(head_logits, torch.float32, "head_logits", 3), M, Kh,
        _ptr(head_row, torch.int32, "head_row"), float(temperature_q), _ptr(u_accept, torch.float32, "u_accept", 2),
        _ptr(u_residual, torch.float32, "u_residual", 2), _ptr(accept_len, torch.int32, "accept_len"),
        _ptr(path, torch.int32, "path", 2), _ptr(bonus, torch.int32, "bonus"), _stream(stream))
    _check(rc, "md_tree_accept_rejection")


def tree_commit(k_cache, v_cache, tree: Tree, prefix_len, accept_len, path, bonus, new_prefix_len, next_root,
                next_head_row, stream=None):
    """md_tree_commit: move the accepted path's K/V next to the prefix (in place)
    and produce the next step's prefix lengths, root tokens and head rows."""
    B, Hkv, S_max, dh = k_cache.shape
    K = path.shape[1] - 1
    _same("tree_commit", v_cache=(tuple(v_cache.shape), (B, Hkv, S_max, dh)), path_rows=(path.shape[0], B),
          prefix_len=(tuple(prefix_len.shape), (B,)), accept_len=(tuple(accept_len.shape), (B,)),
          bonus=(tuple(bonus.shape), (B,)), new_prefix_len=(tuple(new_prefix_len.shape), (B,)),
          next_root=(tuple(next_root.shape), (B,)), next_head_row=(tuple(next_head_row.shape), (B,)))
    rc = lib().md_tree_commit(
        _ptr(k_cache, torch.bfloat16, "k_cache", 4), _ptr(v_cache, torch.bfloat16, "v_cache", 4), S_max, Hkv, dh,
        tree.handle, B, _ptr(prefix_len, torch.int32, "prefix_len"), _ptr(accept_len, torch.int32, "accept_len"),
        _ptr(path, torch.int32, "path", 2), K, _ptr(bonus, torch.int32, "bonus"),
        _ptr(new_prefix_len, torch.int32, "new_prefix_len"), _ptr(next_root, torch.int32, "next_root"),
        _ptr(next_head_row, torch.int32, "next_head_row"), _stream(stream))
    _check(rc, "md_tree_commit")


def device_status(clear: bool = True, stream=None) -> int:
    """Synchronise and read (optionally clear) the MD_DEV_* status bits."""
    v = _I()
    _check(lib().md_get_device_status(_stream(stream), ctypes.byref(v), int(bool(clear))), "md_get_device_status")
    return v.value


def set_wait_limit(ns: int = 0):
    """md_set_wait_limit: bound (ns) on every pipeline wait; 0 restores the 2 s default."""
    _check(lib().md_set_wait_limit(int(ns)), "md_set_wait_limit")


def withhold_attention_chunk_for_test(chunk: int):
    """md_test_withhold_attention_chunk: the timeout-path test hook (-1 = off)."""
    _check(lib().md_test_withhold_attention_chunk(int(chunk)), "md_test_withhold_attention_chunk")


def stream_read(buf, sink, stream=None):
    """md_stream_read: one read-only pass over a contiguous CUDA tensor (the
    read-bandwidth diagnostic); sink is a CUDA int32 tensor of >= 1 element."""
    if not (buf.is_cuda and buf.is_contiguous()):
        raise ValueError("buf: must be a contiguous CUDA tensor")
    sp = _ptr(sink, torch.int32, "sink")
    _check(lib().md_stream_read(buf.data_ptr(), buf.numel() * buf.element_size(), sp, _stream(stream)),
           "md_stream_read")


def version() -> int:
    return lib().md_version()
