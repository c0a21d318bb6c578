"""Out-of-bounds write check of every C-ABI call (the stand-in for a memory
sanitizer): each output and workspace buffer is the head of a larger
allocation whose last 4 KB hold a sentinel byte, and after the call (tiny,
ragged and full-size shapes, every kernel path) the sentinel must be intact
and the device status clean. Outputs are prefilled too, so a cell the call
should have written but did not is caught by the parity tests, and a write
past the end is caught here."""
import numpy as np
import pytest

import medusa_draft_heads_b200 as md
from oracle import tree as ot
from seeded_inputs import device, synth
from seeded_inputs.workloads import LLAMA70B, TREE_ACCEPT

from .helpers import bf16_tensor, head_weights, i32, kv_inputs

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

GUARD = 4096
SENTINEL = 0xA5


class Guarded:
    """A contiguous CUDA tensor followed in memory by GUARD sentinel bytes."""

    def __init__(self, shape, dtype, fill=None):
        shape = tuple(int(x) for x in shape)
        n = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
        self.n = max(n, 1)
        self.buf = torch.full((self.n + GUARD,), SENTINEL, dtype=torch.uint8, device="cuda")
        self.t = self.buf[:n].view(dtype).view(shape)
        if fill is not None:
            self.t.fill_(fill)

    def intact(self) -> bool:
        return bool((self.buf[self.n:] == SENTINEL).all().item())


def _ws(nbytes):
    return Guarded((max(int(nbytes), 256),), torch.uint8, fill=0x3C)


def _assert_intact(**bufs):
    torch.cuda.synchronize()
    assert md.device_status() == 0
    bad = [name for name, g in bufs.items() if not g.intact()]
    assert not bad, f"writes past the end of {bad}"


def _tree(kph, n):
    accept = TREE_ACCEPT if len(kph) == 4 else (0.8,) * len(kph)
    parent, rank, _ = ot.spec_from_tuples(ot.select_tree(kph, accept, n))
    return parent, rank


@pytest.mark.parametrize("M,d,V,kph", [
    (1, 256, 1024, (4, 3, 2, 2)),            # streaming, tiny
    (3, 320, 1000, (10, 1, 7, 3)),           # weights as M, ragged column tile
    (20, 256, 2056, (16, 16, 16, 16)),       # weights as M, ragged rows and columns
    (100, 256, 2056, (16, 16, 16, 16)),      # single-CTA row-tile GEMM, ragged rows and columns
    (160, 192, 1288, (10, 10, 10, 10)),      # CTA-pair GEMM, second pair half-empty
])
def test_heads_write_nothing_past_their_buffers(M, d, V, kph):
    K = len(kph)
    kmax = max(kph)
    h, W1, b1, Wv = (bf16_tensor(x) for x in head_weights(3 + M, d, V, K, M))
    ids = Guarded((M, K, kmax), torch.int32, fill=-7)
    vals = Guarded((M, K, kmax), torch.float32, fill=float("nan"))
    logits = Guarded((M, K, V), torch.float32, fill=float("nan"))
    ws = _ws(md.heads_workspace_bytes(M, d, V, K, kmax))
    md.medusa_heads(h, W1, b1, Wv, kph, ids.t, vals.t, ws.t, logits_dbg=logits.t)
    _assert_intact(ids=ids, vals=vals, logits=logits, ws=ws)
    assert torch.isfinite(logits.t).all()
    # shared projection on the same shapes
    Wv1 = Wv[0].contiguous()
    ws2 = _ws(md.heads_shared_workspace_bytes(M, d, V, K, kmax))
    md.medusa_heads_shared(h, W1, b1, Wv1, kph, ids.t, vals.t, ws2.t, logits_dbg=logits.t)
    _assert_intact(ids=ids, vals=vals, logits=logits, ws=ws2)


@pytest.mark.parametrize("kph,n,B", [((4, 3, 2, 2), 16, 1), ((10, 10, 10, 10), 64, 3), ((8, 4, 2, 2, 2, 1, 1, 1), 127, 2)])
def test_tree_build_writes_nothing_past_its_outputs(kph, n, B):
    parent, rank = _tree(kph, n)
    T = len(parent)
    K = len(kph)
    tree = md.Tree(parent, rank, kph)
    W = (T + 31) // 32
    topk = np.random.default_rng(n).integers(0, 5000, (B, K, 16)).astype(np.int32)
    tok = Guarded((B, T), torch.int32, fill=-9)
    par = Guarded((T,), torch.int32, fill=-9)
    anc = Guarded((T, W), torch.int32, fill=-9)
    pos = Guarded((B, T), torch.int32, fill=-9)
    md.tree_build(tree, i32(topk), i32(np.arange(B) + 3), i32(np.full(B, 50)), tok.t, par.t, anc.t, pos.t)
    _assert_intact(tokens=tok, parent=par, anc=anc, pos=pos)


@pytest.mark.parametrize("kph,n,B,Hq,Hkv,dh,P,S_max", [
    ((4, 3, 2, 2), 16, 1, 4, 2, 64, [128], 192),            # tensor cores, one ragged tile
    ((10, 10, 10, 10), 64, 2, 32, 8, 128, [900, 33], 1024),  # KV splits merged in a cluster
    ((4, 3, 2, 2), 16, 2, 6, 2, 128, [77, 300], 384),       # CUDA-core fallback (group of 3)
])
def test_attention_writes_nothing_past_its_buffers(kph, n, B, Hq, Hkv, dh, P, S_max):
    parent, rank = _tree(kph, n)
    T = len(parent)
    tree = md.Tree(parent, rank, [16] * 4)
    q, k, v = (bf16_tensor(x) for x in kv_inputs(n + B, B, T, Hq, Hkv, dh, S_max))
    out = Guarded((B, T, Hq, dh), torch.float32, fill=float("nan"))
    ws = _ws(md.attention_workspace_bytes(B, T, Hq, Hkv, dh, S_max))
    md.tree_attention(q, k, v, i32(P), tree, out.t, ws.t)
    _assert_intact(out=out, ws=ws)
    assert torch.isfinite(out.t).all()


@pytest.mark.parametrize("mode", ["greedy", "typical", "sampled"])
@pytest.mark.parametrize("kph,n,B,V", [((4, 3, 2, 2), 16, 3, 1000), ((10, 10, 10, 10), 64, 2, 128256)])
def test_accept_writes_nothing_past_its_buffers(mode, kph, n, B, V):
    parent, rank = _tree(kph, n)
    T = len(parent)
    tree = md.Tree(parent, rank, [16] * 4)
    tokens = synth.synthetic_tree_tokens(n, B, parent, V)
    logits = torch.from_numpy(synth.planted_logits(n, parent, tokens, V, TREE_ACCEPT)).cuda()
    acc = Guarded((B,), torch.int32, fill=-9)
    path = Guarded((B, 5), torch.int32, fill=-9)
    bonus = Guarded((B,), torch.int32, fill=-9)
    ws = _ws(md.accept_workspace_bytes(B, T, V))
    if mode == "sampled":
        u = torch.rand((B, T), generator=torch.Generator().manual_seed(n)).cuda()
        md.tree_accept_sampled(logits, i32(tokens), tree, u, acc.t, path.t, bonus.t, ws.t, temperature=0.7)
    else:
        md.tree_accept(logits, i32(tokens), tree, acc.t, path.t, bonus.t, ws.t, mode=mode, temperature=0.7)
    _assert_intact(accept_len=acc, path=path, bonus=bonus, ws=ws)
    assert (acc.t >= 0).all() and (bonus.t >= 0).all()


def test_commit_writes_nothing_past_the_cache_or_outputs():
    parent, rank = _tree((10, 10, 10, 10), 64)
    T = len(parent)
    B, Hkv, dh = 3, 8, 128
    S_max = 300 + T
    tree = md.Tree(parent, rank, [16] * 4)
    kc = Guarded((B, Hkv, S_max, dh), torch.bfloat16, fill=0.5)
    vc = Guarded((B, Hkv, S_max, dh), torch.bfloat16, fill=-0.5)
    # request b accepts the depth-b node on the leftmost path
    path = np.array([[0, -1, -1, -1, -1], [0, 1, -1, -1, -1], [0, 1, 11, -1, -1]], dtype=np.int32)
    assert parent[1] == 0 and parent[11] == 1
    newp = Guarded((B,), torch.int32, fill=-9)
    root = Guarded((B,), torch.int32, fill=-9)
    row = Guarded((B,), torch.int32, fill=-9)
    md.tree_commit(kc.t, vc.t, tree, i32([300, 7, 100]), i32([0, 1, 2]), i32(path), i32([5, 6, 7]), newp.t, root.t,
                   row.t)
    _assert_intact(k_cache=kc, v_cache=vc, new_prefix_len=newp, next_root=root, next_head_row=row)


def test_hydra_writes_nothing_past_its_buffers():
    kph, n, B, d, V = (4, 3, 2, 2), 16, 2, 256, 1000
    parent, rank = _tree(kph, n)
    T = len(parent)
    tree = md.Tree(parent, rank, kph)
    h, W1, b1, Wv = (bf16_tensor(x) for x in head_weights(21, d, V, 4, B))
    E = bf16_tensor(head_weights(22, d, V, 1, V)[0])
    W = (T + 31) // 32
    tok = Guarded((B, T), torch.int32, fill=-9)
    par = Guarded((T,), torch.int32, fill=-9)
    anc = Guarded((T, W), torch.int32, fill=-9)
    pos = Guarded((B, T), torch.int32, fill=-9)
    rows = md.hydra_logit_rows(tree, B)[1]
    logits = Guarded((rows, V), torch.float32, fill=float("nan"))
    ws = _ws(md.hydra_workspace_bytes(tree, B, d, V, 4))
    md.hydra_draft(tree, h, E, W1, b1, Wv, i32([3, 4]), i32([10, 20]), tok.t, par.t, anc.t, pos.t, ws.t,
                   logits_dbg=logits.t)
    _assert_intact(tokens=tok, parent=par, anc=anc, pos=pos, logits=logits, ws=ws)


def test_full_size_70b_calls_write_nothing_past_their_buffers():
    """The benchmark's 70B B = 1 heads call (fused, no logits) and its
    attention call, with guarded outputs and workspaces."""
    w = LLAMA70B
    bf = dict(dtype=torch.bfloat16, device="cuda")
    W1 = device.fill_normal(torch.empty((w.K, w.d, w.d), **bf), w.seed, "W1", w.w_sigma)
    b1 = device.fill_normal(torch.empty((w.K, w.d), **bf), w.seed, "b1", w.w_sigma)
    Wv = device.fill_normal(torch.empty((w.K, w.d, w.V), **bf), w.seed, "Wv", w.w_sigma)
    h = device.fill_normal(torch.empty((1, w.d), **bf), w.seed, "h", 1.0)
    ids = Guarded((1, w.K, w.kmax), torch.int32, fill=-7)
    vals = Guarded((1, w.K, w.kmax), torch.float32, fill=float("nan"))
    ws = _ws(md.heads_workspace_bytes(1, w.d, w.V, w.K, w.kmax))
    md.medusa_heads(h, W1, b1, Wv, w.k_per_head, ids.t, vals.t, ws.t)
    _assert_intact(ids=ids, vals=vals, ws=ws)
    del W1, b1, Wv
    parent, rank = _tree(w.k_per_head, w.n_nodes)
    tree = md.Tree(parent, rank, w.k_per_head)
    q = device.fill_normal(torch.empty((1, w.T, w.Hq, w.dh), **bf), w.seed, "q", 1.0)
    kc = device.fill_normal(torch.empty((1, w.Hkv, w.S_max, w.dh), **bf), w.seed, "k_cache", 1.0)
    vc = device.fill_normal(torch.empty((1, w.Hkv, w.S_max, w.dh), **bf), w.seed, "v_cache", 1.0)
    out = Guarded((1, w.T, w.Hq, w.dh), torch.float32, fill=float("nan"))
    ws2 = _ws(md.attention_workspace_bytes(1, w.T, w.Hq, w.Hkv, w.dh, w.S_max))
    md.tree_attention(q, kc, vc, i32([4096]), tree, out.t, ws2.t)
    _assert_intact(out=out, ws=ws2)
    assert torch.isfinite(out.t).all()
