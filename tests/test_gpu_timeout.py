"""The bounded-wait failure path, made to happen without a GPU fault: with the
wait bound lowered to 1 ms, md_tree_attention's producers are told (test hook)
to withhold one chunk's K/V copies, so the waits that need them run out. The
call must flag MD_DEV_TIMEOUT and return, and the very next call without the
hook must be correct: the context is usable, every issued copy landed and TMEM
was released. Two launch shapes: 70B-shaped tiles whose key range is cut into
three splits (merged through the cluster's shared memory), and a small case
with one chunk per CTA (every CTA's only chunk withheld)."""
import numpy as np
import pytest

import medusa_draft_heads_b200 as md
from oracle import attention as oa
from oracle import tree as ot
from seeded_inputs.workloads import TREE_ACCEPT

from .helpers import ATTN_RTOL, bf16_tensor, i32, kv_inputs, normwise

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,kph,n,B,Hq,Hkv,dh,P,chunk", [
    ("70b-three-splits", (10, 10, 10, 10), 64, 1, 64, 8, 128, [4096], 2),
    ("one-chunk-per-cta", (4, 3, 2, 2), 16, 2, 4, 2, 64, [900, 300], 0),
])
def test_attention_timeout_flags_and_recovers(name, kph, n, B, Hq, Hkv, dh, P, chunk):
    parent, rank, _ = ot.spec_from_tuples(ot.select_tree(kph, TREE_ACCEPT, n))
    T = len(parent)
    tree = md.Tree(parent, rank, [16] * 4)
    S_max = (max(P) + T + 63) // 64 * 64
    qh, kh, vh = kv_inputs(7, B, T, Hq, Hkv, dh, S_max)
    q, k, v = bf16_tensor(qh), bf16_tensor(kh), bf16_tensor(vh)
    out = torch.full((B, T, Hq, dh), np.nan, dtype=torch.float32, device="cuda")
    ws = md.workspace(md.attention_workspace_bytes(B, T, Hq, Hkv, dh, S_max))
    md.device_status(clear=True)
    md.set_wait_limit(1_000_000)
    md.binding.withhold_attention_chunk_for_test(chunk)
    try:
        md.tree_attention(q, k, v, i32(P), tree, out, ws)
        torch.cuda.synchronize()
        status = md.device_status(clear=True)
    finally:
        md.binding.withhold_attention_chunk_for_test(-1)
        md.set_wait_limit(0)
    assert status & md.binding.DEV_TIMEOUT, status
    # the next call, without the hook, is correct
    out.fill_(np.nan)
    md.tree_attention(q, k, v, i32(P), tree, out, ws)
    torch.cuda.synchronize()
    assert md.device_status() == 0
    ref = oa.tree_attention(qh, kh, vh, np.array(P), parent, rows=[(b, t, h) for b in range(B) for t in (0, T - 1)
                                                                    for h in (0, Hq - 1)])
    got = out.cpu().numpy()
    for b in range(B):
        for t in (0, T - 1):
            for h in (0, Hq - 1):
                assert normwise(got[b, t, h], ref[b, t, h]) <= ATTN_RTOL
