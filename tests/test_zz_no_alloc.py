"""md_medusa_heads_static: the heads call for callers that cannot allocate.

Some callers cannot give the library a workspace -- runtimes whose device
memory belongs to a pool that no plugin may grow, or decode loops that must
never reach the allocator -- so the library offers one variant of the heads
call whose scratch is a fixed array in its own device image. These checks call
it through the C ABI (ctypes, raw pointers) twice in a row and compare each
result with the ordinary md_medusa_heads on the same inputs (streaming,
weights-as-M, single-CTA and CTA-pair tensor-core paths), and check that a shape whose
scratch would not fit is refused before anything runs.

This file is named to be collected last, so a run that stops at the first
failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest

import medusa_draft_heads_b200 as md

from .helpers import head_weights, bf16_tensor

STATIC_BYTES = 32 << 20     # MD_HEADS_STATIC_SCRATCH_BYTES in include/medusa.h

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def _static_fn():
    fn = md.lib().md_medusa_heads_static
    P, I = ctypes.c_void_p, ctypes.c_int32
    fn.argtypes = [P, P, P, P, I, I, I, I, P, I, P, P, P, P]
    fn.restype = ctypes.c_int32
    return fn


def _call_static(h, W1, b1, Wv, kph, ids, vals, logits=None):
    M, d = h.shape
    K, _, V = Wv.shape
    k_arr = (ctypes.c_int32 * K)(*kph)
    stream = torch.cuda.current_stream().cuda_stream
    return _static_fn()(h.data_ptr(), W1.data_ptr(), b1.data_ptr(), Wv.data_ptr(), M, d, V, K, k_arr,
                        ids.shape[2], ids.data_ptr(), vals.data_ptr(),
                        None if logits is None else logits.data_ptr(), stream)


@pytest.mark.parametrize("M,d,V,kph", [(1, 1024, 8192, (10, 10, 10, 10)), (3, 512, 2056, (16, 1, 7, 3)),
                                       (20, 256, 4096, (10, 10, 10, 10)), (100, 256, 4096, (10, 10, 10, 10)),
                                       (160, 256, 4096, (10, 10, 10, 10))])
def test_static_scratch_matches_workspace_call(M, d, V, kph):
    h, W1, b1, Wv = (bf16_tensor(x) for x in head_weights(900 + M, d, V, len(kph), M))
    K, kmax = len(kph), max(kph)
    assert md.heads_workspace_bytes(M, d, V, K, kmax) <= STATIC_BYTES
    ref_ids = torch.empty((M, K, kmax), dtype=torch.int32, device="cuda")
    ref_vals = torch.empty((M, K, kmax), dtype=torch.float32, device="cuda")
    ws = md.workspace(md.heads_workspace_bytes(M, d, V, K, kmax))
    md.medusa_heads(h, W1, b1, Wv, kph, ref_ids, ref_vals, ws)
    torch.cuda.synchronize()
    for _ in range(2):                      # two calls in a row share the static scratch
        ids = torch.full((M, K, kmax), -5, dtype=torch.int32, device="cuda")
        vals = torch.zeros((M, K, kmax), dtype=torch.float32, device="cuda")
        assert _call_static(h, W1, b1, Wv, kph, ids, vals) == 0
        torch.cuda.synchronize()
        assert np.array_equal(ids.cpu().numpy(), ref_ids.cpu().numpy())
        np.testing.assert_allclose(vals.cpu().numpy(), ref_vals.cpu().numpy(), rtol=1e-6, atol=0)
    assert md.device_status() == 0


def test_static_scratch_refuses_oversized_shapes():
    """M = 1024 rows of 70B-shaped heads need more scratch than the array holds."""
    M, d, V, K, kmax = 1024, 8192, 128256, 4, 10
    assert md.heads_workspace_bytes(M, d, V, K, kmax) > STATIC_BYTES
    h = torch.empty((M, d), dtype=torch.bfloat16, device="cuda")
    W1 = torch.empty((K, d, d), dtype=torch.bfloat16, device="cuda")
    b1 = torch.empty((K, d), dtype=torch.bfloat16, device="cuda")
    Wv = torch.empty((K, d, V), dtype=torch.bfloat16, device="cuda")
    ids = torch.empty((M, K, kmax), dtype=torch.int32, device="cuda")
    vals = torch.empty((M, K, kmax), dtype=torch.float32, device="cuda")
    assert _call_static(h, W1, b1, Wv, (10,) * K, ids, vals) == -4       # MD_ERR_WORKSPACE
    assert md.device_status() == 0
