"""GPU parity of md_medusa_heads against the oracle (B200 only)."""
import numpy as np
import pytest

from oracle import heads as oh
from seeded_inputs import gen

from .helpers import HEADS_RTOL, bf16_tensor, check_topk_row, head_weights, normwise

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def _run(h, W1, b1, Wv, kph, kmax=None, dbg=True):
    import medusa_draft_heads_b200 as md
    M, d = h.shape
    K, _, V = Wv.shape
    kmax = kmax or max(kph)
    ids = torch.full((M, K, kmax), -7, dtype=torch.int32, device="cuda")
    vals = torch.zeros((M, K, kmax), dtype=torch.float32, device="cuda")
    logits = torch.zeros((M, K, V), dtype=torch.float32, device="cuda") if dbg else None
    ws = md.workspace(md.heads_workspace_bytes(M, d, V, K, kmax))
    md.medusa_heads(bf16_tensor(h), bf16_tensor(W1), bf16_tensor(b1), bf16_tensor(Wv), kph, ids, vals, ws,
                    logits_dbg=logits)
    torch.cuda.synchronize()
    assert md.device_status() == 0
    return ids.cpu().numpy(), vals.cpu().numpy(), (logits.cpu().numpy() if dbg else None)


@pytest.mark.parametrize("M,d,V,kph", [(1, 256, 1024, (4, 3, 2, 2)), (2, 512, 1000, (10, 10, 10, 10)),
                                       (8, 320, 2056, (16, 1, 7, 3)), (3, 1024, 4096, (5, 5, 5, 5))])
def test_heads_match_oracle_small(M, d, V, kph):
    h, W1, b1, Wv = head_weights(11 + M, d, V, len(kph), M)
    kmax = min(16, max(kph) + 1)           # one spare slot where the stride allows it
    ids, vals, logits = _run(h, W1, b1, Wv, kph, kmax=kmax)
    rid, rval, rlog, _ = oh.medusa_heads(h, W1, b1, Wv, kph, kmax)
    err = normwise(logits, rlog)
    assert err.max() <= HEADS_RTOL, err.max()
    # fp32 accumulation sits far inside the stated bound; single rows can move by
    # one bf16 step of z (a value on a rounding boundary), so check the bulk
    assert np.median(err) <= 1e-5, np.median(err)
    for m in range(M):
        for k, kk in enumerate(kph):
            check_topk_row(ids[m, k], vals[m, k], rlog[m, k], kk)
            assert np.all(ids[m, k, kk:] == -1) and np.all(np.isneginf(vals[m, k, kk:]))


def _integer_heads(seed, M, d, V, K):
    """h, Wv small integers and W1 = b1 = 0: z = h exactly and every logit is
    an integer both sides compute exactly, with many exact ties."""
    rng = np.random.default_rng(seed)
    hv = rng.integers(-2, 3, (M, d)).astype(np.float32)
    wv = rng.integers(-1, 2, (K, d, V)).astype(np.float32)
    h = gen.f32_to_bf16_bits(hv)
    Wv = gen.f32_to_bf16_bits(wv)
    W1 = np.zeros((K, d, d), dtype=np.uint16)
    b1 = np.zeros((K, d), dtype=np.uint16)
    return h, W1, b1, Wv


@pytest.mark.parametrize("M,d,V,kph", [(1, 128, 1024, (16, 10, 1, 5)), (4, 256, 1000, (3, 16, 2, 9)),
                                       (8, 64, 776, (16, 16, 16, 16))])
def test_topk_bit_exact_on_exact_integer_logits(M, d, V, kph):
    h, W1, b1, Wv = _integer_heads(M * 7 + d, M, d, V, len(kph))
    ids, vals, logits = _run(h, W1, b1, Wv, kph)
    rid, rval, rlog, _ = oh.medusa_heads(h, W1, b1, Wv, kph)
    assert np.array_equal(logits, rlog.astype(np.float32))
    assert np.array_equal(ids, rid)
    assert np.array_equal(vals, rval.astype(np.float32))
    # ties really were exercised
    ties = sum(int(np.sum(rlog[m, k] == rval[m, k, kk - 1])) > 1
               for m in range(M) for k, kk in enumerate(kph))
    assert ties > 0


@pytest.mark.parametrize("M,K,kk", [(1, 4, 10), (4, 4, 10), (40, 2, 16)])
def test_topk_exact_when_most_candidates_pass_the_threshold(M, K, kk):
    """Every 256-column tile holds kk - 1 columns of the top value: each list's
    first kk - 1 entries tie at the top and its kk-th is lower, so the best of
    the lists' kk-th entries lets hundreds of tied entries through and the
    kk-th best of the lists' first entries (ties to the lower id) decides."""
    d, V = 128, 256 * 32
    rng = np.random.default_rng(40 + M)
    hv = rng.choice(np.array([-1.0, 1.0], dtype=np.float32), size=d)
    c = rng.integers(0, 2, (K, V)).astype(np.float32)
    c[:, (np.arange(V) % 256) < kk - 1] = 3.0
    h = gen.f32_to_bf16_bits(np.tile(hv, (M, 1)))
    Wv = gen.f32_to_bf16_bits(hv[None, :, None] * c[:, None, :])     # logit = c * d exactly
    W1 = np.zeros((K, d, d), dtype=np.uint16)
    b1 = np.zeros((K, d), dtype=np.uint16)
    kph = (kk,) * K
    ids, vals, logits = _run(h, W1, b1, Wv, kph)
    rid, rval, rlog, _ = oh.medusa_heads(h, W1, b1, Wv, kph)
    assert np.array_equal(logits, rlog.astype(np.float32))
    assert np.array_equal(ids, rid)
    assert np.array_equal(vals, rval.astype(np.float32))
    assert np.all(rval[:, :, kk - 1] == 3 * d)


@pytest.mark.parametrize("M", [1, 10])
@pytest.mark.parametrize("fill", ["zeros", "ones", "random"])
def test_heads_need_no_cleared_workspace(M, fill):
    """The tickets of the one-row and weights-as-M paths carry a per-call
    epoch: a workspace holding anything at all, and the same workspace reused
    call after call, give the same results bit for bit (cut units and split-K
    tiles on both paths)."""
    import medusa_draft_heads_b200 as md
    d, V, kph = 1024, 10000, (10, 4, 7, 1)      # one row: 160 units over 148 CTAs, cut units
    h, W1, b1, Wv = head_weights(77 + M, d, V, len(kph), M)
    ref_ids, ref_vals, ref_log = _run(h, W1, b1, Wv, kph)
    K, kmax = len(kph), max(kph)
    ws = md.workspace(md.heads_workspace_bytes(M, d, V, K, kmax))
    if fill == "zeros":
        ws.zero_()
    elif fill == "ones":
        ws.fill_(255)
    else:
        ws.copy_(torch.randint(0, 256, ws.shape, dtype=torch.uint8, device="cuda"))
    hb, W1b, b1b, Wvb = bf16_tensor(h), bf16_tensor(W1), bf16_tensor(b1), bf16_tensor(Wv)
    for _ in range(3):
        ids = torch.full((M, K, kmax), -7, dtype=torch.int32, device="cuda")
        vals = torch.zeros((M, K, kmax), dtype=torch.float32, device="cuda")
        logits = torch.zeros((M, K, V), dtype=torch.float32, device="cuda")
        md.medusa_heads(hb, W1b, b1b, Wvb, kph, ids, vals, ws, logits_dbg=logits)
        torch.cuda.synchronize()
        assert md.device_status() == 0
        assert np.array_equal(ids.cpu().numpy(), ref_ids)
        assert np.array_equal(vals.cpu().numpy(), ref_vals)
        assert np.array_equal(logits.cpu().numpy(), ref_log)


def test_heads_are_deterministic():
    h, W1, b1, Wv = head_weights(5, 512, 2048, 4, 2)
    a = _run(h, W1, b1, Wv, (10, 10, 10, 10))
    b = _run(h, W1, b1, Wv, (10, 10, 10, 10))
    for x, y in zip(a, b):
        assert np.array_equal(x, y)


def test_heads_reject_bad_arguments():
    import medusa_draft_heads_b200 as md
    h, W1, b1, Wv = head_weights(1, 256, 1024, 4, 1)
    ids = torch.zeros((1, 4, 4), dtype=torch.int32, device="cuda")
    vals = torch.zeros((1, 4, 4), dtype=torch.float32, device="cuda")
    ws = md.workspace(64)
    with pytest.raises(md.MedusaError, match="workspace"):
        md.medusa_heads(bf16_tensor(h), bf16_tensor(W1), bf16_tensor(b1), bf16_tensor(Wv), (4, 3, 2, 2), ids,
                        vals, ws)
    ws = md.workspace(md.heads_workspace_bytes(1, 256, 1024, 4, 4))
    with pytest.raises(md.MedusaError, match="invalid"):
        md.medusa_heads(bf16_tensor(h), bf16_tensor(W1), bf16_tensor(b1), bf16_tensor(Wv), (5, 3, 2, 2), ids,
                        vals, ws)


# ------------- tensor-core paths (M > 1: weights as M up to 32 rows, row tiles up to 128, CTA pairs beyond) -------------

@pytest.mark.parametrize("M,d,V,kph", [(9, 256, 1024, (4, 3, 2, 2)), (40, 320, 1000, (10, 10, 10, 10)),
                                       (130, 512, 2056, (16, 1, 7, 3)), (520, 256, 4096, (10, 10, 10, 10))])
def test_tensor_core_heads_match_oracle(M, d, V, kph):
    h, W1, b1, Wv = head_weights(101 + M, d, V, len(kph), M)
    ids, vals, logits = _run(h, W1, b1, Wv, kph)
    rid, rval, rlog, _ = oh.medusa_heads(h, W1, b1, Wv, kph)
    err = normwise(logits, rlog)
    assert err.max() <= HEADS_RTOL, err.max()
    assert np.median(err) <= 1e-5, np.median(err)
    for m in range(M):
        for k, kk in enumerate(kph):
            check_topk_row(ids[m, k], vals[m, k], rlog[m, k], kk)


@pytest.mark.parametrize("M,d,V,kph", [(17, 128, 1024, (16, 10, 1, 5)), (200, 64, 776, (3, 16, 2, 9)),
                                       (300, 128, 520, (8, 2))])
def test_tensor_core_topk_bit_exact_on_integer_logits(M, d, V, kph):
    h, W1, b1, Wv = _integer_heads(M * 3 + d, M, d, V, len(kph))
    ids, vals, logits = _run(h, W1, b1, Wv, kph)
    rid, rval, rlog, _ = oh.medusa_heads(h, W1, b1, Wv, kph)
    assert np.array_equal(logits, rlog.astype(np.float32))
    assert np.array_equal(ids, rid)
    assert np.array_equal(vals, rval.astype(np.float32))


def test_tensor_core_fused_equals_debug_run():
    """The top-k does not depend on whether the logits are also written."""
    h, W1, b1, Wv = head_weights(77, 512, 4096, 4, 64)
    a = _run(h, W1, b1, Wv, (10, 10, 10, 10), dbg=False)
    b = _run(h, W1, b1, Wv, (10, 10, 10, 10), dbg=True)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


# ------------- tensor cores with the weights as the MMA's M (2 .. 32 rows) -------------

@pytest.mark.parametrize("M,d,V,kph", [
    (2, 512, 2056, (10, 10, 10, 10)),        # the smallest row count of this path
    (5, 1024, 8192, (10,)),                  # one head: 4 phase-1 units over 64 CTAs, 16 parts each
    (10, 4096, 4096, (10,)),                 # a Hydra level's row count; units cut into many parts
    (16, 576, 3000, (4, 3, 2, 2)),           # 9 stages per unit, ragged last vocabulary tile
    (17, 512, 1000, (10, 10, 10, 10)),       # 32-row padding, 17 live rows
    (32, 256, 2056, (16, 1, 7, 3)),          # the largest row count of this path
    (33, 256, 1024, (10, 10, 10, 10)),       # 33 .. 128 rows: one 128-row tile per CTA
])
def test_weights_as_m_heads_match_oracle(M, d, V, kph):
    h, W1, b1, Wv = head_weights(500 + M, d, V, len(kph), M)
    ids, vals, logits = _run(h, W1, b1, Wv, kph)
    ids2, vals2, logits2 = _run(h, W1, b1, Wv, kph)
    # the parts of a cut unit are summed in a fixed order: runs agree bit for bit
    assert np.array_equal(logits, logits2) and np.array_equal(ids, ids2) and np.array_equal(vals, vals2)
    rid, rval, rlog, _ = oh.medusa_heads(h, W1, b1, Wv, kph)
    err = normwise(logits, rlog)
    assert err.max() <= HEADS_RTOL, err.max()
    assert np.median(err) <= 1e-5, np.median(err)
    for m in range(M):
        for k, kk in enumerate(kph):
            check_topk_row(ids[m, k], vals[m, k], rlog[m, k], kk)


# ------------------------- shared vocabulary projection -------------------------

def _run_shared(h, W1, b1, Wv, kph, kmax=None):
    import medusa_draft_heads_b200 as md
    M, d = h.shape
    K, V = W1.shape[0], Wv.shape[1]
    kmax = kmax or max(kph)
    ids = torch.full((M, K, kmax), -7, dtype=torch.int32, device="cuda")
    vals = torch.zeros((M, K, kmax), dtype=torch.float32, device="cuda")
    logits = torch.zeros((M, K, V), dtype=torch.float32, device="cuda")
    ws = md.workspace(md.heads_shared_workspace_bytes(M, d, V, K, kmax))
    md.medusa_heads_shared(bf16_tensor(h), bf16_tensor(W1), bf16_tensor(b1), bf16_tensor(Wv), kph, ids, vals, ws,
                           logits_dbg=logits)
    torch.cuda.synchronize()
    assert md.device_status() == 0
    return ids.cpu().numpy(), vals.cpu().numpy(), logits.cpu().numpy()


@pytest.mark.parametrize("M,d,V,kph", [(1, 256, 1024, (10,)),                      # one row: streaming
                                       (1, 256, 1024, (4, 3, 2, 2)), (1, 512, 2056, (10, 10, 10, 10)),
                                       (2, 320, 1000, (16, 1)), (3, 256, 4096, (10, 10, 10, 10)),
                                       (6, 576, 3000, (16, 7, 3, 1)),              # 24 rows after a 6-row phase 1
                                       (12, 576, 3000, (16, 7, 3, 1)),             # 48 rows: row-tile GEMMs
                                       (130, 256, 1024, (7, 3, 2))])
def test_shared_projection_matches_oracle(M, d, V, kph):
    K = len(kph)
    h, W1, b1, _ = head_weights(300 + M, d, V, K, M)
    Wv = gen.normal_bf16(300 + M, "Wv", (d, V), 0.02)
    ids, vals, logits = _run_shared(h, W1, b1, Wv, kph)
    rid, rval, rlog, _ = oh.medusa_heads_shared(h, W1, b1, Wv, kph)
    err = normwise(logits, rlog)
    assert err.max() <= HEADS_RTOL and np.median(err) <= 1e-5, err.max()
    for m in range(M):
        for k, kk in enumerate(kph):
            check_topk_row(ids[m, k], vals[m, k], rlog[m, k], kk)


@pytest.mark.parametrize("M,kph", [(1, (16, 10, 1, 5)), (5, (3, 16, 2, 9))])
def test_shared_projection_bit_exact_on_integer_logits(M, kph):
    K = len(kph)
    h, W1, b1, Wv = _integer_heads(M * 11, M, 128, 1024, 1)
    W1 = np.zeros((K, 128, 128), dtype=np.uint16)
    b1 = np.zeros((K, 128), dtype=np.uint16)
    ids, vals, logits = _run_shared(h, W1, b1, Wv[0], kph)
    rid, rval, rlog, _ = oh.medusa_heads_shared(h, W1, b1, Wv[0], kph)
    assert np.array_equal(logits, rlog.astype(np.float32))
    assert np.array_equal(ids, rid) and np.array_equal(vals, rval.astype(np.float32))
