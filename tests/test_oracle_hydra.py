"""Pins of the Hydra drafting oracle against closed forms, a reduction to the
Medusa tree and invariants of sequential dependence."""
import numpy as np
import pytest

from oracle import heads as oh
from oracle import hydra as ohy
from oracle import tree as ot
from seeded_inputs import gen
from seeded_inputs.workloads import TREE_ACCEPT

ONE = 0x3F80          # bf16 bits of 1.0


def _spec(kph=(4, 3, 2, 2), n=16):
    return ot.spec_from_tuples(ot.select_tree(kph, TREE_ACCEPT, n))


def _random_case(seed, B, d, V, K=4, E_sigma=1.0):
    h = gen.normal_bf16(seed, "h", (B + 1, d), 1.0)
    E = gen.normal_bf16(seed, "E", (V, d), E_sigma)
    W1 = gen.normal_bf16(seed, "W1", (K, d, d), 0.05)
    b1 = gen.normal_bf16(seed, "b1", (K, d), 0.05)
    Wv = gen.normal_bf16(seed, "Wv", (K, d, V), 0.05)
    return h, E, W1, b1, Wv


def test_zero_embedding_reduces_to_medusa_tree():
    """E = 0: every head reads h itself, so each depth's candidates no longer
    depend on the parent and the tree is the Medusa one."""
    parent, rank, _ = _spec()
    B, d, V = 2, 64, 256
    h, _, W1, b1, Wv = _random_case(1, B, d, V)
    E = np.zeros((V, d), dtype=np.uint16)
    root = np.array([5, 200])
    P = np.array([10, 33])
    row = np.array([2, 0])
    tok, par, anc, pos, _ = ohy.hydra_draft(parent, rank, h, E, W1, b1, Wv, root, P, head_row=row)
    ids, _, _, _ = oh.medusa_heads(h, W1, b1, Wv, (4, 3, 2, 2))
    rtok, rpar, ranc, rpos = ot.tree_build(parent, rank, ids, root, P, head_row=row)
    assert np.array_equal(tok, rtok)
    assert np.array_equal(par, rpar) and np.array_equal(anc, ranc) and np.array_equal(pos, rpos)


def _shift_weights(V, K):
    """h = 0, W1 = 0, b1 = 0 (so z = x), E[t] = one-hot at (t + 1) mod V and
    Wv_k = the permutation i -> (i + k) mod V (d = V)."""
    d = V
    h = np.zeros((1, d), dtype=np.uint16)
    E = np.zeros((V, d), dtype=np.uint16)
    E[np.arange(V), (np.arange(V) + 1) % V] = ONE
    W1 = np.zeros((K, d, d), dtype=np.uint16)
    b1 = np.zeros((K, d), dtype=np.uint16)
    Wv = np.zeros((K, d, V), dtype=np.uint16)
    for k in range(K):
        Wv[k, np.arange(d), (np.arange(d) + k) % V] = ONE
    return h, E, W1, b1, Wv


def _shift_expected(parent, rank, depth, root, V):
    """Closed form of the shift construction: head k on parent token t scores
    1 at c = (t + 1 + k) mod V and 0 elsewhere, so rank 0 is c and rank r >= 1
    is the (r - 1)-th smallest id other than c."""
    tok = np.zeros(len(parent), dtype=np.int64)
    tok[0] = root
    for j in range(1, len(parent)):
        t = int(tok[parent[j]])
        k = int(depth[j]) - 1
        c = (t + 1 + k) % V
        r = int(rank[j])
        tok[j] = c if r == 0 else ((r - 1) if (r - 1) < c else r)
    return tok


@pytest.mark.parametrize("kph,n,root", [((4, 3, 2, 2), 16, 7), ((10, 10, 10, 10), 64, 60), ((1, 1, 1, 1), 4, 63),
                                        ((10, 10, 10, 10), 64, 0)])
def test_shift_construction_closed_form(kph, n, root):
    V = 64
    parent, rank, depth = ot.spec_from_tuples(ot.select_tree(kph, TREE_ACCEPT, n))
    h, E, W1, b1, Wv = _shift_weights(V, 4)
    tok, _, _, _, _ = ohy.hydra_draft(parent, rank, h, E, W1, b1, Wv, np.array([root]), np.array([0]))
    assert np.array_equal(tok[0], _shift_expected(parent, rank, depth, root, V))
    # the top-1 chain walks root + 1, root + 3, root + 6, root + 10 (mod V)
    if kph == (1, 1, 1, 1):
        assert tok[0].tolist() == [root, (root + 1) % V, (root + 3) % V, (root + 6) % V, (root + 10) % V]


def test_changing_one_embedding_row_moves_only_that_tokens_descendants():
    parent, rank, _ = _spec()
    B, d, V = 2, 64, 256
    h, E, W1, b1, Wv = _random_case(3, B, d, V)
    root = np.array([11, 97])
    P = np.array([4, 4])
    tok, *_ = ohy.hydra_draft(parent, rank, h, E, W1, b1, Wv, root, P)
    t_star = int(tok[0, 1])                      # the rank-0 draft of depth 1, request 0
    assert t_star not in (int(root[0]), int(root[1]))
    E2 = E.copy()
    E2[t_star] = oh.f64_to_bf16(-3.0 * oh.bf16_to_f64(E[t_star]))
    tok2, *_ = ohy.hydra_draft(parent, rank, h, E2, W1, b1, Wv, root, P)
    anc = ot.ancestors(parent)
    changed = 0
    for b in range(B):
        for j in range(len(parent)):
            strict = anc[j] - {j}
            if any(int(tok[b, a]) == t_star for a in strict):
                changed += int(tok[b, j] != tok2[b, j])
            else:
                assert tok[b, j] == tok2[b, j], (b, j)
    assert changed > 0


def test_children_follow_their_parents_logits():
    """Siblings are distinct, and a child of rank r holds the rank-r entry of
    its parent's logit row under (value desc, id asc)."""
    parent, rank, depth = _spec((10, 10, 10, 10), 64)
    B, d, V = 1, 64, 512
    h, E, W1, b1, Wv = _random_case(4, B, d, V)
    tok, _, _, _, logits = ohy.hydra_draft(parent, rank, h, E, W1, b1, Wv, np.array([3]), np.array([0]))
    kids = {}
    for j in range(1, len(parent)):
        kids.setdefault(int(parent[j]), []).append(j)
    assert set(p for (_, p) in logits) == set(kids)
    for p, js in kids.items():
        row = logits[(0, p)]
        order = sorted(range(V), key=lambda v: (-row[v], v))
        toks = [int(tok[0, j]) for j in js]
        assert len(set(toks)) == len(toks)
        for j in js:
            assert int(tok[0, j]) == order[int(rank[j])]
    # the rows differ between parents: the heads see the parent's token
    d2 = [p for p in kids if depth[p] == 1]
    assert not np.allclose(logits[(0, d2[0])], logits[(0, d2[1])])


def test_head_input_rounds_the_exact_sum_to_nearest_even():
    d = 4
    E = np.zeros((1, d), dtype=np.uint16)
    h = np.zeros(d, dtype=np.uint16)
    # h = [1, 1 + 2^-7, 1, 3], E = [2^-8, 2^-8, 2^-8 + 2^-15, -3] (all bf16 values)
    h[:] = gen.f32_to_bf16_bits(np.array([1.0, 1.0 + 2.0 ** -7, 1.0, 3.0], dtype=np.float32))
    E[0] = gen.f32_to_bf16_bits(np.array([2.0 ** -8, 2.0 ** -8, 2.0 ** -8 + 2.0 ** -15, -3.0], dtype=np.float32))
    assert oh.bf16_to_f64(E[0])[2] == 2.0 ** -8 + 2.0 ** -15
    x = oh.bf16_to_f64(ohy.head_input(h, E, 0))
    # a tie goes to the even neighbour; above the tie rounds up; exact zero stays zero
    assert x.tolist() == [1.0, 1.0 + 2.0 ** -6, 1.0 + 2.0 ** -7, 0.0]


def _random_tree(rng, T, kph):
    """A tree of T nodes of any shape the library accepts: parent[j] < j,
    depth <= len(kph), distinct ranks below one parent."""
    parent, rank, depth = [-1], [0], [0]
    used = {0: set()}
    while len(parent) < T:
        p = int(rng.integers(0, len(parent)))
        if depth[p] >= len(kph):
            continue
        free = [r for r in range(kph[depth[p]]) if r not in used[p]]
        if not free:
            continue
        r = int(rng.choice(free))
        used[p].add(r)
        used[len(parent)] = set()
        parent.append(p)
        rank.append(r)
        depth.append(depth[p] + 1)
    return np.array(parent), np.array(rank), np.array(depth)


@pytest.mark.parametrize("seed", range(4))
def test_random_tree_shapes(seed):
    """Trees not made by the tree selection (siblings out of rank order,
    skipped ranks, uneven depths): the shift closed form and the reduction to
    the Medusa tree both still hold."""
    rng = np.random.default_rng(100 + seed)
    kph = (5, 4, 3, 2)
    parent, rank, depth = _random_tree(rng, 24, kph)
    V = 64
    h, E, W1, b1, Wv = _shift_weights(V, 4)
    root = int(rng.integers(0, V))
    tok, par, anc, pos, _ = ohy.hydra_draft(parent, rank, h, E, W1, b1, Wv, np.array([root]), np.array([3]))
    assert np.array_equal(tok[0], _shift_expected(parent, rank, depth, root, V))
    assert np.array_equal(pos[0], 3 + depth)
    B, d, V2 = 1, 64, 256
    hh, _, W1r, b1r, Wvr = _random_case(seed, B, d, V2)
    Ez = np.zeros((V2, d), dtype=np.uint16)
    t0, *_ = ohy.hydra_draft(parent, rank, hh, Ez, W1r, b1r, Wvr, np.array([7]), np.array([0]))
    ids, _, _, _ = oh.medusa_heads(hh, W1r, b1r, Wvr, kph)
    rtok, _, _, _ = ot.tree_build(parent, rank, ids, np.array([7]), np.array([0]))
    assert np.array_equal(t0, rtok)
