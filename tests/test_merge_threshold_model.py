"""The top-k merge's selection argument, checked on a plain model (CPU).

The heads kernels leave, per (row, head), one sorted candidate list per
producer CTA; the merge keeps only the candidates at or above the stricter of
two thresholds -- the best of the lists' k-th entries, and the k-th best of the
lists' first entries -- and places each kept entry by counting the kept
entries ahead of it. This model restates those steps in numpy and checks,
against a brute-force sort of every candidate, that the kept set always holds
the true top-k, that it never exceeds k * k entries once the second threshold
applies, and that the placement reproduces the sorted top-k. Ties are broken
by the lower id, as everywhere in the library.
"""
import numpy as np
import pytest


def _key(v, i):
    return (-v, i)            # sort key of the top-k order: value descending, then id ascending


def _lists(rng, n_lists, per_list, kk, ties):
    """Disjoint column ranges, each list the sorted top-kk of its range."""
    out, col = [], 0
    for _ in range(n_lists):
        n = int(rng.integers(0, per_list + 1))
        ids = np.arange(col, col + n)
        col += n
        vals = rng.integers(-3, 4, n).astype(np.float32) if ties else rng.standard_normal(n).astype(np.float32)
        order = sorted(range(n), key=lambda j: _key(vals[j], ids[j]))[:kk]
        out.append([(float(vals[j]), int(ids[j])) for j in order])
    return out


def _merge_model(lists, kk):
    better = lambda a, b: _key(*a) < _key(*b)
    # (a) the best of the lists' kk-th entries
    ta = None
    for l in lists:
        if len(l) >= kk and (ta is None or better(l[kk - 1], ta)):
            ta = l[kk - 1]
    # (b) the kk-th best of the lists' first entries
    heads = sorted((l[0] for l in lists if l), key=lambda e: _key(*e))
    tb = heads[kk - 1] if len(heads) >= kk else None
    t = ta
    if tb is not None and (t is None or better(tb, t)):
        t = tb
    kept = [e for l in lists for e in l if t is None or not better(t, e)]
    # placement: the number of kept entries ahead of each one
    out = [None] * min(kk, len(kept))
    for e in kept:
        place = sum(1 for f in kept if better(f, e))
        if place < kk:
            out[place] = e
    return kept, out, tb is not None


@pytest.mark.parametrize("ties", [False, True])
@pytest.mark.parametrize("seed", range(6))
def test_merge_keeps_the_true_top_k_and_at_most_k_squared(seed, ties):
    rng = np.random.default_rng(1000 + seed + 17 * ties)
    for _ in range(40):
        kk = int(rng.integers(1, 17))
        n_lists = int(rng.integers(1, 160))
        lists = _lists(rng, n_lists, int(rng.integers(0, 60)), kk, ties)
        every = sorted((e for l in lists for e in l), key=lambda e: _key(*e))
        truth = every[:kk]
        kept, out, bounded = _merge_model(lists, kk)
        assert set(truth) <= set(kept)
        assert out == truth
        if bounded:
            assert len(kept) <= kk * kk
        else:   # fewer than kk lists hold anything
            assert len(kept) <= (kk - 1) * kk


def test_first_threshold_alone_keeps_many_more():
    """Random logits over 148 lists of 10: the lists' 10th entries alone let
    hundreds through; with the first-entry threshold a handful remain."""
    rng = np.random.default_rng(5)
    lists = _lists(rng, 148, 867, 10, False)
    ta = max((l[9] for l in lists if len(l) >= 10), key=lambda e: (e[0], -e[1]))
    only_a = sum(1 for l in lists for e in l if (e[0], -e[1]) >= (ta[0], -ta[1]))
    kept, out, bounded = _merge_model(lists, 10)
    assert bounded and only_a > 200 and len(kept) <= 20
