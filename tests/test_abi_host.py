"""CPU-only checks of the C ABI library and the product's host logic.

No kernel is launched here: the library is loaded, every symbol the header
declares is looked up, and the host-only entry points (tree spec validation,
workspace sizing, status strings) are exercised.
"""
import ctypes
import os
import re

import pytest

from medusa_draft_heads_b200 import build as mdbuild
from medusa_draft_heads_b200 import tree_spec
from oracle import tree as ot
from seeded_inputs.workloads import CHAIN_ACCEPT, TREE_ACCEPT

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def libmedusa():
    path = mdbuild.build()
    return ctypes.CDLL(path)


def _declared_symbols():
    names = set()
    inc = os.path.join(ROOT, "include")
    for f in os.listdir(inc):
        if f.endswith(".h"):
            text = open(os.path.join(inc, f)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"\b(md_[a-z0-9_]+)\s*\(", text))
    return sorted(names)


def test_header_declares_the_four_calls():
    names = _declared_symbols()
    for n in ("md_medusa_heads", "md_tree_build", "md_tree_attention", "md_tree_accept"):
        assert n in names


def test_library_exports_every_declared_symbol(libmedusa):
    for name in _declared_symbols():
        assert hasattr(libmedusa, name), name


def test_status_strings_and_version(libmedusa):
    libmedusa.md_status_string.restype = ctypes.c_char_p
    assert libmedusa.md_status_string(0) == b"ok"
    assert b"workspace" in libmedusa.md_status_string(-4)
    assert libmedusa.md_version() >= 100


def _i32(v):
    return (ctypes.c_int32 * len(v))(*v)


def _create(libmedusa, parent, rank, K, kph):
    h = ctypes.c_void_p()
    rc = libmedusa.md_tree_create(_i32(parent), _i32(rank), len(parent), K, _i32(kph), ctypes.byref(h))
    if rc == 0:
        libmedusa.md_tree_destroy(h)
    return rc


def test_tree_create_validates_spec(libmedusa):
    ok = _create(libmedusa, [-1, 0, 0, 1], [0, 0, 1, 0], 2, [2, 1])
    assert ok == 0
    assert _create(libmedusa, [0, 0], [0, 0], 1, [1]) == -1            # root must have parent -1
    assert _create(libmedusa, [-1, 1], [0, 0], 1, [1]) == -1           # parent[j] < j
    assert _create(libmedusa, [-1, 0, 1], [0, 0, 0], 1, [1]) == -1     # depth 2 > K = 1
    assert _create(libmedusa, [-1, 0], [0, 3], 1, [3]) == -1           # rank < k
    assert _create(libmedusa, [-1, 0, 0], [0, 1, 1], 1, [3]) == -1     # duplicate sibling rank
    assert _create(libmedusa, [-1] + [0] * 128, [0] + list(range(128)), 1, [16]) == -1  # T > 128


def test_tree_info(libmedusa):
    h = ctypes.c_void_p()
    assert libmedusa.md_tree_create(_i32([-1, 0, 1, 1]), _i32([0, 0, 0, 1]), 4, 3, _i32([1, 2, 1]),
                                    ctypes.byref(h)) == 0
    T, d = ctypes.c_int32(), ctypes.c_int32()
    assert libmedusa.md_tree_info(h, ctypes.byref(T), ctypes.byref(d)) == 0
    assert (T.value, d.value) == (4, 2)
    libmedusa.md_tree_destroy(h)


def test_workspace_queries_and_unsupported_sizes(libmedusa):
    n = ctypes.c_size_t()
    assert libmedusa.md_heads_workspace(1, 8192, 128256, 4, 10, ctypes.byref(n)) == 0 and n.value > 0
    assert libmedusa.md_heads_workspace(1, 100, 1024, 4, 10, ctypes.byref(n)) == -2     # d % 64
    assert libmedusa.md_heads_workspace(1, 256, 1020, 4, 10, ctypes.byref(n)) == -2     # V % 8
    assert libmedusa.md_heads_workspace(1, 256, 1024, 9, 10, ctypes.byref(n)) == -2     # K > 8
    assert libmedusa.md_heads_workspace(0, 256, 1024, 4, 10, ctypes.byref(n)) == -1
    assert libmedusa.md_attention_workspace(1, 65, 64, 8, 128, 4224, ctypes.byref(n)) == 0
    assert libmedusa.md_attention_workspace(1, 65, 64, 8, 96, 4224, ctypes.byref(n)) == -2   # dh
    assert libmedusa.md_attention_workspace(1, 65, 60, 8, 128, 4224, ctypes.byref(n)) == -2  # Hq % Hkv
    assert libmedusa.md_accept_workspace(1, 65, 128256, ctypes.byref(n)) == 0
    assert libmedusa.md_accept_workspace(1, 129, 128256, ctypes.byref(n)) == -2


def test_static_heads_checks_arguments_before_scratch_size(libmedusa):
    """md_medusa_heads_static rejects null pointers and bad per-head k as
    md_medusa_heads does, even for a shape whose scratch would not fit; only
    valid arguments reach the size check. Nothing is launched on either path."""
    fn = libmedusa.md_medusa_heads_static
    P, I = ctypes.c_void_p, ctypes.c_int32
    fn.argtypes = [P, P, P, P, I, I, I, I, P, I, P, P, P, P]
    fn.restype = I
    kph = _i32([10, 10, 10, 10])
    fake = ctypes.c_void_p(4096)          # never dereferenced: the call returns before any launch
    big = (1024, 8192, 128256, 4)         # scratch far beyond the 32 MiB array
    assert fn(None, fake, fake, fake, *big, kph, 10, fake, fake, None, None) == -1
    assert fn(fake, fake, fake, fake, *big, None, 10, fake, fake, None, None) == -1
    assert fn(fake, fake, fake, fake, *big, _i32([10, 10, 11, 10]), 10, fake, fake, None, None) == -1
    assert fn(fake, fake, fake, fake, *big, kph, 10, fake, fake, None, None) == -4


@pytest.mark.parametrize("kph,a,n", [((4, 3, 2, 2), TREE_ACCEPT, 16), ((10, 10, 10, 10), TREE_ACCEPT, 64),
                                     ((10, 10, 10, 10), TREE_ACCEPT, 16), ((1, 1, 1, 1), CHAIN_ACCEPT, 4),
                                     ((5, 4, 3), (0.9, 0.5, 0.5), 40), ((3, 3, 3, 3), (1.0, 1.0, 0.5, 0.5), 30)])
def test_product_tree_choice_equals_oracle(kph, a, n):
    """Best-first expansion (product) against brute-force sorting (oracle)."""
    assert tree_spec.select_tree(kph, a, n) == ot.select_tree(kph, a, n)
    parent, rank = tree_spec.tree_arrays(tree_spec.select_tree(kph, a, n))
    p2, r2, _ = ot.spec_from_tuples(ot.select_tree(kph, a, n))
    assert parent == list(p2) and rank[1:] == list(r2[1:])


def _tree_handle(libmedusa, kph, n, accept=TREE_ACCEPT):
    parent, rank = tree_spec.tree_arrays(tree_spec.select_tree(kph, accept, n))
    h = ctypes.c_void_p()
    assert libmedusa.md_tree_create(_i32(parent), _i32(rank), len(parent), len(kph), _i32(list(kph)),
                                    ctypes.byref(h)) == 0
    return h


def test_hydra_workspace_queries(libmedusa):
    n = ctypes.c_size_t()
    h = _tree_handle(libmedusa, (10, 10, 10, 10), 64)
    try:
        assert libmedusa.md_hydra_workspace(h, 1, 8192, 128256, 10, ctypes.byref(n)) == 0
        # at least the head inputs of the widest level (10 rows of d bf16) and
        # the top-k ids and values of all 1 + 10 + 10 + 4 head rows
        assert n.value >= 10 * 8192 * 2 + 2 * 25 * 10 * 4
        one = n.value
        assert libmedusa.md_hydra_workspace(h, 4, 8192, 128256, 10, ctypes.byref(n)) == 0 and n.value > one
        assert libmedusa.md_hydra_workspace(h, 1, 100, 128256, 10, ctypes.byref(n)) == -2   # d % 64
        assert libmedusa.md_hydra_workspace(h, 1, 8192, 128252, 10, ctypes.byref(n)) == -2  # V % 8
        assert libmedusa.md_hydra_workspace(h, 1, 8192, 128256, 9, ctypes.byref(n)) == -1   # kmax < a head's k
        assert libmedusa.md_hydra_workspace(h, 0, 8192, 128256, 10, ctypes.byref(n)) == -1
        assert libmedusa.md_hydra_workspace(None, 1, 8192, 128256, 10, ctypes.byref(n)) == -1
    finally:
        libmedusa.md_tree_destroy(h)
    root_only = ctypes.c_void_p()
    assert libmedusa.md_tree_create(_i32([-1]), _i32([0]), 1, 1, _i32([1]), ctypes.byref(root_only)) == 0
    try:
        assert libmedusa.md_hydra_workspace(root_only, 2, 256, 1024, 1, ctypes.byref(n)) == 0 and n.value > 0
    finally:
        libmedusa.md_tree_destroy(root_only)


def test_hydra_logit_rows_layout():
    """Level by level, then request by request, then the level's nodes with
    children in node order."""
    import medusa_draft_heads_b200 as md
    parent, rank = tree_spec.tree_arrays(tree_spec.select_tree((10, 10, 10, 10), TREE_ACCEPT, 64))
    tree = md.Tree(parent, rank, (10, 10, 10, 10))
    rows, total = md.hydra_logit_rows(tree, 2)
    assert total == 2 * (1 + 10 + 10 + 4)
    assert rows[(0, 0)] == 0 and rows[(1, 0)] == 1
    assert [rows[(0, j)] for j in range(1, 11)] == list(range(2, 12))
    assert [rows[(1, j)] for j in range(1, 11)] == list(range(12, 22))
    with_children = sorted(set(parent[1:]))
    assert sorted(rows) == sorted((b, p) for b in range(2) for p in with_children)
    assert sorted(rows.values()) == list(range(total))


def test_bench_hydra_level_accounting():
    import bench
    from seeded_inputs.workloads import LLAMA70B
    # depths 0, 1, 1, 2, 2, 2, 3; nodes with children: 0 (depth 0), 1 and 2 (depth 1), 3 (depth 2)
    assert bench.hydra_levels([-1, 0, 0, 1, 1, 2, 3]) == [1, 2, 1]
    parent, _ = tree_spec.tree_arrays(tree_spec.select_tree((10, 10, 10, 10), TREE_ACCEPT, 64))
    levels = bench.hydra_levels(parent)
    assert levels == [1, 10, 10, 4]
    w = LLAMA70B
    # every level streams one head's weights once: the same weight bytes as the Medusa heads
    weights = 4 * 2 * (w.d * w.d + w.d + w.d * w.V)
    assert bench.hydra_bytes(w, levels) == weights + sum(4 * n * w.d + 8 * n * w.kmax for n in levels)
