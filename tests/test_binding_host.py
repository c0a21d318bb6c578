"""The binding's argument checks (CPU only): wrong dtypes, devices, layouts
and shapes are refused in Python before any pointer reaches the library."""
import pytest

import medusa_draft_heads_b200 as md
from medusa_draft_heads_b200 import binding
from seeded_inputs.workloads import TREE_ACCEPT

torch = pytest.importorskip("torch")


def _bf(*shape):
    return torch.zeros(shape, dtype=torch.bfloat16)


def test_pointer_checks():
    t = torch.zeros((4, 4), dtype=torch.float32)
    with pytest.raises(TypeError, match="expected torch.bfloat16"):
        binding._ptr(t, torch.bfloat16, "h")
    with pytest.raises(ValueError, match="CUDA tensor"):
        binding._ptr(t, torch.float32, "h")
    with pytest.raises(TypeError, match="torch.Tensor"):
        binding._ptr([1, 2], torch.float32, "h")
    assert binding._ptr(None, torch.float32, "h") is None


def test_heads_shapes_are_checked_before_the_call():
    M, d, V, K = 1, 64, 256, 2
    ids = torch.zeros((M, K, 4), dtype=torch.int32)
    vals = torch.zeros((M, K, 4), dtype=torch.float32)
    with pytest.raises(ValueError, match="W1 has shape"):
        md.medusa_heads(_bf(M, d), _bf(K, d, d + 64), _bf(K, d), _bf(K, d, V), (2, 2), ids, vals, None)
    with pytest.raises(ValueError, match="k_per_head"):
        md.medusa_heads(_bf(M, d), _bf(K, d, d), _bf(K, d), _bf(K, d, V), (2, 2, 2), ids, vals, None)
    with pytest.raises(ValueError, match="topk_ids"):
        md.medusa_heads(_bf(M, d), _bf(K, d, d), _bf(K, d), _bf(K, d, V), (2, 2),
                        torch.zeros((M, K + 1, 4), dtype=torch.int32), vals, None)
    # right shapes, host tensors: refused as non-CUDA before the library sees them
    with pytest.raises(ValueError, match="CUDA tensor"):
        md.medusa_heads(_bf(M, d), _bf(K, d, d), _bf(K, d), _bf(K, d, V), (2, 2), ids, vals,
                        torch.zeros(256, dtype=torch.uint8))


def test_tree_and_hydra_shapes_are_checked():
    tree = md.Tree(*md.tree_arrays(md.select_tree((4, 3, 2, 2), TREE_ACCEPT, 16)), (4, 3, 2, 2))
    assert (tree.T, tree.max_depth, tree.K) == (17, 4, 4)
    B, d, V = 2, 64, 256
    i32 = lambda *s: torch.zeros(s, dtype=torch.int32)         # noqa: E731
    with pytest.raises(ValueError, match="tokens has shape"):
        md.tree_build(tree, i32(B, 4, 4), i32(B), i32(B), i32(B, 16), i32(17), i32(17, 1), i32(B, 17))
    with pytest.raises(ValueError, match="heads"):
        md.hydra_draft(tree, _bf(B, d), _bf(V, d), _bf(3, d, d), _bf(3, d), _bf(3, d, V), i32(B), i32(B),
                       i32(B, 17), i32(17), i32(17, 1), i32(B, 17), torch.zeros(256, dtype=torch.uint8))
    with pytest.raises(ValueError, match="E has shape"):
        md.hydra_draft(tree, _bf(B, d), _bf(V, d + 64), _bf(4, d, d), _bf(4, d), _bf(4, d, V), i32(B), i32(B),
                       i32(B, 17), i32(17), i32(17, 1), i32(B, 17), torch.zeros(256, dtype=torch.uint8))
    rows, n = md.hydra_logit_rows(tree, B)
    with pytest.raises(ValueError, match="logits_dbg"):
        md.hydra_draft(tree, _bf(B, d), _bf(V, d), _bf(4, d, d), _bf(4, d), _bf(4, d, V), i32(B), i32(B),
                       i32(B, 17), i32(17), i32(17, 1), i32(B, 17), torch.zeros(256, dtype=torch.uint8),
                       logits_dbg=torch.zeros((n + 1, V)))
    assert n == B * (1 + 4 + 3 + 1)


def test_tree_spec_errors_surface_as_exceptions():
    with pytest.raises(md.MedusaError, match="invalid argument"):
        md.Tree([-1, 0, 0], [0, 1, 1], (3,))                     # two children with one rank
    with pytest.raises(md.MedusaError, match="invalid argument"):
        md.Tree([-1, 0, 1], [0, 0, 0], (2,))                     # depth 2 with one head
