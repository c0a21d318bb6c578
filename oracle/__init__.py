"""CPU oracle for the Medusa draft-and-verify step (TEST INFRASTRUCTURE ONLY).

A plain, slow, obviously correct restatement of what each step computes,
written from the pages' definitions in fp64 with naive iteration order. It is
used only by ``tests/``, by ``__graft_entry__.smoke()`` and by the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py``. The product path
(``medusa_draft_heads_b200``) never imports it, and this package imports
nothing from the product path; the two share only ``seeded_inputs``.

Sources (page title, then section):

* "Medusa heads versus separate draft model", section "What each one is":
  a head is a residual block applied to the target's last hidden state,
  then a vocabulary projection of its own; head k drafts the token k places
  ahead, and the heads all read the same state in a single parallel pass.
* same page, "Cost per step": a d x d layer with bias inside the block, a
  bias-free d x V projection, d = 8,192, V = 128,256.
* same page, "Acceptance": the tree paragraph (the heads' best candidates are
  combined into a tree, the target checks all branches in a single masked
  pass, decoding follows the branch that matches) and the expected-length
  formula.
* same page, "Training": typical acceptance (more drafts accepted, the target
  distribution not kept) and rejection sampling when it must be kept.
* "Hydra: Sequentially-Dependent Draft Heads for Medusa Decoding" (abstract):
  draft heads whose guesses are conditioned on the earlier tokens of the
  candidate continuation (``hydra.py``; the architecture is a reading).

Pinning: every function here is pinned by ``tests/test_oracle_*.py`` against
closed forms, brute force or printed values; the typical-acceptance rule is
"parity unpinned" against the pages (they name the rule without its formula),
and is pinned only by its limiting cases.
"""
from . import accept, attention, heads, hydra, tree  # noqa: F401
