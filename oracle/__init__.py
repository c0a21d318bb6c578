"""CPU oracle for the Medusa draft-and-verify step (TEST INFRASTRUCTURE ONLY).

A plain, slow, obviously correct restatement of what each step computes,
written from the pages' definitions in fp64 with naive iteration order. It is
used only by ``tests/``, by ``__graft_entry__.smoke()`` and by the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py``. The product path
(``medusa_draft_heads_b200``) never imports it, and this package imports
nothing from the product path; the two share only ``seeded_inputs``.

Sources (page title, then section):

* "Medusa heads versus separate draft model", section "What each one is":
  each head is one residual block on the target's last hidden state followed
  by its own vocabulary projection; head k guesses the token k positions
  ahead; all heads run once, in parallel.
* same page, "Cost per step": residual block d x d + bias, vocabulary
  projection d x V (no bias), d = 8,192, V = 128,256.
* same page, "Acceptance": the tree paragraph (top few candidates per head,
  a tree of their combinations, one verification pass with a tree attention
  mask, advance along a matching branch) and the expected-length formula.
* same page, "Training": typical acceptance, which accepts more drafts and is
  not lossless.

Pinning: every function here is pinned by ``tests/test_oracle_*.py`` against
closed forms, brute force or printed values; the typical-acceptance rule is
"parity unpinned" against the pages (they name the rule without its formula),
and is pinned only by its limiting cases.
"""
from . import accept, attention, heads, tree  # noqa: F401
