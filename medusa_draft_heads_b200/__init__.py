"""B200-native Medusa draft-and-verify step: four CUDA calls behind a C ABI.

    medusa_heads   K draft heads (residual SiLU block + vocabulary projection)
                   fused with a per-head top-k
    tree_build     candidate tree: tokens, parents, ancestor bitsets, positions
    hydra_draft    heads + tree with sequentially dependent (Hydra) heads:
                   each depth's heads read the parent token's embedding too
    tree_attention tree-masked GQA attention over the KV prefix plus the tree
    tree_accept    longest accepted branch (greedy or typical) and bonus token
    tree_accept_sampled  the same under lossless sampling (one draw per row)
    medusa_heads_sampled  the heads with candidates drawn from their own
                   distributions (Gumbel-top-k over caller uniforms)
    tree_accept_rejection lossless acceptance of those drafts: rejection
                   sampling of each node's children against the heads' q
    tree_commit    advance along it: KV compaction and the next step's inputs

The kernels live in ``libmedusa.so`` (built from ``csrc/`` for sm_100a); this
package only marshals arguments to it.
"""
from .binding import (MedusaError, Tree, accept_workspace_bytes, attention_workspace_bytes,  # noqa: F401
                      device_status, heads_shared_workspace_bytes, heads_workspace_bytes, hydra_draft,
                      hydra_logit_rows, hydra_workspace_bytes, lib, medusa_heads, medusa_heads_sampled,
                      medusa_heads_shared, tree_accept, tree_accept_rejection, tree_accept_sampled, tree_attention,
                      set_wait_limit, stream_read, tree_build, tree_commit, version, workspace)
from .tree_spec import select_tree, tree_arrays  # noqa: F401
