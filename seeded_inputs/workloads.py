"""Named synthetic workloads: shapes, value distributions and seeds.

Shapes follow the Llama-3 8B / 70B cases the Medusa pages price ("Medusa heads
versus separate draft model", section "Cost per step": d = 8,192 and
V = 128,256 for the 70B target; the 8B model has d = 4,096 and the same
vocabulary). The per-depth acceptance profile (0.80, 0.65, 0.50, 0.40) is the
"Medusa, tree of top-k" row of that page's acceptance table; the top-1 chain
row is (0.65, 0.50, 0.40, 0.35).
"""
from __future__ import annotations

from dataclasses import dataclass, field, replace

TREE_ACCEPT = (0.80, 0.65, 0.50, 0.40)
CHAIN_ACCEPT = (0.65, 0.50, 0.40, 0.35)


@dataclass(frozen=True)
class Workload:
    name: str
    B: int                      # requests
    d: int                      # hidden size
    V: int                      # vocabulary
    K: int                      # Medusa heads
    k_per_head: tuple           # top-k of each head
    n_nodes: int                # candidate (non-root) tree nodes; T = n_nodes + 1
    Hq: int
    Hkv: int
    dh: int
    prefix: tuple               # (lo, hi) KV prefix length, uniform per request
    heads_rows: str = "B"       # "B": one hidden row per request; "BT": one per tree node
    accept: tuple = TREE_ACCEPT
    w_sigma: float = 0.02       # head weights ~ N(0, 0.02)
    logit_sigma: float = 1.0    # target logits ~ N(0, logit_sigma)
    bump: float = 1.0           # planted argmax margin over the row maximum
    mode: str = "greedy"        # or "typical", "sample", "rejection"
    temperature: float = 0.7
    eps: float = 0.09
    alpha: float = 0.3
    seed: int = 0
    shared_vocab: bool = False  # one vocabulary projection for all heads
    extra: dict = field(default_factory=dict)

    @property
    def T(self) -> int:
        return self.n_nodes + 1

    @property
    def kmax(self) -> int:
        return max(self.k_per_head)

    @property
    def M(self) -> int:
        return self.B if self.heads_rows == "B" else self.B * self.T

    @property
    def S_max(self) -> int:
        """KV slots per request: the longest prefix plus the tree, rounded to 64."""
        s = self.prefix[1] + self.T
        return (s + 63) // 64 * 64

    def head_weight_bytes(self) -> int:
        proj = self.d * self.V * (1 if self.shared_vocab else self.K)
        return 2 * (self.K * (self.d * self.d + self.d) + proj)


TINY = Workload("tiny", B=1, d=256, V=1024, K=4, k_per_head=(4, 3, 2, 2), n_nodes=16,
                Hq=4, Hkv=2, dh=64, prefix=(128, 128))
LLAMA8B = Workload("llama3-8b", B=1, d=4096, V=128256, K=4, k_per_head=(10, 10, 10, 10),
                   n_nodes=64, Hq=32, Hkv=8, dh=128, prefix=(2048, 2048))
LLAMA70B = Workload("llama3-70b", B=1, d=8192, V=128256, K=4, k_per_head=(10, 10, 10, 10),
                    n_nodes=64, Hq=64, Hkv=8, dh=128, prefix=(4096, 4096))
LLAMA70B_CHAIN = replace(LLAMA70B, name="llama3-70b-chain", k_per_head=(1, 1, 1, 1), n_nodes=4,
                         accept=CHAIN_ACCEPT)
BATCHED70B = replace(LLAMA70B, name="llama3-70b-b8", B=8, prefix=(1024, 8192), heads_rows="BT")

# Profiling case for the heads kernels: 8B-shaped with a 32000-token vocabulary,
# so the weights (1.1 GB) exceed L2 while the device footprint stays small.
PROF_HEADS = replace(LLAMA8B, name="prof-8b-v32000", V=32000)
# Profiling case for the weights-as-M tensor-core heads: the same weights on 16 rows.
PROF_SKINNY = replace(PROF_HEADS, name="prof-8b-v32000-b16", B=16)
# Profiling case for the tensor-core heads: the same weights on 8 x 65 = 520 rows.
PROF_GEMM = replace(PROF_HEADS, name="prof-8b-v32000-b8", B=8, heads_rows="BT", prefix=(1024, 8192))

# The same 70B step with one vocabulary projection shared by the four heads.
LLAMA70B_SHARED = replace(LLAMA70B, name="llama3-70b-shared-proj", shared_vocab=True)

# The same 70B step with lossless sampled acceptance (temperature 0.7).
LLAMA70B_SAMPLED = replace(LLAMA70B, name="llama3-70b-sampled", mode="sample", temperature=0.7)

# The same 70B step with candidates drawn from the heads' own distributions and
# lossless acceptance by rejection sampling (temperature 0.7 for both).
LLAMA70B_REJECTION = replace(LLAMA70B, name="llama3-70b-rejection", mode="rejection", temperature=0.7)

WORKLOADS = {w.name: w for w in (TINY, LLAMA8B, LLAMA70B, LLAMA70B_CHAIN, BATCHED70B, PROF_HEADS, PROF_SKINNY, PROF_GEMM,
                                 LLAMA70B_SHARED, LLAMA70B_SAMPLED, LLAMA70B_REJECTION)}


def sweep_8b(B: int, tree: str, prefix: int, mode: str = "greedy") -> Workload:
    """One point of the 8B-shaped sweep: tree in {"chain", "16", "64"}."""
    if tree == "chain":
        kph, n = (1, 1, 1, 1), 4
    else:
        kph, n = (10, 10, 10, 10), int(tree)
    return replace(LLAMA8B, name=f"sweep8b-B{B}-{tree}-P{prefix}-{mode}", B=B, k_per_head=kph,
                   n_nodes=n, prefix=(prefix, prefix), logit_sigma=3.0, bump=3.0, mode=mode)


# Profiling case for the 64-key, two-CTA-per-SM attention shape: the 8B sweep's
# B = 32 point with the 64-node tree and a 1024-token prefix (768 row tiles,
# more than one wave of 128-key CTAs).
PROF_ATTN_B32 = replace(sweep_8b(32, "64", 1024), name="prof-attn-8b-b32")
WORKLOADS[PROF_ATTN_B32.name] = PROF_ATTN_B32
