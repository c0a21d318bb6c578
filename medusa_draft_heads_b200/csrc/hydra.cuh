// Sequentially dependent (Hydra) drafting of the candidate tree.
//
// Sources: "Medusa heads versus separate draft model", section "Acceptance"
// (a Medusa head drafts without seeing the earlier heads' guesses) and
// "Hydra: Sequentially-Dependent Draft Heads for Medusa Decoding" (abstract:
// drop-in draft heads conditioned on the earlier tokens of the candidate
// continuation). The pages give no architecture; this library reads it as the
// Medusa head's own shape applied to x_p = bf16(h + E[token_p]), where p is
// the parent of the node being drafted and E the target's input embedding.
//
// The draft then runs level by level: level l takes every node p at depth l
// that has children, forms x_p (hydra_gather_kernel), runs head l on those
// rows with the heads kernels (one head, B * n_l rows, top-k fused), and the
// top-k of row (b, p) supplies the tokens of p's children. After the last
// level, hydra_tokens_kernel writes every node's token, the parent array,
// the ancestor bitsets and the positions, like tree_build_kernel.
//
// Level l's top-k rows sit at row0[l] + b * n[l] + slot[p] of one [rows, kmax]
// array, where slot[p] is p's index among the depth-l nodes with children.
#pragma once

#include "common.cuh"

namespace md {
namespace hydra {

constexpr int kGatherThreads = 128;

struct GatherArgs {
  const uint16_t* h;          // [M, d] bf16 hidden states
  const uint16_t* E;          // [V, d] bf16 input embedding
  const int32_t* head_row;    // [B] or null (row b)
  const int32_t* root_token;  // [B]
  const int32_t* prev_ids;    // previous level's top-k ids, its first row (null at level 0)
  uint16_t* x;                // [B * n, d] this level's head inputs
  int M, d, V, kmax;
  int n_prev;                 // parents per request at the previous level
  int8_t pslot[MD_MAX_T];     // q -> slot of the q-th parent's own parent (previous level)
  int8_t prank[MD_MAX_T];     // q -> head rank of the q-th parent
};

// One CTA per (parent q, request b): x[b * n + q] = bf16(h[row_b] + E[token of parent q]).
// The sum of two bf16 values is formed in fp32 (correctly rounded) and then
// rounded to bf16; fp32 carries more than 2 * 8 + 2 significant bits, so the
// two roundings equal one rounding of the exact sum (double rounding is
// innocuous at that width: Figueroa, "When is double rounding innocuous?",
// SIGNUM Newsletter 30(3), 1995).
__global__ void __launch_bounds__(kGatherThreads) hydra_gather_kernel(const __grid_constant__ GatherArgs a) {
  pdl_wait_primary();          // the previous level's top-k comes from the kernel before
  pdl_launch_dependents();
  const int q = blockIdx.x, b = blockIdx.y;
  const int n = gridDim.x;
  int tok;
  if (a.prev_ids == nullptr) {
    tok = a.root_token[b];
  } else {
    tok = a.prev_ids[(size_t(b) * a.n_prev + a.pslot[q]) * a.kmax + a.prank[q]];
  }
  const int row = a.head_row ? a.head_row[b] : b;
  const bool tok_ok = tok >= 0 && tok < a.V;
  const bool row_ok = row >= 0 && row < a.M;
  if (threadIdx.x == 0) {
    if (!tok_ok) set_status(MD_DEV_BAD_TOKEN);
    if (!row_ok) set_status(MD_DEV_BAD_ROW);
  }
  // a bad token or row contributes zeros (the status word reports it)
  const uint4* hv = reinterpret_cast<const uint4*>(a.h + size_t(row_ok ? row : 0) * a.d);
  const uint4* ev = reinterpret_cast<const uint4*>(a.E + size_t(tok_ok ? tok : 0) * a.d);
  uint4* xv = reinterpret_cast<uint4*>(a.x + (size_t(b) * n + q) * a.d);
  const uint32_t hm = row_ok ? 0xFFFFFFFFu : 0u, em = tok_ok ? 0xFFFFFFFFu : 0u;
  for (int i = threadIdx.x; i < a.d / 8; i += kGatherThreads) {
    const uint4 hh = __ldg(hv + i), ee = __ldg(ev + i);
    const uint32_t hw[4] = {hh.x & hm, hh.y & hm, hh.z & hm, hh.w & hm};
    const uint32_t ew[4] = {ee.x & em, ee.y & em, ee.z & em, ee.w & em};
    uint32_t o[4];
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const uint16_t lo = f32_to_bf16_rne(__fadd_rn(bf16lo(hw[w]), bf16lo(ew[w])));
      const uint16_t hi = f32_to_bf16_rne(__fadd_rn(bf16hi(hw[w]), bf16hi(ew[w])));
      o[w] = uint32_t(lo) | (uint32_t(hi) << 16);
    }
    xv[i] = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

struct TokenArgs {
  const int32_t* ids;         // every level's top-k ids [rows, kmax]
  const int32_t* root_token;  // [B]
  const int32_t* prefix_len;  // [B]
  int32_t* tokens;            // [B, T]
  int32_t* parent;            // [T]
  uint32_t* anc;              // [T, W]
  int32_t* pos;               // [B, T]
  int kmax;
  int row0[MD_MAX_K];         // first row of level l
  int n[MD_MAX_K];            // parents per request at level l
  int8_t slot[MD_MAX_T];      // node -> its index among the parents at its depth (-1: no children)
};

// One CTA per request, one thread per node.
__global__ void __launch_bounds__(MD_MAX_T) hydra_tokens_kernel(const __grid_constant__ TreeParams tp,
                                                                const __grid_constant__ TokenArgs a) {
  pdl_wait_primary();          // the last level's top-k comes from the kernel before
  pdl_launch_dependents();
  const int b = blockIdx.x;
  const int j = threadIdx.x;
  if (j >= tp.T) return;
  const int d = tp.depth[j];
  int32_t tok;
  if (j == 0) {
    tok = a.root_token[b];
  } else {
    const int l = d - 1;
    const int p = tp.parent[j];
    const size_t row = size_t(param_at(a.row0, l)) + size_t(b) * param_at(a.n, l) + a.slot[p];
    tok = a.ids[row * a.kmax + tp.rank[j]];
  }
  a.tokens[size_t(b) * tp.T + j] = tok;
  a.pos[size_t(b) * tp.T + j] = a.prefix_len[b] + d;
  if (b == 0) {
    a.parent[j] = tp.parent[j];
    for (int w = 0; w < tp.W; ++w) a.anc[size_t(j) * tp.W + w] = tp.anc[j][w];
  }
}

}  // namespace hydra
}  // namespace md
