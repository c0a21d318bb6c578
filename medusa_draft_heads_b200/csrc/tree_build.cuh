// Candidate tree construction.
//
// Source: "Medusa heads versus separate draft model", section "Acceptance",
// tree paragraph: the heads' best-scoring candidates, combined across heads,
// make up the tree. Node j at depth d takes the rank head_rank[j] candidate of head d.
// Latency-bound (a few KB); one CTA per request, one thread per node.
#pragma once

#include "common.cuh"

namespace md {
namespace tree {

struct BuildArgs {
  const int32_t* topk_ids;    // [M, K, kmax]
  const int32_t* head_row;    // [B] or null
  const int32_t* root_token;  // [B]
  const int32_t* prefix_len;  // [B]
  int32_t* tokens;            // [B, T]
  int32_t* parent;            // [T]
  uint32_t* anc;              // [T, W]
  int32_t* pos;               // [B, T]
  int M, K, kmax;
};

__global__ void __launch_bounds__(MD_MAX_T) tree_build_kernel(const __grid_constant__ TreeParams tp, BuildArgs a) {
  pdl_wait_primary();          // top-k ids come from the previous kernel
  pdl_launch_dependents();
  const int b = blockIdx.x;
  const int j = threadIdx.x;
  __shared__ int row_ok;
  if (j == 0) {
    const int row = a.head_row ? a.head_row[b] : b;
    row_ok = (row >= 0 && row < a.M) ? row : -1;
    if (row_ok < 0) set_status(MD_DEV_BAD_ROW);
  }
  __syncthreads();
  if (j >= tp.T) return;
  const int d = tp.depth[j];
  int32_t tok;
  if (j == 0) {
    tok = a.root_token[b];
  } else if (row_ok < 0) {
    tok = -1;
  } else {
    tok = a.topk_ids[(size_t(row_ok) * a.K + (d - 1)) * a.kmax + tp.rank[j]];
  }
  a.tokens[size_t(b) * tp.T + j] = tok;
  a.pos[size_t(b) * tp.T + j] = a.prefix_len[b] + d;
  if (b == 0) {
    a.parent[j] = tp.parent[j];
    for (int w = 0; w < tp.W; ++w) a.anc[size_t(j) * tp.W + w] = tp.anc[j][w];
  }
}

}  // namespace tree
}  // namespace md
