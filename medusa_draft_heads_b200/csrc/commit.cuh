// Advancing along the accepted branch: KV compaction and next-step handoff.
//
// Source: "Medusa heads versus separate draft model", section "Acceptance",
// tree paragraph (decoding continues along the branch that matches). The accepted path's tokens
// join the sequence, so their K/V move next to the prefix: slot P + i receives
// slot P + path[i] (i = 0..L). Moves are tiny (at most K + 1 rows per KV head)
// and latency-bound: one CTA per (KV head, request) stages the source rows in
// shared memory first, because a destination slot can be another row's source
// (path = 0, 2, 5: slot P+2 is read for i = 1 and written for i = 2).
#pragma once

#include "common.cuh"

namespace md {
namespace commit {

constexpr int kThreads = 128;

struct Args {
  uint16_t* kc;                // [B, Hkv, S_max, dh]
  uint16_t* vc;
  const int32_t* prefix_len;   // [B]
  const int32_t* accept_len;   // [B]
  const int32_t* path;         // [B, K + 1]
  const int32_t* bonus;        // [B]
  int32_t* new_prefix_len;     // [B]
  int32_t* next_root;          // [B]
  int32_t* next_head_row;      // [B]
  int S_max, Hkv, dh, K;
};

__global__ void __launch_bounds__(kThreads) tree_commit_kernel(const __grid_constant__ TreeParams tp, Args a) {
  pdl_wait_primary();          // path and lengths come from the acceptance kernels
  pdl_launch_dependents();
  extern __shared__ __align__(16) uint8_t smem[];
  const int hk = blockIdx.x, b = blockIdx.y;
  const int T = tp.T;
  const int P = a.prefix_len[b];
  const int L = a.accept_len[b];
  __shared__ int src[MD_MAX_K + 1];
  __shared__ int valid;
  if (threadIdx.x == 0) {
    bool ok = P >= 0 && P + T <= a.S_max && L >= 0 && L <= tp.max_depth && L <= a.K;
    for (int i = 0; ok && i <= L; ++i) {
      const int n = a.path[size_t(b) * (a.K + 1) + i];
      // the path must run from the root through parents to a depth-L node
      ok = n >= 0 && n < T && tp.depth[n] == i && (i == 0 || tp.parent[n] == src[i - 1] - P);
      src[i] = P + n;
    }
    valid = ok;
    if (!ok && hk == 0) set_status(MD_DEV_BAD_PATH);
  }
  __syncthreads();
  if (!valid) {
    if (hk == 0 && threadIdx.x == 0) {
      a.new_prefix_len[b] = P;
      a.next_root[b] = a.bonus[b];
      a.next_head_row[b] = -1;
    }
    return;
  }
  const int row16 = a.dh / 8;             // 16-byte chunks per row
  uint4* ks = reinterpret_cast<uint4*>(smem);
  uint4* vs = ks + (MD_MAX_K + 1) * row16;
  const size_t base = (size_t(b) * a.Hkv + hk) * a.S_max;
  const uint4* kg = reinterpret_cast<const uint4*>(a.kc);
  const uint4* vg = reinterpret_cast<const uint4*>(a.vc);
  for (int idx = threadIdx.x; idx < (L + 1) * row16; idx += kThreads) {
    const int i = idx / row16, c = idx % row16;
    ks[idx] = kg[(base + src[i]) * row16 + c];
    vs[idx] = vg[(base + src[i]) * row16 + c];
  }
  __syncthreads();
  uint4* kw = reinterpret_cast<uint4*>(a.kc);
  uint4* vw = reinterpret_cast<uint4*>(a.vc);
  for (int idx = threadIdx.x; idx < (L + 1) * row16; idx += kThreads) {
    const int i = idx / row16, c = idx % row16;
    kw[(base + P + i) * row16 + c] = ks[idx];
    vw[(base + P + i) * row16 + c] = vs[idx];
  }
  if (hk == 0 && threadIdx.x == 0) {
    a.new_prefix_len[b] = P + L + 1;
    a.next_root[b] = a.bonus[b];
    a.next_head_row[b] = b * T + (src[L] - P);
  }
}

}  // namespace commit
}  // namespace md
