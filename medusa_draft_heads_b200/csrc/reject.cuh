// Lossless acceptance of drafts sampled from the heads (rejection sampling).
//
// Source: "Medusa heads versus separate draft model", section "Training":
// when the output must follow the target's distribution exactly, rejection
// sampling is used. With drafts drawn from head d's distribution q without
// replacement (md_medusa_heads_sampled), the children c_1 .. c_m of a tree
// node t (ranks 0 .. m-1, tokens y_1 .. y_m) are tested in rank order against
// the target row p = softmax(z_t / tau):
//
//   r_1 = p;  q_i = q without y_1 .. y_{i-1}, renormalised;
//   accept c_i iff u_acc[c_i] < r_i(y_i) / q_i(y_i), else
//   r_{i+1} = max(0, r_i - q_i) / sum max(0, r_i - q_i);
//   no child accepted (or no child): bonus ~ r_{m+1} by inverse CDF (u_res[t]).
//
// Carried as scalars. Every r_i has the form max(0, p - A_i q) / B_i with
//   A_1 = 0, B_1 = 1,  A_{i+1} = A_i + B_i / S_i,  B_{i+1} = F(A_{i+1}),
//   F(A) = sum_v max(0, p(v) - A q(v)),  S_i = 1 - sum_{j<i} q(y_j)
// (the rejected y_j fall to zero in the residual, so removing them from q_i
// changes only its normaliser S_i). A rejection therefore costs one pass
// over the vocabulary (F at the new A), and a test needs p and q at y_i only.
//
// Layout: one cluster of kCtas CTAs per request, CTA r holding vocabulary
// slice r of the target row e = exp((z - max z) / tau) and of the head row
// eq = exp((x - max x) / tau_q) in shared memory (p = e / Se, q = eq / Sq).
// Sums over the vocabulary are block reductions followed by a fixed-order sum
// of the CTAs' partials read through distributed shared memory, so every CTA
// holds the same value and takes the same decisions.
#pragma once

#include "common.cuh"

namespace md {
namespace rej {

constexpr int kCtas = 8;                 // CTAs per request (one cluster, portable size)
constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxSlice = 24576;         // floats per CTA and row: V <= 8 * 24576
constexpr int kSmem = 2 * kMaxSlice * 4;

struct Args {
  const float* logits;       // target [B, T, V]
  const float* head_logits;  // [M, Kh, V]
  const int32_t* head_row;   // [B] or null (request b uses row b)
  const int32_t* tokens;     // [B, T]
  const float* u_acc;        // [B, T]
  const float* u_res;        // [B, T]
  int32_t* accept_len;       // [B]
  int32_t* path;             // [B, K + 1]
  int32_t* bonus;            // [B]
  int V, T, K, M, Kh, slice;
  float inv_tau, inv_tau_q;
};

// Sum (or max) of one value per thread over the CTA, then over the cluster's
// CTAs in rank order. `part` is this CTA's 2-slot exchange area; consecutive
// reductions alternate slots, so a slot is rewritten only after every CTA has
// passed the cluster barrier of the reduction in between.
struct ClusterReduce {
  float* warp_red;   // [kWarps]
  float* part;       // [2]
  float* result;     // [kCtas]: the combined value (result[0]) or the CTAs' partials
  int flip;
  // CTA partial of v (fixed warp order) into part[flip], then a cluster barrier.
  __device__ __forceinline__ void publish(float v, bool is_max) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float w = __shfl_xor_sync(0xffffffffu, v, o);
      v = is_max ? fmaxf(v, w) : v + w;
    }
    if (lane == 0) warp_red[warp] = v;
    __syncthreads();
    if (threadIdx.x == 0) {
      float t = warp_red[0];
      for (int w = 1; w < kWarps; ++w) t = is_max ? fmaxf(t, warp_red[w]) : t + warp_red[w];
      part[flip] = t;
    }
    cluster_sync();
  }
  // Lane c of warp 0 reads CTA c's partial (one round of remote loads in
  // parallel); warp 0 stores them, or their fixed-order combination, for the
  // whole CTA.
  __device__ __forceinline__ void gather(bool is_max, bool combine) {
    if (threadIdx.x < 32) {
      const int lane = threadIdx.x;
      const float x = lane < kCtas ? ld_cluster_f1(mapa_shared(smem_u32(&part[flip]), uint32_t(lane))) : 0.f;
      if (combine) {
        float r = 0.f;
#pragma unroll
        for (int c = 0; c < kCtas; ++c) {
          const float y = __shfl_sync(0xffffffffu, x, c);
          r = c == 0 ? y : (is_max ? fmaxf(r, y) : r + y);
        }
        if (lane == 0) result[0] = r;
      } else if (lane < kCtas) {
        result[lane] = x;
      }
    }
    __syncthreads();
    flip ^= 1;
  }
  __device__ __forceinline__ float run(float v, bool is_max) {
    publish(v, is_max);
    gather(is_max, true);
    return result[0];
  }
  // The kCtas partials themselves (for the inverse-CDF search).
  __device__ __forceinline__ void partials(float v, float (&out)[kCtas]) {
    publish(v, false);
    gather(false, false);
#pragma unroll
    for (int c = 0; c < kCtas; ++c) out[c] = result[c];
  }
};

// Orders this thread's earlier generic-proxy shared-memory accesses (after a
// block barrier: the block's) before later async-proxy (bulk copy) writes.
__device__ __forceinline__ void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// e = exp2((x - mx) * scale) with scale = log2(e) / tau: the one formula used
// for the slices and for single entries, so both give the same bits.
__device__ __forceinline__ float expw(float x, float mx, float scale) { return exp2f((x - mx) * scale); }

// Load a row's slice into smem and turn it into e = exp((x - max) / tau);
// returns (max over the row, sum of e over the row). The slice arrives as one
// bulk copy (a single DRAM round trip) when its address and length allow,
// else through per-thread loads. Every thread of the block calls this with
// the block's earlier reads of `s` finished (the caller's last reduction).
__device__ __forceinline__ float2 load_exp_row(const float* row, float* s, int lo, int n, float scale,
                                               ClusterReduce& cr, uint64_t* bar, uint32_t& phase) {
  float mx = -INFINITY;
  const float* src = row + lo;
  const bool bulk = n > 0 && (n & 3) == 0 && ((reinterpret_cast<uintptr_t>(src) | reinterpret_cast<uintptr_t>(s)) & 15) == 0;
  if (bulk) {
    if (threadIdx.x == 0) {
      fence_proxy_async_smem();             // the exp values written over s before
      mbar_arrive_expect_tx(smem_u32(bar), uint32_t(n) * 4u);
      bulk_load(smem_u32(s), src, uint32_t(n) * 4u, smem_u32(bar));
    }
    if (!mbar_wait(smem_u32(bar), phase)) set_status(MD_DEV_TIMEOUT);
    phase ^= 1u;
    for (int i = threadIdx.x; i < n; i += kThreads) mx = fmaxf(mx, s[i]);
  } else {
    for (int i = threadIdx.x; i < n; i += kThreads) {
      const float x = __ldg(src + i);
      s[i] = x;
      mx = fmaxf(mx, x);
    }
  }
  mx = cr.run(mx, true);
  float sum = 0.f;
  for (int i = threadIdx.x; i < n; i += kThreads) {
    const float e = expw(s[i], mx, scale);
    s[i] = e;
    sum += e;
  }
  sum = cr.run(sum, false);
  return make_float2(mx, sum);
}

__global__ void __launch_bounds__(kThreads, 1) reject_accept_kernel(const __grid_constant__ TreeParams tp, Args a) {
  extern __shared__ float sm[];
  float* se = sm;                           // target slice e
  float* sq = sm + kMaxSlice;               // head slice eq
  __shared__ float warp_red[kWarps];
  __shared__ float part[2];
  __shared__ float red_out[kCtas];
  __shared__ float scan_tot[kWarps];
  __shared__ int found_id;
  __shared__ int ch_node[MD_MAX_KMAX];       // children of the current node, by rank
  __shared__ float ch_p[MD_MAX_KMAX], ch_q[MD_MAX_KMAX];   // p(y) and q(y) of each child's token
  __shared__ int n_ch;
  __shared__ __align__(8) uint64_t load_bar;  // completes each row slice's bulk copy
  ClusterReduce cr{warp_red, part, red_out, 0};
  uint32_t load_phase = 0;

  const int crank = int(cluster_ctarank());
  const int b = blockIdx.y;
  const int lo = min(a.V, crank * a.slice), n = min(a.V, lo + a.slice) - lo;
  const float sc_t = 1.4426950408889634f * a.inv_tau;
  const float sc_q = 1.4426950408889634f * a.inv_tau_q;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&load_bar), 1);
    fence_barrier_init();
  }
  __syncthreads();
  pdl_wait_primary();
  pdl_launch_dependents();

  const int hrow = a.head_row ? a.head_row[b] : b;
  const bool row_ok = hrow >= 0 && hrow < a.M;
  if (!row_ok && crank == 0 && threadIdx.x == 0) set_status(MD_DEV_BAD_ROW);

  int node = 0, depth = 0, L = 0;
  int steps[MD_MAX_K + 1];
  steps[0] = 0;
  int qdepth = -1;                          // head row held in sq
  float q_max = 0.f, q_sum = 1.f;
  float A = 0.f, Bc = 1.f;                  // r = max(0, p - A q) / Bc over the walk at `node`
  for (;;) {
    const float* zrow = a.logits + (size_t(b) * a.T + node) * a.V;
    const float2 zs = load_exp_row(zrow, se, lo, n, sc_t, cr, &load_bar, load_phase);
    const float inv_se = 1.f / zs.y;
    A = 0.f;
    Bc = 1.f;
    int accepted = -1;
    // children of this node by rank (thread r finds rank r), with p(y) of their tokens
    if (threadIdx.x == 0) n_ch = 0;
    __syncthreads();
    if (threadIdx.x < MD_MAX_KMAX) {
      const int r = threadIdx.x;
      int c = -1;
      for (int j = 1; j < tp.T; ++j)
        if (tp.parent[j] == node && tp.rank[j] == r) c = j;
      ch_node[r] = c;
      float pY = 0.f;
      if (c >= 0) {
        atomicMax(&n_ch, r + 1);
        const int y = a.tokens[size_t(b) * a.T + c];
        if (y >= 0 && y < a.V) pY = expw(__ldg(zrow + y), zs.x, sc_t) * inv_se;
      }
      ch_p[r] = pY;
    }
    __syncthreads();
    const bool has_child = depth < a.K && row_ok && n_ch > 0;
    if (has_child) {
      if (qdepth != depth) {
        const float* xrow = a.head_logits + (size_t(hrow) * a.Kh + depth) * a.V;
        const float2 xs = load_exp_row(xrow, sq, lo, n, sc_q, cr, &load_bar, load_phase);
        q_max = xs.x;
        q_sum = xs.y;
        qdepth = depth;
      }
      const float inv_sq = 1.f / q_sum;
      if (threadIdx.x < MD_MAX_KMAX) {
        const int c = ch_node[threadIdx.x];
        float qY = 0.f;
        if (c >= 0) {
          const int y = a.tokens[size_t(b) * a.T + c];
          if (y >= 0 && y < a.V)
            qY = expw(__ldg(a.head_logits + (size_t(hrow) * a.Kh + depth) * a.V + y), q_max, sc_q) * inv_sq;
          else if (crank == 0)
            set_status(MD_DEV_BAD_TOKEN);
        }
        ch_q[threadIdx.x] = qY;
      }
      __syncthreads();
      float S = 1.f;                       // q mass of the tokens not yet rejected
      for (int r = 0; r < n_ch && accepted < 0; ++r) {
        const int c = ch_node[r];          // children carry the ranks 0 .. m-1
        const float pY = ch_p[r], qY = ch_q[r];
        // accept iff u < r(y) / q_i(y) = S * max(0, p(y) - A q(y)) / (Bc * q(y))
        const float num = S * fmaxf(0.f, pY - A * qY);
        const float u = a.u_acc[size_t(b) * a.T + c];
        if (Bc <= 0.f || u * (Bc * qY) < num) {
          accepted = c;
          break;
        }
        // rejected: r_{i+1} = max(0, p - A' q) / F(A'), A' = A + Bc / S
        A = A + (S > 0.f ? Bc / S : 0.f);
        S = fmaxf(0.f, S - qY);
        float f = 0.f;
        for (int i = threadIdx.x; i < n; i += kThreads) f += fmaxf(0.f, se[i] * inv_se - A * (sq[i] * inv_sq));
        Bc = cr.run(f, false);
      }
    }
    if (accepted < 0) {
      // bonus token: inverse CDF of w = max(0, p - A q) (p itself when A = 0), u_res[node]
      const float inv_sq = 1.f / q_sum;
      const bool useq = A > 0.f;
      auto w_at = [&](int i) -> float {
        const float p = se[i] * inv_se;
        return useq ? fmaxf(0.f, p - A * (sq[i] * inv_sq)) : p;
      };
      float f = 0.f;
      for (int i = threadIdx.x; i < n; i += kThreads) f += w_at(i);
      float pc[kCtas];
      cr.partials(f, pc);
      float total = 0.f;
#pragma unroll
      for (int c = 0; c < kCtas; ++c) total += pc[c];
      const float target = a.u_res[size_t(b) * a.T + node] * total;
      // owner CTA: the first whose running total passes the target; if rounding
      // leaves the target at or past the total, the last CTA with mass
      int owner = -1, last = 0;
      float before = 0.f, run = 0.f;
#pragma unroll
      for (int c = 0; c < kCtas; ++c) {
        if (pc[c] > 0.f) last = c;
        if (owner < 0 && run + pc[c] > target) {
          owner = c;
          before = run;
        }
        run += pc[c];
      }
      const bool past = owner < 0;
      if (past) {
        owner = last;
        before = run - pc[last];
      }
      if (crank == owner) {
        // warps take contiguous ranges of the slice; the warp holding the
        // crossing walks its range 32 entries at a time
        const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
        const int per = (n + kWarps - 1) / kWarps;
        const int w0 = min(n, warp * per), w1 = min(n, w0 + per);
        float ws = 0.f;
        for (int i = w0 + lane; i < w1; i += 32) ws += w_at(i);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ws += __shfl_xor_sync(0xffffffffu, ws, o);
        if (lane == 0) scan_tot[warp] = ws;
        if (threadIdx.x == 0) found_id = -1;
        __syncthreads();
        float wbefore = before;
        int wsel = -1, wlast = -1;
        for (int w = 0; w < kWarps; ++w) {
          if (scan_tot[w] > 0.f) wlast = w;
          if (wsel < 0 && !past && wbefore + scan_tot[w] > target) wsel = w;
          if (wsel < 0) wbefore += scan_tot[w];
        }
        if (wsel < 0) wsel = wlast;
        if (warp == wsel) {
          float acc = wbefore;
          int pick = -1, last_pos = -1;
          for (int i0 = w0; i0 < w1 && pick < 0; i0 += 32) {
            const int i = i0 + lane;
            const float w = i < w1 ? w_at(i) : 0.f;
            float incl = w;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
              const float t = __shfl_up_sync(0xffffffffu, incl, o);
              if (lane >= o) incl += t;
            }
            const unsigned pos = __ballot_sync(0xffffffffu, i < w1 && w > 0.f);
            if (pos) last_pos = i0 + 31 - __clz(pos);
            const unsigned hit = __ballot_sync(0xffffffffu, !past && i < w1 && w > 0.f && acc + incl > target);
            if (hit) pick = i0 + __ffs(hit) - 1;
            acc += __shfl_sync(0xffffffffu, incl, 31);
          }
          // past the total (rounding): the last entry with mass
          if (pick < 0) pick = last_pos >= 0 ? last_pos : w1 - 1;
          if (lane == 0) found_id = pick;
        }
        __syncthreads();
        if (threadIdx.x == 0) a.bonus[b] = lo + found_id;
      }
      break;
    }
    steps[++L] = accepted;
    node = accepted;
    ++depth;
  }
  if (crank == 0 && threadIdx.x == 0) {
    a.accept_len[b] = L;
    for (int i = 0; i <= a.K; ++i) a.path[size_t(b) * (a.K + 1) + i] = i <= L ? steps[i] : -1;
  }
  cluster_sync();                          // peers are done reading this CTA's shared memory
}

}  // namespace rej
}  // namespace md
