// Acceptance of the longest matching branch.
//
// Source: "Medusa heads versus separate draft model", section "Acceptance",
// tree paragraph (advance along the branch that matches), and section
// "Training" (typical acceptance, which accepts more drafts under sampling and
// is not lossless).
//
//   accept_rows_kernel  one pass over a chunk of one target-logit row: the
//                       argmax (lowest id on ties) and, for the typical rule,
//                       the online max m, S = sum e^(x-m), W = sum (x-m) e^(x-m)
//                       of x = logits / temperature (HBM-bound, 16-byte loads)
//   accept_walk_kernel  per request: merge the chunks, test every node against
//                       its parent's row, propagate acceptance down the tree
//                       level by level, pick the deepest accepted node (lowest
//                       index on ties), emit its path and the bonus token.
//   accept_sample_kernel (sampled rule) one draw per row by inverse CDF from a
//                       supplied uniform; the walk then tests each node against
//                       its parent's draw instead of the argmax.
//
// Sampled rule (same section: rejection sampling is the page's choice when the
// target distribution must be kept exactly; it gives no algorithm for a tree
// of deterministic candidates):
// rejection sampling of a candidate chosen with certainty accepts it with
// probability p(c) and otherwise samples p with c removed, which over a node's
// candidate children is one draw y ~ p of the node's row, accepting the child
// whose token is y; the bonus token is the last accepted node's draw.
#pragma once

#include "common.cuh"

namespace md {
namespace acc {

constexpr int kRowThreads = 256;
constexpr int kPartFloats = 8;  // best value, best id (bits), m, S, W, pad

struct Args {
  const float* logits;     // [B, T, V]
  const int32_t* tokens;   // [B, T]
  int32_t* accept_len;     // [B]
  int32_t* path;           // [B, K + 1]
  int32_t* bonus;          // [B]
  float* part;             // [B * T, nchunks, 8]
  const int32_t* ysamp;    // [B * T] per-row draws (sampled rule), else null
  int T, V, K, nchunks, chunk_len, mode;
  float inv_temp, log_eps, log_alpha;
};

struct Soft {
  float m, S, W;
};

// Combine two (max, sum e^(x-max), sum (x-max) e^(x-max)) summaries.
__device__ __forceinline__ Soft soft_merge(Soft a, Soft b) {
  if (a.S == 0.f) return b;
  if (b.S == 0.f) return a;
  const float m = fmaxf(a.m, b.m);
  const float ea = expf(a.m - m), eb = expf(b.m - m);
  Soft r;
  r.m = m;
  r.S = a.S * ea + b.S * eb;
  r.W = ea * (a.W + (a.m - m) * a.S) + eb * (b.W + (b.m - m) * b.S);
  return r;
}

__device__ __forceinline__ void soft_add(Soft& s, float y) {
  if (s.S == 0.f) {
    s.m = y;
    s.S = 1.f;
    s.W = 0.f;
    return;
  }
  if (y > s.m) {
    const float sc = expf(s.m - y);
    s.W = sc * (s.W + (s.m - y) * s.S);
    s.S *= sc;
    s.m = y;
  }
  const float e = expf(y - s.m);
  s.S += e;
  s.W = fmaf(y - s.m, e, s.W);
}

__global__ void __launch_bounds__(kRowThreads) accept_rows_kernel(Args a) {
  pdl_wait_primary();          // logits and tokens may come from earlier kernels
  pdl_launch_dependents();
  const int row = blockIdx.y, c = blockIdx.x;
  const int v0 = c * a.chunk_len;
  const int v1 = min(a.V, v0 + a.chunk_len);
  const float* x = a.logits + size_t(row) * a.V;
  float bv = -INFINITY;
  int bi = INT_MAX;
  Soft sm{-INFINITY, 0.f, 0.f};
  const bool typical = a.mode == MD_ACCEPT_TYPICAL;
  // kUnroll independent 16-byte loads in flight per thread before any use.
  constexpr int kUnroll = 8;
  constexpr int kStep = kRowThreads * 4;
  for (int base = v0 + threadIdx.x * 4; base < v1; base += kStep * kUnroll) {
    float4 f[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int v = base + u * kStep;
      f[u] = v < v1 ? ld_stream_f4(x + v) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int v = base + u * kStep;
      if (v < v1) {
        const float fv[4] = {f[u].x, f[u].y, f[u].z, f[u].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          if (better(fv[e], v + e, bv, bi)) {
            bv = fv[e];
            bi = v + e;
          }
          if (typical) soft_add(sm, fv[e] * a.inv_temp);
        }
      }
    }
  }
  // Block reduction (fixed shuffle tree, then warps in order).
  __shared__ float sv[kRowThreads / 32];
  __shared__ int si[kRowThreads / 32];
  __shared__ Soft ss[kRowThreads / 32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
    const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
    if (better(ov, oi, bv, bi)) {
      bv = ov;
      bi = oi;
    }
    if (typical) {
      Soft o;
      o.m = __shfl_xor_sync(0xffffffffu, sm.m, off);
      o.S = __shfl_xor_sync(0xffffffffu, sm.S, off);
      o.W = __shfl_xor_sync(0xffffffffu, sm.W, off);
      sm = (lane & off) ? soft_merge(o, sm) : soft_merge(sm, o);
    }
  }
  if (lane == 0) {
    sv[warp] = bv;
    si[warp] = bi;
    ss[warp] = sm;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 1; w < kRowThreads / 32; ++w) {
      if (better(sv[w], si[w], bv, bi)) {
        bv = sv[w];
        bi = si[w];
      }
      if (typical) sm = soft_merge(sm, ss[w]);
    }
    float* p = a.part + (size_t(row) * a.nchunks + c) * kPartFloats;
    p[0] = bv;
    p[1] = __int_as_float(bi);
    p[2] = sm.m;
    p[3] = sm.S;
    p[4] = sm.W;
  }
}

__global__ void __launch_bounds__(MD_MAX_T) accept_walk_kernel(const __grid_constant__ TreeParams tp, Args a) {
  pdl_wait_primary();          // row summaries come from accept_rows_kernel
  pdl_launch_dependents();
  const int b = blockIdx.x;
  const int j = threadIdx.x;
  const int T = tp.T;
  __shared__ int amax[MD_MAX_T];
  __shared__ float mrow[MD_MAX_T], logS[MD_MAX_T], Hrow[MD_MAX_T];
  __shared__ int accd[MD_MAX_T];
  __shared__ int wkey[MD_MAX_T / 32];
  const bool typical = a.mode == MD_ACCEPT_TYPICAL;

  if (j < T && a.ysamp) {
    amax[j] = a.ysamp[size_t(b) * T + j];
  } else if (j < T) {
    const float* p = a.part + size_t(b * T + j) * a.nchunks * kPartFloats;
    float bv = p[0];
    int bi = __float_as_int(p[1]);
    Soft sm{p[2], p[3], p[4]};
    for (int c = 1; c < a.nchunks; ++c) {
      const float* q = p + size_t(c) * kPartFloats;
      const int qi = __float_as_int(q[1]);
      if (better(q[0], qi, bv, bi)) {
        bv = q[0];
        bi = qi;
      }
      if (typical) sm = soft_merge(sm, Soft{q[2], q[3], q[4]});
    }
    amax[j] = bi;
    if (typical) {
      mrow[j] = sm.m;
      logS[j] = logf(sm.S);
      Hrow[j] = logS[j] - sm.W / sm.S;
    }
  }
  __syncthreads();
  bool match = false;
  if (j > 0 && j < T) {
    const int par = tp.parent[j];
    const int tok = a.tokens[size_t(b) * T + j];
    if (!typical) {
      match = tok == amax[par];
    } else if (tok >= 0 && tok < a.V) {
      const float y = a.logits[(size_t(b) * T + par) * a.V + tok] * a.inv_temp;
      const float logp = y - mrow[par] - logS[par];
      match = logp > fminf(a.log_eps, a.log_alpha - Hrow[par]);
    } else {
      set_status(MD_DEV_BAD_TOKEN);
    }
  }
  if (j < MD_MAX_T) accd[j] = (j == 0) ? 1 : 0;
  __syncthreads();
  for (int level = 1; level <= tp.max_depth; ++level) {
    if (j < T && tp.depth[j] == level) accd[j] = match && accd[tp.parent[j]];
    __syncthreads();
  }
  // Deepest accepted node, lowest index on ties: max of depth*256 + (255 - j).
  int key = (j < T && accd[j]) ? (tp.depth[j] << 8) | (255 - j) : -1;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) key = max(key, __shfl_xor_sync(0xffffffffu, key, off));
  if ((j & 31) == 0) wkey[j >> 5] = key;
  __syncthreads();
  if (j == 0) {
    for (int w = 1; w < MD_MAX_T / 32; ++w) key = max(key, wkey[w]);
    const int L = key >> 8;
    int node = 255 - (key & 255);
    a.accept_len[b] = L;
    a.bonus[b] = amax[node];
    int32_t* pp = a.path + size_t(b) * (a.K + 1);
    for (int i = a.K; i > L; --i) pp[i] = -1;
    for (int i = L; i >= 0; --i) {
      pp[i] = node;
      node = tp.parent[node];
    }
  }
}

// ---------------------------------------------------------------------------
// Sampled rule: y = min{v : sum_{w <= v} p(w) > u} for p = softmax(x / temp) of
// one row, in id order. One CTA per row: each warp takes 1024-id tiles and
// records the tile maximum and sum of exp(x - max) (fixed order); one thread
// combines the tiles in id order and finds the tile where u * S is crossed;
// warp 0 then walks that tile's ids in order (lane l owns ids 32l .. 32l+31).
// Rounding can leave the crossing just past the end of the tile or of the row:
// then the last id with nonzero weight there is taken.
// ---------------------------------------------------------------------------
constexpr int kSampleTile = 1024;
constexpr int kSampleMaxTiles = 2048;       // V <= 2M
constexpr int kSampleThreads = 1024;        // 32 warps share a row's tiles: one row per CTA

struct SampleArgs {
  const float* logits;     // [B * T, V]
  const float* uniforms;   // [B * T] in [0, 1)
  int32_t* ysamp;          // [B * T]
  int V;
  float inv_temp_log2e;    // log2(e) / temperature
};

__global__ void __launch_bounds__(kSampleThreads) accept_sample_kernel(SampleArgs a) {
  pdl_wait_primary();          // logits may come from earlier kernels
  pdl_launch_dependents();
  __shared__ float tmax[kSampleMaxTiles], tsum[kSampleMaxTiles];
  __shared__ int s_tile;
  __shared__ float s_rem, s_max;
  const int row = blockIdx.x;
  const float* x = a.logits + size_t(row) * a.V;
  const int ntile = (a.V + kSampleTile - 1) / kSampleTile;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float c = a.inv_temp_log2e;          // work in log2 units: y = x * log2(e) / temp
  // pass 1: tile maxima and sums, one warp per tile
  for (int i = warp; i < ntile; i += kSampleThreads / 32) {
    float v[32];
    float mx = -INFINITY;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int id = i * kSampleTile + j * 128 + lane * 4;
      float4 f = make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
      if (id + 3 < a.V) {
        f = ld_stream_f4(x + id);
      } else {
        if (id < a.V) f.x = x[id];
        if (id + 1 < a.V) f.y = x[id + 1];
        if (id + 2 < a.V) f.z = x[id + 2];
      }
      v[4 * j] = f.x * c;
      v[4 * j + 1] = f.y * c;
      v[4 * j + 2] = f.z * c;
      v[4 * j + 3] = f.w * c;
#pragma unroll
      for (int e = 0; e < 4; ++e) mx = fmaxf(mx, v[4 * j + e]);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    float sm = 0.f;
    if (mx != -INFINITY) {
#pragma unroll
      for (int k = 0; k < 32; ++k) sm += exp2f(v[k] - mx);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sm += __shfl_xor_sync(0xffffffffu, sm, off);
    if (lane == 0) {
      tmax[i] = mx;
      tsum[i] = sm;
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    float M = -INFINITY;
    for (int i = 0; i < ntile; ++i) M = fmaxf(M, tmax[i]);
    float S = 0.f;
    for (int i = 0; i < ntile; ++i) S += (tmax[i] == -INFINITY) ? 0.f : tsum[i] * exp2f(tmax[i] - M);
    const float target = a.uniforms[row] * S;
    float C = 0.f;
    int found = -1, last = -1;
    float rem = INFINITY;
    for (int i = 0; i < ntile; ++i) {
      const float w = (tmax[i] == -INFINITY) ? 0.f : tsum[i] * exp2f(tmax[i] - M);
      if (w > 0.f) last = i;
      if (found < 0 && C + w > target) {
        found = i;
        rem = target - C;
      }
      C += w;
    }
    if (found < 0) found = last;             // rounding left u * S at the end: last tile with weight
    s_tile = found;
    s_rem = rem;
    s_max = M;
  }
  __syncthreads();
  if (warp == 0) {
    const int i = s_tile;
    int y = 0;
    if (i >= 0) {
      const float M = s_max, rem = s_rem;
      float w[32];
      float ls = 0.f;
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const int id = i * kSampleTile + lane * 32 + e;
        w[e] = id < a.V ? exp2f(x[id] * c - M) : 0.f;
        ls += w[e];
      }
      float incl = ls;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const float t = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += t;
      }
      const float excl = incl - ls;
      const unsigned hit = __ballot_sync(0xffffffffu, ls > 0.f && rem < incl);
      const unsigned pos = __ballot_sync(0xffffffffu, ls > 0.f);
      // the first lane whose running sum passes rem, else the last lane with weight
      const int src = hit ? __ffs(hit) - 1 : (pos ? 31 - __clz(pos) : 0);
      int yl = -1, lastpos = -1;
      if (lane == src) {
        float run = excl;
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          run += w[e];
          if (w[e] > 0.f) lastpos = e;
          if (yl < 0 && w[e] > 0.f && run > rem) yl = e;
        }
        if (yl < 0) yl = lastpos;
      }
      yl = __shfl_sync(0xffffffffu, yl, src);
      y = i * kSampleTile + src * 32 + max(yl, 0);
    }
    if (lane == 0) a.ysamp[row] = y;
  }
}

}  // namespace acc
}  // namespace md
