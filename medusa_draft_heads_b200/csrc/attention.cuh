// Tree-masked attention over the KV prefix plus the tree (CUDA-core path).
//
// Source: "Medusa heads versus separate draft model", section "Acceptance",
// tree paragraph: every branch is verified in one target pass with a tree
// attention mask. A tree token attends to the whole prefix and, inside the
// tree, to its ancestors and itself; the ancestor sets travel as bitsets in
// the kernel parameter space.
//
// Split-KV: CTA (chunk c, KV head g, request b) takes 128 consecutive key
// slots of [0, P_b + T) and every query row that reads KV head g (T tree
// tokens x Hq/Hkv query heads). It writes a chunk-local max, sum and
// weighted V per row; attn_merge_kernel combines the chunks in fixed order.
#pragma once

#include "common.cuh"

namespace md {
namespace attn {

constexpr int kChunk = 128;
constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

struct Args {
  const uint16_t* q;          // [B, T, Hq, dh]
  const uint16_t* kc;         // [B, Hkv, S_max, dh]
  const uint16_t* vc;
  const int32_t* prefix_len;  // [B]
  float* part_acc;            // [B, Hkv, max_chunks, R, dh]
  float2* part_ml;            // [B, Hkv, max_chunks, R]  (max, sum) in log2 units
  float* out;                 // [B, T, Hq, dh]
  int S_max, Hq, Hkv, G, R, max_chunks;
  float scale_log2;           // softmax scale * log2(e)
};

template <int DH>
constexpr int smem_bytes() {
  return kChunk * (DH + 2) * 2 + kChunk * DH * 2 + kWarps * DH * 4;
}

template <int DH>
__global__ void __launch_bounds__(kThreads) attn_chunk_kernel(const __grid_constant__ TreeParams tp, Args a) {
  extern __shared__ __align__(16) uint8_t smem[];
  constexpr int LK = DH + 2;  // odd word stride: lanes reading different keys hit different banks
  uint16_t* Ks = reinterpret_cast<uint16_t*>(smem);
  uint16_t* Vs = Ks + kChunk * LK;
  float* qs = reinterpret_cast<float*>(Vs + kChunk * DH);
  const int c = blockIdx.x, hk = blockIdx.y, b = blockIdx.z;
  const int T = tp.T;
  pdl_wait_primary();
  pdl_launch_dependents();
  const int P = a.prefix_len[b];
  if (P < 0 || P + T > a.S_max) {
    if (c == 0 && hk == 0 && threadIdx.x == 0) set_status(MD_DEV_BAD_PREFIX);
    return;
  }
  const int nkeys = P + T;
  const int c0 = c * kChunk;
  if (c0 >= nkeys) return;
  const int nk = min(kChunk, nkeys - c0);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const size_t kvbase = ((size_t(b) * a.Hkv + hk) * a.S_max + c0) * DH;
  for (int idx = threadIdx.x; idx < kChunk * (DH / 8); idx += kThreads) {
    const int row = idx / (DH / 8), c8 = idx % (DH / 8);
    uint4 kv = make_uint4(0, 0, 0, 0), vv = make_uint4(0, 0, 0, 0);
    if (row < nk) {
      kv = *reinterpret_cast<const uint4*>(a.kc + kvbase + size_t(row) * DH + c8 * 8);
      vv = *reinterpret_cast<const uint4*>(a.vc + kvbase + size_t(row) * DH + c8 * 8);
    }
    uint32_t* kd = reinterpret_cast<uint32_t*>(Ks + row * LK + c8 * 8);
    kd[0] = kv.x; kd[1] = kv.y; kd[2] = kv.z; kd[3] = kv.w;
    *reinterpret_cast<uint4*>(Vs + row * DH + c8 * 8) = vv;
  }
  __syncthreads();

  constexpr int NI = kChunk / 32;   // keys per lane
  constexpr int NE = DH / 32;       // output dims per lane
  float* qw = qs + warp * DH;
  for (int r = warp; r < a.R; r += kWarps) {
    const int t = r / a.G, g = r % a.G;
    const int h = hk * a.G + g;
    const uint16_t* qp = a.q + ((size_t(b) * T + t) * a.Hq + h) * DH;
    for (int e = lane; e < DH; e += 32) qw[e] = bf16_to_f32(qp[e]);
    __syncwarp();

    float s[NI];
#pragma unroll
    for (int i = 0; i < NI; ++i) s[i] = 0.f;
#pragma unroll 4
    for (int e = 0; e < DH; e += 2) {
      const float2 qv = *reinterpret_cast<const float2*>(qw + e);
#pragma unroll
      for (int i = 0; i < NI; ++i) {
        const uint32_t kk = *reinterpret_cast<const uint32_t*>(Ks + (lane + 32 * i) * LK + e);
        s[i] = fmaf(qv.x, bf16lo(kk), s[i]);
        s[i] = fmaf(qv.y, bf16hi(kk), s[i]);
      }
    }
    float mloc = -INFINITY;
#pragma unroll
    for (int i = 0; i < NI; ++i) {
      const int j = lane + 32 * i;
      const int slot = c0 + j;
      bool vis = j < nk;
      if (vis && slot >= P) {
        const int node = slot - P;
        vis = (tp.anc[t][node >> 5] >> (node & 31)) & 1u;
      }
      s[i] = vis ? s[i] * a.scale_log2 : -INFINITY;
      mloc = fmaxf(mloc, s[i]);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mloc = fmaxf(mloc, __shfl_xor_sync(0xffffffffu, mloc, off));
    float lsum = 0.f;
#pragma unroll
    for (int i = 0; i < NI; ++i) {
      s[i] = (s[i] == -INFINITY) ? 0.f : exp2f(s[i] - mloc);
      lsum += s[i];
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) lsum += __shfl_xor_sync(0xffffffffu, lsum, off);

    float o[NE];
#pragma unroll
    for (int e = 0; e < NE; ++e) o[e] = 0.f;
#pragma unroll
    for (int i = 0; i < NI; ++i) {
      for (int jj = 0; jj < 32; ++jj) {
        const int j = 32 * i + jj;
        const float pj = __shfl_sync(0xffffffffu, s[i], jj);
        if (j < nk) {
          const uint16_t* vr = Vs + j * DH + lane * NE;
          if constexpr (NE == 4) {
            const uint2 vv = *reinterpret_cast<const uint2*>(vr);
            o[0] = fmaf(pj, bf16lo(vv.x), o[0]);
            o[1] = fmaf(pj, bf16hi(vv.x), o[1]);
            o[2] = fmaf(pj, bf16lo(vv.y), o[2]);
            o[3] = fmaf(pj, bf16hi(vv.y), o[3]);
          } else {
            const uint32_t vv = *reinterpret_cast<const uint32_t*>(vr);
            o[0] = fmaf(pj, bf16lo(vv), o[0]);
            o[1] = fmaf(pj, bf16hi(vv), o[1]);
          }
        }
      }
    }
    const size_t prow = ((size_t(b) * a.Hkv + hk) * a.max_chunks + c) * a.R + r;
    if (lane == 0) a.part_ml[prow] = make_float2(mloc, lsum);
#pragma unroll
    for (int e = 0; e < NE; ++e) a.part_acc[prow * DH + lane * NE + e] = o[e];
    __syncwarp();
  }
}

// out[b, t, h, :] from the chunk partials, combined in chunk order.
// grid (T * Hq, B), DH threads (one output dimension each).
template <int DH>
__global__ void __launch_bounds__(DH) attn_merge_kernel(const __grid_constant__ TreeParams tp, Args a) {
  pdl_wait_primary();
  pdl_launch_dependents();
  const int b = blockIdx.y;
  const int th = blockIdx.x;
  const int t = th / a.Hq, h = th % a.Hq;
  const int hk = h / a.G, g = h % a.G;
  const int r = t * a.G + g;
  const int e = threadIdx.x;
  const int T = tp.T;
  const int P = a.prefix_len[b];
  float* o = a.out + ((size_t(b) * T + t) * a.Hq + h) * DH;
  if (P < 0 || P + T > a.S_max) {
    o[e] = 0.f;
    return;
  }
  const int nch = (P + T + kChunk - 1) / kChunk;
  const size_t base = (size_t(b) * a.Hkv + hk) * a.max_chunks;
  float mx = -INFINITY;
  for (int c = 0; c < nch; ++c) mx = fmaxf(mx, a.part_ml[(base + c) * a.R + r].x);
  float L = 0.f, acc = 0.f;
  for (int c = 0; c < nch; ++c) {
    const float2 ml = a.part_ml[(base + c) * a.R + r];
    if (ml.x == -INFINITY) continue;
    const float w = exp2f(ml.x - mx);
    L = fmaf(ml.y, w, L);
    acc = fmaf(a.part_acc[((base + c) * a.R + r) * DH + e], w, acc);
  }
  o[e] = acc / L;
}

}  // namespace attn
}  // namespace md
