// Medusa draft heads with a fused per-head top-k, small-M streaming path.
//
// Source: "Medusa heads versus separate draft model", sections "What each one
// is" and "Cost per step": head k = a residual block around a d x d layer with
// bias, then a bias-free d x V vocabulary projection of its own; all heads read
// the same hidden state, once per step. At small batch the heads are bound by
// the bytes of their weights (8.94 GB of them for four heads at d = 8,192,
// V = 128,256), so both phases stream the weights once from HBM with 16-byte or TMA loads and do the
// arithmetic in fp32 on the CUDA cores.
//
//   phase 1  heads_w1_kernel       u = h W1_k + b1_k, z_k = bf16(h + SiLU(u))
//   phase 2  heads_vocab_kernel    logits tile = z_k Wv_k[:, tile] and its top-k
//   phase 3  heads_merge_kernel    top-k over every tile's candidates
#pragma once

#include <algorithm>

#include "common.cuh"

namespace md {
namespace heads {

constexpr int kTileV = 256;         // vocabulary columns of one phase-2 work unit
constexpr int kStageRows = 64;      // hidden rows per TMA stage
constexpr int kConsumerWarps = 8;   // phase-2 math warps (one more warp feeds TMA)
constexpr int kZPad = 8;            // z row i is stored as 8 bf16 (one per m), 16 B
constexpr int kW1Threads = 256;
constexpr int kW1TileO = 256;       // phase-1 output columns per CTA
constexpr int kW1MaxRows = 2048;    // phase-1 hidden rows per CTA (split-K)
constexpr int kMaxM = 4;        // rows these kernels support; the launchers use them for one row (the
                                // tensor-core weight stream is faster from two)
constexpr uint32_t kStageWBytes = kStageRows * kTileV * 2;  // 32 KB
constexpr uint32_t kStageZBytes = kStageRows * kZPad * 2;   // 1 KB
constexpr int kSmemBudget = 227 * 1024;

struct Plan {
  int M, d, V, K, kmax;
  int ntile_o;  // phase-1 column tiles
  int splits;   // phase-1 split-K factor
  int rows;     // phase-1 rows per split
  int ntiles;   // phase-2 vocabulary tiles
  int units;    // K * ntiles
  int nstages;  // phase-2 pipeline depth
  int grid;     // phase-2 CTAs (one candidate list per row, head and CTA)
  int stream_k; // phase 2 split by 64-row stages (balanced) instead of whole units
  size_t off_zt, off_part, off_cnt, off_tick, off_spart, off_cval, off_cid, bytes;
};

inline size_t align256(size_t x) { return (x + 255) / 256 * 256; }

// Phase-1 CTAs resident per SM (the kernel's launch bounds): the split-K grid
// is sized to one wave of them, so no partial second wave trails the stream.
__host__ __device__ constexpr int w1_blocks_per_sm(int M) { return M <= 2 ? 4 : 3; }

inline int vocab_smem_bytes(int M, int nstages) {
  // stages + mbarriers + cross-warp reduction + reduced logits + 1 KB alignment slack
  return nstages * int(kStageWBytes + kStageZBytes) + 2 * nstages * 8 + kConsumerWarps * M * kTileV * 4 +
         M * kTileV * 4 + 1024 + 64;
}

inline Plan make_plan(int M, int d, int V, int K, int kmax, int num_sms) {
  Plan p{};
  p.M = M; p.d = d; p.V = V; p.K = K; p.kmax = kmax;
  p.ntile_o = (d + kW1TileO - 1) / kW1TileO;
  int splits = 1;
  while (d / splits > kW1MaxRows) splits *= 2;
  const int w1_slots = w1_blocks_per_sm(M) * num_sms;
  while (p.ntile_o * K * splits * 2 <= w1_slots && d / (splits * 2) >= 64 && (d / (splits * 2)) % 8 == 0)
    splits *= 2;
  p.splits = splits;
  p.rows = d / splits;
  p.ntiles = (V + kTileV - 1) / kTileV;
  p.units = K * p.ntiles;
  int ns = 8;
  while (ns > 2 && vocab_smem_bytes(M, ns) > kSmemBudget) --ns;
  p.nstages = ns;
  size_t o = 0;
  p.off_zt = o;   o = align256(o + size_t(K) * d * kZPad * 2);
  p.off_part = o; o = align256(o + size_t(splits) * K * M * d * 4);
  p.off_cnt = o;  o = align256(o + size_t(K) * p.ntile_o * 8);      // epoch tickets (epoch_arrive)
  p.grid = std::min(num_sms, p.units);
  // Whole units over the CTAs leave a tail when they do not divide evenly
  // (2004 units of a 70B call over 148 CTAs: 13 or 14 each; 501 for one head:
  // 3 or 4). With at least one unit per CTA, cut the (unit, stage) items
  // instead: a unit then spans at most two CTAs, whose partial logits the
  // second to finish adds up.
  p.stream_k = (p.units > p.grid && p.units % p.grid != 0) ? 1 : 0;
  p.off_tick = o; o = align256(o + size_t(p.units) * 8);            // one epoch ticket per unit
  p.off_spart = o; o = align256(o + size_t(p.grid) * 2 * M * kTileV * 4);
  p.off_cval = o; o = align256(o + size_t(M) * K * p.grid * kmax * 4);
  p.off_cid = o;  o = align256(o + size_t(M) * K * p.grid * kmax * 4);
  p.bytes = o;
  return p;
}

// ---------------------------------------------------------------------------
// Tickets that need no clearing between calls. A ticket word holds a call's
// epoch (high 32 bits; every call of these kernels draws a new nonzero one on
// the host) and that call's arrivals so far (low 32 bits). An arrival that
// finds another epoch there (an earlier call's, zero, or whatever the
// workspace held) starts the count afresh. Returns this arrival's index
// within the call (0, 1, ...). The loop only retries while other CTAs of the
// call are arriving at the same word, so it ends after at most as many
// rounds as there are arrivals.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t epoch_arrive(unsigned long long* p, uint32_t epoch) {
  unsigned long long cur = *reinterpret_cast<volatile unsigned long long*>(p);
  for (;;) {
    const unsigned long long want =
        uint32_t(cur >> 32) == epoch ? cur + 1ull : ((unsigned long long)epoch << 32) | 1ull;
    const unsigned long long prev = atomicCAS(p, cur, want);
    if (prev == cur) return uint32_t(want) - 1u;
    cur = prev;
  }
}

// ---------------------------------------------------------------------------
// Phase 1: residual block, split over hidden rows, deterministic finish.
// grid (ntile_o, splits, K), 256 threads. Each warp owns rows w, w+8, ...
// of the split, each lane 8 output columns; partial sums go to `part`, and
// the last CTA of a (head, column tile) sums the splits in order and applies
// bias, SiLU and the residual.
// ---------------------------------------------------------------------------
struct W1Args {
  const uint16_t* h;   // [M, d]
  const uint16_t* W1;  // [K, d, d]
  const uint16_t* b1;  // [K, d]
  uint16_t* zt;        // [K, d, 8]
  float* part;         // [splits, K, M, d]
  unsigned long long* counters;   // [K, ntile_o] epoch tickets (epoch_arrive)
  int d, K, splits, rows, ntile_o;
  uint32_t epoch;      // this call's epoch
  int shared;          // 1: one projection for all heads: z row (m, k) goes to slot m*K + k of zt[0]
};

template <int M>
__global__ void __launch_bounds__(kW1Threads, w1_blocks_per_sm(M)) heads_w1_kernel(W1Args a) {
  extern __shared__ __align__(16) uint8_t smem[];
  uint4* hs = reinterpret_cast<uint4*>(smem);                          // [rows] x 8 bf16
  float* red = reinterpret_cast<float*>(smem + size_t(a.rows) * 16);   // [8 warps][M][256]
  __shared__ int is_last;

  pdl_launch_dependents();
  pdl_wait_primary();   // h may come from the work before (dependent launch)

  const int k = blockIdx.z, s = blockIdx.y, ct = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int d = a.d;
  const int i0 = s * a.rows;
  const int o = ct * kW1TileO + lane * 8;
  const bool col_ok = o < d;

  for (int r = threadIdx.x; r < a.rows; r += kW1Threads) {
    uint16_t v[8];
#pragma unroll
    for (int m = 0; m < 8; ++m) v[m] = (m < M) ? a.h[size_t(m) * d + i0 + r] : uint16_t(0);
    hs[r] = make_uint4(v[0] | (uint32_t(v[1]) << 16), v[2] | (uint32_t(v[3]) << 16), v[4] | (uint32_t(v[5]) << 16),
                       v[6] | (uint32_t(v[7]) << 16));
  }
  __syncthreads();

  float acc[M][8];
#pragma unroll
  for (int m = 0; m < M; ++m)
#pragma unroll
    for (int c = 0; c < 8; ++c) acc[m][c] = 0.f;

  if (col_ok) {
    const uint16_t* wrow = a.W1 + (size_t(k) * d + i0) * d + o;
    constexpr int U = M <= 2 ? 8 : 4;      // 16-byte loads in flight per lane
    int r = warp;
    for (; r + (U - 1) * kConsumerWarps < a.rows; r += U * kConsumerWarps) {
      uint4 w[U];
#pragma unroll
      for (int u = 0; u < U; ++u) w[u] = ld_stream_v4(wrow + size_t(r + u * kConsumerWarps) * d);
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const uint4 hv = hs[r + u * kConsumerWarps];
        const uint32_t hw[4] = {hv.x, hv.y, hv.z, hv.w};
        const uint32_t ww[4] = {w[u].x, w[u].y, w[u].z, w[u].w};
#pragma unroll
        for (int m = 0; m < M; ++m) {
          const float hm = (m & 1) ? bf16hi(hw[m >> 1]) : bf16lo(hw[m >> 1]);
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            acc[m][2 * c] = fmaf(hm, bf16lo(ww[c]), acc[m][2 * c]);
            acc[m][2 * c + 1] = fmaf(hm, bf16hi(ww[c]), acc[m][2 * c + 1]);
          }
        }
      }
    }
    for (; r < a.rows; r += kConsumerWarps) {
      const uint4 w = ld_stream_v4(wrow + size_t(r) * d);
      const uint4 hv = hs[r];
      const uint32_t hw[4] = {hv.x, hv.y, hv.z, hv.w};
      const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int m = 0; m < M; ++m) {
        const float hm = (m & 1) ? bf16hi(hw[m >> 1]) : bf16lo(hw[m >> 1]);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          acc[m][2 * c] = fmaf(hm, bf16lo(ww[c]), acc[m][2 * c]);
          acc[m][2 * c + 1] = fmaf(hm, bf16hi(ww[c]), acc[m][2 * c + 1]);
        }
      }
    }
  }

#pragma unroll
  for (int m = 0; m < M; ++m) {
    float4* dst = reinterpret_cast<float4*>(red + (size_t(warp) * M + m) * kW1TileO + lane * 8);
    dst[0] = make_float4(acc[m][0], acc[m][1], acc[m][2], acc[m][3]);
    dst[1] = make_float4(acc[m][4], acc[m][5], acc[m][6], acc[m][7]);
  }
  __syncthreads();

  const int t = threadIdx.x;
  const int col = ct * kW1TileO + t;
  if (col < d) {
#pragma unroll
    for (int m = 0; m < M; ++m) {
      float v = 0.f;
#pragma unroll
      for (int w = 0; w < kConsumerWarps; ++w) v += red[(size_t(w) * M + m) * kW1TileO + t];
      a.part[((size_t(s) * a.K + k) * M + m) * d + col] = v;
    }
  }
  __threadfence();
  __syncthreads();
  if (t == 0) {
    const uint32_t ticket = epoch_arrive(&a.counters[k * a.ntile_o + ct], a.epoch);
    is_last = (ticket == uint32_t(a.splits - 1));
  }
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  if (col < d) {
    const float bias = bf16_to_f32(a.b1[size_t(k) * d + col]);
    uint16_t zv[8];
#pragma unroll
    for (int m = 0; m < 8; ++m) {
      if (m < M) {
        float u = 0.f;
        for (int sp = 0; sp < a.splits; ++sp) u += __ldcg(&a.part[((size_t(sp) * a.K + k) * M + m) * d + col]);
        u += bias;
        const float hval = bf16_to_f32(a.h[size_t(m) * d + col]);
        zv[m] = f32_to_bf16_rne(hval + u / (1.0f + expf(-u)));
      } else {
        zv[m] = 0;
      }
    }
    if (a.shared) {
#pragma unroll
      for (int m = 0; m < M; ++m) a.zt[size_t(col) * kZPad + m * a.K + k] = zv[m];
    } else {
      reinterpret_cast<uint4*>(a.zt)[size_t(k) * d + col] =
          make_uint4(zv[0] | (uint32_t(zv[1]) << 16), zv[2] | (uint32_t(zv[3]) << 16),
                     zv[4] | (uint32_t(zv[5]) << 16), zv[6] | (uint32_t(zv[7]) << 16));
    }
  }
}

// ---------------------------------------------------------------------------
// Phase 2: persistent vocabulary stream with the top-k fused in.
// grid = min(#SMs, K * ntiles), 288 threads: warps 0..7 do the math, warp 8
// issues the TMA loads. A work unit is (head k, 256-column tile); it walks
// d / 64 stages of [64 rows x 256 cols] of Wv_k plus the matching 64 rows of
// z_k. CTA c owns the contiguous units [c*U/G, (c+1)*U/G). Warp w multiplies
// rows 8w..8w+7 of each stage, lane l columns 8l..8l+7, fp32 accumulate; the
// eight warps' partials are summed in fixed order, then warp m folds the
// tile's 256 logits of row m into a running top-k of (row m, head k), which
// is written out once per (CTA, head): one candidate list per CTA and head.
// ---------------------------------------------------------------------------
struct VocabArgs {
  const uint16_t* zt;  // [K, d, 8]
  float* cand_val;     // [M, K, gridDim.x, kmax]: one list per (row, head, CTA)
  int* cand_id;
  float* logits_dbg;   // [M, K, V] or null
  const float* gumbel_u;  // [M, K, V] uniforms (sampled drafts) or null (top-k of the logits)
  float inv_tau;          // 1 / draft temperature (sampled drafts)
  int stream_k;           // CTA ranges in (unit, stage) items instead of whole units
  unsigned long long* tickets;   // [units] epoch tickets: a split unit's second finisher adds the parts
  uint32_t epoch;         // this call's epoch
  float* spart;           // [gridDim.x][2][M][256]: partial logits of the units a CTA range cuts
  int d, V, K, kmax, ntiles, units, nstages;
  int shared, kh;      // shared projection: K == 1 and row m is (m / kh, head m % kh)
  int kph[MD_MAX_K];
};

// This CTA's (unit, stage) items [i0, i1): whole units, or (stream_k) an
// equal share of the units x stages items.
__device__ __forceinline__ void item_range(const VocabArgs& a, int S, long long& i0, long long& i1) {
  if (a.stream_k) {
    const long long W = (long long)a.units * S;
    i0 = (long long)blockIdx.x * W / gridDim.x;
    i1 = (long long)(blockIdx.x + 1) * W / gridDim.x;
  } else {
    i0 = (long long)blockIdx.x * a.units / gridDim.x * S;
    i1 = (long long)(blockIdx.x + 1) * a.units / gridDim.x * S;
  }
}

template <int M>
__global__ void __launch_bounds__((kConsumerWarps + 1) * 32, 1)
    heads_vocab_kernel(const __grid_constant__ CUtensorMap wv_map, VocabArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  const int ns = a.nstages;
  uint8_t* stage_w = smem;                                              // ns x 32 KB
  uint8_t* stage_z = smem + size_t(ns) * kStageWBytes;                  // ns x 1 KB
  uint64_t* full = reinterpret_cast<uint64_t*>(stage_z + size_t(ns) * kStageZBytes);
  uint64_t* empty = full + ns;
  float* red = reinterpret_cast<float*>(empty + ns);                    // [8][M][256]
  float* lg = red + kConsumerWarps * M * kTileV;                        // [M][256]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int stages_per_unit = a.d / kStageRows;
  pdl_launch_dependents();

  if (threadIdx.x == 0) {
    for (int i = 0; i < ns; ++i) {
      mbar_init(smem_u32(&full[i]), 1);
      mbar_init(smem_u32(&empty[i]), kConsumerWarps);
    }
    fence_barrier_init();
  }
  __syncthreads();

  if (warp == kConsumerWarps) {
    // ------------------------------ producer ------------------------------
    if (lane == 0) {
      prefetch_tensormap(&wv_map);
      const uint64_t pol = policy_evict_first();
      long long i0, i1;                    // this CTA's (unit, stage) items
      item_range(a, stages_per_unit, i0, i1);
      auto load_w = [&](long long w, int slot) {
        const int unit = int(w / stages_per_unit), s = int(w % stages_per_unit);
        const int k = unit / a.ntiles, tile = unit % a.ntiles;
        tma_load_2d_hint(smem_u32(stage_w + size_t(slot) * kStageWBytes), &wv_map, tile * kTileV,
                         k * a.d + s * kStageRows, smem_u32(&full[slot]), pol);
      };
      auto load_z = [&](long long w, int slot) {
        const int unit = int(w / stages_per_unit), s = int(w % stages_per_unit);
        const int k = unit / a.ntiles;
        bulk_load(smem_u32(stage_z + size_t(slot) * kStageZBytes),
                  a.zt + (size_t(k) * a.d + size_t(s) * kStageRows) * kZPad, kStageZBytes, smem_u32(&full[slot]));
      };
      // The first stages' weights do not depend on phase 1: request them
      // before waiting for it; z (phase 1's output) only after.
      const int pre = int(min((long long)ns, i1 - i0));
      for (int j = 0; j < pre; ++j) {
        mbar_arrive_expect_tx(smem_u32(&full[j]), kStageWBytes + kStageZBytes);
        load_w(i0 + j, j);
      }
      pdl_wait_primary();
      for (int j = 0; j < pre; ++j) load_z(i0 + j, j);
      int it = pre;
      for (long long w = i0 + pre; w < i1; ++w, ++it) {
        const int slot = it % ns;
        if (!mbar_wait(smem_u32(&empty[slot]), ((it / ns) - 1) & 1)) {
          set_status(MD_DEV_TIMEOUT);
          break;
        }
        mbar_arrive_expect_tx(smem_u32(&full[slot]), kStageWBytes + kStageZBytes);
        load_w(w, slot);
        load_z(w, slot);
      }
      // Drain: wait until the consumers have released every issued stage so
      // no copy is in flight into shared memory when the CTA exits.
      for (int j = (it > ns ? it - ns : 0); j < it; ++j) {
        if (!mbar_wait(smem_u32(&empty[j % ns]), (j / ns) & 1)) {
          set_status(MD_DEV_TIMEOUT);
          break;
        }
      }
    }
    return;
  }

  // -------------------------------- consumers --------------------------------
  __shared__ int s_ticket;
  int it = 0;
  bool ok = true;
  long long i0, i1;
  item_range(a, stages_per_unit, i0, i1);
  // Running top-k of (row m = warp, current head): lane r holds entry r.
  float rv = -INFINITY;
  int ri = INT_MAX;
  // One part = the stages of one unit that lie in this CTA's range.
  for (long long w = i0; w < i1;) {
    const int unit = int(w / stages_per_unit);
    const int s_lo = int(w % stages_per_unit);
    const int s_hi = int(min((long long)stages_per_unit, s_lo + (i1 - w)));
    const int k = unit / a.ntiles, tile = unit % a.ntiles;
    float acc[M][8];
#pragma unroll
    for (int m = 0; m < M; ++m)
#pragma unroll
      for (int c = 0; c < 8; ++c) acc[m][c] = 0.f;

    for (int s = s_lo; s < s_hi; ++s, ++it) {
      const int slot = it % ns;
      if (ok && !mbar_wait(smem_u32(&full[slot]), (it / ns) & 1)) {
        set_status(MD_DEV_TIMEOUT);
        ok = false;
      }
      if (ok) {
        const uint8_t* wb = stage_w + size_t(slot) * kStageWBytes + warp * 8 * (kTileV * 2) + lane * 16;
        const uint8_t* zb = stage_z + size_t(slot) * kStageZBytes + warp * 8 * 16;
#pragma unroll
        for (int r = 0; r < 8; ++r) {
          const uint4 wv = *reinterpret_cast<const uint4*>(wb + r * (kTileV * 2));
          const uint4 zv = *reinterpret_cast<const uint4*>(zb + r * 16);
          const uint32_t zw[4] = {zv.x, zv.y, zv.z, zv.w};
          const uint32_t ww[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
          for (int m = 0; m < M; ++m) {
            const float zm = (m & 1) ? bf16hi(zw[m >> 1]) : bf16lo(zw[m >> 1]);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              acc[m][2 * c] = fmaf(zm, bf16lo(ww[c]), acc[m][2 * c]);
              acc[m][2 * c + 1] = fmaf(zm, bf16hi(ww[c]), acc[m][2 * c + 1]);
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&empty[slot]));
    }
    w += s_hi - s_lo;
    const bool whole = s_lo == 0 && s_hi == stages_per_unit;

    // Cross-warp reduction in fixed warp order.
#pragma unroll
    for (int m = 0; m < M; ++m) {
      float4* dst = reinterpret_cast<float4*>(red + (size_t(warp) * M + m) * kTileV + lane * 8);
      dst[0] = make_float4(acc[m][0], acc[m][1], acc[m][2], acc[m][3]);
      dst[1] = make_float4(acc[m][4], acc[m][5], acc[m][6], acc[m][7]);
    }
    named_bar_sync(1, kConsumerWarps * 32);
    const int t = threadIdx.x;  // 0..255: one column each
    float v[M];
#pragma unroll
    for (int m = 0; m < M; ++m) {
      float x = 0.f;
#pragma unroll
      for (int wp = 0; wp < kConsumerWarps; ++wp) x += red[(size_t(wp) * M + m) * kTileV + t];
      v[m] = x;
    }
    bool fold = whole;
    if (!whole) {
      // A unit cut by the range: the part holding stage 0 sits at the end of
      // one CTA's range (its slot 1), the rest at the start of the next CTA's
      // (its slot 0). Each writes its partial logits; the second to finish
      // adds first part + second part, in that order, and folds the unit.
      const bool head_part = s_lo == 0;
      float* mine = a.spart + ((size_t(blockIdx.x) * 2 + (head_part ? 1 : 0)) * M) * kTileV;
#pragma unroll
      for (int m = 0; m < M; ++m) mine[m * kTileV + t] = v[m];
      __threadfence();
      named_bar_sync(1, kConsumerWarps * 32);
      if (t == 0) s_ticket = int(epoch_arrive(&a.tickets[unit], a.epoch));
      named_bar_sync(1, kConsumerWarps * 32);
      fold = s_ticket == 1;
      if (fold) {
        __threadfence();
        const float* other = a.spart + ((size_t(blockIdx.x + (head_part ? 1 : -1)) * 2 + (head_part ? 0 : 1)) * M) *
                                           kTileV;
#pragma unroll
        for (int m = 0; m < M; ++m) {
          const float o = __ldcg(other + m * kTileV + t);
          v[m] = head_part ? v[m] + o : o + v[m];
        }
      }
    }
    if (fold) {
      const int col = tile * kTileV + t;
#pragma unroll
      for (int m = 0; m < M; ++m) {
        if (col < a.V) {
          const size_t idx = (size_t(m) * a.K + k) * a.V + col;
          if (a.logits_dbg) a.logits_dbg[idx] = v[m];
          // sampled drafts rank the Gumbel keys logit / tau - ln(-ln u) instead
          lg[m * kTileV + t] = a.gumbel_u ? fmaf(v[m], a.inv_tau, gumbel_noise(__ldg(a.gumbel_u + idx))) : v[m];
        } else {
          lg[m * kTileV + t] = -INFINITY;
        }
      }
    }
    named_bar_sync(1, kConsumerWarps * 32);

    // Warp m folds the tile into its running top-k: k rounds, each taking the
    // best entry strictly after the previous winner in (value desc, id asc)
    // order among the tile's 256 logits and the running list.
    if (warp < M) {
      const int m = warp;
      const int kk = param_at(a.kph, a.shared ? m % a.kh : k);
      if (fold) {
        float vv[kTileV / 32];
        int id[kTileV / 32];
#pragma unroll
        for (int i = 0; i < kTileV / 32; ++i) {
          const int c = lane + 32 * i;
          vv[i] = lg[m * kTileV + c];
          id[i] = (tile * kTileV + c < a.V) ? tile * kTileV + c : INT_MAX;
        }
        float pv = INFINITY;
        int pid = -1;
        float nrv = -INFINITY;
        int nri = INT_MAX;
        for (int r = 0; r < kk; ++r) {
          float bv = -INFINITY;
          int bi = INT_MAX;
#pragma unroll
          for (int i = 0; i < kTileV / 32; ++i) {
            if (better(pv, pid, vv[i], id[i]) && better(vv[i], id[i], bv, bi)) {
              bv = vv[i];
              bi = id[i];
            }
          }
          if (better(pv, pid, rv, ri) && better(rv, ri, bv, bi)) {
            bv = rv;
            bi = ri;
          }
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
            const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
            if (better(ov, oi, bv, bi)) {
              bv = ov;
              bi = oi;
            }
          }
          if (lane == r) {
            nrv = bv;
            nri = bi;
          }
          pv = bv;
          pid = bi;
        }
        rv = nrv;
        ri = nri;
      }
      // flush the list when the range moves to another head (or ends): every
      // CTA whose range meets head k writes a list for it, empty or not
      if (w >= i1 || int(w / stages_per_unit) / a.ntiles != k) {
        if (lane < kk) {
          const size_t cb = ((size_t(m) * a.K + k) * gridDim.x + blockIdx.x) * a.kmax + lane;
          a.cand_val[cb] = rv;
          a.cand_id[cb] = (ri == INT_MAX) ? -1 : ri;
        }
        rv = -INFINITY;
        ri = INT_MAX;
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Phase 3: merge candidate lists into each head's top-k.
// grid (M * K), 256 threads. The candidates of (m, k) are `nslots` lists of
// up to kmax entries. In "partitioned" mode slot c is CTA c of the kernel that
// produced them (the CTAs that worked on row m): that kernel split `units`
// work units, ordered (head, column tile of `ntiles`), into contiguous CTA
// ranges, so the slots that hold a list for head k form one contiguous range
// [slot_lo[k], slot_hi[k]), which the host works out with the producer's own
// partition arithmetic (set_merge_ranges). Every list is sorted, so the
// head's top kk lie at or above two thresholds: the best of the lists' kk-th
// entries (each list holds kk entries at or above its own), and the kk-th
// best of the lists' first entries (kk distinct candidates reach it). Only
// entries at or above the stricter one are kept: a few more than kk, where
// the first threshold alone keeps hundreds when there are many lists. Each
// kept entry's position in the top-k order (value descending, then id
// ascending) is the number of kept entries ahead of it, counted in shared
// memory; an entry whose position is below kk writes itself there.
// ---------------------------------------------------------------------------
struct MergeArgs {
  const float* cand_val;
  const int* cand_id;
  int32_t* topk_ids;   // [M, K, kmax]
  float* topk_vals;
  int K, kmax, nslots;
  int partitioned, units, ntiles;   // producer partition (partitioned == 1)
  int stages;          // > 0: the producer cut units x stages items (stages per unit), not whole units
  int kh;              // heads for the top-k size: row mk uses kph[mk % kh]
  int kph[MD_MAX_K];
  int slot_lo[MD_MAX_K], slot_hi[MD_MAX_K];   // slots holding head k's lists (set_merge_ranges)
};

// The slot range of each head. Slot c covered the producer's items
// [c W / nslots, (c + 1) W / nslots) of W = units x stages (or whole units),
// in the same 64-bit arithmetic as the producer; head k owns the items
// [k ntiles S, (k + 1) ntiles S). Both ends are non-decreasing in c, so the
// slots touching head k are contiguous.
inline void set_merge_ranges(MergeArgs& a) {
  for (int k = 0; k < MD_MAX_K; ++k) {
    a.slot_lo[k] = 0;
    a.slot_hi[k] = 0;
  }
  const long long S = a.stages > 0 ? a.stages : 1;
  const long long W = (long long)a.units * S;
  for (int k = 0; k < a.K && k < MD_MAX_K; ++k) {
    if (!a.partitioned) {
      a.slot_hi[k] = a.nslots;
      continue;
    }
    int lo = a.nslots, hi = 0;
    for (int c = 0; c < a.nslots; ++c) {
      const long long w0 = a.stages > 0 ? (long long)c * W / a.nslots : (long long)c * a.units / a.nslots;
      const long long w1 = a.stages > 0 ? (long long)(c + 1) * W / a.nslots : (long long)(c + 1) * a.units / a.nslots;
      if (w1 > (long long)k * a.ntiles * S && w0 < (long long)(k + 1) * a.ntiles * S) {
        lo = c < lo ? c : lo;
        hi = c + 1;
      }
    }
    a.slot_lo[k] = lo < hi ? lo : 0;
    a.slot_hi[k] = lo < hi ? hi : 0;
  }
}

constexpr int kMergeCap = 4096;          // candidates per (row, head): nslots * kmax <= kMergeCap
constexpr int kMergeThreads = 256;
constexpr int kMergeWarps = kMergeThreads / 32;
constexpr int kMergePer = kMergeCap / kMergeThreads;   // candidates per thread
static_assert(kMergePer * kMergeWarps == 4 * 32, "the count scan gives each lane four counts");

__global__ void __launch_bounds__(kMergeThreads) heads_merge_kernel(MergeArgs a) {
  pdl_wait_primary();          // candidates come from the previous kernel (no-op in plain stream order)
  pdl_launch_dependents();
  __shared__ float sv[kMergeCap];
  __shared__ int si[kMergeCap];
  __shared__ int pass_cnt[kMergePer * kMergeWarps];   // [pass][warp]: kept counts, then offsets
  __shared__ float red_v[kMergeWarps];
  __shared__ int red_i[kMergeWarps];
  __shared__ int n_keep;
  __shared__ float head_v[kMergeThreads];      // each list's first entry
  __shared__ int head_i[kMergeThreads];
  __shared__ float first_v;                    // the kk-th best of them
  __shared__ int first_i;
  const int mk = blockIdx.x;
  const int k = mk % a.K;
  const int kk = param_at(a.kph, mk % a.kh);
  const int lo = param_at(a.slot_lo, k), hi = param_at(a.slot_hi, k);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const size_t base = (size_t(mk) * a.nslots + lo) * a.kmax;
  const int n = (hi - lo) * kk;        // candidates: the first kk entries of each list

  // 1. every candidate this thread owns (e = pass * threads + thread) is
  // loaded at once. Its list is e / kk, taken as floor((e + 1/2) / kk) in
  // fp32: the quotient sits at least 1/(2 kk) >= 1/32 from an integer and
  // its rounding error is below 4096 x 2^-23, so the floor is exact.
  const float rkk = 1.0f / float(kk);
  float cv[kMergePer];
  int ci[kMergePer];
  int lr[kMergePer];     // the candidate's place in its list (-1: none)
  int li[kMergePer];     // its list
#pragma unroll
  for (int q = 0; q < kMergePer; ++q) {
    const int e = q * kMergeThreads + threadIdx.x;
    cv[q] = -INFINITY;
    ci[q] = -1;
    lr[q] = -1;
    li[q] = 0;
    if (e < n) {
      const int l = __float2int_rd((float(e) + 0.5f) * rkk);
      const int r = e - l * kk;
      const size_t at = base + size_t(l) * a.kmax + r;
      ci[q] = a.cand_id[at];
      cv[q] = a.cand_val[at];
      lr[q] = r;
      li[q] = l;
    }
  }

  // 2. the threshold, the stricter of two that no member of the head's top
  // kk falls below: (a) the best of the lists' kk-th entries (each list holds
  // kk entries at or above its own kk-th); (b) the kk-th best of the lists'
  // first entries (kk distinct candidates reach it). With many lists (a)
  // alone keeps hundreds of entries, (b) a few more than kk.
  const int n_lists = hi - lo;
  const bool use_first = n_lists <= kMergeThreads;
  if (threadIdx.x == 0) {
    first_v = -INFINITY;
    first_i = INT_MAX;
  }
  {
    float bv = -INFINITY;
    int bi = INT_MAX;
#pragma unroll
    for (int q = 0; q < kMergePer; ++q) {
      if (lr[q] == kk - 1 && ci[q] >= 0 && better(cv[q], ci[q], bv, bi)) {
        bv = cv[q];
        bi = ci[q];
      }
      if (lr[q] == 0 && use_first) {
        head_v[li[q]] = ci[q] >= 0 ? cv[q] : -INFINITY;
        head_i[li[q]] = ci[q] >= 0 ? ci[q] : INT_MAX;
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
      if (better(ov, oi, bv, bi)) {
        bv = ov;
        bi = oi;
      }
    }
    if (lane == 0) {
      red_v[warp] = bv;
      red_i[warp] = bi;
    }
  }
  __syncthreads();
  float tv = red_v[0];
  int ti = red_i[0];
#pragma unroll
  for (int w = 1; w < kMergeWarps; ++w)
    if (better(red_v[w], red_i[w], tv, ti)) {
      tv = red_v[w];
      ti = red_i[w];
    }
  // (b): list l's first entry is the kk-th best of the first entries when
  // exactly kk - 1 of them are ahead of it (an identical pair counts as
  // ahead when its list comes first, so the places are a permutation)
  if (use_first && threadIdx.x < n_lists && head_i[threadIdx.x] != INT_MAX) {
    const int t = threadIdx.x;
    const float v = head_v[t];
    const int x = head_i[t];
    int place = 0;
#pragma unroll 4
    for (int j = 0; j < n_lists; ++j) {
      const float vj = head_v[j];
      const int xj = head_i[j];
      place += (better(vj, xj, v, x) || (vj == v && xj == x && j < t)) ? 1 : 0;
    }
    if (place == kk - 1) {
      first_v = v;
      first_i = x;
    }
  }
  __syncthreads();
  if (better(first_v, first_i, tv, ti)) {
    tv = first_v;
    ti = first_i;
  }

  // 3. keep the entries at or above the threshold: per-pass ballots, one
  // exclusive scan of the (pass, warp) counts by warp 0, then each kept
  // entry stores itself at its offset (the candidates' order)
  unsigned bal[kMergePer];
#pragma unroll
  for (int q = 0; q < kMergePer; ++q) {
    const bool keep = ci[q] >= 0 && (better(cv[q], ci[q], tv, ti) || (cv[q] == tv && ci[q] == ti));
    bal[q] = __ballot_sync(0xffffffffu, keep);
    if (lane == 0) pass_cnt[q * kMergeWarps + warp] = __popc(bal[q]);
  }
  __syncthreads();
  if (warp == 0) {
    int c[4], s = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      c[j] = pass_cnt[4 * lane + j];
      s += c[j];
    }
    int incl = s;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    int run = incl - s;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      pass_cnt[4 * lane + j] = run;
      run += c[j];
    }
    if (lane == 31) n_keep = incl;
  }
  __syncthreads();
  const unsigned below = (1u << lane) - 1u;
#pragma unroll
  for (int q = 0; q < kMergePer; ++q)
    if ((bal[q] >> lane) & 1u) {
      const int at = pass_cnt[q * kMergeWarps + warp] + __popc(bal[q] & below);
      sv[at] = cv[q];
      si[at] = ci[q];
    }
  const int nk = n_keep;
  __syncthreads();

  // 4. each kept entry's place is the number of kept entries ahead of it in
  // the top-k order (an identical pair counts as ahead when it was stored
  // earlier, so the places are a permutation). Sorted lists keep at most
  // kk^2 <= 256 entries, one per thread: only the kk lists whose first entry
  // reaches the threshold can hold an entry that does (or fewer than kk
  // lists hold any); the loop covers any count all the same.
  for (int t = threadIdx.x; t < nk; t += kMergeThreads) {
    const float v = sv[t];
    const int x = si[t];
    int place = 0;
#pragma unroll 4
    for (int j = 0; j < nk; ++j) {
      const float vj = sv[j];
      const int xj = si[j];
      place += (better(vj, xj, v, x) || (vj == v && xj == x && j < t)) ? 1 : 0;
    }
    if (place < kk) {
      a.topk_vals[size_t(mk) * a.kmax + place] = v;
      a.topk_ids[size_t(mk) * a.kmax + place] = x;
    }
  }
  const int filled = nk < kk ? nk : kk;      // the rest of the kmax slots are empty
  if (threadIdx.x >= filled && threadIdx.x < a.kmax) {
    a.topk_vals[size_t(mk) * a.kmax + threadIdx.x] = -INFINITY;
    a.topk_ids[size_t(mk) * a.kmax + threadIdx.x] = -1;
  }
}

}  // namespace heads
}  // namespace md
