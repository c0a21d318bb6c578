// Medusa draft heads on the tensor cores (tcgen05), for many hidden rows.
//
// Source: "Medusa heads versus separate draft model", sections "What each one
// is" and "Cost per step" (the same head computation as heads.cuh). Once the
// heads run on many rows at once -- every tree node of a batch of requests,
// e.g. 8 x 65 = 520 rows -- the projection stops being a weight stream and
// becomes a dense GEMM (the page's tree paragraph: past the ridge point the
// verification width turns the step compute-bound). Both phases then run as
// one persistent tcgen05 GEMM each:
//
//   phase 1  D = h   . W1_k   (M x d x d)   epilogue: z = bf16(h + SiLU(D + b1))
//   phase 2  D = z_k . Wv_k   (M x d x V)   epilogue: per-row top-k of the tile
//
// CTA tile 128 x 256 (UMMA M = 128, N = 256, K = 16 per instruction), 64-deep
// K stages of A (16 KB, K-major) and B (4 x 8 KB, N-major, straight from the
// input-major weights) brought in by TMA with 128-byte swizzle. Warp 0 feeds
// TMA, one thread of warp 1 issues tcgen05.mma into one of two 128 x 256 fp32
// accumulators in tensor memory (512 columns), warps 2..5 drain the other
// accumulator through tcgen05.ld (one TMEM lane = one row per thread).
//
// Work split: the grid is mtiles groups of per_mt CTAs, group g takes row
// tile g, and CTA j of every group takes the same contiguous range
// [j*U/per_mt, (j+1)*U/per_mt) of the U = K * ntiles (head, column tile)
// units, so the CTAs that share a weight strip read it at about the same time
// and the strips in flight at any moment number per_mt. (Contiguous ranges
// over all tiles put the CTAs of different row tiles on different strips and
// measured 5x the weight bytes from HBM at 520 rows.) The launcher uses this
// kernel up to 128 rows (one row tile); beyond that the CTA-pair kernel of
// heads_gemm2.cuh. In phase 2 each row keeps one running top-k across the
// CTA's column tiles: after the first tiles nearly every logit is rejected by
// one compare against the current k-th best.
#pragma once

#include "common.cuh"

namespace md {
namespace gemm {

constexpr int kBM = 128, kBN = 256, kBK = 64;
constexpr int kStages = 4;
constexpr uint32_t kABytes = kBM * kBK * 2;     // 16 KB
constexpr uint32_t kBBox = kBK * 64 * 2;        // 8 KB: 64 k-rows x 64 n-columns
constexpr uint32_t kBBytes = 4 * kBBox;         // 32 KB
constexpr uint32_t kStageBytes = kABytes + kBBytes;
constexpr int kThreads = 192;
constexpr int kSmem = kStages * kStageBytes + 1024 + 256 + MD_MAX_KMAX * 128 * 8;   // + running lists
constexpr uint32_t kTmemCols = 512;
constexpr int kMaxM = 4096;

enum { EPI_SILU = 0, EPI_TOPK = 1 };

struct Args {
  int M, d, N, K;                 // rows, reduction length, output columns, heads
  int ntiles;                     // column tiles per head
  int per_mt;                     // CTAs (pairs) per row tile (pair) group
  int groups;                     // CTA-pair kernel: row-pair groups (grid = 2 x groups x per_mt)
  int a_shared;                   // A is one matrix for every head (phase 1: h)
  const uint16_t* h;              // [M, d]      phase 1 residual
  const uint16_t* b1;             // [K, d]      phase 1 bias
  uint16_t* zg;                   // [K, M, d]   phase 1 output
  float* cand_val;                // [M, K, per_mt, kmax]  phase 2: one list per (row, head, CTA of the row tile)
  int* cand_id;
  float* logits_dbg;              // [M, K, N] or null
  const float* gumbel_u;          // phase 2: [M, K, N] uniforms (sampled drafts) or null
  float inv_tau;                  // phase 2: 1 / draft temperature (sampled drafts)
  int kmax;
  int zg_mk;                      // phase 1: write z rows in (row, head) order [M*K, d]
  int kh;                         // phase 2: row m uses kph[m % kh] when K == 1 (shared projection)
  int kph[MD_MAX_K];
};

// Running top-k of one row in shared memory: entry j of thread t at
// [j * 128 + t] (conflict-free across a warp); sorted, best first.
struct SmemList {
  float* v;
  int* i;
  int kk;
  float tv;   // the current k-th best (the admission threshold)
  int ti;
  __device__ __forceinline__ void reset() {
    for (int j = 0; j < kk; ++j) {
      v[j * 128] = -INFINITY;
      i[j * 128] = INT_MAX;
    }
    tv = -INFINITY;
    ti = INT_MAX;
  }
  __device__ __forceinline__ void insert(float x, int id) {
    int pos = kk - 1;
    while (pos > 0 && better(x, id, v[(pos - 1) * 128], i[(pos - 1) * 128])) {
      v[pos * 128] = v[(pos - 1) * 128];
      i[pos * 128] = i[(pos - 1) * 128];
      --pos;
    }
    v[pos * 128] = x;
    i[pos * 128] = id;
    tv = v[(kk - 1) * 128];
    ti = i[(kk - 1) * 128];
  }
};

// Phase-1 epilogue for 32 columns o0.. of row m, head k: z = bf16(h + SiLU(acc + b1)).
__device__ __forceinline__ void silu_residual_store(const Args& a, int m, int k, int o0, const float (&v)[32]) {
  const uint4* hp = reinterpret_cast<const uint4*>(a.h + size_t(m) * a.d + o0);
  const uint4* bp = reinterpret_cast<const uint4*>(a.b1 + size_t(k) * a.d + o0);
  uint4* zp = reinterpret_cast<uint4*>(a.zg + (a.zg_mk ? size_t(m) * a.K + k : size_t(k) * a.M + m) * a.d + o0);
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    const uint4 hv = hp[g], bv = __ldg(bp + g);
    const uint32_t hw[4] = {hv.x, hv.y, hv.z, hv.w};
    const uint32_t bw[4] = {bv.x, bv.y, bv.z, bv.w};
    uint32_t zw[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float u0 = v[g * 8 + 2 * e] + bf16lo(bw[e]);
      const float u1 = v[g * 8 + 2 * e + 1] + bf16hi(bw[e]);
      const uint16_t z0 = f32_to_bf16_rne(bf16lo(hw[e]) + u0 / (1.0f + expf(-u0)));
      const uint16_t z1 = f32_to_bf16_rne(bf16hi(hw[e]) + u1 / (1.0f + expf(-u1)));
      zw[e] = uint32_t(z0) | (uint32_t(z1) << 16);
    }
    zp[g] = make_uint4(zw[0], zw[1], zw[2], zw[3]);
  }
}

// Phase-2 epilogue for 32 logits of row m, head k, columns c0..: fold them
// into the running top-k (and copy them out when the debug logits are kept).
// Sampled drafts fold the Gumbel keys logit / tau - ln(-ln u) instead.
__device__ __forceinline__ void topk_tile_columns(const Args& a, SmemList& L, int m, int k, int c0,
                                                  const float (&v)[32]) {
  const size_t base = (size_t(m) * a.K + k) * a.N + c0;
  if (a.logits_dbg) {
    float* lp = a.logits_dbg + base;
#pragma unroll
    for (int j = 0; j < 32; j += 4)
      if (c0 + j < a.N) *reinterpret_cast<float4*>(lp + j) = make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
  }
  if (a.gumbel_u) {
#pragma unroll
    for (int j = 0; j < 32; j += 4) {
      if (c0 + j >= a.N) break;
      const float4 u = __ldg(reinterpret_cast<const float4*>(a.gumbel_u + base + j));
      const float key[4] = {fmaf(v[j], a.inv_tau, gumbel_noise(u.x)), fmaf(v[j + 1], a.inv_tau, gumbel_noise(u.y)),
                            fmaf(v[j + 2], a.inv_tau, gumbel_noise(u.z)), fmaf(v[j + 3], a.inv_tau, gumbel_noise(u.w))};
#pragma unroll
      for (int e = 0; e < 4; ++e)
        if (better(key[e], c0 + j + e, L.tv, L.ti)) L.insert(key[e], c0 + j + e);
    }
    return;
  }
#pragma unroll
  for (int j = 0; j < 32; ++j)
    if (c0 + j < a.N && better(v[j], c0 + j, L.tv, L.ti)) L.insert(v[j], c0 + j);
}

// Write a running list to candidate slot `slot` of (row m, head k).
__device__ __forceinline__ void flush_list(const Args& a, const SmemList& L, int m, int k, int slot) {
  const size_t cb = ((size_t(m) * a.K + k) * a.per_mt + slot) * a.kmax;
  for (int j = 0; j < L.kk; ++j) {
    a.cand_val[cb + j] = L.v[j * 128];
    a.cand_id[cb + j] = L.i[j * 128] == INT_MAX ? -1 : L.i[j * 128];
  }
}

template <int EPI, int KK>
__global__ void __launch_bounds__(kThreads, 1)
    heads_gemm_kernel(const __grid_constant__ CUtensorMap amap, const __grid_constant__ CUtensorMap bmap, Args a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes);
  uint64_t* empty = full + kStages;
  uint64_t* acc_full = empty + kStages;
  uint64_t* acc_empty = acc_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);
  float* lv = reinterpret_cast<float*>(smem + kStages * kStageBytes + 256);    // [kmax][128] running lists
  int* li = reinterpret_cast<int*>(lv + MD_MAX_KMAX * 128);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nk = a.d / kBK;
  const int mt = blockIdx.x / a.per_mt, cj = blockIdx.x % a.per_mt;
  const int units = a.K * a.ntiles;
  const int t_begin = int((long long)cj * units / a.per_mt);
  const int t_end = int((long long)(cj + 1) * units / a.per_mt);
  pdl_launch_dependents();

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&acc_full[b]), 1);
      mbar_init(smem_u32(&acc_empty[b]), 4);
    }
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------- TMA producer -------------------------------
    if (lane == 0) {
      prefetch_tensormap(&amap);
      prefetch_tensormap(&bmap);
      pdl_wait_primary();   // A may be the previous kernel's output
      const uint64_t pol = policy_evict_first();
      int it = 0;
      bool ok = true;
      for (int tile = t_begin; tile < t_end && ok; ++tile) {
        const int nt = tile % a.ntiles, k = tile / a.ntiles;
        for (int s = 0; s < nk; ++s, ++it) {
          const int slot = it % kStages;
          if (it >= kStages && !mbar_wait(smem_u32(&empty[slot]), ((it / kStages) - 1) & 1)) {
            set_status(MD_DEV_TIMEOUT);
            ok = false;
            break;
          }
          const uint32_t fb = smem_u32(&full[slot]);
          uint8_t* st = smem + size_t(slot) * kStageBytes;
          mbar_arrive_expect_tx(fb, kStageBytes);
          tma_load_3d(smem_u32(st), &amap, s * kBK, mt * kBM, a.a_shared ? 0 : k, fb);
          // A weight strip is read once per row tile: stream it evict-first only when
          // there is a single row tile, otherwise keep it in L2 for the other tiles.
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            if (gridDim.x == a.per_mt)
              tma_load_3d_hint(smem_u32(st + kABytes + j * kBBox), &bmap, nt * kBN + j * 64, s * kBK, k, fb, pol);
            else
              tma_load_3d(smem_u32(st + kABytes + j * kBBox), &bmap, nt * kBN + j * 64, s * kBK, k, fb);
          }
        }
      }
      for (int j = (it > kStages ? it - kStages : 0); j < it; ++j) {
        if (!mbar_wait(smem_u32(&empty[j % kStages]), (j / kStages) & 1)) {
          set_status(MD_DEV_TIMEOUT);
          break;
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------- MMA issuer ---------------------------------
    if (lane == 0) {
      constexpr uint32_t idesc = umma_idesc_bf16(kBM, kBN, 0, 1);
      int it = 0, lt = 0;
      bool ok = true;
      for (int tile = t_begin; tile < t_end && ok; ++tile, ++lt) {
        const int buf = lt & 1;
        if (lt >= 2 && !mbar_wait(smem_u32(&acc_empty[buf]), ((lt >> 1) - 1) & 1)) {
          set_status(MD_DEV_TIMEOUT);
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem + uint32_t(buf * kBN);
        for (int s = 0; s < nk; ++s, ++it) {
          const int slot = it % kStages;
          if (!mbar_wait(smem_u32(&full[slot]), (it / kStages) & 1)) {
            set_status(MD_DEV_TIMEOUT);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + size_t(slot) * kStageBytes);
          const uint64_t adesc = umma_desc_sw128(sa, 16, 1024);
          const uint64_t bdesc = umma_desc_sw128(sa + kABytes, kBBox, 1024);
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk)
            umma_f16(d_tmem, adesc + uint64_t((kk * 32) >> 4), bdesc + uint64_t((kk * 2048) >> 4), idesc,
                     (s | kk) != 0);
          umma_commit(smem_u32(&empty[slot]));
        }
        umma_commit(smem_u32(&acc_full[buf]));
      }
    }
  } else {
    // -------------------------------- epilogue ----------------------------------
    const int q = warp & 3;   // TMEM lanes 32q .. 32q+31 belong to this warp
    const int row = q * 32 + lane;
    SmemList L;
    L.v = lv + row;
    L.i = li + row;
    int lt = 0;
    int cur_k = -1;
    for (int tile = t_begin; tile < t_end; ++tile, ++lt) {
      const int nt = tile % a.ntiles, k = tile / a.ntiles;
      const int buf = lt & 1;
      if (!mbar_wait(smem_u32(&acc_full[buf]), (lt >> 1) & 1)) {
        set_status(MD_DEV_TIMEOUT);
        break;
      }
      tc_fence_after();
      const int m = mt * kBM + row;
      const bool live = m < a.M;
      const uint32_t tbase = tmem + (uint32_t(q * 32) << 16) + uint32_t(buf * kBN);
      if constexpr (EPI == EPI_SILU) {
        for (int c = 0; c < kBN; c += 32) {
          float v[32];
          tmem_ld32(tbase + c, v);
          const int o0 = nt * kBN + c;
          if (live && o0 < a.d) silu_residual_store(a, m, k, o0, v);
        }
      } else {
        if (k != cur_k) {         // a new head starts: fresh lists
          L.kk = param_at(a.kph, a.kh > 0 ? m % a.kh : k);
          L.reset();
          cur_k = k;
        }
        for (int c = 0; c < kBN; c += 32) {
          float v[32];
          tmem_ld32(tbase + c, v);
          const int c0 = nt * kBN + c;
          if (live) topk_tile_columns(a, L, m, k, c0, v);
        }
        // flush at the end of the CTA's run of this head
        const bool last = tile + 1 == t_end || (tile + 1) / a.ntiles != tile / a.ntiles;
        if (last) {
          if (live) flush_list(a, L, m, k, cj);
          cur_k = -1;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&acc_empty[buf]));
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace gemm
}  // namespace md
