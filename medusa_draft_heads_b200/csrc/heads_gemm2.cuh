// Medusa draft heads on CTA pairs (tcgen05.mma cta_group::2), for many rows.
//
// Source: "Medusa heads versus separate draft model", sections "What each one
// is" and "Cost per step" -- the same two GEMM phases as heads_gemm.cuh
// (z = bf16(h + SiLU(h W1_k + b1_k)), then logits = z_k Wv_k with a per-row
// top-k in the epilogue), for M > 128 rows.
//
// Why pairs: with one SM per 128 x 256 tile, every 64-deep K step moves 48 KB
// into shared memory (16 KB of rows, 32 KB of weights) for 4.2 MFLOP, and four
// such stages are all that fit: at the L2 latency of a weight strip that is
// being read by CTAs on both dies the tensor pipe starves. A CTA pair on the
// two SMs of a TPC computes a 256 x 256 tile with one instruction stream: each
// CTA loads its own 128 rows and HALF of the weight columns (16 + 16 KB per
// stage), and the pair MMA reads the other half from the partner's shared
// memory. Per SM that is 2/3 of the bytes per FLOP and six stages in flight.
//
// Roles (192 threads per CTA): warp 0 issues TMA in both CTAs, each CTA's
// loads completing on the LEADER's full barrier; one thread of the
// leader's warp 1 issues the pair MMAs and commits to the empty / accumulator
// barriers of both CTAs; warps 2..5 of each CTA drain that CTA's 128 rows of
// the accumulator from its own TMEM and arrive on the leader's accumulator-
// empty barrier (4 warps x 2 CTAs).
//
// Work split: as in heads_gemm.cuh, but per row PAIR: the grid is `groups`
// row-pair tiles x per_mt pairs, pair j of every group taking the same
// contiguous range of the K * ntiles (head, column tile) units, so the pairs
// sharing a weight strip read it at about the same time. Block order is (j,
// group, CTA of the pair). The kernel works in clusters of any even size (the
// pair partner is the CTA whose cluster rank differs in bit 0; the even one
// leads); the launcher uses clusters of two.
#pragma once

#include "heads_gemm.cuh"

namespace md {
namespace gemm {

constexpr int kStagesP = 6;
constexpr uint32_t kBHalfBytes = 2 * kBBox;                    // 16 KB: 64 k-rows x 128 columns
constexpr uint32_t kStagePBytes = kABytes + kBHalfBytes;       // 32 KB per CTA
constexpr int kSmemP = kStagesP * kStagePBytes + 1024 + 256 + MD_MAX_KMAX * 128 * 8;

template <int EPI, int KK>
__global__ void __launch_bounds__(kThreads, 1)
    heads_gemm_pair_kernel(const __grid_constant__ CUtensorMap amap, const __grid_constant__ CUtensorMap bmap,
                           Args a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStagesP * kStagePBytes);
  uint64_t* empty = full + kStagesP;
  uint64_t* acc_full = empty + kStagesP;
  uint64_t* acc_empty = acc_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);
  float* lv = reinterpret_cast<float*>(smem + kStagesP * kStagePBytes + 256);    // [kmax][128] running lists
  int* li = reinterpret_cast<int*>(lv + MD_MAX_KMAX * 128);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t crank = cluster_ctarank();
  const uint32_t lead = crank & ~1u;            // cluster rank of the pair's leader (issues the MMAs)
  const uint32_t rank = crank & 1u;             // 0: leader, 1: partner
  const uint16_t pair_mask = uint16_t(3u << lead);
  const int nk = a.d / kBK;
  const int pair = blockIdx.x >> 1;
  const int mp = pair % a.groups, cj = pair / a.groups;
  const int mt = mp * 2 + int(rank);           // this CTA's 128-row tile
  const int units = a.K * a.ntiles;
  const int t_begin = int((long long)cj * units / a.per_mt);
  const int t_end = int((long long)(cj + 1) * units / a.per_mt);
  pdl_launch_dependents();

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStagesP; ++s) {
      mbar_init(smem_u32(&full[s]), 1);       // the leader's arrive + both CTAs' bytes
      mbar_init(smem_u32(&empty[s]), 1);      // the leader's MMA commit
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&acc_full[b]), 1);
      mbar_init(smem_u32(&acc_empty[b]), 8);  // 4 epilogue warps in each CTA
    }
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncwarp();
  cluster_sync();      // barriers of both CTAs initialised, TMEM allocated in both
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------- TMA producer -------------------------------
    if (lane == 0) {
      prefetch_tensormap(&amap);
      prefetch_tensormap(&bmap);
      pdl_wait_primary();   // A may be the previous kernel's output
      const uint32_t full_lead = mapa_shared(smem_u32(&full[0]), lead);
      // the row tiles (M x d per head, re-read for every column tile) stay in L2
      const uint64_t keep = policy_evict_last();
      int it = 0;
      bool ok = true;
      for (int tile = t_begin; tile < t_end && ok; ++tile) {
        const int nt = tile % a.ntiles, k = tile / a.ntiles;
        for (int s = 0; s < nk; ++s, ++it) {
          const int slot = it % kStagesP;
          if (it >= kStagesP && !mbar_wait(smem_u32(&empty[slot]), ((it / kStagesP) - 1) & 1)) {
            set_status(MD_DEV_TIMEOUT);
            ok = false;
            break;
          }
          const uint32_t fb = full_lead + uint32_t(slot) * 8;
          uint8_t* st = smem + size_t(slot) * kStagePBytes;
          if (rank == 0) mbar_arrive_expect_tx(smem_u32(&full[slot]), 2 * kStagePBytes);
          tma_load_3d_pair_hint(smem_u32(st), &amap, s * kBK, mt * kBM, a.a_shared ? 0 : k, fb, keep);
#pragma unroll
          for (int j = 0; j < 2; ++j)
            tma_load_3d_pair(smem_u32(st + kABytes + j * kBBox), &bmap, nt * kBN + int(rank) * 128 + j * 64,
                             s * kBK, k, fb);
        }
      }
      // the partner's MMAs read this CTA's stages: wait until the last ones are consumed
      for (int j = (it > kStagesP ? it - kStagesP : 0); j < it; ++j) {
        if (!mbar_wait(smem_u32(&empty[j % kStagesP]), (j / kStagesP) & 1)) {
          set_status(MD_DEV_TIMEOUT);
          break;
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------- MMA issuer (leader only) -------------------------
    if (lane == 0 && rank == 0) {
      constexpr uint32_t idesc = umma_idesc_bf16(2 * kBM, kBN, 0, 1);
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
          const int slot = it % kStagesP;
          if (!mbar_wait(smem_u32(&full[slot]), (it / kStagesP) & 1)) {
            set_status(MD_DEV_TIMEOUT);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + size_t(slot) * kStagePBytes);
          const uint64_t adesc = umma_desc_sw128(sa, 16, 1024);
          const uint64_t bdesc = umma_desc_sw128(sa + kABytes, kBBox, 1024);
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk)
            umma_f16_pair(d_tmem, adesc + uint64_t((kk * 32) >> 4), bdesc + uint64_t((kk * 2048) >> 4), idesc,
                          (s | kk) != 0);
          umma_commit_pair(smem_u32(&empty[slot]), pair_mask);
        }
        umma_commit_pair(smem_u32(&acc_full[buf]), pair_mask);
      }
    }
  } else {
    // -------------------------------- epilogue ----------------------------------
    const int q = warp & 3;   // TMEM lanes 32q .. 32q+31 belong to this warp
    const int row = q * 32 + lane;
    const uint32_t acc_empty_lead = mapa_shared(smem_u32(&acc_empty[0]), lead);
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
      if (lane == 0) {
        if (rank == 0)
          mbar_arrive(smem_u32(&acc_empty[buf]));
        else
          mbar_arrive_cluster(acc_empty_lead + uint32_t(buf) * 8);
      }
    }
  }
  tc_fence_before();
  __syncwarp();
  cluster_sync();      // every pair MMA has completed and no CTA signals the other any more
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, kTmemCols);
  }
}

}  // namespace gemm
}  // namespace md
