// Tree-masked attention on the tensor cores (tcgen05).
//
// Source: "Medusa heads versus separate draft model", section "Acceptance",
// tree paragraph: every branch is verified in one target pass with a tree
// attention mask. With grouped-query attention every KV head serves
// T x (Hq/Hkv) query rows (65 x 8 = 520 for the 70B tree), so the scores and
// the weighted sum are dense products: S = Q K^T and O += P V run on tcgen05.
//
// CTA = (KV split, 128-row query tile, KV head, request); the grid is sized to
// one wave. The 128 query rows are (tree token, query head of the group) pairs,
// loaded by one 3-D TMA box straight out of q[B, T, Hq, dh]. The CTA walks its
// share of 128-key chunks:
//
//   warp 0     TMA: the Q tile once, then K and V chunks into two 2-deep rings
//              (a K slot frees when its S is done, a V slot when its P V is)
//   warp 1     one thread issues S_c = Q K_c^T into TMEM (double-buffered, two
//              chunks ahead) and O += P_c V_c into one TMEM accumulator that
//              lives across chunks
//   warps 2-9  two warps per TMEM lane quarter, each taking half of the keys of
//              a row (row maxima are exchanged through shared memory): read
//              S_c from TMEM, apply the scale
//              and -- only in chunks that reach the tree slots -- the tree
//              mask (a key at slot >= P_b is tree node slot - P_b, visible iff
//              it is an ancestor-or-self), then P_c = exp2(S - m) against a
//              running row maximum m, split into bf16 hi + lo parts in
//              swizzled shared memory (P V runs as P_hi V + P_lo V, keeping
//              ~16 significant bits of each weight). m only moves when a chunk
//              exceeds it by more than 2^8; O and the row sum are then rescaled
//              in place.
//
// Each CTA writes its split's (m, sum, unnormalised O) per row; the last CTA of
// a (request, KV head, row tile) to finish combines the splits in split order
// and writes the output rows.
#pragma once

#include "common.cuh"

namespace md {
namespace attn_tc {

constexpr int kBM = 128;        // query rows per CTA
constexpr int kBN = 128;        // keys per chunk
constexpr int kSoftWarps = 8;
constexpr int kThreads = 64 + kSoftWarps * 32;
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleLog2 = 8.0f;   // lazy rescale threshold (factor 256)
constexpr int kMaxSplits = 16;

template <int DH>
struct Cfg {
  static constexpr int KB = DH / 64;                          // 64-element blocks of the head dim
  static constexpr uint32_t kQBytes = KB * kBM * 128;         // Q tile, K-major SW128
  static constexpr uint32_t kKBytes = KB * kBN * 128;         // K chunk, K-major SW128
  static constexpr uint32_t kVBytes = KB * kBN * 128;         // V chunk, N(dh)-major SW128
  static constexpr uint32_t kStage = kKBytes + kVBytes;
  static constexpr uint32_t kPBytes = 2 * kBM * 128;          // P tile: 128 rows x 128 keys bf16
  static constexpr int kSmem = kQBytes + 2 * kStage + 2 * kPBytes + 1024 + 256 + 1024;  // P hi/lo, maxima
};

struct Args {
  const int32_t* prefix_len;  // [B]
  float* part_o;              // [B, Hkv, rtiles, splits, 128, dh]
  float2* part_ml;            // [B, Hkv, rtiles, splits, 128]   (max, sum) in log2 units
  int* counters;              // [B, Hkv, rtiles], zero before the launch
  float* out;                 // [B, T, Hq, dh]
  int B, S_max, Hq, Hkv, G, R, rtiles, splits, chunks_per_split;
  float scale_log2;
};

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ bool tree_visible(const TreeParams& tp, int t, int node) {
  return (tp.anc[t][node >> 5] >> (node & 31)) & 1u;
}

template <int DH>
__global__ void __launch_bounds__(kThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
                   const __grid_constant__ CUtensorMap vmap, const __grid_constant__ TreeParams tp, Args a) {
  using C = Cfg<DH>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint8_t* sQ = smem;
  uint8_t* sKV = smem + C::kQBytes;                     // 2 stages of (K, V)
  uint8_t* sP = sKV + 2 * C::kStage;                    // P hi
  uint8_t* sPl = sP + C::kPBytes;                       // P lo
  uint64_t* bars = reinterpret_cast<uint64_t*>(sPl + C::kPBytes);
  uint64_t* q_full = bars;            // 1
  uint64_t* k_full = bars + 1;        // 2
  uint64_t* k_empty = bars + 3;       // 2
  uint64_t* v_full = bars + 5;        // 2
  uint64_t* v_empty = bars + 7;       // 2
  uint64_t* s_full = bars + 9;        // 2
  uint64_t* s_empty = bars + 11;      // 2
  uint64_t* p_full = bars + 13;       // 1
  uint64_t* o_full = bars + 14;       // 1
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 15);
  int* last_flag = reinterpret_cast<int*>(bars + 16);
  float* xmax = reinterpret_cast<float*>(bars + 17);    // [2 halves][128 rows] chunk maxima

  const int split = blockIdx.x, rt = blockIdx.y % a.rtiles, hk = blockIdx.y / a.rtiles, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int T = tp.T;
  pdl_wait_primary();          // inputs may come from earlier kernels
  pdl_launch_dependents();
  const int P = a.prefix_len[b];
  const bool bad = P < 0 || P + T > a.S_max;
  const int nkeys = bad ? 0 : P + T;
  const int nch_total = (nkeys + kBN - 1) / kBN;
  const int c_begin = split * a.chunks_per_split;
  const int c_end = min(nch_total, c_begin + a.chunks_per_split);
  const int nch = max(0, c_end - c_begin);
  if (bad && split == 0 && blockIdx.y == 0 && threadIdx.x == 0) set_status(MD_DEV_BAD_PREFIX);

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(q_full), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&k_full[i]), 1);
      mbar_init(smem_u32(&k_empty[i]), 1);
      mbar_init(smem_u32(&v_full[i]), 1);
      mbar_init(smem_u32(&v_empty[i]), 1);
      mbar_init(smem_u32(&s_full[i]), 1);
      mbar_init(smem_u32(&s_empty[i]), kSoftWarps);
    }
    mbar_init(smem_u32(p_full), kSoftWarps);
    mbar_init(smem_u32(o_full), 1);
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
  const uint32_t tS = tmem;                 // S_c at columns [128*(c&1), +128)
  const uint32_t tO = tmem + 2 * kBN;       // O at columns [256, 256 + DH)
  const int kvrow = b * a.Hkv + hk;
  const int tpt = kBM / a.G;                // tree tokens per query tile

  if (warp == 0) {
    // ---------------------------------- TMA ----------------------------------
    if (lane == 0 && nch > 0) {
      prefetch_tensormap(&qmap);
      prefetch_tensormap(&kmap);
      prefetch_tensormap(&vmap);
      const uint32_t qb = smem_u32(q_full);
      mbar_arrive_expect_tx(qb, C::kQBytes);
#pragma unroll
      for (int kb = 0; kb < C::KB; ++kb)
        tma_load_3d(smem_u32(sQ + kb * kBM * 128), &qmap, kb * 64, hk * a.G, b * T + rt * tpt, qb);
      bool ok = true;
      for (int c = 0; c < nch && ok; ++c) {
        const int st = c & 1;
        const int key0 = (c_begin + c) * kBN;
        uint8_t* sk = sKV + st * C::kStage;
        uint8_t* sv = sk + C::kKBytes;
        if (c >= 2 && !mbar_wait(smem_u32(&k_empty[st]), ((c >> 1) - 1) & 1)) { ok = false; break; }
        const uint32_t kb_ = smem_u32(&k_full[st]);
        mbar_arrive_expect_tx(kb_, C::kKBytes);
#pragma unroll
        for (int kb = 0; kb < C::KB; ++kb) tma_load_3d(smem_u32(sk + kb * kBN * 128), &kmap, kb * 64, key0, kvrow, kb_);
        if (c >= 2 && !mbar_wait(smem_u32(&v_empty[st]), ((c >> 1) - 1) & 1)) { ok = false; break; }
        const uint32_t vb_ = smem_u32(&v_full[st]);
        mbar_arrive_expect_tx(vb_, C::kVBytes);
#pragma unroll
        for (int kb = 0; kb < C::KB; ++kb) tma_load_3d(smem_u32(sv + kb * kBN * 128), &vmap, kb * 64, key0, kvrow, vb_);
      }
      // drain: every issued copy has been consumed before the CTA can exit
      for (int c = max(0, nch - 2); c < nch && ok; ++c) {
        if (!mbar_wait(smem_u32(&k_empty[c & 1]), (c >> 1) & 1) ||
            !mbar_wait(smem_u32(&v_empty[c & 1]), (c >> 1) & 1))
          ok = false;
      }
      if (!ok) set_status(MD_DEV_TIMEOUT);
    }
  } else if (warp == 1) {
    // ---------------------------------- MMA ----------------------------------
    if (lane == 0 && nch > 0) {
      constexpr uint32_t idesc_s = umma_idesc_bf16(kBM, kBN, 0, 0);
      constexpr uint32_t idesc_o = umma_idesc_bf16(kBM, DH, 0, 1);
      bool ok = mbar_wait(smem_u32(q_full), 0);
      const uint32_t aq = smem_u32(sQ);
      // S_c = Q K_c^T into TMEM buffer c & 1; frees K slot c & 1 when done
      auto issue_s = [&](int c) -> bool {
        const int st = c & 1;
        if (!mbar_wait(smem_u32(&k_full[st]), (c >> 1) & 1)) return false;
        if (c >= 2 && !mbar_wait(smem_u32(&s_empty[st]), ((c >> 1) - 1) & 1)) return false;
        tc_fence_after();
        const uint32_t sk = smem_u32(sKV + st * C::kStage);
        const uint32_t d = tS + uint32_t(st * kBN);
#pragma unroll
        for (int kb = 0; kb < C::KB; ++kb) {
          const uint64_t ad = umma_desc_sw128(aq + kb * kBM * 128, 16, 1024);
          const uint64_t bd = umma_desc_sw128(sk + kb * kBN * 128, 16, 1024);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_f16(d, ad + uint64_t((kk * 32) >> 4), bd + uint64_t((kk * 32) >> 4), idesc_s, (kb | kk) != 0);
        }
        umma_commit(smem_u32(&s_full[st]));
        umma_commit(smem_u32(&k_empty[st]));
        return true;
      };
      if (ok) ok = issue_s(0);
      if (ok && nch > 1) ok = issue_s(1);
      for (int c = 0; c < nch && ok; ++c) {
        // O += P_c V_c (hi and lo parts); frees V slot c & 1 and P when done
        if (!mbar_wait(smem_u32(p_full), c & 1) || !mbar_wait(smem_u32(&v_full[c & 1]), (c >> 1) & 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t sv = smem_u32(sKV + (c & 1) * C::kStage + C::kKBytes);
#pragma unroll
        for (int part = 0; part < 2; ++part) {
          const uint32_t sp = smem_u32(part == 0 ? sP : sPl);
#pragma unroll
          for (int kk = 0; kk < kBN / 16; ++kk) {
            const uint64_t ad =
                umma_desc_sw128(sp + (kk >> 2) * kBM * 128, 16, 1024) + uint64_t(((kk & 3) * 32) >> 4);
            const uint64_t bd = umma_desc_sw128(sv, kBN * 128, 1024) + uint64_t((kk * 2048) >> 4);
            umma_f16(tO, ad, bd, idesc_o, (c | part | kk) != 0);
          }
        }
        umma_commit(smem_u32(o_full));
        umma_commit(smem_u32(&v_empty[c & 1]));
        if (c + 2 < nch) ok = issue_s(c + 2);
      }
      if (!ok) set_status(MD_DEV_TIMEOUT);
    }
  } else {
    // ------------------------------- softmax rows -------------------------------
    const int sw = warp - 2;                     // 0..7
    const int q = warp & 3;                      // TMEM lane quarter
    const int half = sw >> 2;                    // which 64 keys of the chunk (and of O's columns)
    const int r = q * 32 + lane;                 // row of the tile = TMEM lane
    const int grow = rt * kBM + r;               // row within (request, KV head)
    const bool live = grow < a.R;
    const int t = live ? grow / a.G : 0;
    const uint32_t lane_off = uint32_t(q * 32) << 16;
    const float sc = a.scale_log2;
    constexpr int kHalf = kBN / 2;
    float run_m = -INFINITY, run_l = 0.f;
    bool ok = true;
    // Every iteration runs both named barriers, so a wait that gives up (ok =
    // false) only skips work and never leaves a partner warp at a barrier.
    for (int c = 0; c < nch; ++c) {
      if (ok && !mbar_wait(smem_u32(&s_full[c & 1]), (c >> 1) & 1)) ok = false;
      ok = __all_sync(0xffffffffu, ok);          // tcgen05.ld below is warp-collective
      tc_fence_after();
      const uint32_t sb = tS + lane_off + uint32_t((c & 1) * kBN + half * kHalf);
      const int key0 = (c_begin + c) * kBN + half * kHalf;
      const bool plain = key0 + kHalf <= P;      // every key of this half is in the prefix
      // this half of the row's scores: one 64-column TMEM load, kept for both passes
      float s[kHalf];
      float mx = -INFINITY;
      if (ok) {
        tmem_ld64(sb, s);
        if (plain) {
#pragma unroll
          for (int j = 0; j < kHalf; ++j) mx = fmaxf(mx, s[j]);
        } else {
#pragma unroll
          for (int j = 0; j < kHalf; ++j) {
            const int slot = key0 + j;
            const bool vis = slot < P || (slot < nkeys && live && tree_visible(tp, t, slot - P));
            s[j] = vis ? s[j] : -INFINITY;
            mx = fmaxf(mx, s[j]);
          }
        }
      }
      // exchange the half maxima with the partner warp (same lane quarter)
      xmax[half * kBM + r] = mx;
      named_bar_sync(1 + q, 64);
      mx = fmaxf(mx, xmax[(half ^ 1) * kBM + r]);
      named_bar_sync(1 + q, 64);                 // both have read before the slots are reused
      mx = (mx == -INFINITY) ? -INFINITY : mx * sc;
      // The previous P V must be done before P is overwritten or O rescaled.
      if (ok && c >= 1 && !mbar_wait(smem_u32(o_full), (c - 1) & 1)) ok = false;
      if (!__all_sync(0xffffffffu, ok)) ok = false;   // warp-uniform from here on
      if (!ok) continue;
      tc_fence_after();
      const bool grow_m = mx > run_m + kRescaleLog2 || (run_m == -INFINITY && mx != -INFINITY);
      const float m_new = grow_m ? mx : run_m;
      const float fold = (grow_m && run_m != -INFINITY) ? exp2f(run_m - m_new) : 1.f;
      if (__any_sync(0xffffffffu, fold != 1.f)) {   // warp-wide: tcgen05.ld/st are collective
#pragma unroll
        for (int e0 = half * (DH / 2); e0 < (half + 1) * (DH / 2); e0 += 32) {
          float o[32];
          tmem_ld32(tO + lane_off + e0, o);
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] *= fold;
          tmem_st32(tO + lane_off + e0, o);
        }
      }
      run_l *= fold;
      run_m = m_new;
      // P = exp2(S*scale - m) as bf16 hi + lo into swizzled smem (K-major over keys);
      // masked keys hold -inf and give exactly 0
      const float mb = (run_m == -INFINITY) ? 0.f : run_m;
      float sum = 0.f;
#pragma unroll
      for (int c32 = 0; c32 < kHalf; c32 += 32) {
        uint32_t ph[16], pl[16];
#pragma unroll
        for (int j = 0; j < 32; j += 2) {
          const float p0 = exp2f(fmaf(s[c32 + j], sc, -mb));
          const float p1 = exp2f(fmaf(s[c32 + j + 1], sc, -mb));
          sum += p0 + p1;
          const uint32_t h2 = pack_bf16x2(p0, p1);
          ph[j >> 1] = h2;
          pl[j >> 1] = pack_bf16x2(p0 - bf16lo(h2), p1 - bf16hi(h2));
        }
        // row r, keys (half*64 + c32) .. +31 -> block `half`, 16-byte chunks c32/8 .. +3, swizzled by r%8
        const uint32_t roff = half * kBM * 128 + r * 128;
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          const int ch = (c32 >> 3) + g;
          const uint32_t off = roff + ((ch ^ (r & 7)) << 4);
          *reinterpret_cast<uint4*>(sP + off) = make_uint4(ph[4 * g], ph[4 * g + 1], ph[4 * g + 2], ph[4 * g + 3]);
          *reinterpret_cast<uint4*>(sPl + off) = make_uint4(pl[4 * g], pl[4 * g + 1], pl[4 * g + 2], pl[4 * g + 3]);
        }
      }
      run_l += sum;
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(smem_u32(&s_empty[c & 1]));
        mbar_arrive(smem_u32(p_full));
      }
    }
    // this split's partial for the row: (m, l, O); each half writes its half of O
    const size_t tile = (size_t(b) * a.Hkv + hk) * a.rtiles + rt;
    const size_t prow = (tile * a.splits + split) * kBM + r;
    float* po = a.part_o + prow * DH;
    if (ok && nch > 0) {
      if (__all_sync(0xffffffffu, mbar_wait(smem_u32(o_full), (nch - 1) & 1))) {
        tc_fence_after();
#pragma unroll
        for (int e0 = half * (DH / 2); e0 < (half + 1) * (DH / 2); e0 += 32) {
          float o[32];
          tmem_ld32(tO + lane_off + e0, o);
#pragma unroll
          for (int e = 0; e < 32; e += 4)
            *reinterpret_cast<float4*>(po + e0 + e) = make_float4(o[e], o[e + 1], o[e + 2], o[e + 3]);
        }
      } else {
        ok = false;
      }
    }
    if (!ok) set_status(MD_DEV_TIMEOUT);
    xmax[half * kBM + r] = run_l;
    named_bar_sync(1 + q, 64);
    if (half == 0)
      a.part_ml[prow] = make_float2((ok && nch > 0) ? run_m : -INFINITY, run_l + xmax[kBM + r]);

    // The last CTA of this (request, KV head, row tile) merges the splits in order.
    __threadfence();
    named_bar_sync(5, kSoftWarps * 32);   // ids 1..4: partner pairs
    if (sw == 0 && lane == 0) *last_flag = (atomicAdd(&a.counters[tile], 1) == a.splits - 1);
    named_bar_sync(5, kSoftWarps * 32);   // ids 1..4: partner pairs
    if (*last_flag && live && half == 0) {
      __threadfence();
      const int g = grow - t * a.G;
      float* orow = a.out + ((size_t(b) * T + t) * a.Hq + hk * a.G + g) * DH;
      if (bad) {
        for (int e = 0; e < DH; e += 4) *reinterpret_cast<float4*>(orow + e) = make_float4(0.f, 0.f, 0.f, 0.f);
      } else {
        const size_t base = tile * a.splits;
        float w[kMaxSplits];
        float mx = -INFINITY;
#pragma unroll
        for (int s = 0; s < kMaxSplits; ++s)
          if (s < a.splits) mx = fmaxf(mx, __ldcg(&a.part_ml[(base + s) * kBM + r]).x);
        float L = 0.f;
#pragma unroll
        for (int s = 0; s < kMaxSplits; ++s) {
          w[s] = 0.f;
          if (s < a.splits) {
            const float2 ml = __ldcg(&a.part_ml[(base + s) * kBM + r]);
            w[s] = (ml.x == -INFINITY) ? 0.f : exp2f(ml.x - mx);
            L = fmaf(ml.y, w[s], L);
          }
        }
        const float inv = 1.f / L;
        for (int e = 0; e < DH; e += 4) {
          float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
          for (int s = 0; s < kMaxSplits; ++s) {
            if (s < a.splits && w[s] != 0.f) {
              const float4 v = __ldcg(reinterpret_cast<const float4*>(a.part_o + ((base + s) * kBM + r) * DH + e));
              acc.x = fmaf(v.x, w[s], acc.x);
              acc.y = fmaf(v.y, w[s], acc.y);
              acc.z = fmaf(v.z, w[s], acc.z);
              acc.w = fmaf(v.w, w[s], acc.w);
            }
          }
          *reinterpret_cast<float4*>(orow + e) = make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace attn_tc
}  // namespace md
