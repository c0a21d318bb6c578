// Tree-masked attention on the tensor cores (tcgen05).
//
// Source: "Medusa heads versus separate draft model", section "Acceptance",
// tree paragraph: every branch is verified in one target pass with a tree
// attention mask. With grouped-query attention every KV head serves
// T x (Hq/Hkv) query rows (65 x 8 = 520 for the 70B tree), so the scores and
// the weighted sum are dense products: S = Q K^T and O = P V run on tcgen05.
//
// CTA = (KV split, 128-row query tile, KV head, request). The 128 query rows
// are (tree token, query head of the group) pairs, loaded by one 3-D TMA box
// straight out of q[B, T, Hq, dh]. The CTA walks its share of 128-key chunks:
//
//   warp 0     TMA: the Q tile once, then K and V chunks into a 2-deep ring
//   warp 1     one thread issues S_c = Q K_c^T into TMEM (double-buffered)
//              and O_c = P_c V_c into TMEM
//   warps 2-5  one query row per thread: read S_c from TMEM, apply the scale
//              and the tree mask (keys >= P_b are tree nodes; visible iff an
//              ancestor-or-self), chunk max, P_c = exp2(S - max) split into
//              bf16 hi + lo parts in swizzled shared memory (P V then runs as
//              P_hi V + P_lo V, so the weights keep ~16 significant bits), and
//              fold O_{c-1} into a running (max, sum, O) kept in registers.
//
// Each CTA writes its split's (max, sum, unnormalised O) per row;
// attn_tc_merge_kernel combines the splits in order.
#pragma once

#include "common.cuh"

namespace md {
namespace attn_tc {

constexpr int kBM = 128;        // query rows per CTA
constexpr int kBN = 128;        // keys per chunk
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 512;

template <int DH>
struct Cfg {
  static constexpr int KB = DH / 64;                          // 64-element blocks of the head dim
  static constexpr uint32_t kQBytes = KB * kBM * 128;         // Q tile, K-major SW128
  static constexpr uint32_t kKBytes = KB * kBN * 128;         // K chunk, K-major SW128
  static constexpr uint32_t kVBytes = KB * kBN * 128;         // V chunk, N(dh)-major SW128
  static constexpr uint32_t kStage = kKBytes + kVBytes;
  static constexpr uint32_t kPBytes = 2 * kBM * 128;          // P tile: 128 rows x 128 keys bf16
  static constexpr int kSmem = kQBytes + 2 * kStage + 2 * kPBytes + 1024 + 256;   // P hi and P lo
};

struct Args {
  const int32_t* prefix_len;  // [B]
  float* part_o;              // [B, Hkv, splits, rtiles*128, dh]
  float2* part_ml;            // [B, Hkv, splits, rtiles*128]   (max, sum) in log2 units
  float* out;                 // [B, T, Hq, dh]
  int B, S_max, Hq, Hkv, G, R, rtiles, splits, chunks_per_split;
  float scale_log2;
};

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
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
  uint8_t* sPl = sP + C::kPBytes;                        // P lo
  uint64_t* bars = reinterpret_cast<uint64_t*>(sPl + C::kPBytes);
  uint64_t* q_full = bars;            // 1
  uint64_t* kv_full = bars + 1;       // 2
  uint64_t* kv_empty = bars + 3;      // 2
  uint64_t* s_full = bars + 5;        // 2
  uint64_t* s_empty = bars + 7;       // 2
  uint64_t* p_full = bars + 9;        // 1
  uint64_t* o_full = bars + 10;       // 1
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 11);

  const int split = blockIdx.x, rt = blockIdx.y % a.rtiles, hk = blockIdx.y / a.rtiles, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int T = tp.T;
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
      mbar_init(smem_u32(&kv_full[i]), 1);
      mbar_init(smem_u32(&kv_empty[i]), 1);
      mbar_init(smem_u32(&s_full[i]), 1);
      mbar_init(smem_u32(&s_empty[i]), 4);
    }
    mbar_init(smem_u32(p_full), 4);
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
  const uint32_t tO = tmem + 2 * kBN;       // O_c at columns [256, 256 + DH)
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
      for (int c = 0; c < nch; ++c) {
        const int st = c & 1;
        if (c >= 2 && !mbar_wait(smem_u32(&kv_empty[st]), ((c >> 1) - 1) & 1)) {
          set_status(MD_DEV_TIMEOUT);
          break;
        }
        const uint32_t fb = smem_u32(&kv_full[st]);
        uint8_t* sk = sKV + st * C::kStage;
        uint8_t* sv = sk + C::kKBytes;
        const int key0 = (c_begin + c) * kBN;
        mbar_arrive_expect_tx(fb, C::kStage);
#pragma unroll
        for (int kb = 0; kb < C::KB; ++kb) {
          tma_load_3d(smem_u32(sk + kb * kBN * 128), &kmap, kb * 64, key0, kvrow, fb);
          tma_load_3d(smem_u32(sv + kb * kBN * 128), &vmap, kb * 64, key0, kvrow, fb);
        }
      }
      for (int c = max(0, nch - 2); c < nch; ++c) {
        if (!mbar_wait(smem_u32(&kv_empty[c & 1]), (c >> 1) & 1)) {
          set_status(MD_DEV_TIMEOUT);
          break;
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------- MMA ----------------------------------
    if (lane == 0 && nch > 0) {
      constexpr uint32_t idesc_s = umma_idesc_bf16(kBM, kBN, 0, 0);
      constexpr uint32_t idesc_o = umma_idesc_bf16(kBM, DH, 0, 1);
      bool ok = mbar_wait(smem_u32(q_full), 0);
      const uint32_t aq = smem_u32(sQ);
      for (int c = 0; c <= nch && ok; ++c) {
        if (c < nch) {
          const int st = c & 1;
          if (!mbar_wait(smem_u32(&kv_full[st]), (c >> 1) & 1)) { ok = false; break; }
          if (c >= 2 && !mbar_wait(smem_u32(&s_empty[c & 1]), ((c >> 1) - 1) & 1)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sk = smem_u32(sKV + st * C::kStage);
          const uint32_t d = tS + uint32_t((c & 1) * kBN);
#pragma unroll
          for (int kb = 0; kb < C::KB; ++kb) {
            const uint64_t ad = umma_desc_sw128(aq + kb * kBM * 128, 16, 1024);
            const uint64_t bd = umma_desc_sw128(sk + kb * kBN * 128, 16, 1024);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              umma_f16(d, ad + uint64_t((kk * 32) >> 4), bd + uint64_t((kk * 32) >> 4), idesc_s, (kb | kk) != 0);
          }
          umma_commit(smem_u32(&s_full[c & 1]));
        }
        if (c >= 1) {
          const int cp = c - 1;
          if (!mbar_wait(smem_u32(p_full), cp & 1)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sv = smem_u32(sKV + (cp & 1) * C::kStage + C::kKBytes);
#pragma unroll
          for (int part = 0; part < 2; ++part) {
            const uint32_t sp = smem_u32(part == 0 ? sP : sPl);
#pragma unroll
            for (int kk = 0; kk < kBN / 16; ++kk) {
              const uint64_t ad =
                  umma_desc_sw128(sp + (kk >> 2) * kBM * 128, 16, 1024) + uint64_t(((kk & 3) * 32) >> 4);
              const uint64_t bd = umma_desc_sw128(sv, kBN * 128, 1024) + uint64_t((kk * 2048) >> 4);
              umma_f16(tO, ad, bd, idesc_o, (part | kk) != 0);
            }
          }
          umma_commit(smem_u32(o_full));
          umma_commit(smem_u32(&kv_empty[cp & 1]));
        }
      }
      if (!ok) set_status(MD_DEV_TIMEOUT);
    }
  } else {
    // ------------------------------- softmax rows -------------------------------
    const int q = warp & 3;
    const int r = q * 32 + lane;                 // row of the tile = TMEM lane
    const int grow = rt * kBM + r;               // row within (request, KV head)
    const int t = grow / a.G;
    const bool live = grow < a.R;
    const uint32_t lane_off = uint32_t(q * 32) << 16;
    float run_m = -INFINITY, run_l = 0.f;
    float o[DH];
#pragma unroll
    for (int e = 0; e < DH; ++e) o[e] = 0.f;
    float cm = -INFINITY, cl = 0.f;              // previous chunk's max and sum
    bool ok = true;
    auto fold = [&](float m_c, float l_c) {      // fold O_c (in TMEM) into the running state
      float vv[32];
      const float mn = fmaxf(run_m, m_c);
      const float fa = (run_m == -INFINITY) ? 0.f : exp2f(run_m - mn);
      const float fb = (m_c == -INFINITY) ? 0.f : exp2f(m_c - mn);
#pragma unroll
      for (int e0 = 0; e0 < DH; e0 += 32) {
        tmem_ld32(tO + lane_off + e0, vv);
#pragma unroll
        for (int e = 0; e < 32; ++e) o[e0 + e] = o[e0 + e] * fa + vv[e] * fb;
      }
      run_l = run_l * fa + l_c * fb;
      run_m = mn;
    };
    for (int c = 0; c < nch && ok; ++c) {
      if (!mbar_wait(smem_u32(&s_full[c & 1]), (c >> 1) & 1)) { ok = false; break; }
      tc_fence_after();
      const uint32_t sb = tS + lane_off + uint32_t((c & 1) * kBN);
      const int key0 = (c_begin + c) * kBN;
      // pass 1: masked, scaled chunk maximum
      float mx = -INFINITY;
      for (int c32 = 0; c32 < kBN; c32 += 32) {
        float s[32];
        tmem_ld32(sb + c32, s);
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int slot = key0 + c32 + j;
          bool vis = slot < nkeys;
          if (vis && slot >= P) {
            const int node = slot - P;
            vis = live && ((tp.anc[t < T ? t : 0][node >> 5] >> (node & 31)) & 1u);
          }
          if (vis) mx = fmaxf(mx, s[j] * a.scale_log2);
        }
      }
      // O_{c-1} must be folded (and P released) before P_c is written
      if (c >= 1) {
        if (!mbar_wait(smem_u32(o_full), (c - 1) & 1)) { ok = false; break; }
        tc_fence_after();
        fold(cm, cl);
      }
      // pass 2: P = exp2(S - max) as bf16 hi + lo into swizzled smem (K-major over keys)
      float sum = 0.f;
      for (int c32 = 0; c32 < kBN; c32 += 32) {
        float s[32];
        tmem_ld32(sb + c32, s);
        uint32_t ph[16], pl[16];
#pragma unroll
        for (int j = 0; j < 32; j += 2) {
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int slot = key0 + c32 + j + u;
            bool vis = slot < nkeys;
            if (vis && slot >= P) {
              const int node = slot - P;
              vis = live && ((tp.anc[t < T ? t : 0][node >> 5] >> (node & 31)) & 1u);
            }
            const float p = (vis && mx != -INFINITY) ? exp2f(s[j + u] * a.scale_log2 - mx) : 0.f;
            const uint16_t hb = f32_to_bf16_rne(p);
            const float hf = bf16_to_f32(hb);
            const uint16_t lb = f32_to_bf16_rne(p - hf);
            sum += hf + bf16_to_f32(lb);   // the weights the two MMAs apply
            if (u == 0) {
              ph[j >> 1] = hb;
              pl[j >> 1] = lb;
            } else {
              ph[j >> 1] |= uint32_t(hb) << 16;
              pl[j >> 1] |= uint32_t(lb) << 16;
            }
          }
        }
        // row r, keys c32 .. c32+31 -> block c32/64, 16-byte chunks (c32%64)/8 .. +3, swizzled by r%8
        const uint32_t roff = (c32 >> 6) * kBM * 128 + r * 128;
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          const int ch = ((c32 & 63) >> 3) + g;
          const uint32_t off = roff + ((ch ^ (r & 7)) << 4);
          *reinterpret_cast<uint4*>(sP + off) = make_uint4(ph[4 * g], ph[4 * g + 1], ph[4 * g + 2], ph[4 * g + 3]);
          *reinterpret_cast<uint4*>(sPl + off) = make_uint4(pl[4 * g], pl[4 * g + 1], pl[4 * g + 2], pl[4 * g + 3]);
        }
      }
      cm = mx;
      cl = sum;
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(smem_u32(&s_empty[c & 1]));
        mbar_arrive(smem_u32(p_full));
      }
    }
    if (ok && nch > 0) {
      if (mbar_wait(smem_u32(o_full), (nch - 1) & 1)) {
        tc_fence_after();
        fold(cm, cl);
      } else {
        ok = false;
      }
    }
    if (!ok) set_status(MD_DEV_TIMEOUT);
    // split partial for this row
    const size_t prow = ((size_t(b) * a.Hkv + hk) * a.splits + split) * (size_t(a.rtiles) * kBM) + grow;
    a.part_ml[prow] = make_float2(nch > 0 ? run_m : -INFINITY, run_l);
    float4* po = reinterpret_cast<float4*>(a.part_o + prow * DH);
#pragma unroll
    for (int e = 0; e < DH; e += 4) po[e >> 2] = make_float4(o[e], o[e + 1], o[e + 2], o[e + 3]);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// out[b, t, h, :] = sum_s O_s 2^(m_s - M) / sum_s l_s 2^(m_s - M), splits in order.
// grid (T * Hq, B), DH threads.
template <int DH>
__global__ void __launch_bounds__(DH) attn_tc_merge_kernel(const __grid_constant__ TreeParams tp, Args a) {
  const int b = blockIdx.y;
  const int th = blockIdx.x;
  const int t = th / a.Hq, h = th % a.Hq;
  const int hk = h / a.G, g = h % a.G;
  const int grow = t * a.G + g;
  const int e = threadIdx.x;
  const int T = tp.T;
  const int P = a.prefix_len[b];
  float* o = a.out + ((size_t(b) * T + t) * a.Hq + h) * DH;
  if (P < 0 || P + T > a.S_max) {
    o[e] = 0.f;
    return;
  }
  const size_t rows = size_t(a.rtiles) * kBM;
  const size_t base = (size_t(b) * a.Hkv + hk) * a.splits;
  float mx = -INFINITY;
  for (int s = 0; s < a.splits; ++s) mx = fmaxf(mx, a.part_ml[(base + s) * rows + grow].x);
  float L = 0.f, acc = 0.f;
  for (int s = 0; s < a.splits; ++s) {
    const float2 ml = a.part_ml[(base + s) * rows + grow];
    if (ml.x == -INFINITY) continue;
    const float w = exp2f(ml.x - mx);
    L = fmaf(ml.y, w, L);
    acc = fmaf(a.part_o[((base + s) * rows + grow) * DH + e], w, acc);
  }
  o[e] = acc / L;
}

}  // namespace attn_tc
}  // namespace md
