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
// share of CH-key chunks (CH = 64 or 128, see Cfg):
//
//   warp 0     TMA: the Q tile once, then K and V chunks into two rings
//              (a K slot frees when its S is done, a V slot when its P V is)
//   warp 1     one thread issues S_c = Q K_c^T into TMEM (one buffer per ring
//              slot, that many chunks ahead) and O += P_c V_c into one TMEM
//              accumulator that lives across chunks, with P_c read from TMEM
//   softmax    one warp per TMEM lane quarter and 64 keys of the chunk (two per
//              quarter for 128-key chunks; row maxima are then exchanged
//              through shared memory): read
//              S_c from TMEM, apply the scale and -- only in chunks that reach
//              the tree slots -- the tree mask (a key at slot >= P_b is tree
//              node slot - P_b, visible iff it is an ancestor-or-self), then
//              P_c = exp2(S - m) against a running row maximum m, split into
//              bf16 hi + lo parts (P V runs as P_hi V + P_lo V, keeping ~16
//              significant bits of each weight) and written back over S_c's
//              own TMEM columns. m only moves when a chunk exceeds it by more
//              than 2^8; O and the row sum are then rescaled in place.
//
// Because P_c lives in S_c's buffer, the softmax of chunk c + 1 never waits for
// P_c V_c (only a rescale of O does), and the next buffers' S are computed
// while the softmax works on c: the softmax warps and the tensor pipe work on
// different chunks at the same time.
//
// The KV splits of one (request, KV head, row tile) are the CTAs of one
// cluster. Each stages its split's unnormalised O and per-row (m, sum) in its
// shared memory; after a cluster barrier every CTA combines its share of the
// rows from all splits' shared memory (distributed shared memory loads, in
// split order) and writes them; a second cluster barrier keeps each CTA's
// shared memory alive until its peers are done reading it.
#pragma once

#include "common.cuh"

namespace md {
namespace attn_tc {

constexpr int kBM = 128;        // query rows per CTA
constexpr int kKeysPerWarp = 64;   // keys of a chunk one softmax warp takes for its 32 rows
constexpr float kRescaleLog2 = 8.0f;   // lazy rescale threshold (factor 256)
constexpr int kMaxSplits = 8;    // KV splits of one tile = CTAs of one cluster (portable size)

// Two shapes of the same pipeline. CH = 128: 128-key chunks, two softmax warps
// per TMEM lane quarter (64 keys each, row maxima exchanged), three S/P buffers
// and a 3-deep K/V ring, all 512 TMEM columns: one CTA per SM. CH = 64: 64-key
// chunks, one softmax warp per lane quarter, two S/P buffers, a 2-deep ring and
// 256 TMEM columns, small enough for two CTAs per SM, so that one CTA's
// prologue and split merge overlap the other's chunk loop.
template <int DH, int CH>
struct Cfg {
  static constexpr int kBN = CH;                              // keys per chunk
  static constexpr int kWPQ = CH / kKeysPerWarp;              // softmax warps per TMEM lane quarter
  static constexpr int kSoftWarps = 4 * kWPQ;
  static constexpr int kThreads = 64 + kSoftWarps * 32;
  static constexpr int kStages = CH == 128 ? 3 : 2;           // K / V ring depth
  static constexpr int kSBufs = CH == 128 ? 3 : 2;            // S / P buffers in TMEM (+ O)
  static constexpr uint32_t kTmemCols = CH == 128 ? 512 : 256;
  static constexpr int kMinBlocks = CH == 128 ? 1 : 2;        // resident CTAs per SM
  static constexpr int KB = DH / 64;                          // 64-element blocks of the head dim
  static constexpr uint32_t kQBytes = KB * kBM * 128;         // Q tile, K-major SW128
  static constexpr uint32_t kKBytes = KB * kBN * 128;         // K chunk, K-major SW128
  static constexpr uint32_t kVBytes = KB * kBN * 128;         // V chunk, N(dh)-major SW128
  static constexpr uint32_t kStage = kKBytes + kVBytes;
  static constexpr int kSmem = kQBytes + kStages * kStage + 1024 + 256 + 1024;  // + barriers, maxima
  // the epilogue stages O, the merge weights and (m, l) over the idle Q tile and K/V ring
  static_assert(kBM * (DH + 4) * 4 + kBM * (kMaxSplits + 1) * 4 + kBM * 8 <= kQBytes + kStages * kStage,
                "staging");
  static_assert(kSBufs * kBN + DH <= int(kTmemCols), "TMEM");
};

struct Args {
  const int32_t* prefix_len;  // [B]
  float* out;                 // [B, T, Hq, dh]
  int B, S_max, Hq, Hkv, G, R, rtiles, splits, chunks_per_split;
  float scale_log2;
};

// 2^x on the special-function unit; results below 2^-126 flush to zero (a
// weight that small is far below the bf16 hi/lo resolution of the row's sum).
__device__ __forceinline__ float exp2_sfu(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Visibility of the 64 keys n0 .. n0 + 63 (n = slot - P: negative n is a
// prefix key, always visible; tree node n is visible iff it is an ancestor-or-
// self of the row's token) as bit j, from the row's 128-bit ancestor set
// (lo = nodes 0..63, hi = nodes 64..127; bits of nodes >= T are zero).
__device__ __forceinline__ uint64_t visible_bits(uint64_t lo, uint64_t hi, int n0) {
  if (n0 <= -64) return ~0ull;
  if (n0 >= 128) return 0ull;
  if (n0 < 0) return (lo << (-n0)) | ((1ull << (-n0)) - 1ull);
  if (n0 == 0) return lo;
  if (n0 < 64) return (lo >> n0) | (hi << (64 - n0));
  if (n0 == 64) return hi;
  return hi >> (n0 - 64);
}

template <int DH, int CH>
__global__ void __launch_bounds__(Cfg<DH, CH>::kThreads, Cfg<DH, CH>::kMinBlocks)
    attn_tc_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
                   const __grid_constant__ CUtensorMap vmap, const __grid_constant__ TreeParams tp, Args a) {
  using C = Cfg<DH, CH>;
  constexpr int kBN = C::kBN, kStages = C::kStages, kSBufs = C::kSBufs, kSoftWarps = C::kSoftWarps;
  constexpr uint32_t kTmemCols = C::kTmemCols;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint8_t* sQ = smem;
  uint8_t* sKV = smem + C::kQBytes;                     // kStages stages of (K, V)
  uint64_t* bars = reinterpret_cast<uint64_t*>(sKV + kStages * C::kStage);
  uint64_t* q_full = bars;                      // 1
  uint64_t* k_full = q_full + 1;                // kStages
  uint64_t* k_empty = k_full + kStages;         // kStages
  uint64_t* v_full = k_empty + kStages;         // kStages
  uint64_t* v_empty = v_full + kStages;         // kStages
  uint64_t* s_full = v_empty + kStages;         // kSBufs
  uint64_t* p_full = s_full + kSBufs;           // kSBufs
  uint64_t* o_full = p_full + kSBufs;           // 2: P_c V_c commits to o_full[c & 1]
  uint64_t* o_last = o_full + 2;                // 1: every P V done
  uint64_t* mma_done = o_last + 1;              // 1: every MMA this CTA issued has completed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  int* req = reinterpret_cast<int*>(tmem_slot + 2);   // request served by this CTA
  float* xmax = reinterpret_cast<float*>(bars + 32);    // [2 halves][128 rows] chunk maxima

  const int split = blockIdx.x, rt = blockIdx.y % a.rtiles, hk = blockIdx.y / a.rtiles;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int T = tp.T;
  // Set-up that reads no input (mbarriers, TMEM) runs before the wait for the
  // previous kernel, overlapping its tail.
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(q_full), 1);
    for (int i = 0; i < kStages; ++i) {
      mbar_init(smem_u32(&k_full[i]), 1);
      mbar_init(smem_u32(&k_empty[i]), 1);
      mbar_init(smem_u32(&v_full[i]), 1);
      mbar_init(smem_u32(&v_empty[i]), 1);
    }
    for (int i = 0; i < kSBufs; ++i) {
      mbar_init(smem_u32(&s_full[i]), 1);
      mbar_init(smem_u32(&p_full[i]), kSoftWarps);
    }
    for (int i = 0; i < 2; ++i) mbar_init(smem_u32(&o_full[i]), 1);
    mbar_init(smem_u32(o_last), 1);
    mbar_init(smem_u32(mma_done), 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  pdl_wait_primary();          // inputs may come from earlier kernels
  pdl_launch_dependents();
  // Blocks are launched in index order, so blockIdx.z walks the requests from
  // the longest prefix down (ties by index): long tiles start first and short
  // ones fill the tail. Warp 0 finds the request of rank blockIdx.z.
  if (warp == 0) {
    for (int c = lane; c < a.B; c += 32) {
      const int pc = a.prefix_len[c];
      int rank = 0;
      for (int j = 0; j < a.B; ++j) {
        const int pj = a.prefix_len[j];
        rank += (pj > pc || (pj == pc && j < c)) ? 1 : 0;
      }
      if (rank == int(blockIdx.z)) *req = c;
    }
  }
  __syncthreads();
  const int b = *req;
  const int P = a.prefix_len[b];
  const bool bad = P < 0 || P + T > a.S_max;
  const int nkeys = bad ? 0 : P + T;
  const int nch_total = (nkeys + kBN - 1) / kBN;
  const int c_begin = split * a.chunks_per_split;
  const int c_end = min(nch_total, c_begin + a.chunks_per_split);
  const int nch = max(0, c_end - c_begin);
  if (bad && split == 0 && blockIdx.y == 0 && threadIdx.x == 0) set_status(MD_DEV_BAD_PREFIX);

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // S_c at columns [128*(c%3), +128); P_c overwrites them: hi parts in the
  // first 64 columns, lo parts in the last 64 (two bf16 keys per column)
  const uint32_t tS = tmem;
  const uint32_t tO = tmem + kSBufs * kBN;  // O at columns [384, 384 + DH)
  const int kvrow = b * a.Hkv + hk;
  const int tpt = kBM / a.G;                // tree tokens per query tile
  // epilogue staging over the Q tile and the K/V ring: O [128][kLd] (padded rows: conflict-free
  // 16-byte accesses), merge weights [128][kMaxSplits + 1] (1/L last), (m, l) [128]
  constexpr int kLd = DH + 4;
  float* sO = reinterpret_cast<float*>(smem);   // over the Q tile and the K/V ring
  float* sW = sO + kBM * kLd;
  float2* sML = reinterpret_cast<float2*>(sW + kBM * (kMaxSplits + 1));

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
      int nk = 0, nv = 0;                    // chunks whose K / V copies were issued
      const int withhold = *const_cast<volatile int*>(&g_withhold_chunk);   // test hook, normally -1
      for (int c = 0; c < nch && ok; ++c) {
        if (c == withhold) continue;         // test hook: this chunk's copies never come
        const int st = c % kStages, ph = ((c / kStages) - 1) & 1;
        const int key0 = (c_begin + c) * kBN;
        uint8_t* sk = sKV + st * C::kStage;
        uint8_t* sv = sk + C::kKBytes;
        if (c >= kStages && !mbar_wait(smem_u32(&k_empty[st]), ph)) { ok = false; break; }
        const uint32_t kb_ = smem_u32(&k_full[st]);
        mbar_arrive_expect_tx(kb_, C::kKBytes);
#pragma unroll
        for (int kb = 0; kb < C::KB; ++kb) tma_load_3d(smem_u32(sk + kb * kBN * 128), &kmap, kb * 64, key0, kvrow, kb_);
        nk = c + 1;
        if (c >= kStages && !mbar_wait(smem_u32(&v_empty[st]), ph)) { ok = false; break; }
        const uint32_t vb_ = smem_u32(&v_full[st]);
        mbar_arrive_expect_tx(vb_, C::kVBytes);
#pragma unroll
        for (int kb = 0; kb < C::KB; ++kb) tma_load_3d(smem_u32(sv + kb * kBN * 128), &vmap, kb * 64, key0, kvrow, vb_);
        nv = c + 1;
      }
      // Before the CTA may exit, every copy issued into its shared memory has
      // landed: wait for the last phase of each ring slot's full barriers (TMA
      // completion, whatever the consumers did) and of the Q barrier. Earlier
      // copies were consumed before their slot was refilled.
      bool drained = mbar_wait(smem_u32(q_full), 0);
      for (int c = (nk > kStages ? nk - kStages : 0); c < nk; ++c)
        drained = mbar_wait(smem_u32(&k_full[c % kStages]), (c / kStages) & 1) && drained;
      for (int c = (nv > kStages ? nv - kStages : 0); c < nv; ++c)
        drained = mbar_wait(smem_u32(&v_full[c % kStages]), (c / kStages) & 1) && drained;
      if (!ok || !drained) set_status(MD_DEV_TIMEOUT);
    }
  } else if (warp == 1) {
    // ---------------------------------- MMA ----------------------------------
    if (lane == 0 && nch > 0) {
      constexpr uint32_t idesc_s = umma_idesc_bf16(kBM, kBN, 0, 0);
      constexpr uint32_t idesc_o = umma_idesc_bf16(kBM, DH, 0, 1);
      bool ok = mbar_wait(smem_u32(q_full), 0);
      const uint32_t aq = smem_u32(sQ);
      // S_c = Q K_c^T into TMEM buffer c % 3; frees K slot c % kStages when done.
      // Buffer c % 3 last held P_{c-3}: P_{c-3} V_{c-3} was issued before this,
      // and tcgen05.mma runs in issue order.
      auto issue_s = [&](int c) -> bool {
        const int st = c % kStages;
        if (!mbar_wait(smem_u32(&k_full[st]), (c / kStages) & 1)) return false;
        tc_fence_after();
        const uint32_t sk = smem_u32(sKV + st * C::kStage);
        const uint32_t d = tS + uint32_t((c % kSBufs) * kBN);
#pragma unroll
        for (int kb = 0; kb < C::KB; ++kb) {
          const uint64_t ad = umma_desc_sw128(aq + kb * kBM * 128, 16, 1024);
          const uint64_t bd = umma_desc_sw128(sk + kb * kBN * 128, 16, 1024);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_f16(d, ad + uint64_t((kk * 32) >> 4), bd + uint64_t((kk * 32) >> 4), idesc_s, (kb | kk) != 0);
        }
        umma_commit(smem_u32(&s_full[c % kSBufs]));
        umma_commit(smem_u32(&k_empty[st]));
        return true;
      };
      for (int c = 0; c < kSBufs && c < nch && ok; ++c) ok = issue_s(c);
      for (int c = 0; c < nch && ok; ++c) {
        // O += P_c V_c (hi and lo parts, P from TMEM); frees V slot c % kStages when done
        const int st = c % kStages;
        if (!mbar_wait(smem_u32(&p_full[c % kSBufs]), (c / kSBufs) & 1) ||
            !mbar_wait(smem_u32(&v_full[st]), (c / kStages) & 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t sv = smem_u32(sKV + st * C::kStage + C::kKBytes);
        const uint32_t tp_ = tS + uint32_t((c % kSBufs) * kBN);
#pragma unroll
        for (int part = 0; part < 2; ++part) {
#pragma unroll
          for (int kk = 0; kk < kBN / 16; ++kk) {
            const uint64_t bd = umma_desc_sw128(sv, kBN * 128, 1024) + uint64_t((kk * 2048) >> 4);
            umma_f16_tmem_a(tO, tp_ + uint32_t(part * (kBN / 2) + kk * 8), bd, idesc_o, (c | part | kk) != 0);
          }
        }
        umma_commit(smem_u32(&o_full[c & 1]));
        umma_commit(smem_u32(&v_empty[st]));
        if (c + kSBufs < nch) ok = issue_s(c + kSBufs);
      }
      if (ok) umma_commit(smem_u32(o_last));
      // TMEM is released after this CTA's last barrier: every MMA issued so far
      // (all of them, or those before a wait gave up) must have completed
      umma_commit(smem_u32(mma_done));
      if (!mbar_wait(smem_u32(mma_done), 0)) ok = false;
      if (!ok) set_status(MD_DEV_TIMEOUT);
    }
  } else {
    // ------------------------------- softmax rows -------------------------------
    const int sw = warp - 2;                     // 0 .. kSoftWarps-1
    const int q = warp & 3;                      // TMEM lane quarter
    const int half = sw >> 2;                    // which 64 keys of the chunk (and which part of O's
                                                 // columns); 0 when one warp takes the whole chunk
    const int r = q * 32 + lane;                 // row of the tile = TMEM lane
    const int grow = rt * kBM + r;               // row within (request, KV head)
    const bool live = grow < a.R;
    const int t = live ? grow / a.G : 0;
    const uint32_t lane_off = uint32_t(q * 32) << 16;
    const uint64_t anc_lo = (uint64_t(tp.anc[t][1]) << 32) | tp.anc[t][0];
    const uint64_t anc_hi = (uint64_t(tp.anc[t][3]) << 32) | tp.anc[t][2];
    const float sc = a.scale_log2;
    constexpr int kHalf = kKeysPerWarp;
    constexpr int kOCols = DH / C::kWPQ;         // O columns this warp rescales and stages
    float run_m = -INFINITY, run_l = 0.f;
    bool ok = true;
    // Every iteration runs both named barriers, so a wait that gives up (ok =
    // false) only skips work and never leaves a partner warp at a barrier.
    for (int c = 0; c < nch; ++c) {
      if (ok && !mbar_wait(smem_u32(&s_full[c % kSBufs]), (c / kSBufs) & 1)) ok = false;
      ok = __all_sync(0xffffffffu, ok);          // tcgen05.ld below is warp-collective
      tc_fence_after();
      const uint32_t sbuf = tS + lane_off + uint32_t((c % kSBufs) * kBN);
      const int key0 = (c_begin + c) * kBN + half * kHalf;
      const bool plain = key0 + kHalf <= P;      // every key of this half is in the prefix
      // this half of the row's scores: one 64-column TMEM load, kept for both passes
      float s[kHalf];
      float mx = -INFINITY;
      if (ok) {
        tmem_ld64(sbuf + uint32_t(half * kHalf), s);
        if (!plain) {
          const uint64_t vis = visible_bits(anc_lo, anc_hi, key0 - P);
#pragma unroll
          for (int j = 0; j < kHalf; ++j) s[j] = ((vis >> j) & 1ull) ? s[j] : -INFINITY;
        }
        // maximum as a tree of independent pairs (short dependency chains)
        float m8[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) m8[i] = s[i];
#pragma unroll
        for (int j = 8; j < kHalf; j += 8)
#pragma unroll
          for (int i = 0; i < 8; ++i) m8[i] = fmaxf(m8[i], s[j + i]);
        mx = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])), fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
      }
      if constexpr (C::kWPQ == 2) {
        // exchange the half maxima with the partner warp (same lane quarter);
        // after the first barrier both warps have read their S columns, so
        // either may overwrite the buffer with P
        xmax[half * kBM + r] = mx;
        named_bar_sync(1 + q, 64);
        mx = fmaxf(mx, xmax[(half ^ 1) * kBM + r]);
        named_bar_sync(1 + q, 64);               // both have read before the slots are reused
      }
      mx = (mx == -INFINITY) ? -INFINITY : mx * sc;
      if (!ok) continue;
      const bool grow_m = mx > run_m + kRescaleLog2 || (run_m == -INFINITY && mx != -INFINITY);
      const float m_new = grow_m ? mx : run_m;
      const float fold = (grow_m && run_m != -INFINITY) ? exp2f(run_m - m_new) : 1.f;
      if (__any_sync(0xffffffffu, fold != 1.f)) {   // warp-wide: tcgen05.ld/st are collective
        // O is read and written in place: P_{c-1} V_{c-1} must have landed.
        // S_c landing implies P_{c-3} V_{c-3} did, so o_full[(c-1) & 1] is at
        // most one phase behind the one waited for.
        if (c >= 1 && !__all_sync(0xffffffffu, mbar_wait(smem_u32(&o_full[(c - 1) & 1]), ((c - 1) >> 1) & 1))) {
          ok = false;
          continue;
        }
        tc_fence_after();
#pragma unroll
        for (int e0 = half * kOCols; e0 < (half + 1) * kOCols; e0 += 32) {
          float o[32];
          tmem_ld32(tO + lane_off + e0, o);
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] *= fold;
          tmem_st32(tO + lane_off + e0, o);
        }
      }
      run_l *= fold;
      run_m = m_new;
      // P = exp2(S*scale - m) as bf16 hi + lo pairs into the S buffer; masked
      // keys hold -inf and give exactly 0. hi is p truncated to bf16 and lo is
      // the exact remainder p - hi truncated to bf16 (|p - hi - lo| < 2^-14 p),
      // both taken with byte permutes instead of conversions.
      const float mb = (run_m == -INFINITY) ? 0.f : run_m;
      float sum4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int g = 0; g < kHalf / 32; ++g) {     // 32 keys -> 16 columns of hi and of lo
        uint32_t ph[16], pl[16];
#pragma unroll
        for (int j = 0; j < 32; j += 2) {
          const float p0 = exp2_sfu(fmaf(s[32 * g + j], sc, -mb));
          const float p1 = exp2_sfu(fmaf(s[32 * g + j + 1], sc, -mb));
          sum4[(j >> 1) & 3] += p0 + p1;
          const uint32_t u0 = __float_as_uint(p0), u1 = __float_as_uint(p1);
          ph[j >> 1] = __byte_perm(u0, u1, 0x7632);
          const float r0 = p0 - __uint_as_float(u0 & 0xFFFF0000u);
          const float r1 = p1 - __uint_as_float(u1 & 0xFFFF0000u);
          pl[j >> 1] = __byte_perm(__float_as_uint(r0), __float_as_uint(r1), 0x7632);
        }
        tmem_st16u(sbuf + uint32_t(half * (kHalf / 2) + 16 * g), ph);
        tmem_st16u(sbuf + uint32_t(kBN / 2 + half * (kHalf / 2) + 16 * g), pl);
      }
      tmem_st_wait();
      run_l += (sum4[0] + sum4[1]) + (sum4[2] + sum4[3]);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&p_full[c % kSBufs]));
    }
    // This split's unnormalised O and (m, l) per row, staged in shared memory
    // (the K/V ring is idle once the last P V has landed).
    const bool have_o = ok && nch > 0;
    if (have_o) {
      if (__all_sync(0xffffffffu, mbar_wait(smem_u32(o_last), 0))) {
        tc_fence_after();
#pragma unroll
        for (int e0 = half * kOCols; e0 < (half + 1) * kOCols; e0 += 32) {
          float o[32];
          tmem_ld32(tO + lane_off + e0, o);
#pragma unroll
          for (int e = 0; e < 32; e += 4)
            *reinterpret_cast<float4*>(sO + r * kLd + e0 + e) = make_float4(o[e], o[e + 1], o[e + 2], o[e + 3]);
        }
      } else {
        ok = false;
      }
    }
    if (!ok) set_status(MD_DEV_TIMEOUT);
    float l_row = run_l;
    if constexpr (C::kWPQ == 2) {
      xmax[half * kBM + r] = run_l;
      named_bar_sync(1 + q, 64);
      l_row += xmax[(half ^ 1) * kBM + r];
    }
    const int tid = threadIdx.x - 64;     // 0..255 over the softmax warps
    constexpr int kF4 = DH / 4;           // float4 per row
    if (a.splits == 1) {
      // one split: the tile's rows are final, written straight from shared memory
      if (half == 0) sW[r * (kMaxSplits + 1) + kMaxSplits] = 1.f / l_row;
      named_bar_sync(5, kSoftWarps * 32);   // ids 1..4: partner pairs
      for (int i = tid; i < kBM * kF4; i += kSoftWarps * 32) {
        const int row = i / kF4, c4 = i % kF4;
        const int gr = rt * kBM + row;
        if (gr >= a.R) continue;
        const int tt = gr / a.G, g = gr - tt * a.G;
        float* orow = a.out + ((size_t(b) * T + tt) * a.Hq + hk * a.G + g) * DH;
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (ok && nch > 0 && !bad) {
          const float inv = sW[row * (kMaxSplits + 1) + kMaxSplits];
          v = *reinterpret_cast<const float4*>(sO + row * kLd + c4 * 4);
          v = make_float4(v.x * inv, v.y * inv, v.z * inv, v.w * inv);
        }
        *reinterpret_cast<float4*>(orow + c4 * 4) = v;
      }
    } else if (half == 0) {
      sML[r] = make_float2(have_o ? run_m : -INFINITY, l_row);
    }
  }

  if (a.splits > 1) {
    // ------------------- split merge through distributed shared memory -------------------
    __syncwarp();
    cluster_sync();                      // every split of the tile is staged
    if (warp >= 2) {
      const int tid = threadIdx.x - 64;
      const uint32_t crank = cluster_ctarank();
      const int r0 = int(crank) * kBM / a.splits, r1 = int(crank + 1) * kBM / a.splits;
      // per-row weights of each split and 1/L for this CTA's rows
      for (int i = tid; i < r1 - r0; i += kSoftWarps * 32) {
        const int row = r0 + i;
        float2 ml[kMaxSplits];
#pragma unroll
        for (int sp = 0; sp < kMaxSplits; ++sp)
          ml[sp] = sp < a.splits ? ld_cluster_f2(mapa_shared(smem_u32(&sML[row]), uint32_t(sp)))
                                 : make_float2(-INFINITY, 0.f);
        float mx = -INFINITY;
#pragma unroll
        for (int sp = 0; sp < kMaxSplits; ++sp) mx = fmaxf(mx, ml[sp].x);
        float L = 0.f;
#pragma unroll
        for (int sp = 0; sp < kMaxSplits; ++sp) {
          const float w = (ml[sp].x == -INFINITY) ? 0.f : exp2f(ml[sp].x - mx);
          sW[row * (kMaxSplits + 1) + sp] = w;
          L = fmaf(ml[sp].y, w, L);
        }
        sW[row * (kMaxSplits + 1) + kMaxSplits] = 1.f / L;
      }
      named_bar_sync(5, kSoftWarps * 32);
      constexpr int kF4 = DH / 4;
      constexpr int kU = 2;               // float4 outputs per thread and pass: all loads of a pass in flight
      const int n4 = (r1 - r0) * kF4;
      for (int i0 = tid; i0 < n4; i0 += kU * kSoftWarps * 32) {
        float4 v[kMaxSplits][kU];
        float w[kMaxSplits][kU];
#pragma unroll
        for (int sp = 0; sp < kMaxSplits; ++sp)
#pragma unroll
          for (int u = 0; u < kU; ++u) {
            const int i = i0 + u * kSoftWarps * 32;
            const int row = r0 + i / kF4, c4 = i % kF4;
            w[sp][u] = (sp < a.splits && i < n4 && !bad) ? sW[row * (kMaxSplits + 1) + sp] : 0.f;
            v[sp][u] = w[sp][u] != 0.f ? ld_cluster_f4(mapa_shared(smem_u32(sO + row * kLd + c4 * 4), uint32_t(sp)))
                                       : make_float4(0.f, 0.f, 0.f, 0.f);
          }
#pragma unroll
        for (int u = 0; u < kU; ++u) {
          const int i = i0 + u * kSoftWarps * 32;
          if (i >= n4) continue;
          const int row = r0 + i / kF4, c4 = i % kF4;
          const int gr = rt * kBM + row;
          if (gr >= a.R) continue;
          float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
          for (int sp = 0; sp < kMaxSplits; ++sp) {
            acc.x = fmaf(v[sp][u].x, w[sp][u], acc.x);
            acc.y = fmaf(v[sp][u].y, w[sp][u], acc.y);
            acc.z = fmaf(v[sp][u].z, w[sp][u], acc.z);
            acc.w = fmaf(v[sp][u].w, w[sp][u], acc.w);
          }
          const float inv = bad ? 0.f : sW[row * (kMaxSplits + 1) + kMaxSplits];
          const int tt = gr / a.G, g = gr - tt * a.G;
          *reinterpret_cast<float4*>(a.out + ((size_t(b) * T + tt) * a.Hq + hk * a.G + g) * DH + c4 * 4) =
              make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
        }
      }
    }
    __syncwarp();
    cluster_sync();                      // peers are done reading this CTA's shared memory
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
