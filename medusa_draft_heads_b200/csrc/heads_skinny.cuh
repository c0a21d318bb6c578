// Medusa draft heads on the tensor cores for a few hidden rows (2 .. 32),
// with the weights on the MMA's M side.
//
// Source: "Medusa heads versus separate draft model", sections "What each one
// is" and "Cost per step" -- the computation of heads.cuh and heads_gemm.cuh:
//
//   phase 1  u = h W1_k (d x d)      z = bf16(h + SiLU(u + b1_k))
//   phase 2  logits = z_k Wv_k (d x V), each row's top-k (or Gumbel top-k)
//
// With a handful of rows the call is still a weight stream: every weight byte
// is used M times. On CUDA cores the M FMAs per weight element slow the stream
// from two rows on, and a 128-row MMA tile pads M to 128. Here
// the product is computed transposed, D^T = W^T x^T: 128 output columns of the
// weights form the MMA's M (the weight tile is N-major as TMA brings it from
// the input-major matrix) and the rows form its N (NR = 16 or 32, rows
// K-major). A 64-deep stage moves 32 KB of weights plus NR x 128 B of rows and
// costs 8 MMAs of 128 x NR x 16, well below the time of its bytes.
//
// Work split (as the streaming vocabulary kernel): the (unit, stage) items --
// unit = (head, 256-column tile), d / 64 stages each -- are cut into equal
// contiguous ranges, one per CTA and one CTA per SM. A unit cut by range
// boundaries is accumulated in parts, one per CTA that it spans (the TMEM
// accumulator restarts for each part). Each part goes to a slot of its CTA in
// global memory; the CTA whose part arrives last (one ticket per unit) sums
// the parts in CTA order -- a fixed order, so results do not depend on timing
// -- and runs the epilogue.
//
// Roles (192 threads): warp 0 issues TMA, the first stages' weights before
// waiting for the previous kernel (whose output the rows may be); one thread
// of warp 1 issues the MMAs into one of two accumulators in TMEM (2 buffers x
// 2 column blocks x NR columns); warps 2..5 drain them, TMEM lane = output
// column, 16 rows per tcgen05.ld. Phase 1 writes z; phase 2 passes 16 rows at a
// time through a [16 x 256] shared tile from which warp w folds the rows
// r = w (mod 4) into running top-k lists kept in shared memory.
#pragma once

#include "common.cuh"
#include "heads.cuh"   // epoch_arrive

namespace md {
namespace skinny {

constexpr int kTile = 256;                   // output columns per unit
constexpr int kBK = 64;                      // reduction rows per stage
constexpr uint32_t kWBox = 64 * kBK * 2;     // 8 KB: 64 reduction rows x 64 columns, 128-byte swizzle
constexpr uint32_t kWBytes = 4 * kWBox;      // 32 KB per stage
constexpr int kThreads = 192;
constexpr int kChunk = 16;                   // rows per tcgen05.ld in the epilogue
constexpr int kMinRows = 2, kMaxRows = 32;   // the launcher's range of rows for this path

enum { EPI_SILU = 0, EPI_TOPK = 1 };

template <int NR>
struct Cfg {
  static constexpr uint32_t kXBytes = uint32_t(NR) * kBK * 2;   // NR rows x 64, K-major, 128-byte swizzle
  static constexpr uint32_t kStage = kWBytes + kXBytes;
  static constexpr int kStages = NR <= 16 ? 6 : (NR <= 32 ? 5 : 4);
  static constexpr uint32_t kTmemCols = NR * 4;                 // 64, 128 or 256
  static constexpr int kSmem = 1024 + kStages * int(kStage) + kChunk * kTile * 4 + NR * MD_MAX_KMAX * 8 + 256;
};

struct Args {
  int M;                 // live rows (phase 2: rows of the top-k)
  int d;                 // reduction length
  int N;                 // output columns per head (phase 1: d, phase 2: V)
  int Kh;                // heads of this phase: units = Kh * ntiles
  int ntiles, S;         // column tiles per head, stages per unit (d / 64)
  const uint16_t* h;     // phase 1: [M, d] residual
  const uint16_t* b1;    // phase 1: [Kh, d]
  uint16_t* z;           // phase 1 output: [Kz, NRz, d]
  int NRz;               // rows of each z matrix (the phase-2 row padding)
  int zg_mk;             // phase 1: row m of head k goes to row m * Kh + k of z[0] (shared projection)
  float* part;           // [gridDim.x][2][M][256]: partial sums of the units a CTA range cuts
  unsigned long long* tickets;   // [units] epoch tickets (md::heads::epoch_arrive)
  uint32_t epoch;        // this call's epoch
  float* cand_val;       // phase 2: [M, Kh, gridDim.x, kmax], one list per (row, head, CTA)
  int* cand_id;
  float* logits_dbg;     // phase 2: [M, Kh, N] or null
  const float* gumbel_u; // phase 2: [M, Kh, N] uniforms (sampled drafts) or null
  float inv_tau;
  int kmax;
  int kh;                // phase 2, shared projection: row m uses kph[m % kh]
  int kph[MD_MAX_K];
};

// First item of CTA c's range when W items are cut over G CTAs.
__device__ __forceinline__ long long range_lo(long long W, int G, int c) { return (long long)c * W / G; }

// The CTA whose range holds item i.
__device__ __forceinline__ int cta_of(long long W, int G, long long i) {
  int c = int(i * G / W);
  while (c + 1 < G && range_lo(W, G, c + 1) <= i) ++c;
  while (c > 0 && range_lo(W, G, c) > i) --c;
  return c;
}

// 16 consecutive fp32 columns at two TMEM addresses of this thread's lane
// (both loads in flight, one wait).
__device__ __forceinline__ void tmem_ld16x2(uint32_t ta, uint32_t tb, float (&va)[16], float (&vb)[16]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, "
      "[%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(ta));
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, "
      "[%16];"
      : "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(tb));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    va[i] = __uint_as_float(r[i]);
    vb[i] = __uint_as_float(r[16 + i]);
  }
}

// Phase-1 epilogue: rows r0 .. r0+15 at output columns o and o + 128 of head k.
__device__ __forceinline__ void silu_store(const Args& a, int k, int r0, int o, const float (&v0)[16],
                                           const float (&v1)[16]) {
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int oc = o + half * 128;
    if (oc >= a.d) continue;
    const float bias = bf16_to_f32(__ldg(a.b1 + size_t(k) * a.d + oc));
#pragma unroll
    for (int i = 0; i < kChunk; ++i) {
      const int r = r0 + i;
      const int zrow = a.zg_mk ? r * a.Kh + k : r;
      if (zrow >= a.NRz) continue;
      uint16_t zv = 0;
      if (r < a.M) {
        const float u = (half ? v1[i] : v0[i]) + bias;
        zv = f32_to_bf16_rne(bf16_to_f32(a.h[size_t(r) * a.d + oc]) + u / (1.0f + expf(-u)));
      }
      a.z[(size_t(a.zg_mk ? 0 : k) * a.NRz + zrow) * a.d + oc] = zv;
    }
  }
}

// Phase-2 fold of row r's 256 logits of tile t (trow, shared) into its running
// list (lvr / lir, shared; sorted best first, (value desc, id asc) order),
// warp-wide: lane j holds entry j, lane l the tile's columns l, l+32, ... .
// Tile values that beat the current kk-th entry are inserted best first, one
// per step, the kk-th entry (the threshold) rising after each insertion; a
// step ends the fold once no tile value beats it. After the first tiles of a
// row few values qualify, so most folds cost one pass of compares.
__device__ __forceinline__ void fold_row(const Args& a, const float* trow, float* lvr, int* lir, int r, int k, int t,
                                         int lane) {
  const int kk = param_at(a.kph, a.kh > 0 ? r % a.kh : k);
  const size_t base = (size_t(r) * a.Kh + k) * a.N;
  float vv[kTile / 32];
  int id[kTile / 32];
#pragma unroll
  for (int j = 0; j < kTile / 32; ++j) {
    const int c = lane + 32 * j;
    const int col = t * kTile + c;
    float x = trow[c];
    if (col < a.N) {
      if (a.logits_dbg) a.logits_dbg[base + col] = x;
      // sampled drafts rank the Gumbel keys logit / tau - ln(-ln u) instead
      if (a.gumbel_u) x = fmaf(x, a.inv_tau, gumbel_noise(__ldg(a.gumbel_u + base + col)));
      vv[j] = x;
      id[j] = col;
    } else {
      vv[j] = -INFINITY;
      id[j] = INT_MAX;
    }
  }
  float rv = lane < kk ? lvr[lane] : -INFINITY;
  int ri = lane < kk ? lir[lane] : INT_MAX;
  float tv = __shfl_sync(0xffffffffu, rv, kk - 1);
  int ti = __shfl_sync(0xffffffffu, ri, kk - 1);
  unsigned cand = 0;                       // this lane's tile values that beat the threshold
#pragma unroll
  for (int j = 0; j < kTile / 32; ++j)
    if (better(vv[j], id[j], tv, ti)) cand |= 1u << j;
  if (!__any_sync(0xffffffffu, cand != 0)) return;
  while (__any_sync(0xffffffffu, cand != 0)) {
    // the best remaining candidate of the warp
    float bv = -INFINITY;
    int bi = INT_MAX;
#pragma unroll
    for (int j = 0; j < kTile / 32; ++j)
      if (((cand >> j) & 1u) && better(vv[j], id[j], bv, bi)) {
        bv = vv[j];
        bi = id[j];
      }
    float wv = bv;
    int wi = bi;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, wv, off);
      const int oi = __shfl_xor_sync(0xffffffffu, wi, off);
      if (better(ov, oi, wv, wi)) {
        wv = ov;
        wi = oi;
      }
    }
    // insert it at its rank: entries ahead of it stay, the rest move down one lane
    const int pos = __popc(__ballot_sync(0xffffffffu, lane < kk && better(rv, ri, wv, wi)));
    const float uv = __shfl_up_sync(0xffffffffu, rv, 1);
    const int ui = __shfl_up_sync(0xffffffffu, ri, 1);
    if (lane < kk && lane > pos) {
      rv = uv;
      ri = ui;
    }
    if (lane == pos) {
      rv = wv;
      ri = wi;
    }
    tv = __shfl_sync(0xffffffffu, rv, kk - 1);
    ti = __shfl_sync(0xffffffffu, ri, kk - 1);
    // drop the inserted value and every value that no longer beats the threshold
#pragma unroll
    for (int j = 0; j < kTile / 32; ++j)
      if (((cand >> j) & 1u) && (id[j] == wi || !better(vv[j], id[j], tv, ti))) cand &= ~(1u << j);
  }
  if (lane < kk) {
    lvr[lane] = rv;
    lir[lane] = ri;
  }
}

template <int EPI, int NR>
__global__ void __launch_bounds__(kThreads, 1)
    heads_skinny_kernel(const __grid_constant__ CUtensorMap wmap, const __grid_constant__ CUtensorMap xmap, Args a) {
  using C = Cfg<NR>;
  constexpr int ns = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  float* tile = reinterpret_cast<float*>(smem + ns * C::kStage);        // [kChunk][256]
  float* lv = tile + kChunk * kTile;                                     // [NR][MD_MAX_KMAX] running lists
  int* li = reinterpret_cast<int*>(lv + NR * MD_MAX_KMAX);
  uint64_t* full = reinterpret_cast<uint64_t*>(li + NR * MD_MAX_KMAX);
  uint64_t* empty = full + ns;
  uint64_t* acc_full = empty + ns;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* mma_done = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  __shared__ int s_ok[2];
  __shared__ int s_ticket[2];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = gridDim.x;
  const int S = a.S;
  const long long W = (long long)a.Kh * a.ntiles * S;
  const long long i0 = range_lo(W, G, blockIdx.x), i1 = range_lo(W, G, blockIdx.x + 1);
  pdl_launch_dependents();

  if (threadIdx.x == 0) {
    for (int s = 0; s < ns; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&acc_full[b]), 1);
      mbar_init(smem_u32(&acc_empty[b]), 4);   // the four epilogue warps
    }
    mbar_init(smem_u32(mma_done), 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------- TMA producer -------------------------------
    if (lane == 0) {
      prefetch_tensormap(&wmap);
      prefetch_tensormap(&xmap);
      const uint64_t pol_w = policy_evict_first();   // weights: read once
      const uint64_t pol_x = policy_evict_last();    // rows: read by every CTA
      auto stage = [&](int slot) { return smem_u32(smem + size_t(slot) * C::kStage); };
      auto load_w = [&](long long w, int slot) {
        const int unit = int(w / S), s = int(w % S);
        const int k = unit / a.ntiles, t = unit % a.ntiles;
        const uint32_t fb = smem_u32(&full[slot]);
#pragma unroll
        for (int j = 0; j < 4; ++j)
          tma_load_3d_hint(stage(slot) + j * kWBox, &wmap, t * kTile + j * 64, s * kBK, k, fb, pol_w);
      };
      auto load_x = [&](long long w, int slot) {
        const int unit = int(w / S), s = int(w % S);
        const int xk = EPI == EPI_SILU ? 0 : unit / a.ntiles;
        tma_load_3d_hint(stage(slot) + kWBytes, &xmap, s * kBK, 0, xk, smem_u32(&full[slot]), pol_x);
      };
      // the first stages' weights do not depend on the previous kernel
      const int pre = int(min((long long)ns, i1 - i0));
      for (int j = 0; j < pre; ++j) {
        mbar_arrive_expect_tx(smem_u32(&full[j]), C::kStage);
        load_w(i0 + j, j);
      }
      pdl_wait_primary();
      for (int j = 0; j < pre; ++j) load_x(i0 + j, j);
      int it = pre;
      for (long long w = i0 + pre; w < i1; ++w, ++it) {
        const int slot = it % ns;
        if (!mbar_wait(smem_u32(&empty[slot]), ((it / ns) - 1) & 1)) {
          set_status(MD_DEV_TIMEOUT);
          break;
        }
        mbar_arrive_expect_tx(smem_u32(&full[slot]), C::kStage);
        load_w(w, slot);
        load_x(w, slot);
      }
      // the MMAs read the stages: wait until the last ones are consumed
      for (int j = (it > ns ? it - ns : 0); j < it; ++j) {
        if (!mbar_wait(smem_u32(&empty[j % ns]), (j / ns) & 1)) {
          set_status(MD_DEV_TIMEOUT);
          break;
        }
      }
    }
  } else if (warp == 1) {
    // -------------------------------- MMA issuer --------------------------------
    if (lane == 0) {
      constexpr uint32_t idesc = umma_idesc_bf16(128, NR, 1, 0);   // A (weights) N-major, B (rows) K-major
      int it = 0, lt = 0;
      bool ok = true;
      for (long long w = i0; w < i1 && ok; ++lt) {
        const int s_lo = int(w % S);
        const int s_hi = int(min((long long)S, s_lo + (i1 - w)));
        const int buf = lt & 1;
        if (lt >= 2 && !mbar_wait(smem_u32(&acc_empty[buf]), ((lt >> 1) - 1) & 1)) {
          set_status(MD_DEV_TIMEOUT);
          break;
        }
        tc_fence_after();
        for (int s = s_lo; s < s_hi; ++s, ++it) {
          const int slot = it % ns;
          if (!mbar_wait(smem_u32(&full[slot]), (it / ns) & 1)) {
            set_status(MD_DEV_TIMEOUT);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sb = smem_u32(smem + size_t(slot) * C::kStage);
          const uint64_t xdesc = umma_desc_sw128(sb + kWBytes, 16, 1024);
#pragma unroll
          for (int b = 0; b < 2; ++b) {
            // columns 128b .. 128b+127: two 64-column boxes, 8 KB apart
            const uint64_t wdesc = umma_desc_sw128(sb + b * 2 * kWBox, kWBox, 1024);
            const uint32_t dt = tmem + uint32_t((buf * 2 + b) * NR);
#pragma unroll
            for (int kk = 0; kk < kBK / 16; ++kk)
              umma_f16(dt, wdesc + uint64_t((kk * 2048) >> 4), xdesc + uint64_t((kk * 32) >> 4), idesc,
                       (s > s_lo || kk > 0) ? 1u : 0u);
          }
          umma_commit(smem_u32(&empty[slot]));
        }
        if (ok) umma_commit(smem_u32(&acc_full[buf]));
        w += s_hi - s_lo;
      }
      // every MMA issued has completed before the accumulators are released
      umma_commit(smem_u32(mma_done));
      if (!mbar_wait(smem_u32(mma_done), 0)) set_status(MD_DEV_TIMEOUT);
    }
  } else {
    // --------------------------------- epilogue ---------------------------------
    const int q = warp & 3;              // TMEM lanes 32q .. 32q+31
    const int e = warp - 2;              // rows r = e (mod 4) are this warp's to fold
    const int et = threadIdx.x - 64;     // 0 .. 127
    const int col0 = q * 32 + lane;      // this thread's columns of a unit: col0 and col0 + 128
    if (EPI == EPI_TOPK) {
      for (int r = e; r < NR; r += 4)
        if (lane < MD_MAX_KMAX) {
          lv[r * MD_MAX_KMAX + lane] = -INFINITY;
          li[r * MD_MAX_KMAX + lane] = INT_MAX;
        }
    }
    int lt = 0;
    for (long long w = i0; w < i1; ++lt) {
      const int unit = int(w / S);
      const int s_lo = int(w % S);
      const int s_hi = int(min((long long)S, s_lo + (i1 - w)));
      const int k = unit / a.ntiles, t = unit % a.ntiles;
      const bool whole = s_lo == 0 && s_hi == S;
      const long long wn = w + (s_hi - s_lo);
      const int buf = lt & 1;
      if (et == 0) s_ok[buf] = mbar_wait(smem_u32(&acc_full[buf]), (lt >> 1) & 1) ? 1 : 0;
      named_bar_sync(1, 128);
      if (!s_ok[buf]) {
        if (et == 0) set_status(MD_DEV_TIMEOUT);
        break;
      }
      tc_fence_after();
      const uint32_t tb = tmem + (uint32_t(q * 32) << 16) + uint32_t(buf * 2 * NR);
      bool finish = whole;
      int cf = 0, cl = 0;
      if (!whole) {
        // this CTA's part: slot 0 if it opens the CTA's range, else slot 1
        float* mine = a.part + (size_t(blockIdx.x) * 2 + (w == i0 ? 0 : 1)) * a.M * kTile;
#pragma unroll 1
        for (int ch = 0; ch < NR / kChunk; ++ch) {
          float v0[16], v1[16];
          tmem_ld16x2(tb + ch * kChunk, tb + NR + ch * kChunk, v0, v1);
#pragma unroll
          for (int i = 0; i < kChunk; ++i) {
            if (ch * kChunk + i < a.M) {
              mine[(ch * kChunk + i) * kTile + col0] = v0[i];
              mine[(ch * kChunk + i) * kTile + col0 + 128] = v1[i];
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&acc_empty[buf]));
        __threadfence();
        named_bar_sync(1, 128);
        if (et == 0) s_ticket[buf] = int(md::heads::epoch_arrive(&a.tickets[unit], a.epoch));
        named_bar_sync(1, 128);
        cf = cta_of(W, G, (long long)unit * S);
        cl = cta_of(W, G, (long long)unit * S + S - 1);
        finish = s_ticket[buf] == cl - cf;
        if (finish) __threadfence();
      }
      if (finish) {
#pragma unroll 1
        for (int ch = 0; ch < NR / kChunk; ++ch) {
          float v0[16], v1[16];
          if (whole) {
            tmem_ld16x2(tb + ch * kChunk, tb + NR + ch * kChunk, v0, v1);
            if (ch == NR / kChunk - 1) {
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(smem_u32(&acc_empty[buf]));
            }
          } else {
            // the unit's parts, summed in CTA order; two parts' loads in flight at once
#pragma unroll
            for (int i = 0; i < kChunk; ++i) v0[i] = v1[i] = 0.f;
            for (int c = cf; c <= cl; c += 2) {
              const bool two = c + 1 <= cl;
              const int sl0 = range_lo(W, G, c) >= (long long)unit * S ? 0 : 1;
              const int sl1 = two && range_lo(W, G, c + 1) >= (long long)unit * S ? 0 : 1;
              const float* pp0 = a.part + (size_t(c) * 2 + sl0) * a.M * kTile + size_t(ch) * kChunk * kTile;
              const float* pp1 = a.part + (size_t(two ? c + 1 : c) * 2 + sl1) * a.M * kTile + size_t(ch) * kChunk * kTile;
              float x0[kChunk], x1[kChunk], y0[kChunk], y1[kChunk];
#pragma unroll
              for (int i = 0; i < kChunk; ++i) {
                const bool live = ch * kChunk + i < a.M;
                x0[i] = live ? __ldcg(pp0 + i * kTile + col0) : 0.f;
                x1[i] = live ? __ldcg(pp0 + i * kTile + col0 + 128) : 0.f;
                y0[i] = live && two ? __ldcg(pp1 + i * kTile + col0) : 0.f;
                y1[i] = live && two ? __ldcg(pp1 + i * kTile + col0 + 128) : 0.f;
              }
#pragma unroll
              for (int i = 0; i < kChunk; ++i) {
                v0[i] += x0[i];
                v1[i] += x1[i];
                if (two) {
                  v0[i] += y0[i];
                  v1[i] += y1[i];
                }
              }
            }
          }
          if constexpr (EPI == EPI_SILU) {
            silu_store(a, k, ch * kChunk, t * kTile + col0, v0, v1);
          } else {
#pragma unroll
            for (int i = 0; i < kChunk; ++i) {
              tile[i * kTile + col0] = v0[i];
              tile[i * kTile + col0 + 128] = v1[i];
            }
            named_bar_sync(1, 128);
            for (int i = e; i < kChunk; i += 4) {
              const int r = ch * kChunk + i;
              if (r < a.M) fold_row(a, tile + i * kTile, lv + r * MD_MAX_KMAX, li + r * MD_MAX_KMAX, r, k, t, lane);
            }
            named_bar_sync(1, 128);
          }
        }
      }
      // phase 2: flush the lists when the range moves to another head or ends
      // (every CTA whose range meets head k writes a list for it, empty or not)
      if (EPI == EPI_TOPK && (wn >= i1 || int(wn / S) / a.ntiles != k)) {
        for (int r = e; r < a.M; r += 4) {
          const int kk = param_at(a.kph, a.kh > 0 ? r % a.kh : k);
          if (lane < kk) {
            const size_t cb = ((size_t(r) * a.Kh + k) * G + blockIdx.x) * a.kmax + lane;
            const int x = li[r * MD_MAX_KMAX + lane];
            a.cand_val[cb] = lv[r * MD_MAX_KMAX + lane];
            a.cand_id[cb] = x == INT_MAX ? -1 : x;
            lv[r * MD_MAX_KMAX + lane] = -INFINITY;
            li[r * MD_MAX_KMAX + lane] = INT_MAX;
          }
        }
      }
      w = wn;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

}  // namespace skinny
}  // namespace md
