// Verify attention on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
// VeriCache summary ("Riepilogo Tecnico: VeriCache", section "Algoritmo Principale",
// step 2): one forward pass over the full cache KV_full checks all k drafted tokens in
// parallel.  Query row (i, h) of a (batch, kv head) pair -- block position i in
// [0, n_q), head h of the GQA group -- sits at absolute position P + i and attends every
// key at position <= P + i: the whole prefix plus the block, causal inside the block.
//
// Decomposition.  A CTA owns one pair, one group of <= 256 query rows (two M = 128
// UMMA tiles; row r = i * g + h) and one split of the keys: the intersection of the
// call's key range with an absolute window [s * w, (s + 1) * w) (w a launch parameter:
// 2048-4096 keys chosen from the cache geometry by the entry point, smaller for the
// loop's decode-sized blocks).  Split windows and 64-key tiles sit at fixed absolute
// positions, so a row's result does not depend on n_q or on the other rows (a verify
// row equals the same token decoded alone).
//
// Per CTA (384 threads):
//   warp 0      TMA producer: K and V tiles [64 keys x D] (128-byte swizzle) into a
//               5-stage ring, one mbarrier per stage with the transaction byte count.
//   warp 1      TMEM allocator; one thread of warp 1 (M-tile 0) and one of warp 2
//   warp 2      (M-tile 1) issue the UMMAs: the tile's next S = Q K^T as soon as its
//               softmax has copied the current S out of TMEM, then O += P V once its
//               P is in.  Q of both M-tiles, K and V are read from shared memory (V as
//               an N-major B), P from TMEM.  (Q of M-tile 0 read from TMEM contended
//               with the softmax's TMEM loads: Q K^T took ~3x the time of P V.)
//   warps 4-7   softmax of M-tile 0, warps 8-11 of M-tile 1: one thread per query row
//               (TMEM lane); M-tile 1 keeps row r in lane (r + 64) % 128, so a part-
//               filled second tile lands on sub-partitions 2-3.  Scores in the log2
//               domain, running max kept unless it grows by more than 2^8 (then O in
//               TMEM is rescaled after the previous P.V), P written as bf16 into the
//               M-tile's P columns once the previous P.V has read them.
// TMEM columns: O0 [0,D), O1 [D,2D), S0, S1 (64 each), P0, P1 (32 each).
// Every mbarrier wait is bounded in time (pipeline waits by a launch parameter, 2 s
// unless vc_set_wait_limit changed it; teardown waits by 1 s); on expiry the CTA raises
// the library's device error word, lets its copies and products in flight land,
// releases TMEM and exits.
// The split partials (max, sum, unnormalised O) are merged by a second kernel in
// split order, optionally together with a carried state for chunked (streamed) keys.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <climits>
#include <functional>
#include <mutex>
#include <vector>

#include "tc05.cuh"
#include "vc_common.cuh"
#include "vc_internal.h"

namespace vc {

__device__ int g_vc_dev_error;   // bit 0: a bounded wait in the verify kernel expired

constexpr int kBN = 64;
constexpr int kVThreads = 384;
constexpr int kNSt = 5;
constexpr float kRescaleLog2 = 8.f;

struct VerifyParams {
  const __nv_bfloat16* q;   // [B, n_q, Hq, D]
  int n_q, Hq, Hkv, g, R;   // R = n_q * g rows per pair
  int64_t kv_start, kv_len, P;
  int split0, n_split;
  int split_keys;           // window of one split (absolute positions, multiple of kBN)
  float qk_scale2;          // scale * log2(e)
  float* ws_o;              // [pairs, n_split, R, D]
  float* ws_ml;             // [pairs, n_split, R, 2]
  uint64_t wait_ns;         // limit of every pipeline wait (teardown waits keep their own)
};

template <int D>
struct VLayout {
  static constexpr int kQTile = 128 * D * 2;        // Q of one M-tile (128-byte swizzle)
  static constexpr int kKVTile = kBN * D * 2;
  static constexpr int kQ0 = 0;
  static constexpr int kQ1 = kQ0 + kQTile;
  static constexpr int kK = kQ1 + kQTile;
  static constexpr int kV = kK + kNSt * kKVTile;
  static constexpr int kBar = kV + kNSt * kKVTile;
  static constexpr int kNBar = 2 * kNSt + 2 + 2 + 2 + 2 + 1;
  static constexpr int kTmemSlot = kBar + kNBar * 8;
  static constexpr int kAbort = kTmemSlot + 4;
  static constexpr int kTotal = kAbort + 4;
  static constexpr int kAlloc = kTotal + 1024;
  static constexpr uint32_t kColO = 0;
  static constexpr uint32_t kColS = 2 * D;
  static constexpr uint32_t kColP = 2 * D + 2 * kBN;
  static constexpr uint32_t kTmemCols = 512;
  static_assert(kColP + 2 * (kBN / 2) <= kTmemCols, "TMEM columns");
  static_assert(kQTile % 1024 == 0 && kKVTile % 1024 == 0, "align");
};

template <int D>
__global__ void __launch_bounds__(kVThreads, 1)
    verify_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                  const VerifyParams p) {
  pdl_wait();
  pdl_trigger();
  using L = VLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int s_local = blockIdx.x, rg = blockIdx.y, pair = blockIdx.z;
  const int b = pair / p.Hkv, kvh = pair - b * p.Hkv;
  const int row0 = rg * 256;
  const int rows_here = min(256, p.R - row0);
  const int n_mt = (rows_here + 127) >> 7;
  const int64_t part = (int64_t)pair * p.n_split + s_local;

  // key range of this split seen by this row group
  const int64_t win = (int64_t)(p.split0 + s_local) * p.split_keys;
  const int64_t a0 = max(p.kv_start, win);
  int64_t a1 = min(p.kv_start + p.kv_len, win + p.split_keys);
  a1 = min(a1, p.P + (row0 + rows_here - 1) / p.g + 1);
  const int n_tiles = a1 > a0 ? (int)((a1 - 1) / kBN - a0 / kBN + 1) : 0;
  const int64_t tile0 = a0 / kBN;

  if (n_tiles == 0) {  // nothing visible: empty partials
    for (int rr = threadIdx.x; rr < rows_here; rr += blockDim.x) {
      const int64_t o = part * p.R + row0 + rr;
      p.ws_ml[o * 2] = -INFINITY;
      p.ws_ml[o * 2 + 1] = 0.f;
      for (int d = 0; d < D; ++d) p.ws_o[o * D + d] = 0.f;
    }
    return;
  }

  auto bar = [&](int i) -> uint32_t { return sb + L::kBar + 8 * i; };
  auto b_kv_full = [&](int st) { return bar(st); };
  auto b_kv_empty = [&](int st) { return bar(kNSt + st); };
  auto b_s_full = [&](int mt) { return bar(2 * kNSt + mt); };
  auto b_s_free = [&](int mt) { return bar(2 * kNSt + 2 + mt); };
  auto b_p_full = [&](int mt) { return bar(2 * kNSt + 4 + mt); };
  auto b_o_done = [&](int mt) { return bar(2 * kNSt + 6 + mt); };
  const uint32_t b_teardown = bar(2 * kNSt + 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kAbort);
  auto nw_active = [&](int mt) {
    const int v = min(128, rows_here - mt * 128);
    return v > 0 ? (v + 31) >> 5 : 0;
  };

  if (threadIdx.x == 0) {
    for (int st = 0; st < kNSt; ++st) {
      tc::mbar_init(b_kv_full(st), 1);
      tc::mbar_init(b_kv_empty(st), n_mt);      // released by each M-tile's issuer
    }
    for (int mt = 0; mt < 2; ++mt) {
      tc::mbar_init(b_s_full(mt), 1);
      tc::mbar_init(b_s_free(mt), max(1, nw_active(mt)));
      tc::mbar_init(b_p_full(mt), max(1, nw_active(mt)));
      tc::mbar_init(b_o_done(mt), 1);
    }
    tc::mbar_init(b_teardown, n_mt);
    *abort_flag = 0;
    tc::fence_barrier_init();
  }
  if (warp == 1) tc::tmem_alloc(sb + L::kTmemSlot, L::kTmemCols);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + L::kTmemSlot);

  // Q rows of this group into shared memory (K-major, 128-byte swizzle; M-tile 0 row r at
  // row r, M-tile 1 row r at row (r + 64) % 128); padding rows are zero.
  if (warp >= 4) {
    const int mt = (warp - 4) >> 2, q4 = warp & 3;
    const int rl = 32 * q4 + lane;                       // TMEM lane / UMMA row
    const int grow = row0 + mt * 128 + ((rl + (mt ? 64 : 0)) & 127);
    const bool ok = mt < n_mt && grow < row0 + rows_here;
    const uint4* src = nullptr;
    if (ok) {
      const int i = grow / p.g, hl = grow - i * p.g;
      src = reinterpret_cast<const uint4*>(p.q + (((int64_t)b * p.n_q + i) * p.Hq + kvh * p.g + hl) * D);
    }
    {
      const int qbase = mt == 0 ? L::kQ0 : L::kQ1;
#pragma unroll
      for (int ch = 0; ch < D / 8; ++ch) {
        const uint4 v = ok ? __ldg(src + ch) : make_uint4(0u, 0u, 0u, 0u);
        const int cb = ch >> 3, cc = ch & 7;
        *reinterpret_cast<uint4*>(smem + qbase + cb * (128 * 128) + rl * 128 +
                                  ((cc ^ (rl & 7)) << 4)) = v;
      }
      tc::fence_proxy_async();
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();

  auto raise = [&]() {
    *abort_flag = 1;
    atomicOr(&g_vc_dev_error, 1);
  };

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tc::prefetch_tmap(&tmK);
      tc::prefetch_tmap(&tmV);
      int issued = 0;
      for (int t = 0; t < n_tiles; ++t) {
        const int st = t % kNSt;
        if (t >= kNSt && !tc::mbar_wait(b_kv_empty(st), ((t / kNSt) - 1) & 1, abort_flag, p.wait_ns)) {
          raise();
          break;
        }
        const uint32_t fb = b_kv_full(st);
        tc::mbar_expect_tx(fb, 2 * L::kKVTile);
        const int y = (int)((tile0 + t) * kBN - p.kv_start);
#pragma unroll
        for (int cb = 0; cb < D / 64; ++cb) {
          tc::tma_load_3d(sb + L::kK + st * L::kKVTile + cb * (kBN * 128), &tmK, fb, cb * 64, y,
                          pair);
          tc::tma_load_3d(sb + L::kV + st * L::kKVTile + cb * (kBN * 128), &tmV, fb, cb * 64, y,
                          pair);
        }
        issued = t + 1;
      }
      // loads still in flight must land before shared memory is released
      for (int t = max(0, issued - kNSt); t < issued; ++t)
        tc::mbar_wait(b_kv_full(t % kNSt), (t / kNSt) & 1, nullptr, 1000000000ull);
    }
  } else if (warp == 1 || warp == 2) {
    // ------------------------------------------------------------ UMMA issuers
    // One thread per M-tile (warp 1: M-tile 0, warp 2: M-tile 1), so neither tile's
    // products wait behind the other tile's softmax.
    const int mt = warp - 1;
    if (lane == 0 && mt < n_mt) {
      const uint32_t id_qk = tc::idesc_bf16_f32(128, kBN, false, false);
      const uint32_t id_pv = tc::idesc_bf16_f32(128, D, false, true);
      auto qk = [&](int t) {
        const int st = t % kNSt;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint32_t bb = sb + L::kK + st * L::kKVTile + (ks >> 2) * (kBN * 128) + (ks & 3) * 32;
          const uint64_t bdesc = tc::sdesc_sw128(bb, 16, 1024);
          const uint32_t a = sb + (mt == 0 ? L::kQ0 : L::kQ1) + (ks >> 2) * (128 * 128) +
                             (ks & 3) * 32;
          tc::umma_ss(tmem + L::kColS + mt * kBN, tc::sdesc_sw128(a, 16, 1024), bdesc, id_qk,
                      ks > 0 ? 1u : 0u);
        }
      };
      auto pv = [&](int t) {
        const int st = t % kNSt;
#pragma unroll
        for (int ks = 0; ks < kBN / 16; ++ks) {
          const uint32_t bb = sb + L::kV + st * L::kKVTile + ks * 16 * 128;
          tc::umma_ts(tmem + L::kColO + mt * D, tmem + L::kColP + mt * (kBN / 2) + ks * 8,
                      tc::sdesc_sw128(bb, kBN * 128, 1024), id_pv, (t > 0 || ks > 0) ? 1u : 0u);
        }
      };
      bool ok = tc::mbar_wait(b_kv_full(0), 0, abort_flag, p.wait_ns);
      if (ok) {
        tc::tc_fence_after();
        qk(0);
        tc::umma_commit(b_s_full(mt));
      }
      for (int t = 0; ok && t < n_tiles; ++t) {
        if (t + 1 < n_tiles) {
          // the next Q K^T as soon as the softmax has copied this S out of TMEM
          if (!(ok = tc::mbar_wait(b_kv_full((t + 1) % kNSt), ((t + 1) / kNSt) & 1,
                                   abort_flag, p.wait_ns)))
            break;
          if (!(ok = tc::mbar_wait(b_s_free(mt), t & 1, abort_flag, p.wait_ns))) break;
          tc::tc_fence_after();
          qk(t + 1);
          tc::umma_commit(b_s_full(mt));
        }
        if (!(ok = tc::mbar_wait(b_p_full(mt), t & 1, abort_flag, p.wait_ns))) break;
        tc::tc_fence_after();
        pv(t);
        tc::umma_commit(b_o_done(mt));
        tc::umma_commit(b_kv_empty(t % kNSt));   // one arrival per M-tile
      }
      if (!ok) raise();
      // every UMMA issued must retire before TMEM is released
      tc::umma_commit(b_teardown);
      tc::mbar_wait(b_teardown, 0, nullptr, 1000000000ull);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax
    const int mt = (warp - 4) >> 2, q4 = warp & 3;
    const int valid_mt = min(128, rows_here - mt * 128);
    const int rot = mt ? 64 : 0;
    if (mt < n_mt && ((32 * q4 + rot) & 127) < valid_mt) {
      const int r = (32 * q4 + lane + rot) & 127;
      const int grow = row0 + mt * 128 + r;
      const bool row_ok = r < valid_mt;
      const int64_t limit = p.P + grow / p.g;
      const uint32_t lane_t = tmem + ((uint32_t)(32 * q4) << 16);
      const uint32_t s_t = lane_t + L::kColS + mt * kBN;
      const uint32_t p_t = lane_t + L::kColP + mt * (kBN / 2);
      const uint32_t o_t = lane_t + L::kColO + mt * D;
      float m_used = -INFINITY, lsum = 0.f;
      bool ok = true;
      for (int t = 0; t < n_tiles; ++t) {
        ok = __all_sync(0xffffffffu, tc::mbar_wait(b_s_full(mt), t & 1, abort_flag, p.wait_ns));
        if (!ok) break;
        tc::tc_fence_after();
        uint32_t sr[64];
        tc::tmem_ld32(s_t, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
        tc::tmem_ld32(s_t + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
        tc::tmem_wait_ld();
        // S is in registers: the next Q K^T may overwrite it
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(b_s_free(mt));
        // visible columns j in [lo, hi] of this tile for this row (int32, clamped); a
        // padding row counts as seeing the whole tile (its values are never used)
        const int64_t key0 = (tile0 + t) * kBN;
        const int lo = row_ok ? (int)max((int64_t)0, min((int64_t)kBN, a0 - key0)) : 0;
        const int hi = row_ok
            ? (int)max((int64_t)-1, min((int64_t)(kBN - 1), min(a1 - 1, limit) - key0))
            : kBN - 1;
        // Row max on the raw scores (the scale is positive, so it commutes with max);
        // a tile every row of the warp sees whole skips the per-column mask.
        // (eight independent partial maxima: a short dependency chain)
        float mx8[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) mx8[u] = -INFINITY;
        if (__all_sync(0xffffffffu, lo == 0 && hi == kBN - 1)) {
#pragma unroll
          for (int j = 0; j < 64; ++j) mx8[j & 7] = fmaxf(mx8[j & 7], __uint_as_float(sr[j]));
        } else {
#pragma unroll
          for (int j = 0; j < 64; ++j) {
            const float v = (j >= lo && j <= hi) ? __uint_as_float(sr[j]) : -INFINITY;
            sr[j] = __float_as_uint(v);
            mx8[j & 7] = fmaxf(mx8[j & 7], v);
          }
        }
        const float mraw = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                                 fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
        const float mx = mraw * p.qk_scale2;
        const float m_new = fmaxf(m_used, mx);
        const bool resc = m_new > m_used + kRescaleLog2;
        const float alpha = resc ? ex2(m_used - m_new) : 1.f;
        if (resc) m_used = m_new;
        const float m_safe = m_used == -INFINITY ? 0.f : m_used;
        // P (bf16, keys packed two per column) in registers first -- it does not depend on
        // O -- so the exponentials overlap the previous P.V; row sum in eight partial sums
        // added in a fixed order
        uint32_t pw[32];
        float rs8[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) rs8[u] = 0.f;
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          const float e0 = ex2(fmaf(__uint_as_float(sr[2 * c]), p.qk_scale2, -m_safe));
          const float e1 = ex2(fmaf(__uint_as_float(sr[2 * c + 1]), p.qk_scale2, -m_safe));
          rs8[(2 * c) & 7] += e0;
          rs8[(2 * c + 1) & 7] += e1;
          pw[c] = pack_bf16x2(e0, e1);
        }
        // the previous P.V must be done before O is rescaled or P overwritten
        if (t > 0) {
          ok = __all_sync(0xffffffffu, tc::mbar_wait(b_o_done(mt), (t - 1) & 1, abort_flag, p.wait_ns));
          if (!ok) break;
          tc::tc_fence_after();
        }
        if (t > 0 && __any_sync(0xffffffffu, resc)) {
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t o[32];
            tc::tmem_ld32(o_t + 32 * c, o);
            tc::tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
            tc::tmem_st32(o_t + 32 * c, o);
          }
          tc::tmem_wait_st();
        }
        lsum *= alpha;
        tc::tmem_st32(p_t, pw);
        lsum += ((rs8[0] + rs8[1]) + (rs8[2] + rs8[3])) + ((rs8[4] + rs8[5]) + (rs8[6] + rs8[7]));
        tc::tmem_wait_st();
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(b_p_full(mt));
      }
      if (ok) {
        const int tl = n_tiles - 1;
        ok = __all_sync(0xffffffffu, tc::mbar_wait(b_o_done(mt), tl & 1, abort_flag, p.wait_ns));
      }
      if (!ok) {
        raise();
      } else {
        tc::tc_fence_after();
        const int64_t o_row = part * p.R + grow;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          tc::tmem_ld32(o_t + 32 * c, o);
          tc::tmem_wait_ld();
          if (row_ok) {
            float4* dst = reinterpret_cast<float4*>(p.ws_o + o_row * D + 32 * c);
#pragma unroll
            for (int e = 0; e < 8; ++e)
              dst[e] = make_float4(__uint_as_float(o[4 * e]), __uint_as_float(o[4 * e + 1]),
                                   __uint_as_float(o[4 * e + 2]), __uint_as_float(o[4 * e + 3]));
          }
        }
        if (row_ok) {
          p.ws_ml[o_row * 2] = m_used;
          p.ws_ml[o_row * 2 + 1] = lsum;
        }
      }
    }
  }

  tc::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, L::kTmemCols);
  }
}

// Merge split partials (plus the carried state) for one query row: one warp per row,
// lanes holding D/32 output channels each.  The lanes load the splits' (max, sum) at
// once (kept in registers for up to 64 splits); the unnormalised outputs of 32 (D 64) or
// 16 (D 128) splits are loaded together before any is used, so a row costs a few L2
// round trips, not one per split.  The sums run in split order
// after the carried state, the same order whatever the number of rows, which keeps a
// verify row bit-identical to the same position decoded alone.
constexpr int kVCombWarps = 8;

template <int D, typename OutT>
__global__ void __launch_bounds__(kVCombWarps * 32) verify_combine_kernel(
    const float* __restrict__ ws_o, const float* __restrict__ ws_ml, int n_split, int R, int g,
    int n_q, int Hq, int Hkv, int flags, float* m_state, float* l_state, float* acc_state,
    OutT* __restrict__ out, int rows) {
  pdl_wait();
  pdl_trigger();
  constexpr int DPL = D / 32;
  constexpr int CH = 64 / DPL;                    // splits whose outputs are loaded at once
  const int lane = threadIdx.x & 31;
  const int gr = blockIdx.x * kVCombWarps + (threadIdx.x >> 5);
  if (gr >= rows) return;
  const int pair = gr / R, row = gr - pair * R;
  const int i = row / g, hl = row - i * g;
  const int b = pair / Hkv, kvh = pair - b * Hkv;
  const int64_t sidx = ((int64_t)b * n_q + i) * Hq + kvh * g + hl;
  const bool carry = m_state != nullptr && !(flags & VC_VERIFY_FIRST);
  const int64_t pr0 = (int64_t)pair * n_split * R + row;   // split s: pr0 + s * R
  // (max, sum) of up to 64 splits stay in registers (lane: splits lane and 32 + lane);
  // more splits are read again group by group below
  float2 mlr[2] = {make_float2(-INFINITY, 0.f), make_float2(-INFINITY, 0.f)};
#pragma unroll
  for (int h = 0; h < 2; ++h)
    if (32 * h + lane < n_split)
      mlr[h] = *reinterpret_cast<const float2*>(ws_ml + (pr0 + (int64_t)(32 * h + lane) * R) * 2);
  float M = carry ? m_state[sidx] : -INFINITY;
  M = fmaxf(M, fmaxf(mlr[0].x, mlr[1].x));
  for (int s = 64 + lane; s < n_split; s += 32) M = fmaxf(M, ws_ml[(pr0 + (int64_t)s * R) * 2]);
  M = warp_max_xor(M, 5);
  float Ls = 0.f, O[DPL];
#pragma unroll
  for (int t = 0; t < DPL; ++t) O[t] = 0.f;
  if (carry) {
    const float cm = m_state[sidx];
    if (cm > -INFINITY) {
      const float f = ex2(cm - M);
      Ls = l_state[sidx] * f;
#pragma unroll
      for (int t = 0; t < DPL; ++t) O[t] = acc_state[sidx * D + lane * DPL + t] * f;
    }
  }
  // the splits in order: weight exp2(m_s - M), sums and outputs added one split at a time
  for (int s0 = 0; s0 < n_split; s0 += 32) {
    const int cnt32 = min(32, n_split - s0);
    float2 ml = make_float2(-INFINITY, 0.f);
    if (s0 < 64) {
      ml = s0 == 0 ? mlr[0] : mlr[1];
    } else if (lane < cnt32) {
      ml = *reinterpret_cast<const float2*>(ws_ml + (pr0 + (int64_t)(s0 + lane) * R) * 2);
    }
    float wl = 0.f, ll = 0.f;
    if (lane < cnt32 && ml.x > -INFINITY) {
      wl = ex2(ml.x - M);
      ll = ml.y;
    }
    for (int c0 = 0; c0 < cnt32; c0 += CH) {
      float v[CH][DPL];
#pragma unroll
      for (int j = 0; j < CH; ++j) {
        const int s = s0 + min(c0 + j, cnt32 - 1);
        const float* src = ws_o + (pr0 + (int64_t)s * R) * D + lane * DPL;
        if constexpr (DPL == 4) {
          const float4 t = *reinterpret_cast<const float4*>(src);
          v[j][0] = t.x; v[j][1] = t.y; v[j][2] = t.z; v[j][3] = t.w;
        } else {
          const float2 t = *reinterpret_cast<const float2*>(src);
          v[j][0] = t.x; v[j][1] = t.y;
        }
      }
      asm volatile("" ::: "memory");              // every load of the batch issued first
#pragma unroll
      for (int j = 0; j < CH; ++j) {
        const float w = __shfl_sync(0xffffffffu, wl, (c0 + j) & 31);
        const float lj = __shfl_sync(0xffffffffu, ll, (c0 + j) & 31);
        if (c0 + j < cnt32 && w != 0.f) {         // warp-uniform
          Ls = fmaf(lj, w, Ls);
#pragma unroll
          for (int t = 0; t < DPL; ++t) O[t] = fmaf(v[j][t], w, O[t]);
        }
      }
    }
  }
  if (flags & VC_VERIFY_LAST) {
    const float inv = 1.f / Ls;
#pragma unroll
    for (int t = 0; t < DPL; ++t) store_out(out + sidx * D + lane * DPL + t, O[t] * inv);
  } else {
#pragma unroll
    for (int t = 0; t < DPL; ++t) acc_state[sidx * D + lane * DPL + t] = O[t];
    if (lane == 0) {
      m_state[sidx] = M;
      l_state[sidx] = Ls;
    }
  }
}

// ------------------------------------------------------------------ host side
namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  }
  return fn;
}

// [pairs][L_cap][D] bf16 viewed as a 3-D tensor whose key extent is kv_len, so rows past
// the live range (and negative rows) read as zero.
bool make_kv_map(CUtensorMap* m, const void* base, int D, int64_t kv_len, int64_t L_cap,
                 int pairs) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)kv_len, (cuuint64_t)pairs};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)L_cap * D * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)kBN, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
            es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct Plan {
  int pairs, g, R, split0, n_split, n_rg;
  size_t ws_bytes;
};

Plan plan(int B, int n_q, int Hq, int Hkv, int D, int64_t kv_start, int64_t kv_len,
          int split_keys) {
  Plan pl;
  pl.pairs = B * Hkv;
  pl.g = Hq / Hkv;
  pl.R = n_q * pl.g;
  pl.split0 = (int)(kv_start / split_keys);
  pl.n_split = (int)((kv_start + kv_len - 1) / split_keys) - pl.split0 + 1;
  pl.n_rg = (pl.R + 255) / 256;
  pl.ws_bytes = (size_t)pl.pairs * pl.n_split * pl.R * ((size_t)D + 2) * sizeof(float);
  return pl;
}

}  // namespace

size_t verify_workspace_bytes(int B, int n_q, int Hq, int Hkv, int D, int64_t kv_start,
                              int64_t kv_len, int split_keys) {
  return plan(B, n_q, Hq, Hkv, D, kv_start, kv_len, split_keys).ws_bytes + 256;
}

constexpr int kWindowMin = 2048;

size_t verify_workspace_bytes_any(int B, int n_q, int Hq, int Hkv, int D, int64_t kv_start,
                                  int64_t kv_len) {
  size_t m = 0;
  for (int w = kVerifySplitKeys; w >= kWindowMin; w -= kBN)
    m = std::max(m, verify_workspace_bytes(B, n_q, Hq, Hkv, D, kv_start, kv_len, w));
  return m;
}

// Among the windows of 2048..4096 keys (multiples of 64), the one whose CTAs, placed in
// launch order (pair-major, splits in order) on the SMs as each frees up (one resident
// CTA per SM), finish first, a CTA costing its 64-key tiles plus four for its start; ties
// go to the larger window.  Fewer, larger splits leave the last wave of CTAs half empty
// at some sizes (512 CTAs of 64 tiles on 148 SMs), slightly smaller ones fill it.  The
// choice is cached per (pairs, L_cap, SM count); caches with less than one wave of
// 4096-key CTAs, or very large ones, keep 4096.
int verify_window(int64_t pairs, int64_t L_cap) {
  struct Chosen { int64_t pairs, L_cap; int sms, w; };
  static std::mutex mu;
  static std::vector<Chosen> chosen;
  const int sms = num_sms();
  {
    std::lock_guard<std::mutex> lk(mu);
    for (const Chosen& c : chosen)
      if (c.pairs == pairs && c.L_cap == L_cap && c.sms == sms) return c.w;
  }
  int best = kVerifySplitKeys;
  const int64_t ctas4096 = pairs * ((L_cap + kVerifySplitKeys - 1) / kVerifySplitKeys);
  if (pairs > 0 && L_cap > 0 && ctas4096 >= sms &&
      pairs * ((L_cap + kWindowMin - 1) / kWindowMin) <= 65536) {
    int64_t best_t = INT64_MAX;
    std::vector<int64_t> heap;
    for (int w = kVerifySplitKeys; w >= kWindowMin; w -= kBN) {
      heap.assign(sms, 0);                      // min-heap of SM free times
      const int64_t n_full = L_cap / w, rem = L_cap % w;
      auto place = [&](int64_t cost) {
        std::pop_heap(heap.begin(), heap.end(), std::greater<int64_t>());
        heap.back() += cost;
        std::push_heap(heap.begin(), heap.end(), std::greater<int64_t>());
      };
      for (int64_t pr = 0; pr < pairs; ++pr) {
        for (int64_t sp = 0; sp < n_full; ++sp) place(w / kBN + 4);
        if (rem) place((rem + kBN - 1) / kBN + 4);
      }
      const int64_t t = *std::max_element(heap.begin(), heap.end());
      if (t < best_t) { best_t = t; best = w; }
    }
  }
  std::lock_guard<std::mutex> lk(mu);
  chosen.push_back({pairs, L_cap, sms, best});
  return best;
}

template <int D>
static vc_status run_verify(const Plan& pl, const VerifyParams& vp, const CUtensorMap& mk,
                            const CUtensorMap& mv, int flags, float* m, float* l, float* acc,
                            void* out, cudaStream_t stream) {
  using L = VLayout<D>;
  VC_CUDA(grant_smem((const void*)verify_kernel<D>, L::kAlloc));
  dim3 grid(pl.n_split, pl.n_rg, pl.pairs);
  VC_CUDA(launch_pdl(verify_kernel<D>, grid, dim3(kVThreads), L::kAlloc, stream, 1, mk, mv, vp));
  VC_CUDA(cudaGetLastError());
  const int rows = pl.pairs * pl.R;
  const int cblocks = (rows + kVCombWarps - 1) / kVCombWarps;
  if (flags & VC_OUT_F32)
    VC_CUDA(launch_pdl(verify_combine_kernel<D, float>, dim3(cblocks), dim3(kVCombWarps * 32), 0,
                       stream, 1, (const float*)vp.ws_o, (const float*)vp.ws_ml, pl.n_split, pl.R,
                       pl.g, vp.n_q, vp.Hq, vp.Hkv, flags, m, l, acc, static_cast<float*>(out),
                       rows));
  else
    VC_CUDA(launch_pdl(verify_combine_kernel<D, __nv_bfloat16>, dim3(cblocks),
                       dim3(kVCombWarps * 32), 0, stream, 1, (const float*)vp.ws_o,
                       (const float*)vp.ws_ml, pl.n_split, pl.R, pl.g, vp.n_q, vp.Hq, vp.Hkv,
                       flags, m, l, acc, static_cast<__nv_bfloat16*>(out), rows));
  VC_CUDA(cudaGetLastError());
  return VC_OK;
}

// Limit of the verify kernel's pipeline waits, for the launches that follow.
static std::atomic<uint64_t> g_verify_wait_ns{kDefaultWaitNs};

uint64_t set_verify_wait_ns(uint64_t ns) { return g_verify_wait_ns.exchange(ns); }

vc_status launch_verify(const void* q, int B, int n_q, int Hq, int Hkv, int D, const void* k,
                        const void* v, int64_t L_cap, int64_t kv_start, int64_t kv_len,
                        int64_t P, float* m, float* l, float* acc, int flags, float scale,
                        void* out, void* ws, size_t ws_bytes, cudaStream_t stream,
                        int split_keys) {
  if (split_keys < kBN || split_keys % kBN) return fail(VC_ERR_INVALID, "verify: split window");
  const Plan pl = plan(B, n_q, Hq, Hkv, D, kv_start, kv_len, split_keys);
  if (ws_bytes < pl.ws_bytes) return fail(VC_ERR_INVALID, "verify workspace too small");
  if (P + n_q > (int64_t)1 << 31) return fail(VC_ERR_UNSUPPORTED, "verify: positions >= 2^31");
  CUtensorMap mk, mv;
  if (!make_kv_map(&mk, k, D, kv_len, L_cap, pl.pairs) ||
      !make_kv_map(&mv, v, D, kv_len, L_cap, pl.pairs))
    return fail(VC_ERR_CUDA, "cuTensorMapEncodeTiled failed");
  VerifyParams vp;
  vp.q = static_cast<const __nv_bfloat16*>(q);
  vp.n_q = n_q;
  vp.Hq = Hq;
  vp.Hkv = Hkv;
  vp.g = pl.g;
  vp.R = pl.R;
  vp.kv_start = kv_start;
  vp.kv_len = kv_len;
  vp.P = P;
  vp.split0 = pl.split0;
  vp.n_split = pl.n_split;
  vp.split_keys = split_keys;
  vp.qk_scale2 = scale * kLog2e;
  vp.ws_o = static_cast<float*>(ws);
  vp.ws_ml = vp.ws_o + (size_t)pl.pairs * pl.n_split * pl.R * D;
  vp.wait_ns = g_verify_wait_ns.load();
  if (D == 128) return run_verify<128>(pl, vp, mk, mv, flags, m, l, acc, out, stream);
  return run_verify<64>(pl, vp, mk, mv, flags, m, l, acc, out, stream);
}

vc_status read_device_error(int32_t* value, int clear) {
  int v = 0;
  VC_CUDA(cudaMemcpyFromSymbol(&v, g_vc_dev_error, sizeof(int)));
  if (value) *value = v;
  if (clear) {
    const int z = 0;
    VC_CUDA(cudaMemcpyToSymbol(g_vc_dev_error, &z, sizeof(int)));
  }
  return VC_OK;
}

}  // namespace vc
