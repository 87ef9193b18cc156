// Verify attention on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
// VeriCache summary ("Riepilogo Tecnico: VeriCache", section "Algoritmo Principale",
// step 2): one forward pass over the full cache KV_full checks all k drafted tokens in
// parallel.  Query row (i, h) of a (batch, kv head) pair -- block position i in
// [0, n_q), head h of the GQA group -- sits at absolute position P + i and attends every
// key at position <= P + i: the whole prefix plus the block, causal inside the block.
//
// Decomposition.  A CTA owns one pair, one group of N <= 160 query rows (row r = i * g +
// h; N is the UMMA N, a multiple of 16, the same for every group of a call) and one split
// of the keys: the intersection of the call's key range with an absolute window
// [s * 4096, (s + 1) * 4096).  Split windows and 128-key tiles sit at fixed absolute
// positions, so a row's result does not depend on n_q or on the other rows (a verify row
// equals the same token decoded alone).
//
// Orientation.  Key positions are the UMMA M = 128 and query rows the N: per 128-key tile
//     S^T [128 keys x N] = K [128 x D] . Q^T          (A = K tile, B = Q, both K-major)
//     O^T [D x N]      += V^T [D x 128] . P^T [128 x N]  (A = V tile read MN-major, B = P^T)
// so a group of 132 rows (k = 32 at g = 4) costs 144 columns of tensor work instead of two
// M = 128 tiles, and the softmax of a tile is spread over all four TMEM sub-partitions.
//
// Per CTA (256 threads):
//   warp 0, lane 0   TMA producer of K tiles, warp 3 lane 0 of V tiles ([128 keys x 64
//                    dims] boxes, 128-byte swizzle), each into its own 2-slot ring with a
//                    full / empty mbarrier pair per slot.
//   warp 1           TMEM allocator; lane 0 issues every UMMA: QK of tile t as soon as the
//                    softmax has copied S of tile t-1 out of TMEM, then PV of tile t-1 once
//                    its P^T is in shared memory.
//   warps 4-7        softmax: thread (w, lane) owns key 32 (w - 4) + lane of the tile (its
//                    TMEM lane) and holds that key's N scores.  Scores are in the log2
//                    domain against a per-row reference maximum m_r that is raised only
//                    when a tile's scores exceed it by more than 2^8 (the four warps vote
//                    once per tile; the rare raise finds the exact column maxima with warp
//                    reductions, then rescales O^T and the sums).  p = 2^(s - m_r) is
//                    written as bf16 P^T (MN-major, 128-byte swizzle) and summed per
//                    (key lane, row) in TMEM; the lanes' sums are added in a fixed order at
//                    the end.  A split's partial (m_r, l_r, unnormalised O) goes to the
//                    workspace.
// TMEM columns: O^T [0, 160), S^T [160, 320), per-lane row sums [320, 480).
// Every mbarrier wait is bounded in time (pipeline waits by a launch parameter, 2 s
// unless vc_set_wait_limit changed it; teardown waits by 1 s); on expiry the CTA raises
// the library's device error word, lets its copies and products in flight land,
// releases TMEM and exits.
// The split partials are merged by a second kernel in split order, optionally together
// with a carried state for chunked (streamed) keys.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <climits>

#include "tc05.cuh"
#include "vc_common.cuh"
#include "vc_internal.h"

namespace vc {

__device__ int g_vc_dev_error;   // bit 0: a bounded wait in the verify kernel expired

constexpr int kSplitKeys = 4096;
constexpr int kBN = 128;          // keys per tile (UMMA M)
constexpr int kNMax = 160;        // query rows per CTA (UMMA N <= kNMax)
constexpr int kVThreads = 256;
constexpr float kRescaleLog2 = 8.f;
constexpr float kPadRowMax = 1e30f;   // reference maximum of padding rows: p = 0, no votes

struct VerifyParams {
  const __nv_bfloat16* q;   // [B, n_q, Hq, D]
  int n_q, Hq, Hkv, g, R;   // R = n_q * g rows per pair
  int N;                    // rows per CTA group (multiple of 16, <= kNMax)
  int64_t kv_start, kv_len, P;
  int split0, n_split;
  float qk_scale2;          // scale * log2(e)
  float* ws_o;              // [pairs, n_split, R, D]
  float* ws_ml;             // [pairs, n_split, R, 2]
  uint64_t wait_ns;         // limit of every pipeline wait (teardown waits keep their own)
};

template <int D>
struct VLayout {
  static constexpr int kQBlk = kNMax * 128;             // 64 dims of the group's Q rows
  static constexpr int kKVBlk = kBN * 128;              // 64 dims of a K or V tile
  static constexpr int kKVSlot = (D / 64) * kKVBlk;
  static constexpr int kPBlk = kBN * 128;               // 64 rows of P^T (one 128 B row per key)
  static constexpr int kPBlocks = (kNMax + 63) / 64;
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + (D / 64) * kQBlk;
  static constexpr int kV = kK + 2 * kKVSlot;
  static constexpr int kP = kV + 2 * kKVSlot;
  static constexpr int kBar = kP + kPBlocks * kPBlk;
  static constexpr int kNBar = 17;
  static constexpr int kTmemSlot = kBar + kNBar * 8;
  static constexpr int kAbort = kTmemSlot + 4;
  static constexpr int kFlags = kAbort + 4;              // int [2][4] votes
  static constexpr int kMUsed = kFlags + 48;             // float [kNMax] reference maxima
  static constexpr int kAlpha = kMUsed + kNMax * 4;      // float [kNMax] rescale factors
  static constexpr int kWMax = kAlpha + kNMax * 4;       // float [4][kNMax] warp maxima
  static constexpr int kTotal = kWMax + 4 * kNMax * 4;
  static constexpr int kAlloc = kTotal + 1024;
  static constexpr int kRedStride = kNMax + 1;           // row sums, per key lane (floats)
  static constexpr uint32_t kColO = 0, kColS = kNMax, kColL = 2 * kNMax;
  static constexpr uint32_t kTmemCols = 512;
  static_assert(kColL + kNMax <= kTmemCols, "TMEM columns");
  static_assert(kK % 1024 == 0 && kV % 1024 == 0 && kP % 1024 == 0, "align");
  static_assert(kMUsed % 16 == 0, "align");
  static_assert(kAlloc <= 232448, "shared memory");
  static_assert(128 * kRedStride * 4 <= kBar - kK, "row-sum staging fits the idle K/V/P buffers");
};

// Largest value over the warp (no NaN), through the order-preserving integer image.
__device__ __forceinline__ float warp_max_f32(float v) {
  const int i = __float_as_int(v);
  int key = i >= 0 ? i : (i ^ 0x7fffffff);
  key = __reduce_max_sync(0xffffffffu, key);
  return __int_as_float(key >= 0 ? key : (key ^ 0x7fffffff));
}

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
  const int N = p.N;
  const int row0 = rg * N;
  const int rows_here = min(N, p.R - row0);
  const int64_t part = (int64_t)pair * p.n_split + s_local;

  // key range of this split seen by this row group
  const int64_t win = (int64_t)(p.split0 + s_local) * kSplitKeys;
  const int64_t a0 = max(p.kv_start, win);
  int64_t a1 = min(p.kv_start + p.kv_len, win + kSplitKeys);
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
  auto b_k_full = [&](int s) { return bar(s); };
  auto b_k_empty = [&](int s) { return bar(2 + s); };
  auto b_v_full = [&](int s) { return bar(4 + s); };
  auto b_v_empty = [&](int s) { return bar(6 + s); };
  const uint32_t b_s_full = bar(8), b_s_free = bar(9), b_p_full = bar(10), b_o_done = bar(11);
  const uint32_t b_teardown = bar(12);
  // syncs of the four softmax warps (one arrival per warp): the tile's vote, the raise of
  // the reference maxima (two steps, only in tiles that raise), the end of the row sums
  const uint32_t b_vote = bar(13), b_wmax = bar(14), b_mnew = bar(15), b_sums = bar(16);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kAbort);
  volatile int* votes = reinterpret_cast<volatile int*>(smem + L::kFlags);
  float* m_used = reinterpret_cast<float*>(smem + L::kMUsed);
  float* alpha = reinterpret_cast<float*>(smem + L::kAlpha);
  float* wmax = reinterpret_cast<float*>(smem + L::kWMax);

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(b_k_full(s), 1);
      tc::mbar_init(b_k_empty(s), 1);
      tc::mbar_init(b_v_full(s), 1);
      tc::mbar_init(b_v_empty(s), 1);
    }
    tc::mbar_init(b_s_full, 1);
    tc::mbar_init(b_s_free, 4);
    tc::mbar_init(b_p_full, 4);
    tc::mbar_init(b_o_done, 1);
    tc::mbar_init(b_teardown, 1);
    tc::mbar_init(b_vote, 4);
    tc::mbar_init(b_wmax, 4);
    tc::mbar_init(b_mnew, 4);
    tc::mbar_init(b_sums, 4);
    *abort_flag = 0;
    tc::fence_barrier_init();
  }
  for (int c = threadIdx.x; c < kNMax; c += kVThreads)
    m_used[c] = c < rows_here ? -INFINITY : kPadRowMax;
  // Q rows of this group into shared memory: K-major, 128-byte swizzle, one 128 B row per
  // query row and 64 dims; rows past the group's are zero
  for (int idx = threadIdx.x; idx < kNMax * (D / 8); idx += kVThreads) {
    const int r = idx / (D / 8), ch = idx - r * (D / 8);
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (r < rows_here) {
      const int grow = row0 + r;
      const int i = grow / p.g, hl = grow - i * p.g;
      v = __ldg(reinterpret_cast<const uint4*>(
                    p.q + (((int64_t)b * p.n_q + i) * p.Hq + kvh * p.g + hl) * D) + ch);
    }
    const int cb = ch >> 3, cc = ch & 7;
    *reinterpret_cast<uint4*>(smem + L::kQ + cb * L::kQBlk + r * 128 + ((cc ^ (r & 7)) << 4)) = v;
  }
  tc::fence_proxy_async();
  if (warp == 1) tc::tmem_alloc(sb + L::kTmemSlot, L::kTmemCols);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + L::kTmemSlot);

  auto raise = [&]() {
    *abort_flag = 1;
    atomicOr(&g_vc_dev_error, 1);
  };

  if ((warp == 0 || warp == 3) && lane == 0) {
    // ------------------------------------------------------------ TMA producers
    const bool is_k = warp == 0;
    const CUtensorMap* map = is_k ? &tmK : &tmV;
    const uint32_t base = sb + (is_k ? L::kK : L::kV);
    tc::prefetch_tmap(map);
    int issued = 0;
    for (int t = 0; t < n_tiles; ++t) {
      const int s = t & 1;
      const uint32_t fb = is_k ? b_k_full(s) : b_v_full(s);
      const uint32_t eb = is_k ? b_k_empty(s) : b_v_empty(s);
      if (t >= 2 && !tc::mbar_wait(eb, ((t >> 1) - 1) & 1, abort_flag, p.wait_ns)) {
        raise();
        break;
      }
      tc::mbar_expect_tx(fb, L::kKVSlot);
      const int y = (int)((tile0 + t) * kBN - p.kv_start);
#pragma unroll
      for (int cb = 0; cb < D / 64; ++cb)
        tc::tma_load_3d(base + s * L::kKVSlot + cb * L::kKVBlk, map, fb, cb * 64, y, pair);
      issued = t + 1;
    }
    // loads still in flight must land before shared memory is released
    for (int t = max(0, issued - 2); t < issued; ++t)
      tc::mbar_wait(is_k ? b_k_full(t & 1) : b_v_full(t & 1), (t >> 1) & 1, nullptr,
                    1000000000ull);
  } else if (warp == 1) {
    // ------------------------------------------------------------ UMMA issuer
    if (lane == 0) {
      const uint32_t id_qk = tc::idesc_bf16_f32(128, N, false, false);
      const uint32_t id_pv = tc::idesc_bf16_f32(128, N, true, true);
      auto qk = [&](int t) {
        const int s = t & 1;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint32_t a = sb + L::kK + s * L::kKVSlot + (ks >> 2) * L::kKVBlk + (ks & 3) * 32;
          const uint32_t bq = sb + L::kQ + (ks >> 2) * L::kQBlk + (ks & 3) * 32;
          tc::umma_ss(tmem + L::kColS, tc::sdesc_sw128(a, 16, 1024), tc::sdesc_sw128(bq, 16, 1024),
                      id_qk, ks > 0 ? 1u : 0u);
        }
      };
      auto pv = [&](int t) {
        const int s = t & 1;
#pragma unroll
        for (int ks = 0; ks < kBN / 16; ++ks) {
          // A = V^T: dims contiguous in each key's 128 B row (64 dims per block, blocks
          // L::kKVBlk apart; at D = 64 the second half of M re-reads the first block)
          const uint32_t a = sb + L::kV + s * L::kKVSlot + ks * 16 * 128;
          const uint32_t bp = sb + L::kP + ks * 16 * 128;
          tc::umma_ss(tmem + L::kColO, tc::sdesc_sw128(a, D == 128 ? L::kKVBlk : 0, 1024),
                      tc::sdesc_sw128(bp, L::kPBlk, 1024), id_pv,
                      (t > 0 || ks > 0) ? 1u : 0u);
        }
      };
      bool ok = true;
      for (int t = 0; t < n_tiles && ok; ++t) {
        if (!(ok = tc::mbar_wait(b_k_full(t & 1), (t >> 1) & 1, abort_flag, p.wait_ns))) break;
        if (t > 0 && !(ok = tc::mbar_wait(b_s_free, (t - 1) & 1, abort_flag, p.wait_ns))) break;
        tc::tc_fence_after();
        qk(t);
        tc::umma_commit(b_s_full);
        tc::umma_commit(b_k_empty(t & 1));
        if (t > 0) {
          if (!(ok = tc::mbar_wait(b_p_full, (t - 1) & 1, abort_flag, p.wait_ns))) break;
          if (!(ok = tc::mbar_wait(b_v_full((t - 1) & 1), ((t - 1) >> 1) & 1, abort_flag,
                                   p.wait_ns)))
            break;
          tc::tc_fence_after();
          pv(t - 1);
          tc::umma_commit(b_o_done);
          tc::umma_commit(b_v_empty((t - 1) & 1));
        }
      }
      if (ok) {
        const int t = n_tiles - 1;
        ok = tc::mbar_wait(b_p_full, t & 1, abort_flag, p.wait_ns) &&
             tc::mbar_wait(b_v_full(t & 1), (t >> 1) & 1, abort_flag, p.wait_ns);
        if (ok) {
          tc::tc_fence_after();
          pv(t);
          tc::umma_commit(b_o_done);
          tc::umma_commit(b_v_empty(t & 1));
        }
      }
      if (!ok) raise();
      // every UMMA issued must retire before TMEM is released
      tc::umma_commit(b_teardown);
      tc::mbar_wait(b_teardown, 0, nullptr, 1000000000ull);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax
    const int q4 = warp - 4;
    const int key_lane = 32 * q4 + lane;
    const int tid_s = threadIdx.x - 128;
    const uint32_t lane_t = tmem + ((uint32_t)(32 * q4) << 16);
    const uint32_t s_t = lane_t + L::kColS, o_t = lane_t + L::kColO, l_t = lane_t + L::kColL;
    const int nch = (N + 31) >> 5;
    const float sc2 = p.qk_scale2;
    // the four softmax warps meet on an mbarrier (bounded wait: a warp that gave up never
    // arrives, and the others give up in turn instead of hanging)
    auto sync4 = [&](uint32_t bar4, uint32_t phase) -> bool {
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(bar4);
      return __all_sync(0xffffffffu, tc::mbar_wait(bar4, phase, abort_flag, p.wait_ns));
    };
    // S columns [N, 32 nch) are read with the last 32-column load but never written by
    // the UMMA: zero them once (disjoint from the columns Q K^T writes)
    if (N & 16) {
      tc::tmem_st16_zero(s_t + N);
      tc::tmem_wait_st();
    }
    bool ok = true;
    int n_raise = 0;                          // tiles that raised a reference maximum
    for (int t = 0; t < n_tiles; ++t) {
      ok = __all_sync(0xffffffffu, tc::mbar_wait(b_s_full, t & 1, abort_flag, p.wait_ns));
      if (!ok) break;
      tc::tc_fence_after();
      float s[kNMax];
#pragma unroll
      for (int c = 0; c < kNMax / 32; ++c)
        if (c < nch) tc::tmem_ld32(s_t + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(&s[32 * c]));
      tc::tmem_wait_ld();
      // S is in registers: the next Q K^T may overwrite it
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(b_s_free);

      // the group's columns c >= r_min see this thread's key: row row0 + c sits at
      // position P + (row0 + c) / g (none if the key is outside the split's range)
      const int64_t key = (tile0 + t) * kBN + key_lane;
      const bool kv_ok = key >= a0 && key < a1;
      const int64_t rm = (key - p.P) * p.g - row0;
      const int r_min = !kv_ok ? INT_MAX : rm <= 0 ? 0 : (int)min((int64_t)INT_MAX, rm);
      const bool whole = __all_sync(0xffffffffu, r_min == 0);
      auto valid = [&](int c) { return whole || c >= r_min; };

      // vote: does any score exceed its row's reference maximum by more than 2^8?
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < kNMax; c += 4) {
        if (c < 32 * nch) {
          const float4 m4 = *reinterpret_cast<const float4*>(m_used + c);
          const float e0 = fmaf(s[c], sc2, -m4.x), e1 = fmaf(s[c + 1], sc2, -m4.y);
          const float e2 = fmaf(s[c + 2], sc2, -m4.z), e3 = fmaf(s[c + 3], sc2, -m4.w);
          if (whole) {
            mx = fmaxf(mx, fmaxf(fmaxf(e0, e1), fmaxf(e2, e3)));
          } else {
            if (valid(c)) mx = fmaxf(mx, e0);
            if (valid(c + 1)) mx = fmaxf(mx, e1);
            if (valid(c + 2)) mx = fmaxf(mx, e2);
            if (valid(c + 3)) mx = fmaxf(mx, e3);
          }
        }
      }
      const int vote = __any_sync(0xffffffffu, mx > kRescaleLog2) ? 1 : 0;
      if (lane == 0) votes[(t & 1) * 4 + q4] = vote;
      if (!(ok = sync4(b_vote, t & 1))) break;
      const bool exceed = (votes[(t & 1) * 4] | votes[(t & 1) * 4 + 1] | votes[(t & 1) * 4 + 2] |
                           votes[(t & 1) * 4 + 3]) != 0;
      bool waited_o = false;
      if (exceed) {
        // exact maxima of this tile per row, then raise the rows that need it
#pragma unroll
        for (int c = 0; c < kNMax; ++c) {
          if (c < 32 * nch) {
            const float v = warp_max_f32(valid(c) ? s[c] * sc2 : -INFINITY);
            if (lane == 0) wmax[q4 * kNMax + c] = v;
          }
        }
        if (!(ok = sync4(b_wmax, n_raise & 1))) break;
        for (int c = tid_s; c < 32 * nch; c += 128) {
          const float m_old = m_used[c];
          const float tm = fmaxf(fmaxf(wmax[c], wmax[kNMax + c]),
                                 fmaxf(wmax[2 * kNMax + c], wmax[3 * kNMax + c]));
          const float m_new = fmaxf(m_old, tm);
          float a = 1.f;
          if (m_new > m_old + kRescaleLog2) {
            a = m_old == -INFINITY ? 0.f : ex2(m_old - m_new);
            m_used[c] = m_new;
          }
          alpha[c] = a;
        }
        if (!(ok = sync4(b_mnew, n_raise & 1))) break;
        ++n_raise;
        if (t > 0) {
          // O^T (lane = head dim) scaled per row once the previous P.V is done
          ok = __all_sync(0xffffffffu, tc::mbar_wait(b_o_done, (t - 1) & 1, abort_flag, p.wait_ns));
          if (!ok) break;
          tc::tc_fence_after();
          waited_o = true;
#pragma unroll
          for (int c = 0; c < kNMax / 32; ++c) {
            if (c < nch) {
              uint32_t o[32];
              tc::tmem_ld32(o_t + 32 * c, o);
              tc::tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 32; ++e)
                o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha[32 * c + e]);
              tc::tmem_st32(o_t + 32 * c, o);
            }
          }
          tc::tmem_wait_st();
        }
      }
      // p = 2^(s - m_r), 0 where the key is not visible
#pragma unroll
      for (int c = 0; c < kNMax; c += 4) {
        if (c < 32 * nch) {
          const float4 m4 = *reinterpret_cast<const float4*>(m_used + c);
          const float e0 = ex2(fmaf(s[c], sc2, -m4.x)), e1 = ex2(fmaf(s[c + 1], sc2, -m4.y));
          const float e2 = ex2(fmaf(s[c + 2], sc2, -m4.z)), e3 = ex2(fmaf(s[c + 3], sc2, -m4.w));
          s[c] = valid(c) ? e0 : 0.f;
          s[c + 1] = valid(c + 1) ? e1 : 0.f;
          s[c + 2] = valid(c + 2) ? e2 : 0.f;
          s[c + 3] = valid(c + 3) ? e3 : 0.f;
        }
      }
      // the previous P.V must be done before P^T is overwritten
      if (t > 0 && !waited_o) {
        ok = __all_sync(0xffffffffu, tc::mbar_wait(b_o_done, (t - 1) & 1, abort_flag, p.wait_ns));
        if (!ok) break;
        tc::tc_fence_after();
      }
      // this lane's row sums: L = L * alpha + p
#pragma unroll
      for (int c = 0; c < kNMax / 32; ++c) {
        if (c < nch) {
          uint32_t lr[32];
          if (t > 0) {
            tc::tmem_ld32(l_t + 32 * c, lr);
            tc::tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const float a = exceed ? alpha[32 * c + e] : 1.f;
              lr[e] = __float_as_uint(fmaf(__uint_as_float(lr[e]), a, s[32 * c + e]));
            }
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) lr[e] = __float_as_uint(s[32 * c + e]);
          }
          tc::tmem_st32(l_t + 32 * c, lr);
        }
      }
      // P^T: bf16, MN-major with 128-byte swizzle: 64-row blocks, key k's 64 rows in one
      // 128-byte line of its block, 16-byte chunk j at position j ^ (k & 7)
      uint8_t* pbase = smem + L::kP + key_lane * 128;
#pragma unroll
      for (int c8 = 0; c8 < kNMax / 8; ++c8) {
        if (c8 < (N >> 3)) {
          const int c = 8 * c8;
          const uint4 w = make_uint4(pack_bf16x2(s[c], s[c + 1]), pack_bf16x2(s[c + 2], s[c + 3]),
                                     pack_bf16x2(s[c + 4], s[c + 5]),
                                     pack_bf16x2(s[c + 6], s[c + 7]));
          *reinterpret_cast<uint4*>(pbase + (c8 >> 3) * L::kPBlk +
                                    (((c8 & 7) ^ (key_lane & 7)) << 4)) = w;
        }
      }
      tc::tmem_wait_st();
      tc::fence_proxy_async();
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(b_p_full);
    }
    if (ok)
      ok = __all_sync(0xffffffffu,
                      tc::mbar_wait(b_o_done, (n_tiles - 1) & 1, abort_flag, p.wait_ns));
    if (ok && *abort_flag) ok = false;       // another role gave up: loads may be in flight
    float* red = reinterpret_cast<float*>(smem + L::kK);
    if (ok) {
      tc::tc_fence_after();
      // row sums: each key lane's partial sums to shared memory (the K/V and P buffers are idle
      // now), then every row added over the 128 lanes in order
#pragma unroll
      for (int c = 0; c < kNMax / 32; ++c) {
        if (c < nch) {
          uint32_t lr[32];
          tc::tmem_ld32(l_t + 32 * c, lr);
          tc::tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) red[key_lane * L::kRedStride + 32 * c + e] = __uint_as_float(lr[e]);
        }
      }
      ok = sync4(b_sums, 0);
    }
    if (!ok) {
      raise();
    } else {
      for (int c = tid_s; c < rows_here; c += 128) {
        float l = 0.f;
        for (int k = 0; k < kBN; ++k) l += red[k * L::kRedStride + c];
        const int64_t o_row = part * p.R + row0 + c;
        p.ws_ml[o_row * 2] = m_used[c];
        p.ws_ml[o_row * 2 + 1] = l;
      }
      // O^T: lane = head dim; a warp writes 32 consecutive dims of one row per store
#pragma unroll
      for (int c = 0; c < kNMax / 32; ++c) {
        if (c < nch) {
          uint32_t o[32];
          tc::tmem_ld32(o_t + 32 * c, o);
          tc::tmem_wait_ld();
          if (key_lane < D) {
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const int col = 32 * c + e;
              if (col < rows_here)
                p.ws_o[(part * p.R + row0 + col) * D + key_lane] = __uint_as_float(o[e]);
            }
          }
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
// once; the unnormalised outputs of 8 splits are loaded together before any is used,
// so a row costs a few L2 round trips, not one per split.  The sums run in split order
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
  constexpr int CH = 8;
  const int lane = threadIdx.x & 31;
  const int gr = blockIdx.x * kVCombWarps + (threadIdx.x >> 5);
  if (gr >= rows) return;
  const int pair = gr / R, row = gr - pair * R;
  const int i = row / g, hl = row - i * g;
  const int b = pair / Hkv, kvh = pair - b * Hkv;
  const int64_t sidx = ((int64_t)b * n_q + i) * Hq + kvh * g + hl;
  const bool carry = m_state != nullptr && !(flags & VC_VERIFY_FIRST);
  const int64_t pr0 = (int64_t)pair * n_split * R + row;   // split s: pr0 + s * R
  float M = carry ? m_state[sidx] : -INFINITY;
  for (int s = lane; s < n_split; s += 32) M = fmaxf(M, ws_ml[(pr0 + (int64_t)s * R) * 2]);
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
  for (int s0 = 0; s0 < n_split; s0 += 32) {
    const int cnt32 = min(32, n_split - s0);
    float wl = 0.f, ll = 0.f;
    if (lane < cnt32) {
      const float2 ml = *reinterpret_cast<const float2*>(ws_ml + (pr0 + (int64_t)(s0 + lane) * R) * 2);
      if (ml.x > -INFINITY) {
        wl = ex2(ml.x - M);
        ll = ml.y;
      }
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
#pragma unroll
      for (int j = 0; j < CH; ++j) {
        const float w = __shfl_sync(0xffffffffu, wl, c0 + j);
        const float lj = __shfl_sync(0xffffffffu, ll, c0 + j);
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
  int pairs, g, R, split0, n_split, n_rg, N;
  size_t ws_bytes;
};

Plan plan(int B, int n_q, int Hq, int Hkv, int D, int64_t kv_start, int64_t kv_len) {
  Plan pl;
  pl.pairs = B * Hkv;
  pl.g = Hq / Hkv;
  pl.R = n_q * pl.g;
  pl.split0 = (int)(kv_start / kSplitKeys);
  pl.n_split = (int)((kv_start + kv_len - 1) / kSplitKeys) - pl.split0 + 1;
  // row groups of at most kNMax rows, all of the same size N (a multiple of 16)
  pl.n_rg = (pl.R + kNMax - 1) / kNMax;
  const int per = (pl.R + pl.n_rg - 1) / pl.n_rg;
  pl.N = (per + 15) / 16 * 16;
  pl.ws_bytes = (size_t)pl.pairs * pl.n_split * pl.R * ((size_t)D + 2) * sizeof(float);
  return pl;
}

}  // namespace

size_t verify_workspace_bytes(int B, int n_q, int Hq, int Hkv, int D, int64_t kv_start,
                              int64_t kv_len) {
  return plan(B, n_q, Hq, Hkv, D, kv_start, kv_len).ws_bytes + 256;
}

template <int D>
static vc_status run_verify(const Plan& pl, const VerifyParams& vp, const CUtensorMap& mk,
                            const CUtensorMap& mv, int flags, float* m, float* l, float* acc,
                            void* out, cudaStream_t stream) {
  using L = VLayout<D>;
  VC_CUDA(cudaFuncSetAttribute(verify_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               L::kAlloc));
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
                        void* out, void* ws, size_t ws_bytes, cudaStream_t stream) {
  const Plan pl = plan(B, n_q, Hq, Hkv, D, kv_start, kv_len);
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
  vp.N = pl.N;
  vp.kv_start = kv_start;
  vp.kv_len = kv_len;
  vp.P = P;
  vp.split0 = pl.split0;
  vp.n_split = pl.n_split;
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
