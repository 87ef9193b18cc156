// Draft attention over the compressed cache KV_comp (split-K GQA decode).
//
// VeriCache summary ("Riepilogo Tecnico: VeriCache", section "Algoritmo Principale",
// step 1): the target model drafts by decoding over the compressed cache.  The
// CentroidKV summary ("Riassunto Tecnico: CentroidKV", item 4 "Aggregazione") adds
// the slot degree n_t to the softmax as a logarithmic term:
//     s_t = (q . k_t) * scale + ln n_t,   o = sum_t softmax(s)_t v_t.
//
// Design (HBM-bound: every KV byte is read once per call):
//   The work is the list of (batch, kv head) pairs times their 16-slot tiles (the
//   compressed slots followed by the bf16 tail rows).  A persistent grid of
//   2 CTAs x 4 warps per SM cuts that list into equal contiguous ranges, one per warp,
//   so every warp streams the same number of tiles (to within one) and no wave is left
//   half empty.  Each warp runs its own cp.async ring of K and V rows gathered by slot
//   index (16-byte copies into XOR-swizzled shared rows; no CTA barrier anywhere).  The
//   slot -> row table and log2-degree biases of the next 16 tiles are prefetched into
//   registers and staged into a double-buffered shared table ahead of the copies.
//   q.K^T and P.V run on mma.sync m16n8k16 with the g <= 8 heads of the group as the M
//   rows; rows 8-15 carry P's bf16 low part so P.V keeps ~16 mantissa bits of P.
//   Scores live in the log2 domain: s2 = s * scale * log2(e) + log2(n_t); the online
//   softmax uses ex2.  A warp writes one partial (max, sum, unnormalised o) per pair
//   it touches; a second kernel merges the partials of each head in a fixed order.
//   Both kernels start with pdl_wait() and are launched as programmatic dependents, so
//   the merge's launch overlaps the split kernel's tail (vc_common.cuh).
//   (Measured and rejected: an L2 bulk prefetch of rows beyond the ring, 37% slower;
//   per-lane cp.async.bulk row copies on an mbarrier ring, 20% slower; 3 CTAs per SM
//   with a 2-stage ring, no gain.)
#include <climits>

#include "vc_common.cuh"
#include "vc_internal.h"

namespace vc {

struct DraftIndexedParams {
  const __nv_bfloat16* q;        // [B, Hq, D]
  const __nv_bfloat16* k;        // [B, Hkv, T_cap, D]
  const __nv_bfloat16* v;
  const int32_t* idx;            // [B, Hkv, S_cap] or null
  const int32_t* deg;            // [B, Hkv, S_cap] or null
  const __nv_bfloat16* k_tail;   // [B, Hkv, R_cap, D]
  const __nv_bfloat16* v_tail;
  int64_t T_cap;
  int S, S_cap, R_cap, n_tail;
  int Hq, Hkv, g;
  int tpp;                       // 16-slot tiles per pair
  int64_t T;                     // tiles in all: pairs * tpp
  int W;                         // warps in the grid
  int maxseg;                    // partial slots per pair
  float qk_scale2;               // scale * log2(e)
  float* ws_o;                   // [pairs, maxseg, g, D]
  float* ws_ml;                  // [pairs, maxseg, g, 2]
  int32_t* err_flag;
};

constexpr int kDraftWarps = 4;
constexpr int kTile = 16;       // slots per tile
constexpr int kTB = 16;         // tiles per slot-table batch
constexpr int kTabE = kTB * kTile;

// First tile of warp w, and the warp whose range holds tile x (ranges are the
// equal split of [0, T) into W parts).
__host__ __device__ __forceinline__ int64_t warp_begin(int64_t w, int64_t T, int64_t W) {
  return w * T / W;
}
__host__ __device__ __forceinline__ int64_t warp_of_tile(int64_t x, int64_t T, int64_t W) {
  return ((x + 1) * W - 1) / T;
}

template <int D>
struct DraftSmem {
  static constexpr int kRowB = D * 2;
  static constexpr int kTileB = kTile * kRowB;        // one of K or V
  static constexpr int kStageB = 2 * kTileB;          // K then V
  static constexpr int kTableB = 2 * kTabE * 8;       // 2 batches x (row code, bias)
};

template <int D, int NST>
__global__ void __launch_bounds__(128, 2) draft_indexed_kernel(const DraftIndexedParams p) {
  pdl_wait();
  pdl_trigger();
  using SM = DraftSmem<D>;
  constexpr int CH = D / 8;                 // 16-byte chunks per row
  constexpr int NT = D / 8;                 // n-tiles of the output
  constexpr int32_t kNone = INT_MIN;        // row code of a slot past the end
  extern __shared__ __align__(128) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t gw = (int64_t)blockIdx.x * kDraftWarps + warp;
  const int64_t x0 = warp_begin(gw, p.T, p.W);
  const int n = (int)(warp_begin(gw + 1, p.T, p.W) - x0);
  if (n <= 0) return;

  uint8_t* wbuf = smem + warp * NST * SM::kStageB;
  const uint32_t wbuf_s = smem_u32(wbuf);
  int32_t* trow = reinterpret_cast<int32_t*>(smem + kDraftWarps * NST * SM::kStageB +
                                             warp * SM::kTableB);
  float* tbias = reinterpret_cast<float*>(trow + 2 * kTabE);
  const int total = p.S + p.n_tail;

  // Tile x0 + i lies in pair (x0 + i) / tpp.  The pair and the tile's place in it are
  // carried forward as the tiles advance, so the loop divides nothing in 64 bits.
  const int tpp = p.tpp;
  const int64_t pair_first = x0 / tpp;
  const int rem_first = (int)(x0 - pair_first * tpp);
  auto advance = [&](int64_t& pair, int& rem, int by) {
    rem += by;
    if (rem >= tpp) {
      const int q = rem / tpp;
      pair += q;
      rem -= q * tpp;
    }
  };

  // ---- slot table: raw idx / degree of one batch prefetched into registers, then
  //      validated and staged into shared memory when the copies reach that batch.
  //      Entry e of a batch is slot e % 16 of the batch's tile e / 16.
  int32_t ri[kTabE / 32], rd[kTabE / 32];
  int64_t lb_pair = pair_first, sb_pair = pair_first;   // first tile of the batch being
  int lb_rem = rem_first, sb_rem = rem_first;           // loaded / stored
  auto slot_of = [&](int b, int e, int64_t bpair, int brem, int64_t& pair) -> int {
    const int t = e / kTile;
    if (b * kTB + t >= n) return -1;
    pair = bpair;
    int rem = brem;
    advance(pair, rem, t);
    return rem * kTile + (e % kTile);
  };
  auto load_batch = [&](int b) {
#pragma unroll
    for (int i = 0; i < kTabE / 32; ++i) {
      int64_t pair = 0;
      const int s = slot_of(b, lane + 32 * i, lb_pair, lb_rem, pair);
      ri[i] = 0;
      rd[i] = 1;
      if (s >= 0 && s < p.S) {
        const int64_t o = pair * p.S_cap + s;
        ri[i] = p.idx ? __ldg(p.idx + o) : s;
        rd[i] = p.deg ? __ldg(p.deg + o) : 1;
      }
    }
    advance(lb_pair, lb_rem, kTB);
  };
  auto store_batch = [&](int b) {
    const int buf = b & 1;
    int bad = 0;
#pragma unroll
    for (int i = 0; i < kTabE / 32; ++i) {
      const int e = lane + 32 * i;
      int64_t pair = 0;
      const int s = slot_of(b, e, sb_pair, sb_rem, pair);
      int32_t code = kNone;
      float bias = -INFINITY;
      if (s >= 0 && s < p.S) {
        code = ri[i];
        if (code < 0 || (int64_t)code >= p.T_cap) { bad = 1; code = 0; }
        int dg = rd[i];
        if (dg < 1) { bad = 1; dg = 1; }
        bias = log2f((float)dg);
      } else if (s >= 0 && s < total) {
        code = -(s - p.S) - 1;
        bias = 0.f;
      }
      trow[buf * kTabE + e] = code;
      tbias[buf * kTabE + e] = bias;
    }
    advance(sb_pair, sb_rem, kTB);
    if (bad && p.err_flag) atomicExch(p.err_flag, 1);
    __syncwarp();
  };

  const int nb = (n + kTB - 1) / kTB;
  load_batch(0);
  store_batch(0);
  int pending = 1;                                   // batch whose raw values are in ri/rd
  if (nb > 1) load_batch(1);

  // The table of batch b is staged when the copies first reach it; the compute trails
  // by fewer than kTB tiles, so the other buffer still holds what it reads.
  // Lane l copies chunk l % CH of rows (l / CH) * NI + i, i < NI: its NI row codes are
  // contiguous in the table (two 16-byte shared loads at D = 128).
  constexpr int NI = kTile * CH / 32;
  const int c_ln = lane % CH, r_ln = (lane / CH) * NI;
  int64_t is_pair = pair_first;
  int is_rem = rem_first;
  auto issue = [&](int it, int st) {
    const int b = it / kTB;
    if (b == pending) {
      store_batch(b);
      ++pending;
      if (pending < nb) load_batch(pending);
    }
    const int64_t pair = is_pair;
    advance(is_pair, is_rem, 1);
    const uint64_t kb = reinterpret_cast<uint64_t>(p.k + pair * p.T_cap * D);
    const uint64_t vb = reinterpret_cast<uint64_t>(p.v + pair * p.T_cap * D);
    const uint64_t kt = p.k_tail ? reinterpret_cast<uint64_t>(p.k_tail + pair * p.R_cap * D) : kb;
    const uint64_t vt = p.v_tail ? reinterpret_cast<uint64_t>(p.v_tail + pair * p.R_cap * D) : vb;
    const int e0 = (b & 1) * kTabE + (it % kTB) * kTile;
    int32_t code[NI];
#pragma unroll
    for (int i = 0; i < NI; i += 4) {
      const int4 c4 = *reinterpret_cast<const int4*>(trow + e0 + r_ln + i);
      code[i] = c4.x; code[i + 1] = c4.y; code[i + 2] = c4.z; code[i + 3] = c4.w;
    }
    const uint32_t kd = wbuf_s + st * SM::kStageB;
    const uint32_t vd = kd + SM::kTileB;
#pragma unroll
    for (int i = 0; i < NI; ++i) {
      const int r = r_ln + i;
      const bool ok = code[i] != kNone;
      const bool tail = code[i] < 0;
      // byte offset of the chunk in its row (a masked slot reads nothing: size 0)
      const uint64_t bo = ok ? ((uint64_t)(tail ? -code[i] - 1 : code[i]) * D + c_ln * 8) * 2 : 0;
      const uint32_t off = r * SM::kRowB + ((c_ln ^ (r & 7)) << 4);
      cp_async16(kd + off, reinterpret_cast<const void*>((tail ? kt : kb) + bo), ok ? 16u : 0u);
      cp_async16(vd + off, reinterpret_cast<const void*>((tail ? vt : vb) + bo), ok ? 16u : 0u);
    }
  };

  // ---- query fragments (A operand rows = heads of the group; rows >= g are zero)
  const int qr = lane >> 2, qc = lane & 3;
  uint32_t qa[D / 16][2], qn[D / 16][2];
  auto load_q = [&](int64_t pair, uint32_t (&dst)[D / 16][2]) {
    const int64_t b = pair / p.Hkv, j = pair - b * p.Hkv;
    const bool ok = qr < p.g;
    const uint32_t* qp =
        reinterpret_cast<const uint32_t*>(p.q + (b * p.Hq + j * p.g + (ok ? qr : 0)) * D);
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
      dst[ks][0] = ok ? __ldg(qp + (16 * ks + 2 * qc) / 2) : 0u;
      dst[ks][1] = ok ? __ldg(qp + (16 * ks + 8 + 2 * qc) / 2) : 0u;
    }
  };
  const int64_t pair_last = (x0 + n - 1) / tpp;
  load_q(pair_first, qa);
  if (pair_last > pair_first) load_q(pair_first + 1, qn);

  float o[NT][4];
  float m_run, l_run;
  auto reset = [&]() {
#pragma unroll
    for (int nn = 0; nn < NT; ++nn) o[nn][0] = o[nn][1] = o[nn][2] = o[nn][3] = 0.f;
    m_run = -INFINITY;
    l_run = 0.f;
  };
  auto flush = [&](int64_t pair) {
    float l = l_run + __shfl_xor_sync(0xffffffffu, l_run, 1);
    l += __shfl_xor_sync(0xffffffffu, l, 2);
    const int64_t seg = gw - warp_of_tile(pair * p.tpp, p.T, p.W);
    const int64_t part = (pair * p.maxseg + seg) * p.g;
    if (qr < p.g) {
      float* dst = p.ws_o + (part + qr) * D;
#pragma unroll
      for (int nn = 0; nn < NT; ++nn)
        *reinterpret_cast<float2*>(dst + nn * 8 + 2 * qc) =
            make_float2(o[nn][0] + o[nn][2], o[nn][1] + o[nn][3]);
      if (qc == 0) *reinterpret_cast<float2*>(p.ws_ml + (part + qr) * 2) = make_float2(m_run, l);
    }
  };
  reset();
  int64_t cur = pair_first;

#pragma unroll
  for (int st = 0; st < NST - 1; ++st) {
    if (st < n) issue(st, st);
    cp_async_commit();
  }

  int c_rem = rem_first;
  for (int it = 0; it < n; ++it) {
    if (it + NST - 1 < n) issue(it + NST - 1, (it + NST - 1) % NST);
    cp_async_commit();
    cp_async_wait<NST - 1>();
    __syncwarp();
    if (c_rem == tpp) {                              // segment boundary
      c_rem = 0;
      flush(cur);
      reset();
      ++cur;
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) { qa[ks][0] = qn[ks][0]; qa[ks][1] = qn[ks][1]; }
      if (cur < pair_last) load_q(cur + 1, qn);
    }
    ++c_rem;
    const int st = it % NST;
    const uint32_t ks_base = wbuf_s + st * SM::kStageB;
    const uint32_t vs_base = ks_base + SM::kTileB;
    const int e0 = ((it / kTB) & 1) * kTabE + (it % kTB) * kTile;

    // S = Q K^T over two n-tiles of 8 slots; the two k-halves of each 32-wide step go
    // to separate accumulators (two short MMA chains per n-tile instead of one long one)
    float s[2][4], s2[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
      s2[nt][0] = s2[nt][1] = s2[nt][2] = s2[nt][3] = 0.f;
      const int r = nt * 8 + (lane & 7);
      const int mi = lane >> 3;
#pragma unroll
      for (int kk = 0; kk < D / 32; ++kk) {
        const int c = 4 * kk + mi;
        uint32_t b0, b1, b2, b3;
        ldsm_x4(ks_base + r * SM::kRowB + ((c ^ (r & 7)) << 4), b0, b1, b2, b3);
        mma_bf16(s[nt], qa[2 * kk][0], 0u, qa[2 * kk][1], 0u, b0, b1);
        mma_bf16(s2[nt], qa[2 * kk + 1][0], 0u, qa[2 * kk + 1][1], 0u, b2, b3);
      }
    }
    // log2-domain scores; the bias of a slot past the end is -inf (masked)
    float mx = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const float v2 =
            fmaf(s[nt][e] + s2[nt][e], p.qk_scale2, tbias[e0 + nt * 8 + 2 * qc + e]);
        s[nt][e] = v2;
        mx = fmaxf(mx, v2);
      }
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    const float m_new = fmaxf(m_run, mx);
    // rescale only when some row's running maximum moved (rare after the first tiles)
    if (__any_sync(0xffffffffu, m_new != m_run)) {
      const float alpha = ex2(m_run - m_new);
      l_run *= alpha;
#pragma unroll
      for (int nn = 0; nn < NT; ++nn) {
        o[nn][0] *= alpha; o[nn][1] *= alpha; o[nn][2] *= alpha; o[nn][3] *= alpha;
      }
      m_run = m_new;
    }
    float psum = 0.f;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        s[nt][e] = ex2(s[nt][e] - m_new);
        psum += s[nt][e];
      }
    l_run += psum;
    // P as bf16 high part (A rows 0-7, the heads) plus bf16 low part (A rows 8-15,
    // otherwise padding): the two accumulator halves sum to P.V with P kept to
    // about 16 mantissa bits, at no extra MMA.
    const uint32_t ph0 = pack_bf16x2(s[0][0], s[0][1]);
    const uint32_t ph2 = pack_bf16x2(s[1][0], s[1][1]);
    const uint32_t pl0 = pack_bf16x2(s[0][0] - bf16_lo(ph0), s[0][1] - bf16_hi(ph0));
    const uint32_t pl2 = pack_bf16x2(s[1][0] - bf16_lo(ph2), s[1][1] - bf16_hi(ph2));
#pragma unroll
    for (int n2 = 0; n2 < NT / 2; ++n2) {
      const int mi = lane >> 3;
      const int r = (mi & 1) * 8 + (lane & 7);
      const int c = 2 * n2 + (mi >> 1);
      uint32_t b0, b1, b2, b3;
      ldsm_x4_t(vs_base + r * SM::kRowB + ((c ^ (r & 7)) << 4), b0, b1, b2, b3);
      mma_bf16(o[2 * n2], ph0, pl0, ph2, pl2, b0, b1);
      mma_bf16(o[2 * n2 + 1], ph0, pl0, ph2, pl2, b2, b3);
    }
    __syncwarp();
  }
  cp_async_wait<0>();
  flush(cur);
}

// ------------------------------------------------------------------ int4 cache
// Draft attention over the 4-bit cache (layout in vericache.h): the same persistent
// per-warp ranges, over (pair, 32-token block) units.  A block's packed K and V words
// and its fp16 scales / zeros are five contiguous runs (5 KB at D = 128) copied into a
// per-warp cp.async ring.  The word layout matches the mma.sync fragments, so a thread
// reads exactly its own nibbles: one 16-byte load per token for K, one word per channel
// for V.  The nibbles stay exact (ORed into the mantissa of fp16 1024, then 1024
// subtracted) and the scales move to the other operand, so nothing proportional to a
// dequantised value is ever rounded to fp16:
//   q . k_hat = sum_d (q_d s_d) n_d + sum_d q_d z_d              (K: per channel)
//   sum_t p_t v_hat_t = sum_t (p_t s_t)(n_t - 8) + sum_t p_t (z_t + 8 s_t)
//                                                                 (V: per token, group;
//   centred so that neither sum is much larger than the result)
// q_d s_d and p_t s_t are split into fp16 high and low parts placed in A rows 0-7 and
// 8-15 (rows 8-15 are padding: g <= 8), so one f16 mma.sync carries both and the two
// accumulator halves add up to ~22 mantissa bits.  The zero-point sum over tokens is
// one more mma per 16 tokens; sum_d q_d z_d is an fp32 dot product.
struct DraftInt4Params {
  const __nv_bfloat16* q;
  const uint32_t* kq;            // [pairs, nblk_cap, 32, 4, D/32]
  const __half* ks;              // [pairs, nblk_cap, D]
  const __half* kz;
  const uint32_t* vq;            // [pairs, nblk_cap, D, 4]
  const __half* vs;              // [pairs, nblk_cap, D/32, 32]
  const __half* vz;
  int64_t nblk_cap;
  int nblk;                      // live blocks per pair
  int Hq, Hkv, g;
  int64_t T;                     // pairs * nblk
  int W, maxseg;
  float qk_scale2;
  float* ws_o;
  float* ws_ml;
};

template <int D>
struct Int4Smem {
  static constexpr int kKW = 16 * D;     // 32 tokens x D/2 bytes
  static constexpr int kVW = 16 * D;     // D channels x 4 words
  static constexpr int kSZ = 2 * D;      // one fp16 per channel (K) / per token-group (V)
  static constexpr int kStageB = kKW + kVW + 4 * kSZ;
};

// Nibble pair j of word w as exact fp16x2 integers (n0, n1): nibble j of the low and of
// the high half-word, put into the mantissa of fp16 1024, then 1024 subtracted.
__device__ __forceinline__ uint32_t nib_pair(uint32_t w, int j) {
  const uint32_t x = ((w >> (4 * j)) & 0x000F000Fu) | 0x64006400u;   // 1024 + n
  uint32_t n;
  asm("sub.f16x2 %0, %1, %2;" : "=r"(n) : "r"(x), "r"(0x64006400u));
  return n;
}
// Same pairs centred on the 4-bit range, (n0 - 8, n1 - 8), exact; w8 = w >> 8 is shared
// by the four pairs of a word.  A low nibble of a byte goes into the mantissa of fp16
// 1024 and 1032 is subtracted; a high nibble is masked in place (1024 + 16 n) and one
// fused multiply-add takes x / 16 - 72: two instructions per pair.
__device__ __forceinline__ uint32_t nib_pair_c(uint32_t w, uint32_t w8, int j) {
  const uint32_t src = j < 2 ? w : w8;
  uint32_t n;
  if ((j & 1) == 0) {
    const uint32_t x = (src & 0x000F000Fu) | 0x64006400u;           // 1024 + n
    asm("sub.f16x2 %0, %1, %2;" : "=r"(n) : "r"(x), "r"(0x64086408u));   // - 1032
  } else {
    const uint32_t x = (src & 0x00F000F0u) | 0x64006400u;           // 1024 + 16 n
    asm("fma.rn.f16x2 %0, %1, %2, %3;"                              // x / 16 - 72
        : "=r"(n) : "r"(x), "r"(0x2C002C00u), "r"(0xD480D480u));
  }
  return n;
}
__device__ __forceinline__ float2 h2f(uint32_t h) {
  return __half22float2(*reinterpret_cast<const __half2*>(&h));
}
// (a, b) -> fp16x2 high part and fp16x2 low part (a - hi, b - hi).
__device__ __forceinline__ void split_f16(float a, float b, uint32_t& hi, uint32_t& lo) {
  hi = pack_f16x2(a, b);
  const float2 h = h2f(hi);
  lo = pack_f16x2(a - h.x, b - h.y);
}

template <int D, int NST>
__global__ void __launch_bounds__(128, 3) draft_int4_kernel(const DraftInt4Params p) {
  pdl_wait();
  pdl_trigger();
  using SM = Int4Smem<D>;
  constexpr int NT = D / 8;
  constexpr int NW = D / 32;                 // K words per (token, c); channel groups of V
  extern __shared__ __align__(128) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t gw = (int64_t)blockIdx.x * kDraftWarps + warp;
  const int64_t x0 = warp_begin(gw, p.T, p.W);
  const int n = (int)(warp_begin(gw + 1, p.T, p.W) - x0);
  if (n <= 0) return;
  const uint32_t wbuf_s = smem_u32(smem + warp * NST * SM::kStageB);
  uint8_t* wbuf = smem + warp * NST * SM::kStageB;

  // Block x0 + i lies in pair (x0 + i) / nblk: carried forward, not divided per block.
  const int nblk = p.nblk;
  const int64_t pair_first = x0 / nblk;
  const int rem_first = (int)(x0 - pair_first * nblk);
  int64_t is_pair = pair_first;
  int is_rem = rem_first;
  // Copies of one block: the K and V word runs in 16-byte chunks (lane l takes chunks
  // l, l + 32, ...), then the four 2D-byte scale / zero runs, two chunks per lane.
  constexpr int KWC = SM::kKW / 16, SZC = SM::kSZ / 16;     // chunks per word run / per scale run
  static_assert(KWC % 32 == 0 && (4 * SZC) % 32 == 0, "chunk split");
  const int sz_run = (lane * ((4 * SZC) / 32)) / SZC;        // scale run of this lane's chunks
  const int sz_off = (lane * ((4 * SZC) / 32)) % SZC;
  const __half* sz_base = sz_run == 0 ? p.ks : sz_run == 1 ? p.kz : sz_run == 2 ? p.vs : p.vz;
  auto issue = [&](int it, int st) {
    const int64_t blk = is_pair * p.nblk_cap + is_rem;
    if (++is_rem == nblk) { is_rem = 0; ++is_pair; }
    const uint32_t dst = wbuf_s + st * SM::kStageB;
    const uint8_t* kb = reinterpret_cast<const uint8_t*>(p.kq + blk * (32 * 4 * NW));
    const uint8_t* vb = reinterpret_cast<const uint8_t*>(p.vq + blk * (D * 4));
#pragma unroll
    for (int i = 0; i < KWC / 32; ++i) {
      const int c = lane + 32 * i;
      cp_async16(dst + c * 16, kb + c * 16, 16u);
      cp_async16(dst + SM::kKW + c * 16, vb + c * 16, 16u);
    }
    const uint8_t* zb = reinterpret_cast<const uint8_t*>(sz_base + blk * D) + sz_off * 16;
    const uint32_t zd = dst + SM::kKW + SM::kVW + (sz_run * SZC + sz_off) * 16;
#pragma unroll
    for (int i = 0; i < (4 * SZC) / 32; ++i) cp_async16(zd + i * 16, zb + i * 16, 16u);
  };

  const int qr = lane >> 2, qc = lane & 3;
  uint32_t qa[D / 16][2], qn[D / 16][2];
  auto load_q = [&](int64_t pair, uint32_t (&dst)[D / 16][2]) {
    const int64_t b = pair / p.Hkv, j = pair - b * p.Hkv;
    const bool ok = qr < p.g;
    const uint32_t* qp =
        reinterpret_cast<const uint32_t*>(p.q + (b * p.Hq + j * p.g + (ok ? qr : 0)) * D);
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {       // raw bf16 pairs, widened when used
      dst[ks][0] = ok ? __ldg(qp + (16 * ks + 2 * qc) / 2) : 0u;
      dst[ks][1] = ok ? __ldg(qp + (16 * ks + 8 + 2 * qc) / 2) : 0u;
    }
  };
  const int64_t pair_last = (x0 + n - 1) / nblk;
  load_q(pair_first, qa);
  if (pair_last > pair_first) load_q(pair_first + 1, qn);

  float o[NT][4];
  float zacc[4];
  float m_run, l_run;
  auto reset = [&]() {
#pragma unroll
    for (int nn = 0; nn < NT; ++nn) o[nn][0] = o[nn][1] = o[nn][2] = o[nn][3] = 0.f;
    zacc[0] = zacc[1] = zacc[2] = zacc[3] = 0.f;
    m_run = -INFINITY;
    l_run = 0.f;
  };
  auto flush = [&](int64_t pair) {
    float l = l_run + __shfl_xor_sync(0xffffffffu, l_run, 1);
    l += __shfl_xor_sync(0xffffffffu, l, 2);
    // zero-point term of group G for row qr: columns G of the zacc tile (lane qr*4 + G/2)
    const float zc0 = zacc[0] + zacc[2], zc1 = zacc[1] + zacc[3];
    float zt[NW];
#pragma unroll
    for (int G = 0; G < NW; ++G) {
      const float a = __shfl_sync(0xffffffffu, zc0, qr * 4 + G / 2);
      const float b = __shfl_sync(0xffffffffu, zc1, qr * 4 + G / 2);
      zt[G] = (G & 1) ? b : a;
    }
    const int64_t seg = gw - warp_of_tile(pair * p.nblk, p.T, p.W);
    const int64_t part = (pair * p.maxseg + seg) * p.g;
    if (qr < p.g) {
      float* dst = p.ws_o + (part + qr) * D;
#pragma unroll
      for (int nn = 0; nn < NT; ++nn)
        *reinterpret_cast<float2*>(dst + nn * 8 + 2 * qc) =
            make_float2(o[nn][0] + o[nn][2] + zt[nn / 4], o[nn][1] + o[nn][3] + zt[nn / 4]);
      if (qc == 0) *reinterpret_cast<float2*>(p.ws_ml + (part + qr) * 2) = make_float2(m_run, l);
    }
  };
  reset();
  int64_t cur = pair_first;

#pragma unroll
  for (int st = 0; st < NST - 1; ++st) {
    if (st < n) issue(st, st);
    cp_async_commit();
  }
  int c_rem = rem_first;
  for (int it = 0; it < n; ++it) {
    if (it + NST - 1 < n) issue(it + NST - 1, (it + NST - 1) % NST);
    cp_async_commit();
    cp_async_wait<NST - 1>();
    __syncwarp();
    if (c_rem == nblk) {                             // segment boundary
      c_rem = 0;
      flush(cur);
      reset();
      ++cur;
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) { qa[ks][0] = qn[ks][0]; qa[ks][1] = qn[ks][1]; }
      if (cur < pair_last) load_q(cur + 1, qn);
    }
    ++c_rem;
    const uint8_t* sbase = wbuf + (it % NST) * SM::kStageB;
    const uint32_t* kw = reinterpret_cast<const uint32_t*>(sbase);
    const uint32_t* vw = reinterpret_cast<const uint32_t*>(sbase + SM::kKW);
    const uint32_t* ksc = reinterpret_cast<const uint32_t*>(sbase + SM::kKW + SM::kVW);
    const uint32_t* kzr = ksc + SM::kSZ / 4;
    const uint32_t* vsc = kzr + SM::kSZ / 4;
    const uint32_t* vzr = vsc + SM::kSZ / 4;

    // ---- q'_d = q_d * s_d (per channel of this block) as hi/lo A fragments, and the
    //      zero-point term c = sum_d q_d z_d of this thread's head (fp32)
    uint32_t ah[D / 16][2], al[D / 16][2];
    float cz = 0.f;
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int d0 = 16 * ks + 8 * h + 2 * qc;
        const float2 sc = h2f(ksc[d0 / 2]), zc = h2f(kzr[d0 / 2]);
        const float q0 = bf16_lo(qa[ks][h]), q1 = bf16_hi(qa[ks][h]);
        split_f16(q0 * sc.x, q1 * sc.y, ah[ks][h], al[ks][h]);
        cz = fmaf(q0, zc.x, fmaf(q1, zc.y, cz));
      }
    cz += __shfl_xor_sync(0xffffffffu, cz, 1);
    cz += __shfl_xor_sync(0xffffffffu, cz, 2);

    // ---- S = Q K^T over 4 n-tiles of 8 tokens (B = exact nibbles)
    float s[4][4];
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
      s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
      const int t = nt * 8 + qr;
      uint32_t w[NW];
      if constexpr (NW == 4) {
        const uint4 v4 = *reinterpret_cast<const uint4*>(kw + (t * 4 + qc) * NW);
        w[0] = v4.x; w[1] = v4.y; w[2] = v4.z; w[3] = v4.w;
      } else {
        const uint2 v2 = *reinterpret_cast<const uint2*>(kw + (t * 4 + qc) * NW);
        w[0] = v2.x; w[1] = v2.y;
      }
#pragma unroll
      for (int wi = 0; wi < NW; ++wi)
#pragma unroll
        for (int hk = 0; hk < 2; ++hk) {            // k-step 2wi + hk
          const int ks = 2 * wi + hk;
          mma_f16(s[nt], ah[ks][0], al[ks][0], ah[ks][1], al[ks][1], nib_pair(w[wi], 2 * hk),
                  nib_pair(w[wi], 2 * hk + 1));
        }
    }
    // rows qr (high part) + rows qr+8 (low part) + zero-point term
    float mx = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
      s[nt][0] = (s[nt][0] + s[nt][2] + cz) * p.qk_scale2;
      s[nt][1] = (s[nt][1] + s[nt][3] + cz) * p.qk_scale2;
      mx = fmaxf(mx, fmaxf(s[nt][0], s[nt][1]));
    }
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    const float m_new = fmaxf(m_run, mx);
    // rescale only when some row's running maximum moved (rare after the first blocks)
    if (__any_sync(0xffffffffu, m_new != m_run)) {
      const float alpha = ex2(m_run - m_new);
      l_run *= alpha;
#pragma unroll
      for (int nn = 0; nn < NT; ++nn) {
        o[nn][0] *= alpha; o[nn][1] *= alpha; o[nn][2] *= alpha; o[nn][3] *= alpha;
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) zacc[e] *= alpha;
      m_run = m_new;
    }
    float psum = 0.f;
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
      s[nt][0] = ex2(s[nt][0] - m_new);
      s[nt][1] = ex2(s[nt][1] - m_new);
      psum += s[nt][0] + s[nt][1];
    }
    l_run += psum;

    // ---- zero-point term sum_t p_t z_t: A = p (hi/lo), B = zeros [tokens x groups]
    {
      uint32_t ph[4], pl[4];
#pragma unroll
      for (int nt = 0; nt < 4; ++nt) split_f16(s[nt][0], s[nt][1], ph[nt], pl[nt]);
      // B = z + 8 s, the value of the middle of each group's grid (the nibbles of V
      // enter centred, so both sums stay of the size of the result: no cancellation)
      auto zmid = [&](int t0) -> uint32_t {
        const int o = (qr * 32 + t0) / 2;
        const float2 z = h2f(vzr[o]), sc = h2f(vsc[o]);
        return pack_f16x2(fmaf(8.f, sc.x, z.x), fmaf(8.f, sc.y, z.y));
      };
#pragma unroll
      for (int kt = 0; kt < 2; ++kt) {
        uint32_t z0 = 0u, z1 = 0u;
        if (qr < NW) {
          z0 = zmid(16 * kt + 2 * qc);
          z1 = zmid(16 * kt + 8 + 2 * qc);
        }
        mma_f16(zacc, ph[2 * kt], pl[2 * kt], ph[2 * kt + 1], pl[2 * kt + 1], z0, z1);
      }
    }
    // ---- O += (p s) (N - 8) per channel group, B = exact centred nibbles
#pragma unroll
    for (int G = 0; G < NW; ++G) {
      uint32_t pah[4], pal[4];                      // [kt * 2 + half]
#pragma unroll
      for (int j = 0; j < 4; ++j) {                 // token pair 2qc + 8j: n-tile j
        const float2 sv = h2f(vsc[(G * 32 + 2 * qc + 8 * j) / 2]);
        split_f16(s[j][0] * sv.x, s[j][1] * sv.y, pah[j], pal[j]);
      }
#pragma unroll
      for (int nn = 4 * G; nn < 4 * G + 4; ++nn) {
        const uint32_t wv = vw[(nn * 8 + qr) * 4 + qc], wv8 = wv >> 8;
        mma_f16(o[nn], pah[0], pal[0], pah[1], pal[1], nib_pair_c(wv, wv8, 0),
                nib_pair_c(wv, wv8, 1));
        mma_f16(o[nn], pah[2], pal[2], pah[3], pal[3], nib_pair_c(wv, wv8, 2),
                nib_pair_c(wv, wv8, 3));
      }
    }
    __syncwarp();
  }
  cp_async_wait<0>();
  flush(cur);
}

// ------------------------------------------------------------------ merge
// Partials of one launch: one (max, sum, unnormalised o) per (pair, warp segment, head).
struct PartialSet {
  const float* o;
  const float* ml;
  int upp;          // units per pair
  int64_t T;        // pairs * upp
  int W, maxseg;
};

// Merge of up to two partial sets, one CTA of kCombWarps warps per (pair, head).  The
// pair's segments are cut into one contiguous share per warp; a warp loads the (max,
// sum) of up to 8 segments and their unnormalised outputs all at once (its lanes hold
// D/32 channels each), so a share of <= 8 segments costs one L2 round trip, and folds
// them into its running (m, l, o) with the weights broadcast by shuffle.  The warps'
// states are then merged through shared memory in warp order.  Every sum runs in an
// order fixed by the launch configuration, so results are reproducible.
constexpr int kCombWarps = 4;
constexpr int kCombChunk = 8;

template <int D, typename OutT>
__global__ void __launch_bounds__(kCombWarps * 32) draft_combine_kernel(
    PartialSet a, PartialSet b, int nsets, int g, int Hkv, int Hq, OutT* __restrict__ out,
    float* __restrict__ lse) {
  pdl_wait();
  pdl_trigger();
  constexpr int DPL = D / 32;                 // output channels per lane
  __shared__ float s_o[kCombWarps][D];
  __shared__ float s_m[kCombWarps], s_l[kCombWarps];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t pair = blockIdx.x / g;
  const int r = (int)(blockIdx.x - pair * g);
  float m = -INFINITY, l = 0.f, o[DPL];
#pragma unroll
  for (int j = 0; j < DPL; ++j) o[j] = 0.f;
  // Fold segments [s_begin, s_end) of one set into (m, l, o).  The segments of this pair
  // are warps w0 + s; empty warp ranges wrote no partial and get weight 0.
  auto fold = [&](const PartialSet& ps) {
    const int64_t w0 = warp_of_tile(pair * ps.upp, ps.T, ps.W);
    const int n = (int)(warp_of_tile((pair + 1) * ps.upp - 1, ps.T, ps.W) - w0 + 1);
    const int s_begin = warp * n / kCombWarps, s_end = (warp + 1) * n / kCombWarps;
    for (int c0 = s_begin; c0 < s_end; c0 += kCombChunk) {
      const int cnt = min(kCombChunk, s_end - c0);
      float2 ml = make_float2(-INFINITY, 0.f);
      if (lane < cnt && warp_begin(w0 + c0 + lane, ps.T, ps.W) <
                            warp_begin(w0 + c0 + lane + 1, ps.T, ps.W))
        ml = *reinterpret_cast<const float2*>(ps.ml + ((pair * ps.maxseg + c0 + lane) * g + r) * 2);
      float v[kCombChunk][DPL];
#pragma unroll
      for (int j = 0; j < kCombChunk; ++j) {
        const float* src = ps.o + ((pair * ps.maxseg + c0 + min(j, cnt - 1)) * g + r) * D + lane * DPL;
        if constexpr (DPL == 4) {
          const float4 t = *reinterpret_cast<const float4*>(src);
          v[j][0] = t.x; v[j][1] = t.y; v[j][2] = t.z; v[j][3] = t.w;
        } else {
          const float2 t = *reinterpret_cast<const float2*>(src);
          v[j][0] = t.x; v[j][1] = t.y;
        }
      }
      float mc = ml.x;
#pragma unroll
      for (int x = 1; x < kCombChunk; x <<= 1) mc = fmaxf(mc, __shfl_xor_sync(0xffffffffu, mc, x));
      mc = __shfl_sync(0xffffffffu, mc, 0);
      const float m_new = fmaxf(m, mc);
      if (m_new == -INFINITY) continue;          // nothing live yet
      const float alpha = m == -INFINITY ? 0.f : ex2(m - m_new);
      const float wl = ml.x == -INFINITY ? 0.f : ex2(ml.x - m_new);
      l *= alpha;
#pragma unroll
      for (int t = 0; t < DPL; ++t) o[t] *= alpha;
#pragma unroll
      for (int j = 0; j < kCombChunk; ++j) {
        const float w = __shfl_sync(0xffffffffu, wl, j);
        const float lj = __shfl_sync(0xffffffffu, ml.y, j);
        if (j < cnt && w != 0.f) {               // warp-uniform
          l = fmaf(w, lj, l);
#pragma unroll
          for (int t = 0; t < DPL; ++t) o[t] = fmaf(w, v[j][t], o[t]);
        }
      }
      m = m_new;
    }
  };
  fold(a);
  if (nsets > 1) fold(b);
#pragma unroll
  for (int t = 0; t < DPL; ++t) s_o[warp][lane * DPL + t] = o[t];
  if (lane == 0) { s_m[warp] = m; s_l[warp] = l; }
  __syncthreads();
  const int64_t bb = pair / Hkv, j = pair - bb * Hkv;
  const int64_t h = bb * Hq + j * g + r;
  for (int d = threadIdx.x; d < D; d += kCombWarps * 32) {
    float M = s_m[0];
#pragma unroll
    for (int w = 1; w < kCombWarps; ++w) M = fmaxf(M, s_m[w]);
    float L = 0.f, O = 0.f;
#pragma unroll
    for (int w = 0; w < kCombWarps; ++w) {
      const float f = s_m[w] == -INFINITY ? 0.f : ex2(s_m[w] - M);
      L = fmaf(s_l[w], f, L);
      O = fmaf(s_o[w][d], f, O);
    }
    store_out(out + h * D + d, O / L);
    if (lse && d == 0) lse[h] = (M + __log2f(L)) * kLn2;
  }
}

// ------------------------------------------------------------------ host side
namespace {
constexpr int kNStage = 3;
constexpr int kNStageInt4 = 3;

struct DraftPlan {
  int upp, W, maxseg;
  int64_t T;
  size_t floats(int pairs, int g, int D) const {
    return (size_t)pairs * maxseg * g * ((size_t)D + 2);
  }
};

// Equal contiguous warp ranges over pairs x upp units (upp units per pair), for a grid of
// ctas_per_sm resident CTAs per SM.
DraftPlan draft_plan(int pairs, int upp, int ctas_per_sm = 2) {
  DraftPlan pl;
  pl.upp = upp;
  pl.T = (int64_t)pairs * upp;
  const int64_t ctas = std::min<int64_t>((int64_t)ctas_per_sm * num_sms(),
                                         std::max<int64_t>(1, pl.T / kDraftWarps));
  pl.W = (int)(ctas * kDraftWarps);
  int ms = 1;
  for (int64_t pr = 0; pr < pairs; ++pr) {
    const int64_t a = warp_of_tile(pr * upp, pl.T, pl.W);
    const int64_t b = warp_of_tile((pr + 1) * upp - 1, pl.T, pl.W);
    ms = std::max<int>(ms, (int)(b - a + 1));
  }
  pl.maxseg = ms;
  return pl;
}

int tiles_of(int slots) { return (slots + kTile - 1) / kTile; }

template <int D>
size_t draft_indexed_smem() {
  return (size_t)kDraftWarps * (kNStage * DraftSmem<D>::kStageB + DraftSmem<D>::kTableB);
}
template <int D>
size_t draft_int4_smem() {
  return (size_t)kDraftWarps * kNStageInt4 * Int4Smem<D>::kStageB;
}

PartialSet partials(const DraftPlan& pl, float* base, int pairs, int g, int D) {
  PartialSet ps;
  ps.o = base;
  ps.ml = base + (size_t)pairs * pl.maxseg * g * D;
  ps.upp = pl.upp;
  ps.T = pl.T;
  ps.W = pl.W;
  ps.maxseg = pl.maxseg;
  return ps;
}

template <int D>
vc_status launch_combine(const PartialSet& a, const PartialSet& b, int nsets, int pairs, int g,
                         int Hkv, int Hq, int flags, void* out, float* lse, cudaStream_t stream) {
  const int blocks = pairs * g;
  constexpr int T = kCombWarps * 32;
  if (flags & VC_OUT_F32)
    VC_CUDA(launch_pdl(draft_combine_kernel<D, float>, dim3(blocks), dim3(T), 0, stream, 1, a, b,
                       nsets, g, Hkv, Hq, static_cast<float*>(out), lse));
  else
    VC_CUDA(launch_pdl(draft_combine_kernel<D, __nv_bfloat16>, dim3(blocks), dim3(T), 0, stream,
                       1, a, b, nsets, g, Hkv, Hq, static_cast<__nv_bfloat16*>(out), lse));
  VC_CUDA(cudaGetLastError());
  return VC_OK;
}

// Indexed-kernel parameters for the slots [0, S) and tail rows [0, n_tail) of a cache.
DraftIndexedParams indexed_params(const void* q, const vc_comp_cache* c, int S, int n_tail,
                                  float scale, const DraftPlan& pl, float* ws) {
  const int pairs = c->B * c->Hkv;
  DraftIndexedParams p;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.k = static_cast<const __nv_bfloat16*>(c->k);
  p.v = static_cast<const __nv_bfloat16*>(c->v);
  p.idx = c->idx;
  p.deg = c->deg;
  p.k_tail = static_cast<const __nv_bfloat16*>(c->k_tail);
  p.v_tail = static_cast<const __nv_bfloat16*>(c->v_tail);
  p.T_cap = c->T_cap;
  p.S = S;
  p.S_cap = c->S_cap;
  p.R_cap = c->R_cap;
  p.n_tail = n_tail;
  p.Hq = c->Hq;
  p.Hkv = c->Hkv;
  p.g = c->Hq / c->Hkv;
  p.tpp = pl.upp;
  p.T = pl.T;
  p.W = pl.W;
  p.maxseg = pl.maxseg;
  p.qk_scale2 = scale * kLog2e;
  p.ws_o = ws;
  p.ws_ml = ws + (size_t)pairs * pl.maxseg * p.g * c->D;
  p.err_flag = c->err_flag;
  return p;
}

template <int D>
vc_status run_indexed(const DraftIndexedParams& p, cudaStream_t stream) {
  const size_t sm = draft_indexed_smem<D>();
  VC_CUDA(grant_smem((const void*)draft_indexed_kernel<D, kNStage>, (int)sm));
  VC_CUDA(launch_pdl(draft_indexed_kernel<D, kNStage>, dim3(p.W / kDraftWarps), dim3(128), sm,
                     stream, 1, p));
  VC_CUDA(cudaGetLastError());
  return VC_OK;
}

template <int D>
vc_status run_int4(const DraftInt4Params& p, cudaStream_t stream) {
  const size_t sm = draft_int4_smem<D>();
  VC_CUDA(grant_smem((const void*)draft_int4_kernel<D, kNStageInt4>, (int)sm));
  VC_CUDA(launch_pdl(draft_int4_kernel<D, kNStageInt4>, dim3(p.W / kDraftWarps), dim3(128), sm,
                     stream, 1, p));
  VC_CUDA(cudaGetLastError());
  return VC_OK;
}

// Workspace split of an int4 call: partials of the quantised blocks, then of the tail.
struct Int4Plans {
  DraftPlan q, t;
  bool has_q, has_t;
  size_t floats_q, floats_t;
};
Int4Plans int4_plans(const vc_comp_cache* c) {
  const int pairs = c->B * c->Hkv, g = c->Hq / c->Hkv;
  Int4Plans ip;
  ip.has_q = c->S > 0;
  ip.has_t = c->n_tail > 0;
  ip.q = draft_plan(pairs, ip.has_q ? c->S / 32 : 1, 3);   // 3 CTAs of 4 warps per SM
  ip.t = draft_plan(pairs, ip.has_t ? tiles_of(c->n_tail) : 1);
  ip.floats_q = ip.has_q ? ip.q.floats(pairs, g, c->D) : 0;
  ip.floats_t = ip.has_t ? ip.t.floats(pairs, g, c->D) : 0;
  return ip;
}
}  // namespace

size_t draft_workspace_bytes(const vc_comp_cache* c) {
  const int pairs = c->B * c->Hkv, g = c->Hq / c->Hkv;
  if (c->kind == VC_CACHE_INT4) {
    const Int4Plans ip = int4_plans(c);
    return (ip.floats_q + ip.floats_t) * sizeof(float) + 256;
  }
  const int total = c->S + c->n_tail;
  const DraftPlan pl = draft_plan(pairs, tiles_of(total > 0 ? total : 1));
  return pl.floats(pairs, g, c->D) * sizeof(float) + 256;
}

vc_status launch_draft_indexed(const void* q, const vc_comp_cache* c, float scale, int flags,
                               void* out, float* lse, void* ws, size_t ws_bytes,
                               cudaStream_t stream) {
  const int pairs = c->B * c->Hkv, g = c->Hq / c->Hkv;
  const DraftPlan pl = draft_plan(pairs, tiles_of(c->S + c->n_tail));
  if (ws_bytes < pl.floats(pairs, g, c->D) * sizeof(float))
    return fail(VC_ERR_INVALID, "draft workspace too small");
  float* w = static_cast<float*>(ws);
  const DraftIndexedParams p = indexed_params(q, c, c->S, c->n_tail, scale, pl, w);
  const PartialSet ps = partials(pl, w, pairs, g, c->D);
  vc_status st = c->D == 128 ? run_indexed<128>(p, stream) : run_indexed<64>(p, stream);
  if (st != VC_OK) return st;
  return c->D == 128 ? launch_combine<128>(ps, ps, 1, pairs, g, c->Hkv, c->Hq, flags, out, lse, stream)
                     : launch_combine<64>(ps, ps, 1, pairs, g, c->Hkv, c->Hq, flags, out, lse, stream);
}

vc_status launch_draft_int4(const void* q, const vc_comp_cache* c, float scale, int flags,
                            void* out, float* lse, void* ws, size_t ws_bytes,
                            cudaStream_t stream) {
  const int pairs = c->B * c->Hkv, g = c->Hq / c->Hkv;
  const Int4Plans ip = int4_plans(c);
  if (ws_bytes < (ip.floats_q + ip.floats_t) * sizeof(float))
    return fail(VC_ERR_INVALID, "draft workspace too small");
  float* wq = static_cast<float*>(ws);
  float* wt = wq + ip.floats_q;
  PartialSet sets[2];
  int nsets = 0;
  if (ip.has_q) {
    DraftInt4Params p;
    p.q = static_cast<const __nv_bfloat16*>(q);
    p.kq = c->kq;
    p.ks = static_cast<const __half*>(c->k_scale);
    p.kz = static_cast<const __half*>(c->k_zero);
    p.vq = c->vq;
    p.vs = static_cast<const __half*>(c->v_scale);
    p.vz = static_cast<const __half*>(c->v_zero);
    p.nblk_cap = c->T_cap / 32;
    p.nblk = c->S / 32;
    p.Hq = c->Hq;
    p.Hkv = c->Hkv;
    p.g = g;
    p.T = ip.q.T;
    p.W = ip.q.W;
    p.maxseg = ip.q.maxseg;
    p.qk_scale2 = scale * kLog2e;
    p.ws_o = wq;
    p.ws_ml = wq + (size_t)pairs * ip.q.maxseg * g * c->D;
    vc_status st = c->D == 128 ? run_int4<128>(p, stream) : run_int4<64>(p, stream);
    if (st != VC_OK) return st;
    sets[nsets++] = partials(ip.q, wq, pairs, g, c->D);
  }
  if (ip.has_t) {   // the bf16 tail rows through the indexed kernel (no slots)
    const DraftIndexedParams p = indexed_params(q, c, 0, c->n_tail, scale, ip.t, wt);
    vc_status st = c->D == 128 ? run_indexed<128>(p, stream) : run_indexed<64>(p, stream);
    if (st != VC_OK) return st;
    sets[nsets++] = partials(ip.t, wt, pairs, g, c->D);
  }
  return c->D == 128
             ? launch_combine<128>(sets[0], sets[nsets - 1], nsets, pairs, g, c->Hkv, c->Hq, flags,
                                   out, lse, stream)
             : launch_combine<64>(sets[0], sets[nsets - 1], nsets, pairs, g, c->Hkv, c->Hq, flags,
                                  out, lse, stream);
}

}  // namespace vc

// ------------------------------------------------------------------ fixed-scratch variant
// Some callers hand this library only their input and output buffers and cannot give it
// scratch memory: a plugin inside a host runtime that owns every byte of device memory
// and exposes no allocator, a fixed-budget serving process whose pool is fully reserved
// up front, or a latency-critical path that must not call cudaMalloc (which can block
// and synchronise the device).  For them vc_draft_attn_noalloc runs the same draft
// attention with its split-K partials in the array below, which lives in the library's
// own device image: every GPU that loads the library holds these bytes until the
// process exits, and no call allocates anything.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>
#include <vector>

namespace {
constexpr size_t kNoAllocScratchBytes = 8u << 20;   // 8 MiB per device
static __device__ __align__(256) unsigned char g_draft_noalloc_scratch[kNoAllocScratchBytes];

// Device address of the array, per CUDA context: a context is named by its unique id
// (cuCtxGetId), which is never reused within the process, so a context created after a
// cudaDeviceReset, or a non-primary context, gets its own look-up.
struct NoAllocEntry {
  int dev;
  unsigned long long ctx_id;
  void* ptr;
};
std::mutex g_noalloc_mu;
std::vector<NoAllocEntry> g_noalloc;

// Id of the context current on this thread; 0 when none is current yet (the runtime
// binds the device's primary context at its first call that needs one).
bool current_ctx_id(unsigned long long* id) {
  static PFN_cuCtxGetCurrent_v4000 get_cur = nullptr;
  static PFN_cuCtxGetId_v12000 get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_cur = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(f);
    f = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(f);
  });
  if (!get_cur || !get_id) return false;
  CUcontext ctx = nullptr;
  if (get_cur(&ctx) != CUDA_SUCCESS) return false;
  *id = 0;
  if (ctx && get_id(ctx, id) != CUDA_SUCCESS) return false;
  return true;
}
}  // namespace

extern "C" vc_status vc_draft_attn_noalloc(const void* q, const vc_comp_cache* cache,
                                           float scale, int flags, void* out, float* lse,
                                           cudaStream_t stream) {
  // The size check comes first and needs no device: the partials this call needs must
  // fit the fixed array.
  const size_t need = vc_draft_workspace_size(cache);
  if (need == 0) return VC_ERR_INVALID;   // cache rejected; vc_last_error() says why
  if (need > kNoAllocScratchBytes)
    return vc::fail(VC_ERR_UNSUPPORTED,
                    "draft_noalloc: this cache needs %zu bytes of scratch, the fixed scratch "
                    "holds %zu (use vc_draft_attn with a caller workspace)",
                    need, kNoAllocScratchBytes);
  // Set-up once per device and context, with that device current: in host code the
  // array's name is only a stand-in, so its device address is looked up and kept.
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess)
    return vc::fail(VC_ERR_CUDA, "draft_noalloc: cudaGetDevice: %s", cudaGetErrorString(e));
  unsigned long long ctx = 0;
  if (!current_ctx_id(&ctx))
    return vc::fail(VC_ERR_CUDA, "draft_noalloc: cannot identify the current context");
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    for (const NoAllocEntry& en : g_noalloc)
      if (ctx != 0 && en.dev == dev && en.ctx_id == ctx) scratch = en.ptr;
    if (!scratch) {
      e = cudaGetSymbolAddress(&scratch, g_draft_noalloc_scratch);
      if (e != cudaSuccess || !scratch)
        return vc::fail(VC_ERR_CUDA, "draft_noalloc: cudaGetSymbolAddress: %s",
                        cudaGetErrorString(e));
      // the look-up bound the device's context if none was current: name it now
      if (ctx == 0 && !current_ctx_id(&ctx))
        return vc::fail(VC_ERR_CUDA, "draft_noalloc: cannot identify the current context");
      if (ctx != 0) g_noalloc.push_back({dev, ctx, scratch});
    }
  }
  // Nothing in the partials has to start at zero: every entry a call reads was written
  // earlier in the same call, so the previous call's leftovers are harmless.
  return vc_draft_attn(q, cache, scale, flags, out, lse, scratch, kNoAllocScratchBytes, stream);
}
