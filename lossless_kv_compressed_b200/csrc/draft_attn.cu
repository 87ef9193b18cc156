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
//   (Measured and rejected: L2 bulk prefetch of rows beyond the ring, 37% slower;
//   launching the merge as a programmatic dependent, 4% slower.)
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

  // ---- slot table: raw idx / degree of one batch prefetched into registers, then
  //      validated and staged into shared memory when the copies reach that batch.
  int32_t ri[kTabE / 32], rd[kTabE / 32];
  auto slot_of = [&](int b, int e, int64_t& pair) -> int {
    const int local = b * kTB + e / kTile;
    if (local >= n) return -1;
    const int64_t x = x0 + local;
    pair = x / p.tpp;
    return (int)(x - pair * p.tpp) * kTile + (e % kTile);
  };
  auto load_batch = [&](int b) {
#pragma unroll
    for (int i = 0; i < kTabE / 32; ++i) {
      int64_t pair = 0;
      const int s = slot_of(b, lane + 32 * i, pair);
      ri[i] = 0;
      rd[i] = 1;
      if (s >= 0 && s < p.S) {
        const int64_t o = pair * p.S_cap + s;
        ri[i] = p.idx ? __ldg(p.idx + o) : s;
        rd[i] = p.deg ? __ldg(p.deg + o) : 1;
      }
    }
  };
  auto store_batch = [&](int b) {
    const int buf = b & 1;
    int bad = 0;
#pragma unroll
    for (int i = 0; i < kTabE / 32; ++i) {
      const int e = lane + 32 * i;
      int64_t pair = 0;
      const int s = slot_of(b, e, pair);
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
  auto issue = [&](int it, int st) {
    const int b = it / kTB;
    if (b == pending) {
      store_batch(b);
      ++pending;
      if (pending < nb) load_batch(pending);
    }
    const int64_t x = x0 + it;
    const int64_t pair = x / p.tpp;
    const __nv_bfloat16* kb = p.k + pair * p.T_cap * D;
    const __nv_bfloat16* vb = p.v + pair * p.T_cap * D;
    const __nv_bfloat16* kt = p.k_tail ? p.k_tail + pair * p.R_cap * D : kb;
    const __nv_bfloat16* vt = p.v_tail ? p.v_tail + pair * p.R_cap * D : vb;
    const int e0 = (b & 1) * kTabE + (it % kTB) * kTile;
    const uint32_t kd = wbuf_s + st * SM::kStageB;
    const uint32_t vd = kd + SM::kTileB;
#pragma unroll
    for (int i = 0; i < kTile * CH / 32; ++i) {
      const int lin = lane + 32 * i;
      const int r = lin / CH, c = lin % CH;
      const int32_t code = trow[e0 + r];
      const bool ok = code != kNone;
      const __nv_bfloat16* kp =
          code >= 0 ? kb + (int64_t)code * D : (ok ? kt + (int64_t)(-code - 1) * D : kb);
      const __nv_bfloat16* vp =
          code >= 0 ? vb + (int64_t)code * D : (ok ? vt + (int64_t)(-code - 1) * D : vb);
      const uint32_t off = r * SM::kRowB + ((c ^ (r & 7)) << 4);
      cp_async16(kd + off, kp + c * 8, ok ? 16u : 0u);
      cp_async16(vd + off, vp + c * 8, ok ? 16u : 0u);
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
  const int64_t pair_first = x0 / p.tpp;
  const int64_t pair_last = (x0 + n - 1) / p.tpp;
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

  for (int it = 0; it < n; ++it) {
    if (it + NST - 1 < n) issue(it + NST - 1, (it + NST - 1) % NST);
    cp_async_commit();
    cp_async_wait<NST - 1>();
    __syncwarp();
    const int64_t pair = (x0 + it) / p.tpp;
    if (pair != cur) {                               // segment boundary
      flush(cur);
      reset();
      cur = pair;
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) { qa[ks][0] = qn[ks][0]; qa[ks][1] = qn[ks][1]; }
      if (pair < pair_last) load_q(pair + 1, qn);
    }
    const int st = it % NST;
    const uint32_t ks_base = wbuf_s + st * SM::kStageB;
    const uint32_t vs_base = ks_base + SM::kTileB;
    const int e0 = ((it / kTB) & 1) * kTabE + (it % kTB) * kTile;

    // S = Q K^T over two n-tiles of 8 slots
    float s[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
      const int r = nt * 8 + (lane & 7);
      const int mi = lane >> 3;
#pragma unroll
      for (int kk = 0; kk < D / 32; ++kk) {
        const int c = 4 * kk + mi;
        uint32_t b0, b1, b2, b3;
        ldsm_x4(ks_base + r * SM::kRowB + ((c ^ (r & 7)) << 4), b0, b1, b2, b3);
        mma_bf16(s[nt], qa[2 * kk][0], 0u, qa[2 * kk][1], 0u, b0, b1);
        mma_bf16(s[nt], qa[2 * kk + 1][0], 0u, qa[2 * kk + 1][1], 0u, b2, b3);
      }
    }
    // log2-domain scores; the bias of a slot past the end is -inf (masked)
    float mx = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const float v2 = fmaf(s[nt][e], p.qk_scale2, tbias[e0 + nt * 8 + 2 * qc + e]);
        s[nt][e] = v2;
        mx = fmaxf(mx, v2);
      }
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    const float m_new = fmaxf(m_run, mx);
    const float alpha = ex2(m_run - m_new);
    m_run = m_new;
    float psum = 0.f;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        s[nt][e] = ex2(s[nt][e] - m_new);
        psum += s[nt][e];
      }
    l_run = fmaf(l_run, alpha, psum);
#pragma unroll
    for (int nn = 0; nn < NT; ++nn) {
      o[nn][0] *= alpha; o[nn][1] *= alpha; o[nn][2] *= alpha; o[nn][3] *= alpha;
    }
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

// Fixed-order merge of the partials of one head: block (pair, head), D threads.
template <int D, typename OutT>
__global__ void __launch_bounds__(D) draft_combine_kernel(const DraftIndexedParams p,
                                                          OutT* __restrict__ out,
                                                          float* __restrict__ lse) {
  const int64_t pair = blockIdx.x / p.g;
  const int r = blockIdx.x - (int)(pair * p.g);
  const int d = threadIdx.x;
  const int64_t w0 = warp_of_tile(pair * p.tpp, p.T, p.W);
  const int64_t w1 = warp_of_tile((pair + 1) * p.tpp - 1, p.T, p.W);
  float M = -INFINITY, L = 0.f, O = 0.f;
#pragma unroll 4
  for (int64_t w = w0; w <= w1; ++w) {
    if (warp_begin(w, p.T, p.W) >= warp_begin(w + 1, p.T, p.W)) continue;   // empty range
    const int64_t pr = (pair * p.maxseg + (w - w0)) * p.g + r;
    const float2 ml = *reinterpret_cast<const float2*>(p.ws_ml + pr * 2);
    const float os = p.ws_o[pr * D + d];
    const float Mn = fmaxf(M, ml.x);
    const float a = ex2(M - Mn), c = ex2(ml.x - Mn);
    L = fmaf(L, a, ml.y * c);
    O = fmaf(O, a, os * c);
    M = Mn;
  }
  const int64_t b = pair / p.Hkv, j = pair - b * p.Hkv;
  const int64_t h = b * p.Hq + j * p.g + r;
  store_out(out + h * D + d, O / L);
  if (lse && d == 0) lse[h] = (M + __log2f(L)) * kLn2;
}

// ------------------------------------------------------------------ host side
namespace {
constexpr int kNStage = 3;

struct DraftPlan {
  int tpp, W, maxseg;
  int64_t T;
};

DraftPlan draft_plan(int pairs, int total) {
  DraftPlan pl;
  pl.tpp = (total + kTile - 1) / kTile;
  pl.T = (int64_t)pairs * pl.tpp;
  const int64_t ctas = std::min<int64_t>(2 * (int64_t)num_sms(),
                                         std::max<int64_t>(1, pl.T / kDraftWarps));
  pl.W = (int)(ctas * kDraftWarps);
  int ms = 1;
  for (int64_t pr = 0; pr < pairs; ++pr) {
    const int64_t a = warp_of_tile(pr * pl.tpp, pl.T, pl.W);
    const int64_t b = warp_of_tile((pr + 1) * pl.tpp - 1, pl.T, pl.W);
    ms = std::max<int>(ms, (int)(b - a + 1));
  }
  pl.maxseg = ms;
  return pl;
}

template <int D>
size_t draft_indexed_smem() {
  return (size_t)kDraftWarps * (kNStage * DraftSmem<D>::kStageB + DraftSmem<D>::kTableB);
}
}  // namespace

size_t draft_workspace_bytes(const vc_comp_cache* c) {
  const int pairs = c->B * c->Hkv;
  const int total = c->S + c->n_tail;
  const DraftPlan pl = draft_plan(pairs, total > 0 ? total : 1);
  const int g = c->Hq / c->Hkv;
  return (size_t)pairs * pl.maxseg * g * ((size_t)c->D + 2) * sizeof(float) + 256;
}

template <int D>
static vc_status launch_draft_d(const DraftIndexedParams& p, int flags, void* out, float* lse,
                                cudaStream_t stream) {
  const size_t sm = draft_indexed_smem<D>();
  VC_CUDA(cudaFuncSetAttribute(draft_indexed_kernel<D, kNStage>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm));
  draft_indexed_kernel<D, kNStage><<<p.W / kDraftWarps, 128, sm, stream>>>(p);
  VC_CUDA(cudaGetLastError());
  const int blocks = (int)(p.T / p.tpp) * p.g;   // one per (pair, head)
  if (flags & VC_OUT_F32)
    draft_combine_kernel<D, float><<<blocks, D, 0, stream>>>(p, static_cast<float*>(out), lse);
  else
    draft_combine_kernel<D, __nv_bfloat16><<<blocks, D, 0, stream>>>(
        p, static_cast<__nv_bfloat16*>(out), lse);
  VC_CUDA(cudaGetLastError());
  return VC_OK;
}

vc_status launch_draft_indexed(const void* q, const vc_comp_cache* c, float scale, int flags,
                               void* out, float* lse, void* ws, size_t ws_bytes,
                               cudaStream_t stream) {
  const int pairs = c->B * c->Hkv;
  const int total = c->S + c->n_tail;
  const DraftPlan pl = draft_plan(pairs, total);
  DraftIndexedParams p;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.k = static_cast<const __nv_bfloat16*>(c->k);
  p.v = static_cast<const __nv_bfloat16*>(c->v);
  p.idx = c->idx;
  p.deg = c->deg;
  p.k_tail = static_cast<const __nv_bfloat16*>(c->k_tail);
  p.v_tail = static_cast<const __nv_bfloat16*>(c->v_tail);
  p.T_cap = c->T_cap;
  p.S = c->S;
  p.S_cap = c->S_cap;
  p.R_cap = c->R_cap;
  p.n_tail = c->n_tail;
  p.Hq = c->Hq;
  p.Hkv = c->Hkv;
  p.g = c->Hq / c->Hkv;
  p.tpp = pl.tpp;
  p.T = pl.T;
  p.W = pl.W;
  p.maxseg = pl.maxseg;
  p.qk_scale2 = scale * kLog2e;
  const size_t ws_need = (size_t)pairs * pl.maxseg * p.g * ((size_t)c->D + 2) * sizeof(float);
  if (ws_bytes < ws_need) return fail(VC_ERR_INVALID, "draft workspace too small");
  p.ws_o = static_cast<float*>(ws);
  p.ws_ml = p.ws_o + (size_t)pairs * pl.maxseg * p.g * c->D;
  p.err_flag = c->err_flag;
  if (c->D == 128) return launch_draft_d<128>(p, flags, out, lse, stream);
  return launch_draft_d<64>(p, flags, out, lse, stream);
}

}  // namespace vc

namespace vc {
vc_status launch_draft_int4(const void*, const vc_comp_cache*, float, int, void*, float*, void*,
                            size_t, cudaStream_t) {
  return fail(VC_ERR_UNSUPPORTED, "int4 draft attention not built yet");
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
#include <mutex>
#include <vector>

namespace {
constexpr size_t kNoAllocScratchBytes = 8u << 20;   // 8 MiB per device
static __device__ __align__(256) unsigned char g_draft_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mu;
std::vector<void*> g_noalloc_ptr;   // device address of the array, per device ordinal
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
  // One-time set-up per device, with that device current: in host code the array's
  // name is only a stand-in, so its device address is looked up once and kept.
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess)
    return vc::fail(VC_ERR_CUDA, "draft_noalloc: cudaGetDevice: %s", cudaGetErrorString(e));
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    if ((int)g_noalloc_ptr.size() <= dev) g_noalloc_ptr.resize(dev + 1, nullptr);
    if (!g_noalloc_ptr[dev]) {
      void* p = nullptr;
      e = cudaGetSymbolAddress(&p, g_draft_noalloc_scratch);
      if (e != cudaSuccess || !p)
        return vc::fail(VC_ERR_CUDA, "draft_noalloc: cudaGetSymbolAddress: %s",
                        cudaGetErrorString(e));
      g_noalloc_ptr[dev] = p;
    }
    scratch = g_noalloc_ptr[dev];
  }
  // Nothing in the partials has to start at zero: every entry a call reads was written
  // earlier in the same call, so the previous call's leftovers are harmless.
  return vc_draft_attn(q, cache, scale, flags, out, lse, scratch, kNoAllocScratchBytes, stream);
}
