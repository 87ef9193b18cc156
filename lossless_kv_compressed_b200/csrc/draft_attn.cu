// Draft attention over the compressed cache KV_comp (split-K GQA decode).
//
// VeriCache summary ("Riepilogo Tecnico: VeriCache", section "Algoritmo Principale",
// step 1): the target model drafts by decoding over the compressed cache.  The
// CentroidKV summary ("Riassunto Tecnico: CentroidKV", item 4 "Aggregazione") adds
// the slot degree n_t to the softmax as a logarithmic term:
//     s_t = (q . k_t) * scale + ln n_t,   o = sum_t softmax(s)_t v_t.
//
// Design (HBM-bound: every KV byte is read once per call):
//   grid (n_split, B*Hkv); a CTA owns one (batch, kv head) and a chunk of slots, all
//   g <= 8 query heads of the group share the KV rows it streams.  4 warps, each with
//   its own cp.async ring of 16-slot tiles (K and V rows gathered by slot index,
//   16-byte copies into XOR-swizzled shared rows, no CTA barrier in the main loop).
//   q.K^T and P.V run on mma.sync m16n8k16 with the heads as the M rows (rows >= g are
//   zero padding) so the fp32 pipes only do the softmax.  Scores live in the log2
//   domain: s2 = s * scale * log2(e) + log2(n_t); the online softmax uses ex2.
//   Each CTA writes one partial (max, sum, unnormalised o) per head; a second kernel
//   merges the splits in a fixed order and writes bf16 o (and lse).
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
  int chunk, n_split;
  float qk_scale2;               // scale * log2(e)
  float* ws_o;                   // [pairs, n_split, g, D]
  float* ws_ml;                  // [pairs, n_split, g, 2]
  int32_t* err_flag;
};

constexpr int kDraftWarps = 4;
constexpr int kTile = 16;       // slots per warp tile

template <int D>
struct DraftSmem {
  static constexpr int kRowB = D * 2;
  static constexpr int kTileB = kTile * kRowB;       // one of K or V
  static constexpr int kStageB = 2 * kTileB;          // K then V
};

template <int D, int NST>
__global__ void __launch_bounds__(128, 2) draft_indexed_kernel(const DraftIndexedParams p) {
  using SM = DraftSmem<D>;
  constexpr int CH = D / 8;                 // 16-byte chunks per row
  constexpr int NT = D / 8;                 // n-tiles of the output
  extern __shared__ __align__(128) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int split = blockIdx.x, pair = blockIdx.y;
  const int b = pair / p.Hkv, j = pair - b * p.Hkv;
  const int total = p.S + p.n_tail;
  const int s0 = split * p.chunk;
  const int n_here = min(p.chunk, total - s0);

  int32_t* srow = reinterpret_cast<int32_t*>(smem + kDraftWarps * NST * SM::kStageB);
  float* sbias = reinterpret_cast<float*>(srow + p.chunk);

  // ---- slot -> row table and log2-degree bias for this chunk
  {
    const int32_t* idx = p.idx ? p.idx + (int64_t)pair * p.S_cap : nullptr;
    const int32_t* deg = p.deg ? p.deg + (int64_t)pair * p.S_cap : nullptr;
    int bad = 0;
    for (int i = threadIdx.x; i < n_here; i += blockDim.x) {
      const int s = s0 + i;
      int32_t r;
      float bias = 0.f;
      if (s < p.S) {
        r = idx ? idx[s] : s;
        if (r < 0 || (int64_t)r >= p.T_cap) { bad = 1; r = 0; }
        int dg = deg ? deg[s] : 1;
        if (dg < 1) { bad = 1; dg = 1; }
        bias = log2f((float)dg);
      } else {
        r = -(s - p.S) - 1;
      }
      srow[i] = r;
      sbias[i] = bias;
    }
    if (bad && p.err_flag) atomicExch(p.err_flag, 1);
  }
  __syncthreads();

  const __nv_bfloat16* kb = p.k + (int64_t)pair * p.T_cap * D;
  const __nv_bfloat16* vb = p.v + (int64_t)pair * p.T_cap * D;
  const __nv_bfloat16* kt = p.k_tail ? p.k_tail + (int64_t)pair * p.R_cap * D : kb;
  const __nv_bfloat16* vt = p.v_tail ? p.v_tail + (int64_t)pair * p.R_cap * D : vb;

  uint8_t* wbuf = smem + warp * NST * SM::kStageB;
  const uint32_t wbuf_s = smem_u32(wbuf);
  const int n_tiles = (n_here + kTile - 1) / kTile;
  const int my_tiles = n_tiles > warp ? (n_tiles - warp + kDraftWarps - 1) / kDraftWarps : 0;

  auto issue = [&](int it, int st) {
    const int ts = (warp + it * kDraftWarps) * kTile;
    const uint32_t kd = wbuf_s + st * SM::kStageB;
    const uint32_t vd = kd + SM::kTileB;
#pragma unroll
    for (int i = 0; i < kTile * CH / 32; ++i) {
      const int lin = lane + 32 * i;
      const int r = lin / CH, c = lin % CH;
      const int sl = ts + r;
      const bool ok = sl < n_here;
      const int32_t row = ok ? srow[sl] : 0;
      const __nv_bfloat16* kp = row >= 0 ? kb + (int64_t)row * D : kt + (int64_t)(-row - 1) * D;
      const __nv_bfloat16* vp = row >= 0 ? vb + (int64_t)row * D : vt + (int64_t)(-row - 1) * D;
      const uint32_t off = r * SM::kRowB + ((c ^ (r & 7)) << 4);
      cp_async16(kd + off, kp + c * 8, ok ? 16u : 0u);
      cp_async16(vd + off, vp + c * 8, ok ? 16u : 0u);
    }
  };

  // ---- query fragments (A operand rows = heads of the group; rows >= g are zero)
  const int qr = lane >> 2, qc = lane & 3;
  uint32_t qa[D / 16][2];
  {
    const bool ok = qr < p.g;
    const uint32_t* qp = reinterpret_cast<const uint32_t*>(
        p.q + ((int64_t)b * p.Hq + j * p.g + (ok ? qr : 0)) * D);
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
      qa[ks][0] = ok ? qp[(16 * ks + 2 * qc) / 2] : 0u;
      qa[ks][1] = ok ? qp[(16 * ks + 8 + 2 * qc) / 2] : 0u;
    }
  }

  float o[NT][4];
#pragma unroll
  for (int n = 0; n < NT; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
  float m_run = -INFINITY, l_run = 0.f;

#pragma unroll
  for (int st = 0; st < NST - 1; ++st) {
    if (st < my_tiles) issue(st, st);
    cp_async_commit();
  }

  for (int it = 0; it < my_tiles; ++it) {
    if (it + NST - 1 < my_tiles) issue(it + NST - 1, (it + NST - 1) % NST);
    cp_async_commit();
    cp_async_wait<NST - 1>();
    __syncwarp();
    const int st = it % NST;
    const uint32_t ks_base = wbuf_s + st * SM::kStageB;
    const uint32_t vs_base = ks_base + SM::kTileB;
    const int ts = (warp + it * kDraftWarps) * kTile;

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
    // log2-domain scores with degree bias and the ragged-tile mask
    float mx = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int sl = ts + nt * 8 + 2 * qc + e;
        const float v2 = sl < n_here ? fmaf(s[nt][e], p.qk_scale2, sbias[sl]) : -INFINITY;
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
    for (int n = 0; n < NT; ++n) {
      o[n][0] *= alpha; o[n][1] *= alpha; o[n][2] *= alpha; o[n][3] *= alpha;
    }
    // P as bf16 high part (A rows 0-7, the heads) plus bf16 low part (A rows 8-15,
    // otherwise padding): the two accumulator halves sum to P.V with P kept to
    // about 16 mantissa bits, at no extra MMA.
    const uint32_t ph0 = pack_bf16x2(s[0][0], s[0][1]);
    const uint32_t ph2 = pack_bf16x2(s[1][0], s[1][1]);
    const uint32_t pl0 = pack_bf16x2(s[0][0] - bf16_lo(ph0), s[0][1] - bf16_hi(ph0));
    const uint32_t pl2 = pack_bf16x2(s[1][0] - bf16_lo(ph2), s[1][1] - bf16_hi(ph2));
    // O += P V
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

  // ---- merge the 4 warps of the CTA through shared memory
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 1);
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 2);
  __syncthreads();
  float* red = reinterpret_cast<float*>(smem);          // [4][8][D + 2]
  constexpr int RS = D + 2;
  float* mine = red + (warp * 8 + qr) * RS;
#pragma unroll
  for (int n = 0; n < NT; ++n) {
    mine[n * 8 + 2 * qc] = o[n][0] + o[n][2];
    mine[n * 8 + 2 * qc + 1] = o[n][1] + o[n][3];
  }
  if (qc == 0) { mine[D] = m_run; mine[D + 1] = l_run; }
  __syncthreads();
  const int64_t part = (int64_t)pair * p.n_split + split;
  for (int t = threadIdx.x; t < p.g * D; t += blockDim.x) {
    const int r = t / D, d = t - r * D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kDraftWarps; ++w) M = fmaxf(M, red[(w * 8 + r) * RS + D]);
    float L = 0.f, O = 0.f;
#pragma unroll
    for (int w = 0; w < kDraftWarps; ++w) {
      const float* row = red + (w * 8 + r) * RS;
      const float f = ex2(row[D] - M);
      L = fmaf(row[D + 1], f, L);
      O = fmaf(row[d], f, O);
    }
    p.ws_o[(part * p.g + r) * D + d] = O;
    if (d == 0) {
      p.ws_ml[(part * p.g + r) * 2] = M;
      p.ws_ml[(part * p.g + r) * 2 + 1] = L;
    }
  }
}

// Fixed-order merge of the split partials of every head -> bf16 output (+ lse).
template <int D, typename OutT>
__global__ void __launch_bounds__(256) draft_combine_kernel(const float* __restrict__ ws_o,
                                                            const float* __restrict__ ws_ml,
                                                            int n_split, int g, int Hkv, int Hq,
                                                            OutT* __restrict__ out,
                                                            float* __restrict__ lse) {
  const int pair = blockIdx.x;
  const int b = pair / Hkv, j = pair - b * Hkv;
  for (int t = threadIdx.x; t < g * D; t += blockDim.x) {
    const int r = t / D, d = t - r * D;
    float M = -INFINITY;
    for (int s = 0; s < n_split; ++s)
      M = fmaxf(M, ws_ml[(((int64_t)pair * n_split + s) * g + r) * 2]);
    float L = 0.f, O = 0.f;
    for (int s = 0; s < n_split; ++s) {
      const int64_t pr = ((int64_t)pair * n_split + s) * g + r;
      const float f = ex2(ws_ml[pr * 2] - M);
      L = fmaf(ws_ml[pr * 2 + 1], f, L);
      O = fmaf(ws_o[pr * D + d], f, O);
    }
    const int64_t h = (int64_t)b * Hq + j * g + r;
    store_out(out + h * D + d, O / L);
    if (lse && d == 0) lse[h] = (M + __log2f(L)) * kLn2;
  }
}

// ------------------------------------------------------------------ host side
namespace {
constexpr int kNStage = 3;

int draft_chunk(int pairs, int total, int* n_split_out) {
  const int target = 4 * num_sms();
  int n_split = (target + pairs - 1) / pairs;
  int chunk = (total + n_split - 1) / n_split;
  chunk = ((chunk + 63) / 64) * 64;
  if (chunk < 64) chunk = 64;
  if (chunk > 2048) chunk = 2048;
  *n_split_out = (total + chunk - 1) / chunk;
  return chunk;
}

template <int D>
size_t draft_indexed_smem(int chunk) {
  return (size_t)kDraftWarps * kNStage * DraftSmem<D>::kStageB + (size_t)chunk * 8;
}
}  // namespace

size_t draft_workspace_bytes(const vc_comp_cache* c) {
  const int pairs = c->B * c->Hkv;
  const int total = c->S + c->n_tail;
  int n_split = 1;
  draft_chunk(pairs, total > 0 ? total : 1, &n_split);
  const int g = c->Hq / c->Hkv;
  return (size_t)pairs * n_split * g * ((size_t)c->D + 2) * sizeof(float) + 256;
}

template <int D>
static void launch_draft_combine(const DraftIndexedParams& p, int pairs, int flags, void* out,
                                 float* lse, cudaStream_t stream) {
  if (flags & VC_OUT_F32)
    draft_combine_kernel<D, float><<<pairs, 256, 0, stream>>>(
        p.ws_o, p.ws_ml, p.n_split, p.g, p.Hkv, p.Hq, static_cast<float*>(out), lse);
  else
    draft_combine_kernel<D, __nv_bfloat16><<<pairs, 256, 0, stream>>>(
        p.ws_o, p.ws_ml, p.n_split, p.g, p.Hkv, p.Hq, static_cast<__nv_bfloat16*>(out), lse);
}

vc_status launch_draft_indexed(const void* q, const vc_comp_cache* c, float scale, int flags,
                               void* out, float* lse, void* ws, size_t ws_bytes,
                               cudaStream_t stream) {
  const int pairs = c->B * c->Hkv;
  const int total = c->S + c->n_tail;
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
  p.chunk = draft_chunk(pairs, total, &p.n_split);
  p.qk_scale2 = scale * kLog2e;
  const size_t ws_need = (size_t)pairs * p.n_split * p.g * ((size_t)c->D + 2) * sizeof(float);
  if (ws_bytes < ws_need) return fail(VC_ERR_INVALID, "draft workspace too small");
  p.ws_o = static_cast<float*>(ws);
  p.ws_ml = p.ws_o + (size_t)pairs * p.n_split * p.g * c->D;
  p.err_flag = c->err_flag;
  dim3 grid(p.n_split, pairs);
  if (c->D == 128) {
    const size_t sm = draft_indexed_smem<128>(p.chunk);
    VC_CUDA(cudaFuncSetAttribute(draft_indexed_kernel<128, kNStage>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm));
    draft_indexed_kernel<128, kNStage><<<grid, 128, sm, stream>>>(p);
    VC_CUDA(cudaGetLastError());
    launch_draft_combine<128>(p, pairs, flags, out, lse, stream);
  } else {
    const size_t sm = draft_indexed_smem<64>(p.chunk);
    VC_CUDA(cudaFuncSetAttribute(draft_indexed_kernel<64, kNStage>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm));
    draft_indexed_kernel<64, kNStage><<<grid, 128, sm, stream>>>(p);
    VC_CUDA(cudaGetLastError());
    launch_draft_combine<64>(p, pairs, flags, out, lse, stream);
  }
  VC_CUDA(cudaGetLastError());
  return VC_OK;
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
