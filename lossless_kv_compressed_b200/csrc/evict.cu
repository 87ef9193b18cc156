// Token eviction by attention score: the scores and the top-budget selection.
//
// CentroidKV's summary ("Riassunto Tecnico: CentroidKV", section "Problematica") names
// eviction -- dropping the least important tokens by their attention scores -- as the
// usual way to shrink the KV cache, and keeps attention sinks and recent tokens in every
// compressed cache (section "Metodologia", item 2, "Preservazione").  VeriCache drafts
// over such a token-evicted cache ("Riepilogo Tecnico: VeriCache", section "Supporto
// Architetturale": eviction methods plug into its uniform compression interface).
//
// Score (the plainest reading of "attention score" for a prompt of n tokens): for kv
// head j, the attention probability key t receives, summed over the g query heads of j
// and the last W prompt queries, each query at position p attending keys [0, p]:
//     score[j, t] = sum_{w, h} softmax_{t' <= p_w}(q_{w,h} . k_t' * scale)[t].
// Two kernels: evict_lse_kernel finds each query row's log-sum-exp (one CTA per (query,
// pair) streams the visible keys once with a per-thread online max / sum, merged in a
// fixed order); evict_score_kernel gives each thread one key and sums its probability
// over the pair's W * g rows in row order (q rows and their log-sum-exp in shared
// memory), so every score is a fixed-order fp32 sum.
//
// Selection: keep sinks [0, n_sinks), the recent window [n - n_recent, n) and the
// budget - n_sinks - n_recent highest-scoring positions between (ties to the lower
// position), written in ascending order.  One CTA per row: a 4-pass radix select (8-bit
// digits, shared-memory histograms) finds the score of the last kept position, then two
// ordered block scans take the ties at that score from the lowest positions and compact
// the kept positions in order.  Exact: the result depends only on the scores' order.
#include <climits>

#include "vc_common.cuh"
#include "vc_internal.h"

namespace vc {

constexpr int kEvThreads = 256;

struct EvictParams {
  const __nv_bfloat16* q;   // [B, W, Hq, D]
  const __nv_bfloat16* k;   // [B, Hkv, L_cap, D]
  int W, Hq, Hkv, g;
  int64_t L_cap, n;
  float scale2;             // scale * log2(e)
  float* lse2;              // [B, W, Hq]: log2 sum_t 2^(s2_t)  (s2 = q.k * scale2)
  float* score;             // [B, Hkv, score_cap]
  int64_t score_cap;
};

template <int D>
__device__ __forceinline__ void load_row_f32(const __nv_bfloat16* src, float (&x)[D]) {
  const uint4* s = reinterpret_cast<const uint4*>(src);
#pragma unroll
  for (int c = 0; c < D / 8; ++c) {
    const uint4 u = __ldg(s + c);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      x[8 * c + 2 * e] = bf16_lo(w[e]);
      x[8 * c + 2 * e + 1] = bf16_hi(w[e]);
    }
  }
}

// One CTA per (query w, pair): lse2 of the g rows (w, h) of that pair.
template <int D>
__global__ void __launch_bounds__(kEvThreads) evict_lse_kernel(const EvictParams p) {
  pdl_wait();
  pdl_trigger();
  __shared__ float sq[8][D];
  __shared__ float sm[kEvThreads / 32][8], sl[kEvThreads / 32][8];
  const int w = blockIdx.x;
  const int64_t pair = blockIdx.y;
  const int64_t b = pair / p.Hkv, j = pair - b * p.Hkv;
  const int g = p.g, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int i = tid; i < g * D; i += kEvThreads) {
    const int h = i / D, d = i - h * D;
    sq[h][d] = __bfloat162float(p.q[((b * p.W + w) * p.Hq + j * g + h) * D + d]) * p.scale2;
  }
  __syncthreads();
  const int64_t last = p.n - p.W + w;          // this query's position: keys [0, last]
  float m[8], l[8];
#pragma unroll
  for (int h = 0; h < 8; ++h) { m[h] = -INFINITY; l[h] = 0.f; }
  const __nv_bfloat16* kb = p.k + pair * p.L_cap * D;
  for (int64_t t = tid; t <= last; t += kEvThreads) {
    float x[D];
    load_row_f32<D>(kb + t * D, x);
#pragma unroll
    for (int h = 0; h < 8; ++h) {
      if (h < g) {
        float s = 0.f;
#pragma unroll
        for (int d = 0; d < D; ++d) s = fmaf(sq[h][d], x[d], s);
        if (s > m[h]) {
          l[h] = l[h] * ex2(m[h] - s) + 1.f;
          m[h] = s;
        } else {
          l[h] += ex2(s - m[h]);
        }
      }
    }
  }
  // fixed-order merge: lanes by xor steps, then warps in order
#pragma unroll
  for (int h = 0; h < 8; ++h) {
    if (h >= g) break;
    float mh = m[h], lh = l[h];
    for (int o = 16; o > 0; o >>= 1) {
      const float mo = __shfl_xor_sync(0xffffffffu, mh, o);
      const float lo = __shfl_xor_sync(0xffffffffu, lh, o);
      const float mn = fmaxf(mh, mo);
      lh = (mh == -INFINITY ? 0.f : lh * ex2(mh - mn)) + (mo == -INFINITY ? 0.f : lo * ex2(mo - mn));
      mh = mn;
    }
    if (lane == 0) { sm[warp][h] = mh; sl[warp][h] = lh; }
  }
  __syncthreads();
  if (tid < g) {
    float M = -INFINITY;
    for (int u = 0; u < kEvThreads / 32; ++u) M = fmaxf(M, sm[u][tid]);
    float L = 0.f;
    for (int u = 0; u < kEvThreads / 32; ++u)
      if (sm[u][tid] != -INFINITY) L += sl[u][tid] * ex2(sm[u][tid] - M);
    p.lse2[(b * p.W + w) * p.Hq + j * g + tid] = M + __log2f(L);
  }
}

// One thread per key t of a pair: sum over the pair's W * g rows, row order fixed.
template <int D>
__global__ void __launch_bounds__(kEvThreads) evict_score_kernel(const EvictParams p) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ __align__(16) float ssh[];
  const int64_t pair = blockIdx.y;
  const int64_t b = pair / p.Hkv, j = pair - b * p.Hkv;
  const int g = p.g, rows = p.W * g;
  float* sq = ssh;                    // [rows][D], row r = w * g + h
  float* sl = ssh + rows * D;         // [rows]
  for (int i = threadIdx.x; i < rows * D; i += kEvThreads) {
    const int r = i / D, d = i - r * D;
    const int w = r / g, h = r - w * g;
    sq[i] = __bfloat162float(p.q[((b * p.W + w) * p.Hq + j * g + h) * D + d]) * p.scale2;
  }
  for (int r = threadIdx.x; r < rows; r += kEvThreads) {
    const int w = r / g, h = r - w * g;
    sl[r] = p.lse2[(b * p.W + w) * p.Hq + j * g + h];
  }
  __syncthreads();
  const int64_t t = (int64_t)blockIdx.x * kEvThreads + threadIdx.x;
  if (t >= p.n) return;
  float x[D];
  load_row_f32<D>(p.k + (pair * p.L_cap + t) * D, x);
  const int64_t first_q = p.n - p.W;   // position of query w = 0
  const int w0 = t > first_q ? (int)(t - first_q) : 0;   // queries that see key t
  float acc = 0.f;
  for (int r = w0 * g; r < rows; ++r) {
    const float4* qr = reinterpret_cast<const float4*>(sq + r * D);
    float s0 = 0.f, s1 = 0.f;
#pragma unroll
    for (int c = 0; c < D / 4; c += 2) {
      const float4 a = qr[c], bq = qr[c + 1];
      s0 = fmaf(a.x, x[4 * c], s0);
      s0 = fmaf(a.y, x[4 * c + 1], s0);
      s0 = fmaf(a.z, x[4 * c + 2], s0);
      s0 = fmaf(a.w, x[4 * c + 3], s0);
      s1 = fmaf(bq.x, x[4 * c + 4], s1);
      s1 = fmaf(bq.y, x[4 * c + 5], s1);
      s1 = fmaf(bq.z, x[4 * c + 6], s1);
      s1 = fmaf(bq.w, x[4 * c + 7], s1);
    }
    acc += ex2(s0 + s1 - sl[r]);
  }
  p.score[pair * p.score_cap + t] = acc;
}

// ------------------------------------------------------------------ selection
constexpr int kSelThreads = 1024;

// Order-preserving key: larger score -> larger key (-0 counts as +0).
__device__ __forceinline__ uint32_t score_key(float s) {
  uint32_t u = __float_as_uint(s == 0.f ? 0.f : s);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Inclusive block scan of one int per thread (fixed order); returns the block total.
__device__ __forceinline__ int block_scan(int v, int* s_warp, int& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += y;
  }
  if (lane == 31) s_warp[warp] = v;
  __syncthreads();
  if (warp == 0) {
    int x = lane < kSelThreads / 32 ? s_warp[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    s_warp[lane] = x;
  }
  __syncthreads();
  const int add = warp > 0 ? s_warp[warp - 1] : 0;
  total = s_warp[kSelThreads / 32 - 1];
  __syncthreads();
  return v + add;
}

__global__ void __launch_bounds__(kSelThreads) evict_select_kernel(
    const float* __restrict__ score, int64_t score_cap, int64_t n, int budget, int n_sinks,
    int n_recent, int32_t* __restrict__ idx, int64_t S_cap) {
  pdl_wait();
  pdl_trigger();
  __shared__ int hist[256];
  __shared__ int s_warp[32];
  __shared__ uint32_t s_prefix;
  __shared__ int s_rank;
  const int64_t row = blockIdx.x;
  const float* sc = score + row * score_cap;
  int32_t* out = idx + row * S_cap;
  const int tid = threadIdx.x;
  if ((int64_t)budget >= n) {                       // everything fits: keep all
    for (int64_t t = tid; t < n; t += kSelThreads) out[t] = (int32_t)t;
    return;
  }
  const int64_t lo = n_sinks, hi = n - n_recent;
  const int take = budget - n_sinks - n_recent;     // >= 0 (checked on the host)
  for (int t = tid; t < n_sinks; t += kSelThreads) out[t] = t;
  for (int64_t t = hi + tid; t < n; t += kSelThreads) out[n_sinks + take + (t - hi)] = (int32_t)t;
  if (take == 0) return;
  // ---- radix select: the key of the take-th largest middle score
  uint32_t prefix = 0, mask = 0;
  int rank = take;                                  // 1-based rank still to find
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = tid; i < 256; i += kSelThreads) hist[i] = 0;
    __syncthreads();
    for (int64_t t = lo + tid; t < hi; t += kSelThreads) {
      const uint32_t key = score_key(sc[t]);
      if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255], 1);
    }
    __syncthreads();
    if (tid == 0) {
      int acc = 0, dgt = 255;
      for (; dgt > 0; --dgt) {                      // from the largest digit down
        if (acc + hist[dgt] >= rank) break;
        acc += hist[dgt];
      }
      s_prefix = prefix | ((uint32_t)dgt << shift);
      s_rank = rank - acc;
    }
    __syncthreads();
    prefix = s_prefix;
    rank = s_rank;
    mask |= 255u << shift;
    __syncthreads();
  }
  const uint32_t kth = prefix;                      // key of the last kept position
  const int need_eq = rank;                         // ties at kth to keep, lowest first
  // ---- keep: key > kth, or key == kth among the first need_eq such positions; then
  //      write the kept positions in ascending order after the sinks
  int eq_before = 0, kept_before = 0;
  for (int64_t base = lo; base < hi; base += kSelThreads) {
    const int64_t t = base + tid;
    uint32_t key = 0;
    if (t < hi) key = score_key(sc[t]);
    const int is_eq = (t < hi && key == kth) ? 1 : 0;
    int tot_eq;
    const int eq_incl = block_scan(is_eq, s_warp, tot_eq) + eq_before;
    const int keep = (t < hi && (key > kth || (is_eq && eq_incl <= need_eq))) ? 1 : 0;
    int tot_keep;
    const int pos = block_scan(keep, s_warp, tot_keep) + kept_before;
    if (keep) out[n_sinks + pos - 1] = (int32_t)t;
    eq_before += tot_eq;
    kept_before += tot_keep;
  }
}

// ------------------------------------------------------------------ host side
template <int D>
static vc_status run_evict_scores(const EvictParams& p, int B, cudaStream_t stream) {
  const int pairs = B * p.Hkv;
  VC_CUDA(launch_pdl(evict_lse_kernel<D>, dim3(p.W, pairs), dim3(kEvThreads), 0, stream, 1, p));
  const size_t sm = ((size_t)p.W * p.g * D + (size_t)p.W * p.g) * sizeof(float);
  VC_CUDA(grant_smem((const void*)evict_score_kernel<D>, (int)sm));
  const unsigned nb = (unsigned)((p.n + kEvThreads - 1) / kEvThreads);
  VC_CUDA(launch_pdl(evict_score_kernel<D>, dim3(nb, pairs), dim3(kEvThreads), sm, stream, 1, p));
  VC_CUDA(cudaGetLastError());
  return VC_OK;
}

vc_status launch_evict_scores(const void* q, int B, int W, int Hq, int Hkv, int D,
                              const void* k, int64_t L_cap, int64_t n, float scale,
                              float* score, int64_t score_cap, float* ws, cudaStream_t stream) {
  EvictParams p;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.k = static_cast<const __nv_bfloat16*>(k);
  p.W = W;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.g = Hq / Hkv;
  p.L_cap = L_cap;
  p.n = n;
  p.scale2 = scale * kLog2e;
  p.lse2 = ws;
  p.score = score;
  p.score_cap = score_cap;
  return D == 128 ? run_evict_scores<128>(p, B, stream) : run_evict_scores<64>(p, B, stream);
}

vc_status launch_evict_select(const float* score, int rows, int64_t score_cap, int64_t n,
                              int budget, int n_sinks, int n_recent, int32_t* idx,
                              int64_t S_cap, cudaStream_t stream) {
  VC_CUDA(launch_pdl(evict_select_kernel, dim3(rows), dim3(kSelThreads), 0, stream, 1, score,
                     score_cap, n, budget, n_sinks, n_recent, idx, S_cap));
  VC_CUDA(cudaGetLastError());
  return VC_OK;
}

}  // namespace vc
