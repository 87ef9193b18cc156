// Model glue for the end-to-end draft-then-verify loop (see vericache_glue.h).
// Every kernel computes a row with the same instructions in the same order whatever the
// number of rows, so a block of k+1 tokens and k+1 single tokens agree bit for bit.
#include <math.h>

#include "vc_common.cuh"
#include "vc_internal.h"
#include "vericache_glue.h"

namespace vc {
namespace {

bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

__global__ void embed_kernel(const __nv_bfloat16* __restrict__ table, const int32_t* __restrict__ ids,
                             int n, int d, float* __restrict__ x) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (int64_t)n * d) return;
  const int r = (int)(i / d), c = (int)(i - (int64_t)r * d);
  x[i] = __bfloat162float(table[(int64_t)ids[r] * d + c]);
}

// one warp per row; lane-strided squares summed in a fixed order, butterfly reduction
__global__ void rmsnorm_kernel(const float* __restrict__ x, int n, int d, float eps,
                               __nv_bfloat16* __restrict__ out) {
  const int row = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= n) return;
  const float* xr = x + (int64_t)row * d;
  float ss = 0.f;
  for (int j = lane; j < d; j += 32) ss = fmaf(xr[j], xr[j], ss);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const float inv = 1.0f / sqrtf(ss / (float)d + eps);
  for (int j = lane; j < d; j += 32) out[(int64_t)row * d + j] = __float2bfloat16_rn(xr[j] * inv);
}

// c[16 x 64 tile] (+)= A[16 x K] @ w[K x 64]: 4 warps x (16 rows x 16 cols), k-steps of
// 16 in order.  The CTA's 16 rows of A are built once in shared memory (K * 32 bytes,
// 16-byte chunks XOR-swizzled within each group of 8), from
//   kGemmBf16:    a bf16 matrix (cp.async),
//   kGemmRmsNorm: RMSNorm of fp32 rows x (a row staged in shared memory by all threads,
//                 then the rmsnorm kernel's sum of squares, order and rounding by one
//                 warp, so the product is the same as normalising first),
//   kGemmSwiGLU:  bf16(silu(g) u) of fp32 rows gu = (g | u), as the swiglu kernel,
// while w streams through a 4-stage cp.async ring of 64 k-rows (128-byte rows, swizzled);
// fragments by ldmatrix (w transposed).  The k-steps and their
// order are the same whatever M, so a row's result does not depend on M.
constexpr int kGemmNst = 4;
constexpr int kGemmKs = 64;                  // k-rows per stage
constexpr int kGemmBf16 = 0, kGemmRmsNorm = 1, kGemmSwiGLU = 2;
constexpr int kGemmWBytes = kGemmNst * kGemmKs * 128;

__device__ __forceinline__ uint32_t gemm_a_off(int row, int chunk, int K) {
  const int nch = K >> 3;
  const int c = (chunk | 7) < nch ? (chunk & ~7) | ((chunk ^ row) & 7) : chunk;
  return (uint32_t)(row * K * 2 + c * 16);
}

template <int AMODE>
__global__ void __launch_bounds__(128) gemm_kernel(const void* __restrict__ a_src, float eps,
                                                   const __nv_bfloat16* __restrict__ w, int M,
                                                   int K, int N, float* __restrict__ c,
                                                   int accumulate) {
  extern __shared__ __align__(128) uint8_t gsm[];
  uint8_t* sw = gsm;                                   // [kGemmNst][64 rows x 128 B]
  uint8_t* sa = gsm + kGemmWBytes;                     // [16][K] bf16, swizzled
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qr = lane >> 2, qc = lane & 3;
  const int n0 = blockIdx.x * 64, m0 = blockIdx.y * 16;
  const int ksteps = K / 16;
  const int nstage = (K + kGemmKs - 1) / kGemmKs;
  auto issue = [&](int sg, int st) {
    const int kb = sg * kGemmKs;
#pragma unroll
    for (int i = 0; i < 4; ++i) {                     // w: 64 rows x 8 chunks
      const int e = threadIdx.x + 128 * i;
      const int row = e >> 3, ch = e & 7;
      const bool ok = kb + row < K;
      const __nv_bfloat16* src = w + (int64_t)(ok ? kb + row : 0) * N + n0 + ch * 8;
      cp_async16(smem_u32(sw + st * (kGemmKs * 128) + row * 128 + ((ch ^ (row & 7)) << 4)), src,
                 ok ? 16u : 0u);
    }
  };
  // ---- A rows: bf16 copies join the first copy group; the fp32 modes are computed while
  //      the first w stages are in flight
  if constexpr (AMODE == kGemmBf16) {
    const __nv_bfloat16* a = static_cast<const __nv_bfloat16*>(a_src);
    const int nch = K >> 3;
    for (int e = threadIdx.x; e < 16 * nch; e += 128) {
      const int row = e / nch, ch = e - row * nch;
      const bool ok = m0 + row < M;
      cp_async16(smem_u32(sa + gemm_a_off(row, ch, K)),
                 a + (int64_t)(ok ? m0 + row : 0) * K + ch * 8, ok ? 16u : 0u);
    }
  }
#pragma unroll
  for (int st = 0; st < kGemmNst - 1; ++st) {
    if (st < nstage) issue(st, st);
    cp_async_commit();
  }
  if constexpr (AMODE != kGemmBf16) {
    // all 128 threads build the rows (independent loads in flight together).  Rows past
    // M are left as they are: a row of the product depends on its own row of A only, and
    // rows past M are never stored.
    const float* x = static_cast<const float*>(a_src);
    __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(sa);
    const int rows = min(16, M - m0);
    auto put = [&](int rr, int j, float v) {
      dst[(gemm_a_off(rr, j >> 3, K) >> 1) + (j & 7)] = __float2bfloat16_rn(v);
    };
    if constexpr (AMODE == kGemmRmsNorm) {
      float* xs = reinterpret_cast<float*>(sa + 32 * K);   // one row of x, fp32
      float* inv_s = xs + K;
      for (int rr = 0; rr < rows; ++rr) {
        const float* xr = x + (int64_t)(m0 + rr) * K;
#pragma unroll 4
        for (int j = threadIdx.x; j < K; j += 128) xs[j] = xr[j];
        __syncthreads();
        if (warp == 0) {                               // the rmsnorm kernel's sum, order
          float ss = 0.f;                              // and rounding
          for (int j = lane; j < K; j += 32) ss = fmaf(xs[j], xs[j], ss);
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
          if (lane == 0) *inv_s = 1.0f / sqrtf(ss / (float)K + eps);
        }
        __syncthreads();
        const float inv = *inv_s;
        for (int j = threadIdx.x; j < K; j += 128) put(rr, j, xs[j] * inv);
        __syncthreads();
      }
    } else {
      for (int rr = 0; rr < rows; ++rr) {
        const float* gr = x + (int64_t)(m0 + rr) * 2 * K;
#pragma unroll 4
        for (int j = threadIdx.x; j < K; j += 128) {
          const float g = gr[j], u = gr[K + j];
          put(rr, j, g / (1.0f + expf(-g)) * u);
        }
      }
    }
  }
  float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
  const int mi = lane >> 3;
  const int arow = (lane & 7) + 8 * (mi & 1), achk = mi >> 1;   // a: rows 0-15, k chunk 0/1
  const int krow = (mi & 1) * 8 + (lane & 7);                 // w: k rows of the step
  const int wch = warp * 2 + (mi >> 1);                       // w: 8-column chunk
  for (int sg = 0; sg < nstage; ++sg) {
    if (sg + kGemmNst - 1 < nstage) issue(sg + kGemmNst - 1, (sg + kGemmNst - 1) % kGemmNst);
    cp_async_commit();
    cp_async_wait<kGemmNst - 1>();
    __syncthreads();
    const uint8_t* sws = sw + (sg % kGemmNst) * (kGemmKs * 128);
#pragma unroll
    for (int kk = 0; kk < kGemmKs / 16; ++kk) {
      const int ks = sg * (kGemmKs / 16) + kk;
      if (ks >= ksteps) break;
      uint32_t A0, A1, A2, A3, b0, b1, b2, b3;
      ldsm_x4(smem_u32(sa + gemm_a_off(arow, 2 * ks + achk, K)), A0, A1, A2, A3);
      const int wr = kk * 16 + krow;
      ldsm_x4_t(smem_u32(sws + wr * 128 + ((wch ^ (wr & 7)) << 4)), b0, b1, b2, b3);
      mma_bf16(acc[0], A0, A1, A2, A3, b0, b1);
      mma_bf16(acc[1], A0, A1, A2, A3, b2, b3);
    }
    __syncthreads();
  }
  cp_async_wait<0>();
  const bool r0 = m0 + qr < M, r1 = m0 + qr + 8 < M;
#pragma unroll
  for (int nt = 0; nt < 2; ++nt) {
    const int col = n0 + warp * 16 + nt * 8 + 2 * qc;
    if (r0) {
      float* p = c + (int64_t)(m0 + qr) * N + col;
      p[0] = accumulate ? p[0] + acc[nt][0] : acc[nt][0];
      p[1] = accumulate ? p[1] + acc[nt][1] : acc[nt][1];
    }
    if (r1) {
      float* p = c + (int64_t)(m0 + qr + 8) * N + col;
      p[0] = accumulate ? p[0] + acc[nt][2] : acc[nt][2];
      p[1] = accumulate ? p[1] + acc[nt][3] : acc[nt][3];
    }
  }
}

// one thread per (row, head, i < D/2): rotate-half RoPE in double precision angles
__global__ void rope_store_kernel(const float* __restrict__ qkv, const int32_t* __restrict__ pos,
                                  const int32_t* __restrict__ dst_row, int n, int Hq, int Hkv,
                                  int D, float theta, __nv_bfloat16* __restrict__ q_out,
                                  __nv_bfloat16* __restrict__ kc, __nv_bfloat16* __restrict__ vc_,
                                  int cap) {
  const int half = D / 2;
  const int heads = Hq + 2 * Hkv;
  const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= (int64_t)n * heads * half) return;
  const int row = (int)(t / ((int64_t)heads * half));
  const int rem = (int)(t - (int64_t)row * heads * half);
  const int h = rem / half, i = rem - h * half;
  const float* src = qkv + (int64_t)row * heads * D + (int64_t)h * D;
  const float x1 = src[i], x2 = src[i + half];
  if (h < Hq + Hkv) {
    const double inv = pow((double)theta, -2.0 * i / (double)D);
    double s, co;
    sincos((double)pos[row] * inv, &s, &co);
    const float y1 = (float)(x1 * co - x2 * s), y2 = (float)(x2 * co + x1 * s);
    if (h < Hq) {
      __nv_bfloat16* qo = q_out + ((int64_t)row * Hq + h) * D;
      qo[i] = __float2bfloat16_rn(y1);
      qo[i + half] = __float2bfloat16_rn(y2);
    } else if (dst_row[row] >= 0) {
      __nv_bfloat16* ko = kc + ((int64_t)(h - Hq) * cap + dst_row[row]) * D;
      ko[i] = __float2bfloat16_rn(y1);
      ko[i + half] = __float2bfloat16_rn(y2);
    }
  } else if (dst_row[row] >= 0) {
    __nv_bfloat16* vo = vc_ + ((int64_t)(h - Hq - Hkv) * cap + dst_row[row]) * D;
    vo[i] = __float2bfloat16_rn(x1);
    vo[i + half] = __float2bfloat16_rn(x2);
  }
}

__global__ void swiglu_kernel(const float* __restrict__ gu, int n, int F,
                              __nv_bfloat16* __restrict__ out) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (int64_t)n * F) return;
  const int r = (int)(i / F), j = (int)(i - (int64_t)r * F);
  const float g = gu[(int64_t)r * 2 * F + j], u = gu[(int64_t)r * 2 * F + F + j];
  out[i] = __float2bfloat16_rn(g / (1.0f + expf(-g)) * u);
}

__global__ void append_slots_kernel(int32_t* idx, int32_t* deg, int Hkv, int S_cap, int S,
                                    int start, int count) {
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= Hkv * count) return;
  const int h = t / count, i = t - h * count;
  idx[(int64_t)h * S_cap + S + i] = start + i;
  if (deg) deg[(int64_t)h * S_cap + S + i] = 1;
}

int blocks_for(int64_t n, int t) { return (int)((n + t - 1) / t); }

}  // namespace

template <int AMODE>
static vc_status launch_gemm(const void* a, float eps, const void* w, int M, int K, int N,
                             float* c, int accumulate, cudaStream_t stream) {
  if (!a || !w || !c || M <= 0 || K <= 0 || N <= 0) return fail(VC_ERR_INVALID, "gemm: args");
  if (K % 16 || N % 64) return fail(VC_ERR_UNSUPPORTED, "gemm: K %% 16 and N %% 64 must be 0");
  if (K > 4096) return fail(VC_ERR_UNSUPPORTED, "gemm: K > 4096");
  if (!al16(a) || !al16(w)) return fail(VC_ERR_INVALID, "gemm: misaligned");
  // w ring, A rows (bf16), and for the RMSNorm one fp32 row and its scale
  const int smem = kGemmWBytes + 32 * K + (AMODE == kGemmRmsNorm ? 4 * K + 16 : 0);
  if (smem > 48 * 1024) VC_CUDA(grant_smem((const void*)gemm_kernel<AMODE>, smem));
  dim3 grid(N / 64, (M + 15) / 16);
  gemm_kernel<AMODE><<<grid, 128, smem, stream>>>(a, eps, static_cast<const __nv_bfloat16*>(w),
                                                  M, K, N, c, accumulate);
  VC_CUDA(cudaGetLastError());
  return VC_OK;
}

}  // namespace vc

using namespace vc;

extern "C" {

vc_status vc_glue_embed(const void* table, const int32_t* ids, int n, int d, float* x,
                        cudaStream_t stream) {
  if (!table || !ids || !x || n <= 0 || d <= 0) return fail(VC_ERR_INVALID, "embed: args");
  embed_kernel<<<blocks_for((int64_t)n * d, 256), 256, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(table), ids, n, d, x);
  VC_CUDA(cudaGetLastError());
  return VC_OK;
}

vc_status vc_glue_rmsnorm(const float* x, int n, int d, float eps, void* out,
                          cudaStream_t stream) {
  if (!x || !out || n <= 0 || d <= 0) return fail(VC_ERR_INVALID, "rmsnorm: args");
  rmsnorm_kernel<<<blocks_for(n, 4), 128, 0, stream>>>(x, n, d, eps,
                                                       static_cast<__nv_bfloat16*>(out));
  VC_CUDA(cudaGetLastError());
  return VC_OK;
}


vc_status vc_glue_gemm(const void* a, const void* w, int M, int K, int N, float* c,
                       int accumulate, cudaStream_t stream) {
  return launch_gemm<kGemmBf16>(a, 0.f, w, M, K, N, c, accumulate, stream);
}

vc_status vc_glue_rmsnorm_gemm(const float* x, float eps, const void* w, int M, int K, int N,
                               float* c, int accumulate, cudaStream_t stream) {
  if (K % 256) return fail(VC_ERR_UNSUPPORTED, "rmsnorm_gemm: K %% 256 must be 0");
  return launch_gemm<kGemmRmsNorm>(x, eps, w, M, K, N, c, accumulate, stream);
}

vc_status vc_glue_swiglu_gemm(const float* gu, const void* w, int M, int F, int N, float* c,
                              int accumulate, cudaStream_t stream) {
  return launch_gemm<kGemmSwiGLU>(gu, 0.f, w, M, F, N, c, accumulate, stream);
}

vc_status vc_glue_rope_store(const float* qkv, const int32_t* pos, const int32_t* dst_row,
                             int n, int Hq, int Hkv, int D, float theta, void* q_out,
                             void* k_cache, void* v_cache, int cap, cudaStream_t stream) {
  if (!qkv || !pos || !dst_row || !q_out || !k_cache || !v_cache || n <= 0 || D % 2)
    return fail(VC_ERR_INVALID, "rope_store: args");
  const int64_t total = (int64_t)n * (Hq + 2 * Hkv) * (D / 2);
  rope_store_kernel<<<blocks_for(total, 256), 256, 0, stream>>>(
      qkv, pos, dst_row, n, Hq, Hkv, D, theta, static_cast<__nv_bfloat16*>(q_out),
      static_cast<__nv_bfloat16*>(k_cache), static_cast<__nv_bfloat16*>(v_cache), cap);
  VC_CUDA(cudaGetLastError());
  return VC_OK;
}

vc_status vc_glue_swiglu(const float* gu, int n, int F, void* out, cudaStream_t stream) {
  if (!gu || !out || n <= 0 || F <= 0) return fail(VC_ERR_INVALID, "swiglu: args");
  swiglu_kernel<<<blocks_for((int64_t)n * F, 256), 256, 0, stream>>>(
      gu, n, F, static_cast<__nv_bfloat16*>(out));
  VC_CUDA(cudaGetLastError());
  return VC_OK;
}

vc_status vc_glue_append_slots(int32_t* idx, int32_t* deg, int Hkv, int S_cap, int S, int start,
                               int count, cudaStream_t stream) {
  if (!idx || Hkv <= 0 || count < 0 || S < 0 || S + count > S_cap)
    return fail(VC_ERR_INVALID, "append_slots: args");
  if (count == 0) return VC_OK;
  append_slots_kernel<<<blocks_for((int64_t)Hkv * count, 256), 256, 0, stream>>>(
      idx, deg, Hkv, S_cap, S, start, count);
  VC_CUDA(cudaGetLastError());
  return VC_OK;
}

// ------------------------------------------------------------------ loop drivers
namespace {

vc_status check_model(const vc_tinylm* m) {
  if (!m || m->n_layers <= 0 || !m->wqkv || !m->wo || !m->wgu || !m->wdown || !m->k_full ||
      !m->v_full || !m->positions || !m->x || !m->h || !m->qkv || !m->q || !m->att ||
      !m->gu || !m->act || !m->logits || !m->ws || !m->embed || !m->lm_head)
    return fail(VC_ERR_INVALID, "tinylm: NULL field");
  if (m->Hq % m->Hkv || m->d_model % 256 || (m->D != 64 && m->D != 128))
    return fail(VC_ERR_UNSUPPORTED, "tinylm: shape");
  return VC_OK;
}

// One layer's work after the attention output is in m->att: output projection with the
// residual, the MLP with its residual.
vc_status layer_tail(const vc_tinylm* m, int l, int n, cudaStream_t s) {
  vc_status st;
  if ((st = vc_glue_gemm(m->att, m->wo[l], n, m->Hq * m->D, m->d_model, m->x, 1, s))) return st;
  if ((st = vc_glue_rmsnorm_gemm(m->x, m->rms_eps, m->wgu[l], n, m->d_model, 2 * m->ffn, m->gu,
                                 0, s)))
    return st;
  return vc_glue_swiglu_gemm(m->gu, m->wdown[l], n, m->ffn, m->d_model, m->x, 1, s);
}

vc_status layer_head(const vc_tinylm* m, int l, int n, const int32_t* pos, const int32_t* dst,
                     void* kc, void* vcache, int cap, cudaStream_t s) {
  vc_status st;
  const int nqkv = (m->Hq + 2 * m->Hkv) * m->D;
  if ((st = vc_glue_rmsnorm_gemm(m->x, m->rms_eps, m->wqkv[l], n, m->d_model, nqkv, m->qkv, 0,
                                 s)))
    return st;
  return vc_glue_rope_store(m->qkv, pos, dst, n, m->Hq, m->Hkv, m->D, m->rope_theta, m->q, kc,
                            vcache, cap, s);
}

vc_status logits_of(const vc_tinylm* m, int n, cudaStream_t s) {
  return vc_glue_rmsnorm_gemm(m->x, m->rms_eps, m->lm_head, n, m->d_model, m->vocab, m->logits,
                              0, s);
}

// Key window of the verify calls of decode-sized blocks (at most tail_cap tokens: a
// single greedy step or a block of k + 1): the largest power of two <= 4096, and >= 256,
// that still gives two CTAs per SM over the model's kv heads and cache capacity.  It
// depends on the model only, so a k + 1 block and k + 1 single steps use the same window
// and agree bit for bit.  Longer blocks (the prefill) use the window vc_verify_attn
// chooses for this cache.
int decode_split_keys(const vc_tinylm* m) {
  const int64_t want = 2 * (int64_t)num_sms();
  int w = kVerifySplitKeys;
  while (w > 256 && (int64_t)m->Hkv * ((m->cap + w - 1) / w) < want) w >>= 1;
  return w;
}

vc_status forward_full(const vc_tinylm* m, const int32_t* ids, int n, int pos0, cudaStream_t s) {
  vc_status st;
  const int split = n <= m->tail_cap ? decode_split_keys(m) : verify_window(m->Hkv, m->cap);
  if ((st = vc_glue_embed(m->embed, ids, n, m->d_model, m->x, s))) return st;
  const int g = m->Hq / m->Hkv;
  const int chunk = 1024 / g;
  const size_t qrow = (size_t)m->Hq * m->D * 2;          // bytes of one row of q / att
  for (int l = 0; l < m->n_layers; ++l) {
    const int32_t* pos = m->positions + pos0;
    if ((st = layer_head(m, l, n, pos, pos, m->k_full[l], m->v_full[l], m->cap, s))) return st;
    for (int r0 = 0; r0 < n; r0 += chunk) {
      const int r1 = n < r0 + chunk ? n : r0 + chunk;
      const int nq = r1 - r0;
      const int64_t P = pos0 + r0;
      st = verify_checked(static_cast<const char*>(m->q) + r0 * qrow, 1, nq, m->Hq, m->Hkv,
                          m->D, m->k_full[l], m->v_full[l], m->cap, 0, P + nq, P, nullptr,
                          nullptr, nullptr, 0, 0.f, static_cast<char*>(m->att) + r0 * qrow,
                          m->ws, m->ws_bytes, s, split);
      if (st) return st;
    }
    if ((st = layer_tail(m, l, n, s))) return st;
  }
  return logits_of(m, n, s);
}

}  // namespace

size_t vc_glue_workspace_size(const vc_tinylm* m) {
  if (!m || m->Hkv <= 0 || m->Hq <= 0 || m->Hq % m->Hkv || m->cap <= 0 || m->rows_cap <= 0)
    return 0;
  const int g = m->Hq / m->Hkv;
  const int rows = m->rows_cap < 1024 / g ? m->rows_cap : 1024 / g;
  size_t need = verify_workspace_bytes_any(1, rows, m->Hq, m->Hkv, m->D, 0, m->cap);
  if (m->tail_cap > 0) {
    const size_t dec = verify_workspace_bytes(1, m->tail_cap, m->Hq, m->Hkv, m->D, 0, m->cap,
                                              decode_split_keys(m));
    if (dec > need) need = dec;
  }
  return need;
}

vc_status vc_glue_forward_full(const vc_tinylm* m, const int32_t* ids, int n, int pos0,
                               cudaStream_t stream) {
  vc_status st = check_model(m);
  if (st) return st;
  if (!ids || n <= 0 || n > m->rows_cap || pos0 < 0 || pos0 + n > m->cap)
    return fail(VC_ERR_INVALID, "forward_full: rows or positions");
  return forward_full(m, ids, n, pos0, stream);
}

vc_status vc_glue_draft_steps(const vc_tinylm* m, const vc_comp_cache* caches, int32_t* ids,
                              int k, int P, cudaStream_t stream) {
  vc_status st = check_model(m);
  if (st) return st;
  if (!caches || !ids || k < 0 || k + 1 > m->tail_cap || P < 0 || P + k > m->cap ||
      !m->k_tail || !m->v_tail)
    return fail(VC_ERR_INVALID, "draft_steps: arguments");
  for (int j = 0; j < k; ++j) {
    if ((st = vc_glue_embed(m->embed, ids + j, 1, m->d_model, m->x, stream))) return st;
    for (int l = 0; l < m->n_layers; ++l) {
      // this step's K/V go to row j of the draft tail
      if ((st = layer_head(m, l, 1, m->positions + P + j, m->positions + j, m->k_tail[l],
                           m->v_tail[l], m->tail_cap, stream)))
        return st;
      vc_comp_cache c = caches[l];
      c.k_tail = m->k_tail[l];
      c.v_tail = m->v_tail[l];
      c.R_cap = m->tail_cap;
      c.n_tail = j + 1;
      if ((st = vc_draft_attn(m->q, &c, 0.f, 0, m->att, nullptr, m->ws, m->ws_bytes, stream)))
        return st;
      if ((st = layer_tail(m, l, 1, stream))) return st;
    }
    if ((st = logits_of(m, 1, stream))) return st;
    if ((st = vc_accept(m->logits, nullptr, 1, 1, m->vocab, ids + j + 1, nullptr, nullptr,
                        nullptr, nullptr, stream)))
      return st;
  }
  return VC_OK;
}

vc_status vc_glue_greedy_steps(const vc_tinylm* m, int32_t* ids, int n, int pos0,
                               cudaStream_t stream) {
  vc_status st = check_model(m);
  if (st) return st;
  if (!ids || n < 0 || pos0 < 0 || pos0 + n > m->cap)
    return fail(VC_ERR_INVALID, "greedy_steps: arguments");
  for (int t = 0; t < n; ++t) {
    if ((st = forward_full(m, ids + t, 1, pos0 + t, stream))) return st;
    if ((st = vc_accept(m->logits, nullptr, 1, 1, m->vocab, ids + t + 1, nullptr, nullptr,
                        nullptr, nullptr, stream)))
      return st;
  }
  return VC_OK;
}

}  // extern "C"
