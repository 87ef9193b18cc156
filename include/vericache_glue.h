/*
 * vericache_glue.h -- model glue for running the draft-then-verify loop end to end on a
 * small decoder-only transformer (pre-norm RMSNorm, rotate-half RoPE, GQA attention,
 * SwiGLU MLP, untied LM head).  These are not steps of the method; they let the loop of
 * [VC] "Riepilogo Tecnico: VeriCache", section "Algoritmo Principale" run on the GPU with
 * the attention and acceptance calls of vericache.h.
 *
 * Every kernel here is row-invariant: the result for one token (row) does not depend on
 * how many rows are processed together or what they hold (fixed tiling, fixed
 * reduction order, no split-K).  With the verify attention's fixed absolute split grid
 * this makes one verify pass over k+1 tokens produce, bit for bit, the logits of k+1
 * one-token greedy steps -- so the loop's committed stream equals greedy decoding
 * exactly on the GPU, not only up to rounding.
 *
 * Conventions as in vericache.h: device pointers owned by the caller, row-major,
 * 16-byte aligned, calls enqueue on `stream` and return a status.
 */
#ifndef VERICACHE_GLUE_H
#define VERICACHE_GLUE_H

#include <stdint.h>
#include <cuda_runtime_api.h>

#include "vericache.h"

#ifdef __cplusplus
extern "C" {
#endif

/* x[i, :] = table[ids[i], :] widened to fp32.  table bf16 [vocab, d], ids int32 [n]
 * (device), x fp32 [n, d].  d % 8 == 0. */
vc_status vc_glue_embed(const void* table, const int32_t* ids, int n, int d, float* x,
                        cudaStream_t stream);

/* out[i, :] = bf16(x[i, :] / sqrt(mean_j x[i, j]^2 + eps)) (unit weight).
 * x fp32 [n, d], out bf16 [n, d], d % 256 == 0. */
vc_status vc_glue_rmsnorm(const float* x, int n, int d, float eps, void* out,
                          cudaStream_t stream);

/* c[M, N] (+)= a[M, K] @ w[K, N]: a, w bf16 row-major, c fp32, fp32 accumulation in a
 * fixed K order.  accumulate != 0 adds into c (residual connections).
 * K % 16 == 0, N % 64 == 0. */
vc_status vc_glue_gemm(const void* a, const void* w, int M, int K, int N, float* c,
                       int accumulate, cudaStream_t stream);

/* Split fused projections qkv fp32 [n, (Hq + 2 Hkv) * D] (q | k | v), rotate q and k by
 * rotate-half RoPE at positions pos[i] (theta base), write q_out bf16 [n, Hq, D], and store
 * k, v (bf16) into caches [Hkv, cap, D] at row dst_row[i] (skipped when dst_row[i] < 0).
 * pos, dst_row int32 [n] (device). */
vc_status vc_glue_rope_store(const float* qkv, const int32_t* pos, const int32_t* dst_row,
                             int n, int Hq, int Hkv, int D, float theta, void* q_out,
                             void* k_cache, void* v_cache, int cap, cudaStream_t stream);

/* out[i, j] = bf16(silu(gu[i, j]) * gu[i, F + j]); gu fp32 [n, 2F] (gate | up), out bf16
 * [n, F]. */
vc_status vc_glue_swiglu(const float* gu, int n, int F, void* out, cudaStream_t stream);

/* idx[h, S + i] = start + i for i < count and every kv head h: append consecutive
 * positions to the compressed cache's slot lists (and deg[h, S + i] = 1 if deg != NULL).
 * idx, deg int32 [Hkv, S_cap]. */
vc_status vc_glue_append_slots(int32_t* idx, int32_t* deg, int Hkv, int S_cap, int S,
                               int start, int count, cudaStream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* VERICACHE_GLUE_H */
