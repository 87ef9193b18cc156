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
 * K % 16 == 0, K <= 4096, N % 64 == 0. */
vc_status vc_glue_gemm(const void* a, const void* w, int M, int K, int N, float* c,
                       int accumulate, cudaStream_t stream);

/* vc_glue_gemm with a = the RMSNorm of x's rows (as vc_glue_rmsnorm, the same rounding:
 * bf16(x * 1 / sqrt(mean(x^2) + eps))) formed inside the kernel: x fp32 [M, K],
 * K % 256 == 0, K <= 4096.  The same result as vc_glue_rmsnorm then vc_glue_gemm, bit for
 * bit, in one launch. */
vc_status vc_glue_rmsnorm_gemm(const float* x, float eps, const void* w, int M, int K, int N,
                               float* c, int accumulate, cudaStream_t stream);

/* vc_glue_gemm with a = SwiGLU of gu (as vc_glue_swiglu) formed inside the kernel: gu fp32
 * [M, 2F] (gate | up), w bf16 [F, N], F % 16 == 0, F <= 4096.  The same result as
 * vc_glue_swiglu then vc_glue_gemm, bit for bit, in one launch. */
vc_status vc_glue_swiglu_gemm(const float* gu, const void* w, int M, int F, int N, float* c,
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

/* ----------------------------------------------------------------------------------
 * Host-side drivers of the loop: one call enqueues every kernel of k draft steps, of a
 * verify (or prefill) pass, or of n greedy steps, so a round costs a handful of calls
 * from the host instead of one per kernel.  They run the same kernels as the calls above
 * and the attention / acceptance calls of vericache.h, in the same order.
 *
 * vc_tinylm describes the model and its buffers (batch 1).  Per-layer arrays are HOST
 * arrays of n_layers device pointers.  Weights bf16, matrices [in, out]:
 *   wqkv [d, (Hq + 2 Hkv) D] (q | k | v), wo [Hq D, d], wgu [d, 2 ffn] (gate | up),
 *   wdown [ffn, d], embed [vocab, d], lm_head [d, vocab].
 * Caches: k_full / v_full bf16 [Hkv, cap, D] (position p in row p); k_tail / v_tail bf16
 * [Hkv, tail_cap, D] (draft step j stores its K/V in row j).  positions: device int32
 * [>= cap] with positions[i] = i.  Work buffers for rows_cap rows: x fp32 [rows, d], h
 * bf16 [rows, d], qkv fp32 [rows, (Hq + 2 Hkv) D], q, att bf16 [rows, Hq, D], gu fp32
 * [rows, 2 ffn], act bf16 [rows, ffn], logits fp32 [rows, vocab].  ws: device workspace
 * for the attention calls of one pass, at least vc_glue_workspace_size(m) bytes and
 * vc_draft_workspace_size of every draft cache.
 *
 * Verify attention of blocks of at most tail_cap tokens (a greedy step, a block of k + 1)
 * splits the keys into windows chosen from Hkv and cap only (the largest power of two
 * <= 4096, >= 256, giving two CTAs per SM), so a block and the same tokens stepped one at
 * a time agree bit for bit; longer blocks (the prefill) use the window vc_verify_attn
 * chooses for a cache of Hkv pairs and capacity cap.
 * -------------------------------------------------------------------------------- */
typedef struct vc_tinylm {
  int32_t n_layers, d_model, Hq, Hkv, D, ffn, vocab;
  float rms_eps, rope_theta;
  const void* embed;
  const void* lm_head;
  const void* const* wqkv;
  const void* const* wo;
  const void* const* wgu;
  const void* const* wdown;
  void* const* k_full;
  void* const* v_full;
  int32_t cap;
  void* const* k_tail;
  void* const* v_tail;
  int32_t tail_cap;
  const int32_t* positions;
  float* x;
  void* h;
  float* qkv;
  void* q;
  void* att;
  float* gu;
  void* act;
  float* logits;
  int32_t rows_cap;
  void* ws;
  size_t ws_bytes;
} vc_tinylm;

/* Device workspace the verify calls of vc_glue_forward_full / vc_glue_greedy_steps need
 * for this model (its Hq, Hkv, D, cap, rows_cap and tail_cap); 0 if those are invalid. */
size_t vc_glue_workspace_size(const vc_tinylm* m);

/* Tokens ids[0 .. n-1] (device int32) at positions pos0 .. pos0+n-1 through the whole
 * model over the full cache (their K/V stored at their positions, rows attending
 * causally): logits fp32 [n, vocab] in m->logits.  n <= rows_cap, pos0 + n <= cap. */
vc_status vc_glue_forward_full(const vc_tinylm* m, const int32_t* ids, int n, int pos0,
                               cudaStream_t stream);

/* k draft steps ([VC] "Algoritmo Principale", step 1): step j feeds ids[j] at position
 * P + j through the model, attending layer l's compressed cache caches[l] (a host array
 * of n_layers descriptors; their tail fields are replaced by the model's draft tail with
 * j + 1 rows) and writes the argmax of its logits to ids[j + 1].  ids device int32
 * [k + 1]; k + 1 <= tail_cap; P + k <= cap. */
vc_status vc_glue_draft_steps(const vc_tinylm* m, const vc_comp_cache* caches, int32_t* ids,
                              int k, int P, cudaStream_t stream);

/* n greedy steps over the full cache: step t feeds ids[t] at position pos0 + t and writes
 * the argmax of its logits to ids[t + 1].  ids device int32 [n + 1]. */
vc_status vc_glue_greedy_steps(const vc_tinylm* m, int32_t* ids, int n, int pos0,
                               cudaStream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* VERICACHE_GLUE_H */
