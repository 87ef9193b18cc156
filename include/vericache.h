/*
 * vericache.h -- C ABI of the VeriCache draft/verify hot path for NVIDIA B200 (sm_100a).
 *
 * The operations follow two web summaries:
 *   [VC]  "Riepilogo Tecnico: VeriCache" (gist.science/it/paper/2605.17613; Arabic
 *         translation gist.science/ar/paper/2605.17613): draft over the compressed
 *         cache, verify all drafts in one pass over the full cache, greedy acceptance
 *         with a bonus token, and streaming of the full cache from CPU memory over
 *         PCIe overlapped with other requests' drafting.
 *   [CKV] "Riassunto Tecnico: CentroidKV" (gist.science/it/paper/2506.11418): per-slot
 *         degree n_t that enters the softmax as a logarithmic term.
 *
 * Conventions for every call:
 *   - All tensor pointers are DEVICE pointers owned by the caller, except the host
 *     source of vc_stage_full_kv.  The library allocates nothing; scratch space is a
 *     caller-provided workspace whose size the matching *_workspace_size call gives.
 *   - bf16 tensors are IEEE bfloat16 (2 bytes), fp16 tensors IEEE half.  Shapes are
 *     row-major and contiguous unless a capacity (…_cap) gives the row stride.
 *   - Calls only enqueue work on the given stream and return at once.  The return
 *     code covers argument validation and launch errors; errors found on the device
 *     (out-of-range slot indices, NaN logits) are written to caller-provided flags
 *     that the caller reads after synchronising.
 *   - Every pointer passed to a kernel must be 16-byte aligned.
 *   - There is no fallback path: an unsupported shape returns VC_ERR_UNSUPPORTED.
 */
#ifndef VERICACHE_H
#define VERICACHE_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

#define VC_ABI_VERSION 1

typedef enum {
  VC_OK = 0,
  VC_ERR_INVALID = 1,      /* bad argument: NULL, negative size, misaligned, … */
  VC_ERR_UNSUPPORTED = 2,  /* valid but not implemented (e.g. head dim 96) */
  VC_ERR_CUDA = 3,         /* a CUDA runtime call or launch failed */
  VC_ERR_TIMEOUT = 4       /* a bounded host wait ran out */
} vc_status;

typedef enum {
  VC_CACHE_INDEXED = 0,    /* bf16 rows picked by a slot index list, with degrees */
  VC_CACHE_INT4 = 1        /* 4-bit group-quantised rows (see the layout below) */
} vc_cache_kind;

/* Human-readable name of a status code (static string). */
const char* vc_status_string(int status);
/* Detail of the last failing call in this thread (static thread-local buffer). */
const char* vc_last_error(void);
/* VC_ABI_VERSION of the loaded library. */
int vc_abi_version(void);

/* ------------------------------------------------------------------------------
 * Compressed cache KV_comp of one attention layer ([VC] "Algoritmo Principale",
 * step 1; [VC] "Supporto Architetturale": one interface for eviction and
 * quantisation compressors).
 *
 * Common:  B batch, Hq query heads, Hkv kv heads (Hq % Hkv == 0, g = Hq/Hkv <= 8),
 *          D head dim in {64, 128}.  Query head h reads kv head h / g.
 * Tail:    k_tail, v_tail bf16 [B, Hkv, R_cap, D]; the first n_tail rows are live
 *          (tokens appended while drafting), each of degree 1.  May be NULL when
 *          n_tail == 0.
 *
 * VC_CACHE_INDEXED (token eviction, optionally merged centroids):
 *   k, v      bf16 [B, Hkv, T_cap, D]  base rows (a full cache viewed through idx,
 *                                      or compact slot rows when idx == NULL)
 *   idx       int32 [B, Hkv, S_cap]    base row of slot s, 0 <= idx < T_cap; NULL
 *                                      means slot s is row s (needs S <= T_cap)
 *   deg       int32 [B, Hkv, S_cap]    degree n_s >= 1 of slot s ([CKV] item 4:
 *                                      score += ln n_s); NULL means all 1
 *   S         live slots per (batch, kv head), same for all
 *   err_flag  int32 [1] or NULL: set to 1 when an idx entry is out of range (the
 *             entry is clamped and the result is then meaningless) or a degree < 1
 *
 * VC_CACHE_INT4 (asymmetric 4-bit groups; x_hat = q * scale + zero):
 *   Per (batch, kv head) the S quantised tokens (S % 32 == 0, capacity T_cap tokens,
 *   T_cap % 32 == 0) form blocks of 32.  Words are little-endian uint32 of 8 nibbles
 *   (nibble p at bits 4p..4p+3); pair j (0..3) of a word keeps its first element in
 *   nibble j and its second in nibble j + 4.
 *   kq        uint32 [B, Hkv, T_cap/32, 32, 4, D/32]: pair j of word (token t, c, w)
 *             holds channels e, e+1 of token t, e = 2c + 32w + 16*(j/2) + 8*(j%2)
 *   k_scale, k_zero  fp16 [B, Hkv, T_cap/32, D]: one group per (block, channel)
 *   vq        uint32 [B, Hkv, T_cap/32, D, 4]: pair j of word (channel d, c) holds
 *             channel d of tokens 2c + 8j and 2c + 8j + 1 of the block
 *   v_scale, v_zero  fp16 [B, Hkv, T_cap/32, D/32, 32]: one group per (token,
 *             32 consecutive channels), stored block, channel group, token
 *   All quantised tokens have degree 1.
 * ---------------------------------------------------------------------------- */
typedef struct vc_comp_cache {
  int32_t kind;                 /* vc_cache_kind */
  int32_t B, Hq, Hkv, D;
  int32_t S;                    /* live slots (indexed) or quantised tokens (int4) */
  int32_t S_cap;                /* row stride of idx / deg (indexed) */
  int64_t T_cap;                /* base rows (indexed) or token capacity (int4) */
  /* VC_CACHE_INDEXED */
  const void* k;
  const void* v;
  const int32_t* idx;
  const int32_t* deg;
  /* VC_CACHE_INT4 */
  const uint32_t* kq;
  const void* k_scale;
  const void* k_zero;
  const uint32_t* vq;
  const void* v_scale;
  const void* v_zero;
  /* tail */
  const void* k_tail;
  const void* v_tail;
  int32_t R_cap;
  int32_t n_tail;
  /* device error flag, may be NULL */
  int32_t* err_flag;
} vc_comp_cache;

/* Output precision flag shared by the attention calls: write `out` as fp32 instead of
 * bf16 (the fp32 value is the one the bf16 output is rounded from, to nearest even). */
#define VC_OUT_F32 4

/* ------------------------------------------------------------------------------
 * Draft attention: one decode step of every query head over KV_comp plus the tail
 * ([VC] "Algoritmo Principale", step 1, with the [CKV] log-degree term):
 *   s_t = (q . k_t) * scale + ln n_t ;  o = sum_t softmax(s)_t v_t
 *   q    bf16 [B, Hq, D]            out  bf16 [B, Hq, D] (fp32 with flags & VC_OUT_F32)
 *   lse  fp32 [B, Hq] or NULL: ln sum_t exp(s_t)
 *   scale <= 0 selects D^-1/2.
 * Split-K over slots: ws must hold vc_draft_workspace_size(cache) bytes (device).
 * S + n_tail must be >= 1.
 * ---------------------------------------------------------------------------- */
size_t vc_draft_workspace_size(const vc_comp_cache* cache);
vc_status vc_draft_attn(const void* q, const vc_comp_cache* cache, float scale, int flags,
                        void* out, float* lse, void* ws, size_t ws_bytes,
                        cudaStream_t stream);

/* Draft attention that allocates nothing and takes no workspace (the pages have no
 * counterpart: this serves callers that cannot hand the library scratch memory, such as
 * a plugin whose host runtime owns all device memory and offers no allocator, a process
 * whose memory pool is fully reserved up front, or a path that must not call cudaMalloc
 * because it can block and synchronise the device).  Same arguments and result as
 * vc_draft_attn, without ws / ws_bytes: the split-K partials go to a fixed 8 MiB array in
 * the library's device image, which every GPU that loads the library holds until exit.
 *   - A cache whose partials need more than 8 MiB (vc_draft_workspace_size) is rejected
 *     with VC_ERR_UNSUPPORTED before anything is launched.
 *   - The first call on each device does a one-time set-up (it looks up the array's
 *     device address with that device current); make that first call before any stream
 *     capture begins.  The address is kept per CUDA context, so the set-up runs again
 *     on the first call after a cudaDeviceReset or under another context.
 *   - All calls on a device share the one array and it keeps the last call's contents
 *     (nothing in it needs to start at zero).  Calls that overlap on the GPU -- on
 *     different streams, or from different threads -- race on it: serialise them. */
vc_status vc_draft_attn_noalloc(const void* q, const vc_comp_cache* cache, float scale,
                                int flags, void* out, float* lse, cudaStream_t stream);

/* ------------------------------------------------------------------------------
 * Verify attention ([VC] "Algoritmo Principale", step 2: one pass over KV_full checks
 * all drafted tokens in parallel).  Row i (0 <= i < n_q, n_q = k + 1: the pending
 * token and the k drafts) sits at absolute position P + i and attends every key at
 * position <= P + i: the prefix plus the block, causal inside the block.  No degree
 * term.
 *   q     bf16 [B, n_q, Hq, D]
 *   k, v  bf16 [B, Hkv, L_cap, D]: row r holds the key / value at absolute position
 *         kv_start + r, for r < kv_len (kv_len <= L_cap).  The block's own keys
 *         (positions P .. P+n_q-1) must already be written where they fall.
 *   Single pass (m == l == acc == NULL): kv_start == 0, kv_len == P + n_q; writes out
 *         bf16 [B, n_q, Hq, D] (fp32 with flags & VC_OUT_F32).
 *   Chunked (long context with KV_full streamed from host memory, [VC] "Supporto
 *         Architetturale"): m, l fp32 [B, n_q, Hq] and acc fp32 [B, n_q, Hq, D] carry
 *         the softmax state (running max of s * log2(e), sum of 2^(s*log2(e) - max),
 *         weighted values) between
 *         calls over consecutive key ranges in increasing kv_start.  VC_VERIFY_FIRST
 *         resets the state before adding this range; VC_VERIFY_LAST writes out after
 *         adding it.  Ranges must tile [0, P + n_q) exactly, in order.
 *   Results do not depend on n_q or on other rows: key tiles and split boundaries sit
 *   at fixed absolute positions, and splits are merged in a fixed order.  The split
 *   window (a multiple of 64 keys in [2048, 4096]; 4096 when B * Hkv * L_cap / 4096 is
 *   under one CTA per SM) is chosen from B * Hkv and L_cap only, so that the CTAs fill the
 *   SMs' last wave; every call on one cache uses the same one.
 *   ws: vc_verify_workspace_size(...) bytes of device memory (enough for any window).
 *   Supported: D in {64, 128}, g <= 8, n_q * g <= 1024.
 * ---------------------------------------------------------------------------- */
#define VC_VERIFY_FIRST 1
#define VC_VERIFY_LAST 2
size_t vc_verify_workspace_size(int B, int n_q, int Hq, int Hkv, int D,
                                int64_t kv_start, int64_t kv_len);
vc_status vc_verify_attn(const void* q, int B, int n_q, int Hq, int Hkv, int D,
                         const void* k, const void* v, int64_t L_cap,
                         int64_t kv_start, int64_t kv_len, int64_t P,
                         float* m, float* l, float* acc, int flags, float scale,
                         void* out, void* ws, size_t ws_bytes, cudaStream_t stream);

/* ------------------------------------------------------------------------------
 * Greedy acceptance ([VC] "Algoritmo Principale", step 3).
 *   logits  fp32 [B, n_q, V]; drafts int32 [B, n_q - 1] or NULL
 *   target[b, i] = argmax_v logits[b, i, v] (ties: lowest v; a NaN counts as larger
 *                  than any number, the first NaN wins)           int32 [B, n_q]
 *   accept_len[b] = a = first i < n_q-1 with target[b,i] != drafts[b,i], else n_q-1
 *   commit[b, :] = target[b, 0..a], then -1                        int32 [B, n_q]
 *   n_commit[b] = a + 1 (a == n_q-1: every draft plus the bonus token)
 *   err_flag[b] = 1 if row b had a NaN, else 0                    int32 [B] or NULL
 * With accept_len == commit == n_commit == NULL only target (and err_flag) are written
 * (the argmax of each draft step) and drafts is not read.  Otherwise all three must be
 * set and drafts must be non-NULL unless n_q == 1 (no drafts: a = 0).
 * ---------------------------------------------------------------------------- */
vc_status vc_accept(const float* logits, const int32_t* drafts, int B, int n_q, int V,
                    int32_t* target, int32_t* accept_len, int32_t* commit,
                    int32_t* n_commit, int32_t* err_flag, cudaStream_t stream);

/* ------------------------------------------------------------------------------
 * Staging of KV_full from pinned host memory to HBM over PCIe on a side stream
 * ([VC] "Scaglionamento tra Risorse (P1)" and "Supporto Architetturale": the full
 * cache lives in CPU memory and verification loads it over PCIe while other
 * requests draft).  Copies [0, bytes) of src to dst in chunks of chunk_bytes with
 * one cudaMemcpyAsync each (copy engine, no SMs) and records chunk_done[i] after
 * chunk i, so a verify call on another stream can wait on exactly its chunk.
 *   src_host must be page-locked (cudaHostAlloc / cudaHostRegister): checked.
 *   chunk_done may be NULL (n_events == 0); otherwise n_events >= number of chunks.
 * ---------------------------------------------------------------------------- */
vc_status vc_stage_full_kv(void* dst_dev, const void* src_host, size_t bytes,
                           size_t chunk_bytes, cudaStream_t copy_stream,
                           cudaEvent_t* chunk_done, int n_events);

/* Host wait on an event with a time limit (polls cudaEventQuery).  Returns VC_OK,
 * VC_ERR_TIMEOUT after timeout_s seconds, or VC_ERR_CUDA. */
vc_status vc_event_wait(cudaEvent_t ev, double timeout_s);

/* ----------------------------------------------------------------------------
 * One round of Chunked Soft Matching: CentroidKV's one-pass clustering of a KV cache
 * ([CKV] "Riassunto Tecnico: CentroidKV", section "Metodologia", items 2-4).  For each
 * (batch, kv head) pair, rows [0, n_sinks) and [T - n_recent, T) are kept as they are;
 * the rows between are cut into consecutive chunks of `chunk` rows (the last may be
 * shorter).  In a chunk, A = rows at even offsets, B = rows at odd offsets; each A row is
 * matched to its most similar B row by cosine of the key rows (lowest B row on ties; an
 * all-zero row has cosine 0 with everything); the m = floor(r * |A|) A rows with the
 * highest similarity (lower row on ties) merge into their matches.  A B row and the A
 * rows merged into it become one centroid: K and V = degree-weighted means (fp32 sums,
 * the B row first, then its A rows in ascending order, rounded to bf16 once), degree =
 * the sum.  A one-row chunk (no B row) merges nothing.  Output order: sinks, each chunk's surviving rows in their order (a centroid in
 * its B row's place), recent rows.  The result is a compact cache (idx = NULL, deg =
 * deg_out) for vc_draft_attn.  A decreasing r over successive rounds (r_j = r_init -
 * j * delta_r) is the caller's schedule.  Similarities use bf16 products with fp32
 * accumulation; a near-tie may resolve either way.
 *
 *   k, v      bf16 [pairs, T_cap, D] (device), the cache rows [0, T) of each pair
 *   deg       int32 [pairs, T_cap] degrees >= 1, or NULL (all 1)
 *   k_out, v_out  bf16 [pairs, T_cap_out, D]; deg_out int32 [pairs, T_cap_out]
 *             (must not overlap the inputs); rows [0, vc_csm_out_len(...)) are written
 *   dest      int32 [pairs, T_cap] or NULL: output row of every input row (the
 *             centroid's row for a merged row)
 *   D in {64, 128}; 2 <= chunk <= 256; 0 <= r <= 1; n_sinks + n_recent <= T <= T_cap;
 *   T < 2^31; pairs <= 65535; pointers 16-byte aligned.
 * ---------------------------------------------------------------------------- */
int64_t vc_csm_out_len(int64_t T, int n_sinks, int n_recent, int chunk, double r);
vc_status vc_csm_compress(const void* k, const void* v, const int32_t* deg, int pairs, int D,
                          int64_t T, int64_t T_cap, int n_sinks, int n_recent, int chunk,
                          double r, void* k_out, void* v_out, int32_t* deg_out,
                          int64_t T_cap_out, int32_t* dest, cudaStream_t stream);

/* ----------------------------------------------------------------------------
 * Int4 compressor: quantise whole 32-token blocks of bf16 K/V rows into the
 * VC_CACHE_INT4 layout above ([VC] "Supporto Architetturale": quantisation plugs into
 * the uniform compression interface; [CKV] "Problematica": quantisation among the known
 * KV-cache reductions).  Groups as in the layout: keys per channel over the block's 32
 * tokens, values per token over 32 consecutive channels;
 *     z = fp16(min), s = fp16((max - min) / 15) (1 if that is 0),
 *     n = clamp(rint((x - z) / s), 0, 15), round half to even, in fp64.
 * This is how tokens leaving a bf16 window join the quantised part of the cache: call it
 * on each 32 rows that leave, with blk0 = the next free block.
 *   k, v      bf16 [pairs, src_cap, D]; rows src_t0 .. src_t0 + 32 n_blocks - 1 of every
 *             pair are read
 *   kq, k_scale, k_zero, vq, v_scale, v_zero: the int4 arrays with capacity blk_cap
 *             blocks per pair (T_cap = 32 blk_cap); blocks blk0 .. blk0 + n_blocks - 1
 *             of every pair are written, nothing else
 *   D in {64, 128}; pairs <= 65535; pointers (and row src_t0) 16-byte aligned.
 *   Groups with values beyond the fp16 range cannot be represented (result unspecified).
 * ---------------------------------------------------------------------------- */
vc_status vc_int4_quantize(const void* k, const void* v, int pairs, int D, int64_t src_cap,
                           int64_t src_t0, int n_blocks, uint32_t* kq, void* k_scale,
                           void* k_zero, uint32_t* vq, void* v_scale, void* v_zero,
                           int64_t blk_cap, int64_t blk0, cudaStream_t stream);

/* ----------------------------------------------------------------------------
 * Token eviction by attention score ([CKV] "Problematica": eviction drops the tokens
 * with the lowest attention scores; [CKV] "Metodologia" item 2 "Preservazione": sinks and
 * recent tokens are always kept; [VC] "Supporto Architetturale": eviction compressors
 * plug into the same interface).
 *
 * vc_evict_scores: for a prompt of n tokens, the attention mass each key receives from
 * the last W prompt queries over the g query heads of its kv head:
 *     score[b, j, t] = sum_{w < W, h in group j} softmax_{t' <= n-W+w}(q . k_t' * scale)[t]
 *   q      bf16 [B, W, Hq, D]: the queries of positions n-W .. n-1 (as attention sees
 *          them, i.e. after any rotary embedding)
 *   k      bf16 [B, Hkv, L_cap, D]: keys of positions 0 .. n-1 in rows 0 .. n-1
 *   score  fp32 [B, Hkv, score_cap], entries [0, n) written (each a fixed-order fp32 sum)
 *   ws     device workspace of vc_evict_workspace_size(B, W, Hq) bytes
 *   scale <= 0 selects D^-1/2.  D in {64, 128}, g <= 8, W <= 32, W <= n <= L_cap.
 *
 * vc_evict_select: per row r (e.g. (batch, kv head)) of score [rows, score_cap], the kept
 * positions in ascending order: [0, n_sinks), then the budget - n_sinks - n_recent
 * highest-scoring positions of [n_sinks, n - n_recent) (equal scores: the lower position
 * first), then [n - n_recent, n); budget >= n keeps 0 .. n-1.  Writes idx int32
 * [rows, S_cap], entries [0, min(budget, n)).  Exact: depends only on the scores' order.
 * ---------------------------------------------------------------------------- */
size_t vc_evict_workspace_size(int B, int W, int Hq);
vc_status vc_evict_scores(const void* q, int B, int W, int Hq, int Hkv, int D, const void* k,
                          int64_t L_cap, int64_t n, float scale, float* score,
                          int64_t score_cap, void* ws, size_t ws_bytes, cudaStream_t stream);
vc_status vc_evict_select(const float* score, int rows, int64_t score_cap, int64_t n,
                          int budget, int n_sinks, int n_recent, int32_t* idx, int64_t S_cap,
                          cudaStream_t stream);

/* The library's device error word on the current device (synchronous read; clear != 0
 * resets it).  Bit 0: a bounded wait inside a verify-attention CTA expired (the call's
 * output is then invalid; the CTA released its resources and exited). */
vc_status vc_device_error(int32_t* value, int clear);

/* Failure detection (no counterpart in the pages).  Sets the time limit of every
 * pipeline wait inside the verify-attention kernel for the launches that follow (a
 * process-wide setting; default 2 s; seconds == 0 restores it; at most 60 s) and
 * returns the previous limit in *previous (may be NULL).  A wait that runs out raises
 * bit 0 of the device error word and the CTA exits cleanly, leaving the context usable;
 * a very short limit makes that happen on purpose, which is how the error path is tested
 * without any device fault.
 * Staging has a host-side injection point for the same purpose: with the environment
 * variable VC_FAULT_INJECT=stage_fail, vc_stage_full_kv returns VC_ERR_CUDA before
 * enqueueing anything. */
vc_status vc_set_wait_limit(double seconds, double* previous);

#ifdef __cplusplus
}
#endif
#endif /* VERICACHE_H */
