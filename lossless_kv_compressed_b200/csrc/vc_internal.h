// Host-side internals shared by the translation units of the library.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "vericache.h"

namespace vc {

// Records a message for vc_last_error() and returns the status.
vc_status fail(vc_status st, const char* fmt, ...);
// Number of SMs of the current device (cached per device).
int num_sms();
// Raise a kernel's dynamic shared memory limit to at least bytes on the current device;
// the attribute call is made only when the limit granted so far is smaller.
cudaError_t grant_smem(const void* func, int bytes);

#define VC_CUDA(call)                                                                \
  do {                                                                               \
    cudaError_t e_ = (call);                                                         \
    if (e_ != cudaSuccess)                                                           \
      return ::vc::fail(VC_ERR_CUDA, "%s: %s (%s:%d)", #call, cudaGetErrorString(e_), \
                        __FILE__, __LINE__);                                         \
  } while (0)

size_t draft_workspace_bytes(const vc_comp_cache* c);
vc_status launch_draft_indexed(const void* q, const vc_comp_cache* c, float scale, int flags,
                               void* out, float* lse, void* ws, size_t ws_bytes,
                               cudaStream_t stream);
vc_status launch_draft_int4(const void* q, const vc_comp_cache* c, float scale, int flags,
                            void* out, float* lse, void* ws, size_t ws_bytes,
                            cudaStream_t stream);

// Verify attention splits the keys into absolute windows of split_keys positions (a
// multiple of 64); calls whose rows must agree bit for bit use the same window.  The
// public entry point uses kVerifySplitKeys.
constexpr int kVerifySplitKeys = 4096;
size_t verify_workspace_bytes(int B, int n_q, int Hq, int Hkv, int D, int64_t kv_start,
                              int64_t kv_len, int split_keys = kVerifySplitKeys);
vc_status launch_verify(const void* q, int B, int n_q, int Hq, int Hkv, int D, const void* k,
                        const void* v, int64_t L_cap, int64_t kv_start, int64_t kv_len,
                        int64_t P, float* m, float* l, float* acc, int flags, float scale,
                        void* out, void* ws, size_t ws_bytes, cudaStream_t stream,
                        int split_keys = kVerifySplitKeys);
// The public entry point's window for a cache of pairs (batch x kv head) and capacity
// L_cap: a function of those two only, so every call on one cache uses the same one.
int verify_window(int64_t pairs, int64_t L_cap);
// Workspace bytes enough for any window verify_window can return.
size_t verify_workspace_bytes_any(int B, int n_q, int Hq, int Hkv, int D, int64_t kv_start,
                                  int64_t kv_len);
// vc_verify_attn's argument checks and launch with a chosen window.
vc_status verify_checked(const void* q, int B, int n_q, int Hq, int Hkv, int D, const void* k,
                         const void* v, int64_t L_cap, int64_t kv_start, int64_t kv_len,
                         int64_t P, float* m, float* l, float* acc, int flags, float scale,
                         void* out, void* ws, size_t ws_bytes, cudaStream_t stream,
                         int split_keys);

vc_status read_device_error(int32_t* value, int clear);
constexpr uint64_t kDefaultWaitNs = 2000000000ull;   // 2 s
uint64_t set_verify_wait_ns(uint64_t ns);            // returns the previous limit

int64_t csm_out_len(int64_t T, int n_sinks, int n_recent, int chunk, double r);
vc_status launch_csm(const void* k, const void* v, const int32_t* deg, int pairs, int D,
                     int64_t T, int64_t T_cap, int n_sinks, int n_recent, int chunk, double r,
                     void* k_out, void* v_out, int32_t* deg_out, int64_t T_cap_out,
                     int32_t* dest, cudaStream_t stream);

vc_status launch_int4_quantize(const void* k, const void* v, int pairs, int D, int64_t src_cap,
                               int64_t src_t0, int n_blocks, uint32_t* kq, void* k_scale,
                               void* k_zero, uint32_t* vq, void* v_scale, void* v_zero,
                               int64_t blk_cap, int64_t blk0, cudaStream_t stream);

vc_status launch_evict_scores(const void* q, int B, int W, int Hq, int Hkv, int D,
                              const void* k, int64_t L_cap, int64_t n, float scale,
                              float* score, int64_t score_cap, float* ws, cudaStream_t stream);
vc_status launch_evict_select(const float* score, int rows, int64_t score_cap, int64_t n,
                              int budget, int n_sinks, int n_recent, int32_t* idx,
                              int64_t S_cap, cudaStream_t stream);

vc_status launch_accept(const float* logits, const int32_t* drafts, int B, int n_q, int V,
                        int32_t* target, int32_t* accept_len, int32_t* commit,
                        int32_t* n_commit, int32_t* err_flag, cudaStream_t stream);

}  // namespace vc
