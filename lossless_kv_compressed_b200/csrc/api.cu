// C ABI entry points: argument validation and dispatch.  Every check that can be
// made on the host is made here; nothing is launched on a failed check.
#include <cstdarg>
#include <cstdio>
#include <mutex>
#include <vector>

#include "vc_internal.h"

namespace vc {

namespace {
thread_local char g_err[512] = "";

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }
}  // namespace

vc_status fail(vc_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return st;
}

int num_sms() {
  static std::mutex mu;
  static std::vector<int> cache;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  std::lock_guard<std::mutex> lk(mu);
  if ((int)cache.size() <= dev) cache.resize(dev + 1, 0);
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cache[dev] = n;
  }
  return cache[dev];
}

cudaError_t grant_smem(const void* func, int bytes) {
  struct Granted { const void* func; int dev; int bytes; };
  static std::mutex mu;
  static std::vector<Granted> granted;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lk(mu);
  for (Granted& g : granted) {
    if (g.func == func && g.dev == dev) {
      if (g.bytes >= bytes) return cudaSuccess;
      e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
      if (e == cudaSuccess) g.bytes = bytes;
      return e;
    }
  }
  e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) granted.push_back({func, dev, bytes});
  return e;
}

vc_status stage_full_kv(void* dst, const void* src, size_t bytes, size_t chunk,
                        cudaStream_t stream, cudaEvent_t* done, int n_events);
vc_status event_wait(cudaEvent_t ev, double timeout_s);

static vc_status check_cache(const vc_comp_cache* c) {
  if (!c) return fail(VC_ERR_INVALID, "cache is NULL");
  if (c->B <= 0 || c->Hq <= 0 || c->Hkv <= 0 || c->D <= 0)
    return fail(VC_ERR_INVALID, "B, Hq, Hkv, D must be positive");
  if (c->Hq % c->Hkv) return fail(VC_ERR_INVALID, "Hq %% Hkv != 0");
  if (c->D != 64 && c->D != 128) return fail(VC_ERR_UNSUPPORTED, "D must be 64 or 128");
  if (c->Hq / c->Hkv > 8) return fail(VC_ERR_UNSUPPORTED, "GQA group g > 8");
  if (c->S < 0 || c->n_tail < 0) return fail(VC_ERR_INVALID, "negative S or n_tail");
  if (c->S + c->n_tail < 1) return fail(VC_ERR_INVALID, "no slots (S + n_tail == 0)");
  if (c->n_tail > 0) {
    if (!c->k_tail || !c->v_tail) return fail(VC_ERR_INVALID, "tail pointers NULL");
    if (c->R_cap < c->n_tail) return fail(VC_ERR_INVALID, "n_tail > R_cap");
    if (!aligned16(c->k_tail) || !aligned16(c->v_tail))
      return fail(VC_ERR_INVALID, "tail not 16-byte aligned");
  }
  if (c->kind == VC_CACHE_INDEXED) {
    if (c->S > 0) {
      if (!c->k || !c->v) return fail(VC_ERR_INVALID, "k / v NULL");
      if (!aligned16(c->k) || !aligned16(c->v)) return fail(VC_ERR_INVALID, "k / v misaligned");
      if ((c->idx || c->deg) && c->S_cap < c->S) return fail(VC_ERR_INVALID, "S > S_cap");
      if (!c->idx && c->S > c->T_cap) return fail(VC_ERR_INVALID, "compact cache: S > T_cap");
      if (c->T_cap <= 0 || c->T_cap >= (int64_t)1 << 31)
        return fail(VC_ERR_INVALID, "T_cap out of range");
    }
  } else if (c->kind == VC_CACHE_INT4) {
    if (c->S % 32 || c->T_cap % 32) return fail(VC_ERR_INVALID, "int4: S, T_cap % 32 != 0");
    if (c->S > c->T_cap) return fail(VC_ERR_INVALID, "int4: S > T_cap");
    if (c->S > 0) {
      if (!c->kq || !c->vq || !c->k_scale || !c->k_zero || !c->v_scale || !c->v_zero)
        return fail(VC_ERR_INVALID, "int4: NULL pointer");
      if (!aligned16(c->kq) || !aligned16(c->vq) || !aligned16(c->k_scale) ||
          !aligned16(c->k_zero) || !aligned16(c->v_scale) || !aligned16(c->v_zero))
        return fail(VC_ERR_INVALID, "int4: misaligned pointer");
    }
  } else {
    return fail(VC_ERR_INVALID, "unknown cache kind %d", c->kind);
  }
  return VC_OK;
}

}  // namespace vc

using namespace vc;

extern "C" {

const char* vc_status_string(int s) {
  switch (s) {
    case VC_OK: return "VC_OK";
    case VC_ERR_INVALID: return "VC_ERR_INVALID";
    case VC_ERR_UNSUPPORTED: return "VC_ERR_UNSUPPORTED";
    case VC_ERR_CUDA: return "VC_ERR_CUDA";
    case VC_ERR_TIMEOUT: return "VC_ERR_TIMEOUT";
    default: return "VC_UNKNOWN_STATUS";
  }
}

const char* vc_last_error(void) { return g_err; }

int vc_abi_version(void) { return VC_ABI_VERSION; }

size_t vc_draft_workspace_size(const vc_comp_cache* cache) {
  if (check_cache(cache) != VC_OK) return 0;
  return draft_workspace_bytes(cache);
}

vc_status vc_draft_attn(const void* q, const vc_comp_cache* cache, float scale, int flags,
                        void* out, float* lse, void* ws, size_t ws_bytes, cudaStream_t stream) {
  vc_status st = check_cache(cache);
  if (st != VC_OK) return st;
  if (!q || !out || !ws) return fail(VC_ERR_INVALID, "draft: q / out / ws NULL");
  if (!aligned16(q) || !aligned16(out) || !aligned16(ws))
    return fail(VC_ERR_INVALID, "draft: q / out / ws misaligned");
  if (scale <= 0.f) scale = 1.0f / sqrtf((float)cache->D);
  if (flags & ~VC_OUT_F32) return fail(VC_ERR_INVALID, "draft: unknown flags");
  if (cache->kind == VC_CACHE_INDEXED)
    return launch_draft_indexed(q, cache, scale, flags, out, lse, ws, ws_bytes, stream);
  return launch_draft_int4(q, cache, scale, flags, out, lse, ws, ws_bytes, stream);
}

size_t vc_verify_workspace_size(int B, int n_q, int Hq, int Hkv, int D, int64_t kv_start,
                                int64_t kv_len) {
  if (B <= 0 || n_q <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || kv_start < 0 || kv_len <= 0)
    return 0;
  return verify_workspace_bytes_any(B, n_q, Hq, Hkv, D, kv_start, kv_len);
}

vc_status vc_verify_attn(const void* q, int B, int n_q, int Hq, int Hkv, int D, const void* k,
                         const void* v, int64_t L_cap, int64_t kv_start, int64_t kv_len,
                         int64_t P, float* m, float* l, float* acc, int flags, float scale,
                         void* out, void* ws, size_t ws_bytes, cudaStream_t stream) {
  return verify_checked(q, B, n_q, Hq, Hkv, D, k, v, L_cap, kv_start, kv_len, P, m, l, acc,
                        flags, scale, out, ws, ws_bytes, stream,
                        verify_window((int64_t)B * Hkv, L_cap));
}

}  // extern "C"

namespace vc {
vc_status verify_checked(const void* q, int B, int n_q, int Hq, int Hkv, int D, const void* k,
                         const void* v, int64_t L_cap, int64_t kv_start, int64_t kv_len,
                         int64_t P, float* m, float* l, float* acc, int flags, float scale,
                         void* out, void* ws, size_t ws_bytes, cudaStream_t stream,
                         int split_keys) {
  if (B <= 0 || n_q <= 0 || Hq <= 0 || Hkv <= 0) return fail(VC_ERR_INVALID, "verify: sizes");
  if (Hq % Hkv) return fail(VC_ERR_INVALID, "verify: Hq %% Hkv != 0");
  if (D != 64 && D != 128) return fail(VC_ERR_UNSUPPORTED, "verify: D must be 64 or 128");
  if (Hq / Hkv > 8) return fail(VC_ERR_UNSUPPORTED, "verify: g > 8");
  if ((int64_t)n_q * (Hq / Hkv) > 1024) return fail(VC_ERR_UNSUPPORTED, "verify: n_q * g > 1024");
  if (!q || !k || !v || !ws) return fail(VC_ERR_INVALID, "verify: NULL pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(ws))
    return fail(VC_ERR_INVALID, "verify: misaligned pointer");
  if (kv_start < 0 || kv_len <= 0 || kv_len > L_cap || P < 0)
    return fail(VC_ERR_INVALID, "verify: bad key range");
  if (flags & ~(VC_VERIFY_FIRST | VC_VERIFY_LAST | VC_OUT_F32))
    return fail(VC_ERR_INVALID, "verify: unknown flags");
  const bool chunked = m || l || acc;
  if (chunked) {
    if (!m || !l || !acc) return fail(VC_ERR_INVALID, "verify: m, l, acc must all be set");
    if (kv_start + kv_len > P + n_q) return fail(VC_ERR_INVALID, "verify: range past the block");
    if ((flags & VC_VERIFY_LAST) && kv_start + kv_len != P + n_q)
      return fail(VC_ERR_INVALID, "verify: last range must end at P + n_q");
    if ((flags & VC_VERIFY_FIRST) && kv_start != 0)
      return fail(VC_ERR_INVALID, "verify: first range must start at 0");
    if ((flags & VC_VERIFY_LAST) && !out) return fail(VC_ERR_INVALID, "verify: out NULL");
  } else {
    if (kv_start != 0 || kv_len != P + n_q)
      return fail(VC_ERR_INVALID, "verify: single pass needs kv_start 0, kv_len P + n_q");
    if (!out) return fail(VC_ERR_INVALID, "verify: out NULL");
    flags = (flags & VC_OUT_F32) | VC_VERIFY_FIRST | VC_VERIFY_LAST;
  }
  if (out && !aligned16(out)) return fail(VC_ERR_INVALID, "verify: out misaligned");
  if (scale <= 0.f) scale = 1.0f / sqrtf((float)D);
  return launch_verify(q, B, n_q, Hq, Hkv, D, k, v, L_cap, kv_start, kv_len, P, m, l, acc,
                       flags, scale, out, ws, ws_bytes, stream, split_keys);
}
}  // namespace vc

extern "C" {


vc_status vc_accept(const float* logits, const int32_t* drafts, int B, int n_q, int V,
                    int32_t* target, int32_t* accept_len, int32_t* commit, int32_t* n_commit,
                    int32_t* err_flag, cudaStream_t stream) {
  if (B <= 0 || n_q <= 0 || V <= 0) return fail(VC_ERR_INVALID, "accept: sizes");
  if (!logits || !target) return fail(VC_ERR_INVALID, "accept: logits / target NULL");
  const bool acc = accept_len || commit || n_commit;
  if (acc && (!accept_len || !commit || !n_commit))
    return fail(VC_ERR_INVALID, "accept: accept_len, commit, n_commit must be all set or all NULL");
  if (acc && !drafts && n_q > 1) return fail(VC_ERR_INVALID, "accept: drafts NULL");
  if (!acc) drafts = nullptr;
  return launch_accept(logits, drafts, B, n_q, V, target, accept_len, commit, n_commit,
                       err_flag, stream);
}

vc_status vc_stage_full_kv(void* dst_dev, const void* src_host, size_t bytes, size_t chunk_bytes,
                           cudaStream_t copy_stream, cudaEvent_t* chunk_done, int n_events) {
  return stage_full_kv(dst_dev, src_host, bytes, chunk_bytes, copy_stream, chunk_done, n_events);
}

vc_status vc_event_wait(cudaEvent_t ev, double timeout_s) { return event_wait(ev, timeout_s); }

vc_status vc_device_error(int32_t* value, int clear) { return read_device_error(value, clear); }

vc_status vc_set_wait_limit(double seconds, double* previous) {
  if (!(seconds >= 0.0 && seconds <= 60.0))
    return fail(VC_ERR_INVALID, "wait limit must be in [0, 60] s (0 restores 2 s)");
  const uint64_t ns = seconds == 0.0 ? kDefaultWaitNs : (uint64_t)(seconds * 1e9);
  const uint64_t old = set_verify_wait_ns(ns < 1 ? 1 : ns);
  if (previous) *previous = (double)old * 1e-9;
  return VC_OK;
}

int64_t vc_csm_out_len(int64_t T, int n_sinks, int n_recent, int chunk, double r) {
  if (T < 0 || n_sinks < 0 || n_recent < 0 || (int64_t)n_sinks + n_recent > T || chunk < 2 ||
      chunk > 256 || !(r >= 0.0 && r <= 1.0))
    return -1;
  return csm_out_len(T, n_sinks, n_recent, chunk, r);
}

vc_status vc_csm_compress(const void* k, const void* v, const int32_t* deg, int pairs, int D,
                          int64_t T, int64_t T_cap, int n_sinks, int n_recent, int chunk,
                          double r, void* k_out, void* v_out, int32_t* deg_out,
                          int64_t T_cap_out, int32_t* dest, cudaStream_t stream) {
  if (pairs <= 0 || pairs > 65535) return fail(VC_ERR_INVALID, "csm: pairs");
  if (D != 64 && D != 128) return fail(VC_ERR_UNSUPPORTED, "csm: D must be 64 or 128");
  if (chunk < 2 || chunk > 256) return fail(VC_ERR_UNSUPPORTED, "csm: chunk must be in [2, 256]");
  if (!(r >= 0.0 && r <= 1.0)) return fail(VC_ERR_INVALID, "csm: r must be in [0, 1]");
  if (n_sinks < 0 || n_recent < 0 || (int64_t)n_sinks + n_recent > T || T > T_cap ||
      T >= ((int64_t)1 << 31))
    return fail(VC_ERR_INVALID, "csm: need n_sinks + n_recent <= T <= T_cap, T < 2^31");
  if (!k || !v || !k_out || !v_out || !deg_out)
    return fail(VC_ERR_INVALID, "csm: k, v, k_out, v_out, deg_out must be set");
  if (!aligned16(k) || !aligned16(v) || !aligned16(k_out) || !aligned16(v_out))
    return fail(VC_ERR_INVALID, "csm: k / v / k_out / v_out misaligned");
  const int64_t n_out = csm_out_len(T, n_sinks, n_recent, chunk, r);
  if (n_out > T_cap_out) return fail(VC_ERR_INVALID, "csm: T_cap_out < output rows");
  return launch_csm(k, v, deg, pairs, D, T, T_cap, n_sinks, n_recent, chunk, r, k_out, v_out,
                    deg_out, T_cap_out, dest, stream);
}

vc_status vc_int4_quantize(const void* k, const void* v, int pairs, int D, int64_t src_cap,
                           int64_t src_t0, int n_blocks, uint32_t* kq, void* k_scale,
                           void* k_zero, uint32_t* vq, void* v_scale, void* v_zero,
                           int64_t blk_cap, int64_t blk0, cudaStream_t stream) {
  if (pairs <= 0 || pairs > 65535) return fail(VC_ERR_INVALID, "quantize: pairs");
  if (D != 64 && D != 128) return fail(VC_ERR_UNSUPPORTED, "quantize: D must be 64 or 128");
  if (n_blocks < 0 || src_t0 < 0 || blk0 < 0 || src_t0 + 32 * (int64_t)n_blocks > src_cap ||
      blk0 + n_blocks > blk_cap)
    return fail(VC_ERR_INVALID, "quantize: block range outside the source or the cache");
  if (!k || !v || !kq || !k_scale || !k_zero || !vq || !v_scale || !v_zero)
    return fail(VC_ERR_INVALID, "quantize: NULL pointer");
  if (!aligned16(k) || !aligned16(v) || !aligned16(kq) || !aligned16(vq) ||
      !aligned16(k_scale) || !aligned16(k_zero) || !aligned16(v_scale) || !aligned16(v_zero))
    return fail(VC_ERR_INVALID, "quantize: misaligned pointer");
  if (((src_t0 * D * 2) & 15) != 0) return fail(VC_ERR_INVALID, "quantize: src_t0 misaligned");
  return launch_int4_quantize(k, v, pairs, D, src_cap, src_t0, n_blocks, kq, k_scale, k_zero,
                              vq, v_scale, v_zero, blk_cap, blk0, stream);
}

size_t vc_evict_workspace_size(int B, int W, int Hq) {
  if (B <= 0 || W <= 0 || Hq <= 0) return 0;
  return (size_t)B * W * Hq * sizeof(float) + 256;
}

vc_status vc_evict_scores(const void* q, int B, int W, int Hq, int Hkv, int D, const void* k,
                          int64_t L_cap, int64_t n, float scale, float* score,
                          int64_t score_cap, void* ws, size_t ws_bytes, cudaStream_t stream) {
  if (B <= 0 || W <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv)
    return fail(VC_ERR_INVALID, "evict_scores: sizes");
  if (D != 64 && D != 128) return fail(VC_ERR_UNSUPPORTED, "evict_scores: D must be 64 or 128");
  if (Hq / Hkv > 8) return fail(VC_ERR_UNSUPPORTED, "evict_scores: g > 8");
  if (W > 32) return fail(VC_ERR_UNSUPPORTED, "evict_scores: W > 32");
  if (n < W || n > L_cap || n > score_cap || (int64_t)B * Hkv > 65535)
    return fail(VC_ERR_INVALID, "evict_scores: need W <= n <= L_cap, n <= score_cap");
  if (!q || !k || !score || !ws) return fail(VC_ERR_INVALID, "evict_scores: NULL pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(ws))
    return fail(VC_ERR_INVALID, "evict_scores: misaligned pointer");
  if (ws_bytes < (size_t)B * W * Hq * sizeof(float))
    return fail(VC_ERR_INVALID, "evict_scores: workspace too small");
  if (scale <= 0.f) scale = 1.0f / sqrtf((float)D);
  return launch_evict_scores(q, B, W, Hq, Hkv, D, k, L_cap, n, scale, score, score_cap,
                             static_cast<float*>(ws), stream);
}

vc_status vc_evict_select(const float* score, int rows, int64_t score_cap, int64_t n,
                          int budget, int n_sinks, int n_recent, int32_t* idx, int64_t S_cap,
                          cudaStream_t stream) {
  if (rows <= 0 || n <= 0 || n > score_cap || n >= ((int64_t)1 << 31))
    return fail(VC_ERR_INVALID, "evict_select: sizes");
  if (n_sinks < 0 || n_recent < 0 || budget < 1)
    return fail(VC_ERR_INVALID, "evict_select: budget, n_sinks, n_recent");
  if ((int64_t)budget < n && (int64_t)n_sinks + n_recent > budget)
    return fail(VC_ERR_INVALID, "evict_select: sinks + recent exceed the budget");
  if ((int64_t)budget < n && (int64_t)n_sinks + n_recent > n)
    return fail(VC_ERR_INVALID, "evict_select: sinks + recent exceed n");
  if (S_cap < ((int64_t)budget < n ? (int64_t)budget : n))
    return fail(VC_ERR_INVALID, "evict_select: S_cap too small");
  if (!score || !idx) return fail(VC_ERR_INVALID, "evict_select: NULL pointer");
  return launch_evict_select(score, rows, score_cap, n, budget, n_sinks, n_recent, idx, S_cap,
                             stream);
}

}  // extern "C"
