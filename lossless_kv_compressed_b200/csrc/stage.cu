// Staging of the full cache KV_full from pinned host memory to HBM over PCIe.
//
// VeriCache summary ("Riepilogo Tecnico: VeriCache"): in the long-context scenario the
// full cache sits in CPU memory and verification loads it over PCIe (section
// "Supporto Architetturale"); the runtime staggers requests so this transfer overlaps
// other requests' HBM-bound drafting (section "Scaglionamento tra Risorse (P1)").
//
// The copy runs on the copy engines (cudaMemcpyAsync from page-locked memory, one
// call per chunk, no SM involved) on a caller-given side stream; an event after each
// chunk lets the verify stream start on chunk i while chunk i+1 is in flight.
#include <chrono>
#include <cstdlib>
#include <cstring>
#include <thread>

#include "vc_internal.h"

namespace vc {

// Host-side fault injection for failure-detection tests: with VC_FAULT_INJECT set to
// "stage_fail" in the environment, every staging call fails as a failed copy would,
// before anything is enqueued (no device work, no device fault).
static bool inject_stage_failure() {
  const char* e = std::getenv("VC_FAULT_INJECT");
  return e != nullptr && std::strcmp(e, "stage_fail") == 0;
}

vc_status stage_full_kv(void* dst, const void* src, size_t bytes, size_t chunk,
                        cudaStream_t stream, cudaEvent_t* done, int n_events) {
  if (inject_stage_failure())
    return fail(VC_ERR_CUDA, "stage: injected copy failure (VC_FAULT_INJECT=stage_fail)");
  if (!dst || !src) return fail(VC_ERR_INVALID, "stage: null pointer");
  if (chunk == 0) return fail(VC_ERR_INVALID, "stage: chunk_bytes == 0");
  const size_t n_chunks = bytes == 0 ? 0 : (bytes + chunk - 1) / chunk;
  if (done && (size_t)n_events < n_chunks)
    return fail(VC_ERR_INVALID, "stage: %d events for %zu chunks", n_events, n_chunks);
  cudaPointerAttributes a;
  VC_CUDA(cudaPointerGetAttributes(&a, src));
  if (a.type != cudaMemoryTypeHost)
    return fail(VC_ERR_INVALID, "stage: source is not page-locked host memory");
  cudaPointerAttributes d;
  VC_CUDA(cudaPointerGetAttributes(&d, dst));
  if (d.type != cudaMemoryTypeDevice)
    return fail(VC_ERR_INVALID, "stage: destination is not device memory");
  const char* s = static_cast<const char*>(src);
  char* t = static_cast<char*>(dst);
  for (size_t i = 0; i < n_chunks; ++i) {
    const size_t off = i * chunk;
    const size_t n = bytes - off < chunk ? bytes - off : chunk;
    VC_CUDA(cudaMemcpyAsync(t + off, s + off, n, cudaMemcpyHostToDevice, stream));
    if (done) VC_CUDA(cudaEventRecord(done[i], stream));
  }
  return VC_OK;
}

vc_status event_wait(cudaEvent_t ev, double timeout_s) {
  const auto t0 = std::chrono::steady_clock::now();
  for (;;) {
    const cudaError_t e = cudaEventQuery(ev);
    if (e == cudaSuccess) return VC_OK;
    if (e != cudaErrorNotReady)
      return fail(VC_ERR_CUDA, "cudaEventQuery: %s", cudaGetErrorString(e));
    const double dt =
        std::chrono::duration<double>(std::chrono::steady_clock::now() - t0).count();
    if (dt > timeout_s) return fail(VC_ERR_TIMEOUT, "event not reached after %.3f s", dt);
    std::this_thread::sleep_for(std::chrono::microseconds(20));
  }
}

}  // namespace vc
