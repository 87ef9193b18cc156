// Greedy acceptance over the verify logits (VeriCache summary, "Riepilogo Tecnico:
// VeriCache", section "Algoritmo Principale", step 3): accept drafted tokens up to
// the first disagreement with the full-KV prediction, plus one bonus token when all
// agree.
//
// Kernel 1: float4 streaming argmax of each logits row (ties -> lowest index; NaN
//           larger than any number, first NaN wins); large vocabularies split a row
//           over an 8-CTA cluster merged through distributed shared memory.  The
//           row's NaN bit is parked in bit 31 of its target entry.
// Kernel 2: one warp per batch row: clears the NaN bits into err_flag, finds the first
//           disagreement with a ballot, and writes accept_len / commit / n_commit.
#include <climits>

#include <cooperative_groups.h>

#include "vc_common.cuh"
#include "vc_internal.h"

namespace vc {

struct ArgBest {
  float val;
  int idx;
};

// true if (v, i) should replace the current best (b) -- larger value, or equal
// value at a lower index.
__device__ __forceinline__ bool better(float v, int i, const ArgBest& b) {
  return v > b.val || (v == b.val && i < b.idx);
}

// One row per thread-block cluster of CL CTAs: CTA c scans a contiguous slice of the
// row, the cluster's rank-0 CTA merges the CL partials through distributed shared
// memory (slices in order, so the lowest index still wins ties).
template <int THREADS, int CL>
__global__ void __launch_bounds__(THREADS) argmax_rows_kernel(const float* __restrict__ logits,
                                                              int V, int32_t* __restrict__ target) {
  namespace cg = cooperative_groups;
  const int64_t row = blockIdx.x / CL;
  const int crank = (int)(blockIdx.x % CL);
  const float* x = logits + row * (int64_t)V;
  // slice [lo, hi) of the row, multiples of 4 so float4 loads stay aligned
  const int per = ((V + CL - 1) / CL + 3) & ~3;
  const int lo = min(V, crank * per), hi = min(V, lo + per);
  ArgBest best{-INFINITY, INT_MAX};
  int first_nan = INT_MAX;
  const bool vec = ((V & 3) == 0) && ((reinterpret_cast<uintptr_t>(x) & 15) == 0);
  if (vec) {
    const float4* x4 = reinterpret_cast<const float4*>(x);
    for (int i = (lo >> 2) + threadIdx.x; i < (hi >> 2); i += THREADS) {
      const float4 f = __ldg(x4 + i);
      const float e[4] = {f.x, f.y, f.z, f.w};
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int id = 4 * i + u;
        if (isnan(e[u])) first_nan = min(first_nan, id);
        else if (better(e[u], id, best)) best = {e[u], id};
      }
    }
  } else {
    for (int i = lo + threadIdx.x; i < hi; i += THREADS) {
      const float e = __ldg(x + i);
      if (isnan(e)) first_nan = min(first_nan, i);
      else if (better(e, i, best)) best = {e, i};
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float v = __shfl_xor_sync(0xffffffffu, best.val, o);
    const int i = __shfl_xor_sync(0xffffffffu, best.idx, o);
    if (better(v, i, best)) best = {v, i};
    first_nan = min(first_nan, __shfl_xor_sync(0xffffffffu, first_nan, o));
  }
  __shared__ float sv[THREADS / 32];
  __shared__ int si[THREADS / 32];
  __shared__ int sn[THREADS / 32];
  __shared__ float cv;   // this CTA's result, read by the cluster leader
  __shared__ int ci, cn;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) { sv[warp] = best.val; si[warp] = best.idx; sn[warp] = first_nan; }
  __syncthreads();
  if (warp == 0) {
    constexpr int NW = THREADS / 32;
    best = lane < NW ? ArgBest{sv[lane], si[lane]} : ArgBest{-INFINITY, INT_MAX};
    first_nan = lane < NW ? sn[lane] : INT_MAX;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float v = __shfl_xor_sync(0xffffffffu, best.val, o);
      const int i = __shfl_xor_sync(0xffffffffu, best.idx, o);
      if (better(v, i, best)) best = {v, i};
      first_nan = min(first_nan, __shfl_xor_sync(0xffffffffu, first_nan, o));
    }
    if (lane == 0) { cv = best.val; ci = best.idx; cn = first_nan; }
  }
  if constexpr (CL > 1) {
    cg::cluster_group cluster = cg::this_cluster();
    cluster.sync();
    if (crank == 0 && threadIdx.x == 0) {
      best = {cv, ci};
      first_nan = cn;
      for (int r = 1; r < CL; ++r) {
        const float v = *cluster.map_shared_rank(&cv, r);
        const int i = *cluster.map_shared_rank(&ci, r);
        if (better(v, i, best)) best = {v, i};
        first_nan = min(first_nan, *cluster.map_shared_rank(&cn, r));
      }
      cv = best.val; ci = best.idx; cn = first_nan;
    }
    cluster.sync();   // peers keep their shared memory until the leader has read it
  } else {
    __syncthreads();
  }
  if (crank == 0 && threadIdx.x == 0) {
    // an all -inf row: every entry ties at -inf, lowest index 0 wins
    int t = ci == INT_MAX ? 0 : ci;
    if (cn != INT_MAX) t = cn | (int)0x80000000u;
    target[row] = t;
  }
}

__global__ void accept_kernel(int n_q, const int32_t* __restrict__ drafts,
                              int32_t* __restrict__ target, int32_t* __restrict__ accept_len,
                              int32_t* __restrict__ commit, int32_t* __restrict__ n_commit,
                              int32_t* __restrict__ err_flag) {
  const int b = blockIdx.x;
  const int lane = threadIdx.x;
  int32_t* tg = target + (int64_t)b * n_q;
  const int k = n_q - 1;
  int any_nan = 0;
  int a = k;
  for (int base = 0; base < n_q; base += 32) {
    const int i = base + lane;
    int t = 0;
    if (i < n_q) {
      t = tg[i];
      if (t < 0) { any_nan = 1; t &= 0x7fffffff; tg[i] = t; }
    }
    if (commit) {
      const bool mismatch = (i < k) && (t != drafts[(int64_t)b * k + i]);
      const unsigned bal = __ballot_sync(0xffffffffu, mismatch);
      if (bal && a == k) a = base + __ffs(bal) - 1;
    }
  }
  any_nan = __any_sync(0xffffffffu, any_nan);
  if (err_flag && lane == 0) err_flag[b] = any_nan;
  if (!commit) return;
  __syncwarp();
  if (lane == 0) {
    accept_len[b] = a;
    n_commit[b] = a + 1;
  }
  for (int i = lane; i < n_q; i += 32) commit[(int64_t)b * n_q + i] = i <= a ? tg[i] : -1;
}

vc_status launch_accept(const float* logits, const int32_t* drafts, int B, int n_q, int V,
                        int32_t* target, int32_t* accept_len, int32_t* commit,
                        int32_t* n_commit, int32_t* err_flag, cudaStream_t stream) {
  const int rows = B * n_q;
  if (V >= 16384) {
    constexpr int CL = 8;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(rows * CL);
    cfg.blockDim = dim3(256);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = CL;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    VC_CUDA(cudaLaunchKernelEx(&cfg, argmax_rows_kernel<256, CL>, logits, V, target));
  } else {
    argmax_rows_kernel<128, 1><<<rows, 128, 0, stream>>>(logits, V, target);
  }
  VC_CUDA(cudaGetLastError());
  accept_kernel<<<B, 32, 0, stream>>>(n_q, drafts, target, accept_len, commit, n_commit,
                                      err_flag);
  VC_CUDA(cudaGetLastError());
  return VC_OK;
}

}  // namespace vc
