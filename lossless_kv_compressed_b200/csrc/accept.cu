// Greedy acceptance over the verify logits (VeriCache summary, "Riepilogo Tecnico:
// VeriCache", section "Algoritmo Principale", step 3): accept drafted tokens up to
// the first disagreement with the full-KV prediction, plus one bonus token when all
// agree.
//
// Kernel 1: one CTA per logits row, float4 streaming argmax (ties -> lowest index;
//           NaN larger than any number, first NaN wins).  The row's NaN bit is
//           parked in bit 31 of its target entry.
// Kernel 2: one warp per batch row: clears the NaN bits into err_flag, finds the first
//           disagreement with a ballot, and writes accept_len / commit / n_commit.
#include <climits>

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

template <int THREADS>
__global__ void __launch_bounds__(THREADS) argmax_rows_kernel(const float* __restrict__ logits,
                                                              int V, int32_t* __restrict__ target) {
  const int64_t row = blockIdx.x;
  const float* x = logits + row * (int64_t)V;
  ArgBest best{-INFINITY, INT_MAX};
  int first_nan = INT_MAX;
  const bool vec = ((V & 3) == 0) && ((reinterpret_cast<uintptr_t>(x) & 15) == 0);
  if (vec) {
    const float4* x4 = reinterpret_cast<const float4*>(x);
    const int n4 = V >> 2;
    for (int i = threadIdx.x; i < n4; i += THREADS) {
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
    for (int i = threadIdx.x; i < V; i += THREADS) {
      const float e = __ldg(x + i);
      if (isnan(e)) first_nan = min(first_nan, i);
      else if (better(e, i, best)) best = {e, i};
    }
  }
  // warp reduction
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
    if (lane == 0) {
      // an all -inf row: every entry ties at -inf, lowest index 0 wins
      int t = best.idx == INT_MAX ? 0 : best.idx;
      if (first_nan != INT_MAX) t = first_nan | (int)0x80000000u;
      target[row] = t;
    }
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
  if (V >= 16384) argmax_rows_kernel<512><<<rows, 512, 0, stream>>>(logits, V, target);
  else argmax_rows_kernel<128><<<rows, 128, 0, stream>>>(logits, V, target);
  VC_CUDA(cudaGetLastError());
  accept_kernel<<<B, 32, 0, stream>>>(n_q, drafts, target, accept_len, commit, n_commit,
                                      err_flag);
  VC_CUDA(cudaGetLastError());
  return VC_OK;
}

}  // namespace vc
