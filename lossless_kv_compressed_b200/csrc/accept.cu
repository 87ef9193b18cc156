// Greedy acceptance over the verify logits (VeriCache summary, "Riepilogo Tecnico:
// VeriCache", section "Algoritmo Principale", step 3): accept drafted tokens up to
// the first disagreement with the full-KV prediction, plus one bonus token when all
// agree.
//
// Kernel 1: float4 streaming argmax of each logits row (ties -> lowest index; NaN
//           larger than any number, first NaN wins).  Each thread keeps 8 float4 loads
//           in flight, and a group of 4 values takes the per-element comparison only
//           when it holds a NaN or a value above the thread's best so far (a thread
//           meets its indices in increasing order, so equal values never replace the
//           best).  When the rows are few (a draft step's B rows) each row is split
//           over a cluster of up to 8 CTAs merged through distributed shared memory, so
//           the grid still covers the SMs.  The row's NaN bit is parked in bit 31 of its
//           target entry -- except for one-position rows (n_q == 1), whose outputs this
//           kernel finishes itself (a single launch per draft step).
// Kernel 2 (n_q > 1): one warp per batch row: clears the NaN bits into err_flag, finds
//           the first disagreement with a ballot, and writes accept_len / commit /
//           n_commit.
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

// Outputs of a one-position row (n_q == 1), written by the argmax kernel itself so that
// the draft-time argmax is a single launch: the target without its NaN bit, the row's
// NaN flag, and -- in acceptance mode -- accept_len 0, commit [target], n_commit 1.
struct RowEpilogue {
  int32_t* accept_len;
  int32_t* commit;
  int32_t* n_commit;
  int32_t* err_flag;
  int fused;
};

// One row per thread-block cluster of CL CTAs: CTA c scans a contiguous slice of the
// row, U float4 loads in flight per thread before any is compared, stores its result
// into the cluster leader's shared memory (one cluster barrier), and the leader merges
// the CL results (any order gives the same winner: larger value, then lower index).
template <int THREADS, int CL, int U>
__global__ void __launch_bounds__(THREADS) argmax_rows_kernel(const float* __restrict__ logits,
                                                              int V, int32_t* __restrict__ target,
                                                              RowEpilogue ep) {
  pdl_wait();
  pdl_trigger();
  namespace cg = cooperative_groups;
  const int64_t row = blockIdx.x / CL;
  const int crank = (int)(blockIdx.x % CL);
  const float* x = logits + row * (int64_t)V;
  // Distributed shared memory of a CTA may be written only once that CTA has started:
  // arrive now, wait just before the remote stores (every CTA has long started by then).
  if constexpr (CL > 1) asm volatile("barrier.cluster.arrive.relaxed.aligned;\n" ::: "memory");
  // slice [lo, hi) of the row, multiples of 4 so float4 loads stay aligned
  const int per = ((V + CL - 1) / CL + 3) & ~3;
  const int lo = min(V, crank * per), hi = min(V, lo + per);
  ArgBest best{-INFINITY, INT_MAX};
  int first_nan = INT_MAX;
  auto take = [&](float e, int id) {
    if (isnan(e)) first_nan = min(first_nan, id);
    else if (better(e, id, best)) best = {e, id};
  };
  const bool vec = ((V & 3) == 0) && ((reinterpret_cast<uintptr_t>(x) & 15) == 0);
  if (vec) {
    const float4* x4 = reinterpret_cast<const float4*>(x);
    const int lo4 = lo >> 2, hi4 = hi >> 2;
    for (int base = lo4 + (int)threadIdx.x; base < hi4; base += THREADS * U) {
      float4 f[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int i = base + u * THREADS;
        f[u] = i < hi4 ? __ldcs(x4 + i) : make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
      }
      // A thread meets its indices in increasing order, so an equal value never
      // replaces its best: only a group holding a NaN or a strictly larger value
      // needs the per-element pass (fmaxf ignores NaN; out-of-range lanes are -inf).
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int i = base + u * THREADS;
        const float m4 = fmaxf(fmaxf(f[u].x, f[u].y), fmaxf(f[u].z, f[u].w));
        const bool nan4 = isnan(f[u].x) | isnan(f[u].y) | isnan(f[u].z) | isnan(f[u].w);
        if (nan4 | (m4 > best.val)) {
          take(f[u].x, 4 * i);
          take(f[u].y, 4 * i + 1);
          take(f[u].z, 4 * i + 2);
          take(f[u].w, 4 * i + 3);
        }
      }
    }
  } else {
    for (int i = lo + threadIdx.x; i < hi; i += THREADS) take(__ldg(x + i), i);
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
  __shared__ float cv[CL];   // each CTA's result, gathered in the cluster leader's copy
  __shared__ int ci[CL], cn[CL];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) { sv[warp] = best.val; si[warp] = best.idx; sn[warp] = first_nan; }
  __syncthreads();
  if constexpr (CL > 1) asm volatile("barrier.cluster.wait.aligned;\n" ::: "memory");
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
      // write this CTA's result into the leader's slot `crank` (a remote store through
      // distributed shared memory for the other CTAs of the cluster)
      if constexpr (CL > 1) {
        cg::cluster_group cluster = cg::this_cluster();
        *cluster.map_shared_rank(&cv[crank], 0) = best.val;
        *cluster.map_shared_rank(&ci[crank], 0) = best.idx;
        *cluster.map_shared_rank(&cn[crank], 0) = first_nan;
      } else {
        cv[0] = best.val; ci[0] = best.idx; cn[0] = first_nan;
      }
    }
  }
  if constexpr (CL > 1) {
    cg::this_cluster().sync();   // release the remote stores, acquire them in the leader
  } else {
    __syncthreads();
  }
  int res_i = INT_MAX, res_n = INT_MAX;
  if (crank == 0 && threadIdx.x == 0) {
    best = {cv[0], ci[0]};
    first_nan = cn[0];
#pragma unroll
    for (int r = 1; r < CL; ++r) {
      if (better(cv[r], ci[r], best)) best = {cv[r], ci[r]};
      first_nan = min(first_nan, cn[r]);
    }
    res_i = best.idx;
    res_n = first_nan;
  }
  if (crank == 0 && threadIdx.x == 0) {
    // an all -inf row: every entry ties at -inf, lowest index 0 wins
    int t = res_i == INT_MAX ? 0 : res_i;
    const bool nan = res_n != INT_MAX;
    if (nan) t = res_n;
    if (!ep.fused) {
      target[row] = nan ? (t | (int)0x80000000u) : t;
    } else {
      target[row] = t;
      if (ep.err_flag) ep.err_flag[row] = nan ? 1 : 0;
      if (ep.commit) {
        ep.accept_len[row] = 0;
        ep.commit[row] = t;
        ep.n_commit[row] = 1;
      }
    }
  }
}

__global__ void accept_kernel(int n_q, const int32_t* __restrict__ drafts,
                              int32_t* __restrict__ target, int32_t* __restrict__ accept_len,
                              int32_t* __restrict__ commit, int32_t* __restrict__ n_commit,
                              int32_t* __restrict__ err_flag) {
  pdl_wait();
  pdl_trigger();
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

namespace {
constexpr int kArgThreads = 512;
constexpr int kArgUnroll = 8;

template <int CL>
vc_status launch_argmax(const float* logits, int V, int rows, int32_t* target,
                        const RowEpilogue& ep, cudaStream_t stream) {
  VC_CUDA(launch_pdl(argmax_rows_kernel<kArgThreads, CL, kArgUnroll>, dim3(rows * CL),
                     dim3(kArgThreads), 0, stream, CL, logits, V, target, ep));
  VC_CUDA(cudaGetLastError());
  return VC_OK;
}
}  // namespace

// Cluster size: split rows over more CTAs while the grid still fits in one wave of two
// CTAs per SM and every CTA keeps at least 2048 logits.
int argmax_cluster(int rows, int V) {
  int cl = 1;
  while (cl < 8 && (int64_t)rows * cl * 2 <= 2 * (int64_t)num_sms() && V / (2 * cl) >= 2048)
    cl *= 2;
  return cl;
}

vc_status launch_accept(const float* logits, const int32_t* drafts, int B, int n_q, int V,
                        int32_t* target, int32_t* accept_len, int32_t* commit,
                        int32_t* n_commit, int32_t* err_flag, cudaStream_t stream) {
  const int rows = B * n_q;
  RowEpilogue ep{accept_len, commit, n_commit, err_flag, n_q == 1 ? 1 : 0};
  vc_status st;
  switch (argmax_cluster(rows, V)) {
    case 1: st = launch_argmax<1>(logits, V, rows, target, ep, stream); break;
    case 2: st = launch_argmax<2>(logits, V, rows, target, ep, stream); break;
    case 4: st = launch_argmax<4>(logits, V, rows, target, ep, stream); break;
    default: st = launch_argmax<8>(logits, V, rows, target, ep, stream); break;
  }
  if (st != VC_OK || n_q == 1) return st;
  VC_CUDA(launch_pdl(accept_kernel, dim3(B), dim3(32), 0, stream, 1, n_q, drafts, target,
                     accept_len, commit, n_commit, err_flag));
  VC_CUDA(cudaGetLastError());
  return VC_OK;
}

}  // namespace vc
