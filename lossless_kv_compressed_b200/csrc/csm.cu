// One round of Chunked Soft Matching (CSM), the one-pass KV-cache clustering of the
// CentroidKV summary ("Riassunto Tecnico: CentroidKV", section "Metodologia": item 2,
// sinks and recent tokens kept out of the partition; item 3, chunks, alternating A/B
// partition, bipartite matching, only the most similar fraction r merged; item 4,
// degree-weighted centroids whose degree n_t later enters the draft softmax as ln n_t).
//
// Readings (the page gives no formula): A = rows at even offsets of a chunk, B = odd
// offsets; similarity = cosine of the key rows (0 for an all-zero row); each A row's
// match is its most similar B row (lowest on ties); the m = floor(r |A|) A rows with the
// highest similarity (lower row on ties) merge into their matches; a centroid is the
// degree-weighted mean of K and V with the summed degree and takes its B row's place;
// the output keeps sinks, then the survivors of each chunk in order, then recent rows.
//
// Design: one CTA per (chunk, pair) -- a chunk is <= 256 rows, so its key rows and
// degrees stay in shared memory (3 CTAs per SM).  The key rows land once in a swizzled
// tile (cp.async); the |A| x |B| dot products run on mma.sync (bf16 in, fp32 accumulate,
// each warp one 16-row A tile against all B rows) and every A row keeps its best
// dot / |b| with a quad reduction; the top-m selection is a rank count over the
// chunk's <= 128 candidates.  A scan then lays the chunk's rows out as a source list
// grouped by output row, and the centroids sum in a fixed order (the B row, then its
// merged A rows in ascending order) in fp32 and round to bf16 once; a warp folds a
// contiguous span of the list with eight value-row loads from global memory in
// flight.  One extra CTA per pair copies the sinks and recent rows.  The rows a chunk keeps and their output
// places depend only on that chunk, so every CTA writes its own output rows.
#include <climits>
#include <cmath>
#include <type_traits>

#include "vc_common.cuh"
#include "vc_internal.h"

namespace vc {

constexpr int kCsmThreads = 256;
constexpr int kCsmMaxChunk = 256;

struct CsmParams {
  const __nv_bfloat16* k;    // [pairs, T_cap, D]
  const __nv_bfloat16* v;
  const int32_t* deg;        // [pairs, T_cap] or null (all 1)
  __nv_bfloat16* k_out;      // [pairs, T_cap_out, D]
  __nv_bfloat16* v_out;
  int32_t* deg_out;          // [pairs, T_cap_out]
  int32_t* dest;             // [pairs, T_cap] or null: output row of each input row
  int64_t T_cap, T_cap_out;
  int T, n_sinks, n_recent, chunk, n_chunks;
  int m_full, m_last;        // merges per full chunk / the last chunk
  int out_len;
};

template <int D>
struct CsmSmem {
  static constexpr int kRowB = D * 2;
  static constexpr int kK = 0;                                     // [256][D] bf16
  static constexpr int kInvN = kK + kCsmMaxChunk * kRowB;          // float [256]
  static constexpr int kBestB = kInvN + kCsmMaxChunk * 4;          // int [128]
  static constexpr int kBestS = kBestB + 128 * 4;                  // float [128]
  static constexpr int kMerged = kBestS + 128 * 4;                 // int [128]
  static constexpr int kScan = kMerged + 128 * 4;                  // int [256]
  static constexpr int kDeg = kScan + kCsmMaxChunk * 4;            // int [256]
  static constexpr int kSrc = kDeg + kCsmMaxChunk * 4;             // int [256]
  static constexpr int kNm = kSrc + kCsmMaxChunk * 4;              // int [128]
  static constexpr int kInvB = kNm + 128 * 4;                      // float [128]
  static constexpr int kTotal = kInvB + 128 * 4;
};

template <int D>
__device__ __forceinline__ uint32_t csm_row_addr(uint32_t base, int r, int c) {
  return base + r * CsmSmem<D>::kRowB + ((c ^ (r & 7)) << 4);
}

template <int D>
__global__ void __launch_bounds__(kCsmThreads, 3) csm_kernel(const CsmParams p) {
  pdl_wait();
  pdl_trigger();
  using SM = CsmSmem<D>;
  constexpr int CH = D / 8;                       // 16-byte chunks per row
  extern __shared__ __align__(128) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t pair = blockIdx.y;
  const __nv_bfloat16* kin = p.k + pair * p.T_cap * D;
  const __nv_bfloat16* vin = p.v + pair * p.T_cap * D;
  const int32_t* din = p.deg ? p.deg + pair * p.T_cap : nullptr;
  __nv_bfloat16* kout = p.k_out + pair * p.T_cap_out * D;
  __nv_bfloat16* vout = p.v_out + pair * p.T_cap_out * D;
  int32_t* dout = p.deg_out + pair * p.T_cap_out;
  int32_t* dst = p.dest ? p.dest + pair * p.T_cap : nullptr;
  auto deg_of = [&](int row) { return din ? din[row] : 1; };

  if ((int)blockIdx.x == p.n_chunks) {
    // ---- sinks and recent rows: copied unchanged, eight 16-byte pieces in flight per
    //      thread (piece e: row e / (2 CH), K for the first CH pieces of a row, then V)
    const int n_copy = p.n_sinks + p.n_recent;
    const int total = n_copy * 2 * CH;
    auto in_row = [&](int e) { return e < p.n_sinks ? e : p.T - p.n_recent + (e - p.n_sinks); };
    auto out_row = [&](int e) {
      return e < p.n_sinks ? e : p.out_len - p.n_recent + (e - p.n_sinks);
    };
    constexpr int kInFlight = 8;
    for (int e0 = tid; e0 < total; e0 += kCsmThreads * kInFlight) {
      uint4 w[kInFlight];
#pragma unroll
      for (int u = 0; u < kInFlight; ++u) {
        const int e = e0 + u * kCsmThreads;
        if (e < total) {
          const int r = e / (2 * CH), c = e - r * 2 * CH;
          const __nv_bfloat16* src = c < CH ? kin : vin;
          w[u] = reinterpret_cast<const uint4*>(src + (int64_t)in_row(r) * D)[c % CH];
        }
      }
#pragma unroll
      for (int u = 0; u < kInFlight; ++u) {
        const int e = e0 + u * kCsmThreads;
        if (e < total) {
          const int r = e / (2 * CH), c = e - r * 2 * CH;
          __nv_bfloat16* dst_t = c < CH ? kout : vout;
          reinterpret_cast<uint4*>(dst_t + (int64_t)out_row(r) * D)[c % CH] = w[u];
        }
      }
    }
    for (int e = tid; e < n_copy; e += kCsmThreads) {
      dout[out_row(e)] = deg_of(in_row(e));
      if (dst) dst[in_row(e)] = out_row(e);
    }
    return;
  }

  const int c_idx = blockIdx.x;
  const int r0 = p.n_sinks + c_idx * p.chunk;
  const int len = min(p.chunk, p.T - p.n_recent - r0);
  const int nA = (len + 1) >> 1, nB = len >> 1;
  const int m = nB > 0 ? (c_idx == p.n_chunks - 1 ? p.m_last : p.m_full) : 0;
  const int base = p.n_sinks + c_idx * (p.chunk - p.m_full);
  const uint32_t ks = smem_u32(smem + SM::kK);
  float* invn = reinterpret_cast<float*>(smem + SM::kInvN);
  int* best_b = reinterpret_cast<int*>(smem + SM::kBestB);
  float* best_s = reinterpret_cast<float*>(smem + SM::kBestS);
  int* merged = reinterpret_cast<int*>(smem + SM::kMerged);
  int* scan = reinterpret_cast<int*>(smem + SM::kScan);

  // ---- key rows of the chunk -> shared memory (rows past the chunk zeroed)
  for (int e = tid; e < kCsmMaxChunk * CH; e += kCsmThreads) {
    const int r = e / CH, c = e - r * CH;
    const bool ok = r < len;
    cp_async16(csm_row_addr<D>(ks, r, c), kin + (int64_t)(r0 + (ok ? r : 0)) * D + c * 8,
               ok ? 16u : 0u);
  }
  cp_async_commit();
  int* deg_s = reinterpret_cast<int*>(smem + SM::kDeg);
  deg_s[tid] = tid < len ? deg_of(r0 + tid) : 0;   // kCsmThreads == kCsmMaxChunk
  cp_async_wait<0>();
  __syncthreads();

  // ---- 1 / |k| of every row (0 for an all-zero row: its cosines are 0)
  {
    const int r = tid;
    float ss = 0.f;
    if (r < len) {
      const uint8_t* row = smem + SM::kK + r * SM::kRowB;
#pragma unroll 4
      for (int c = 0; c < CH; ++c) {
        const uint4 w = *reinterpret_cast<const uint4*>(row + ((c ^ (r & 7)) << 4));
        const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float a = bf16_lo(ww[u]), b = bf16_hi(ww[u]);
          ss = fmaf(a, a, ss);
          ss = fmaf(b, b, ss);
        }
      }
    }
    const float in = ss > 0.f ? 1.f / sqrtf(ss) : 0.f;
    invn[r] = in;
    if (r & 1) reinterpret_cast<float*>(smem + SM::kInvB)[r >> 1] = in;   // B rows, compact
    if (r < 128 && r >= nA) best_s[r] = -INFINITY;   // candidates past the chunk never rank
  }
  __syncthreads();

  // ---- best B match of every A row: warp w takes A rows 16w .. 16w+15 (chunk rows
  //      2i), all B rows (chunk rows 2j+1), dot products on mma.sync
  if (16 * warp < nA) {
    const int qr = lane >> 2, qc = lane & 3;
    // A fragments for all k-steps: rows i = 16w + (lane & 15), chunk 2ks + (lane >> 4)
    uint32_t af[D / 16][4];
    {
      const int i = 16 * warp + (lane & 15);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk)
        ldsm_x4(csm_row_addr<D>(ks, 2 * i, 2 * kk + (lane >> 4)), af[kk][0], af[kk][1],
                af[kk][2], af[kk][3]);
    }
    float bv[2] = {-INFINITY, -INFINITY};
    int bj[2] = {INT_MAX, INT_MAX};
    for (int nt = 0; nt < (nB + 7) / 8; ++nt) {
      float s[4] = {0.f, 0.f, 0.f, 0.f};
      const int j = 8 * nt + (lane & 7);              // B row of this lane's ldmatrix row
#pragma unroll
      for (int kk = 0; kk < D / 32; ++kk) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4(csm_row_addr<D>(ks, 2 * j + 1, 4 * kk + (lane >> 3)), b0, b1, b2, b3);
        mma_bf16(s, af[2 * kk][0], af[2 * kk][1], af[2 * kk][2], af[2 * kk][3], b0, b1);
        mma_bf16(s, af[2 * kk + 1][0], af[2 * kk + 1][1], af[2 * kk + 1][2],
                 af[2 * kk + 1][3], b2, b3);
      }
      // accumulator: rows qr, qr + 8; columns (B rows) 8nt + 2qc, +1
      const float2 ib = reinterpret_cast<const float2*>(smem + SM::kInvB)[4 * nt + qc];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int jj = 8 * nt + 2 * qc + (e & 1);
        const int h = e >> 1;
        if (jj < nB) {
          const float val = s[e] * ((e & 1) ? ib.y : ib.x);
          if (val > bv[h] || (val == bv[h] && jj < bj[h])) { bv[h] = val; bj[h] = jj; }
        }
      }
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
#pragma unroll
      for (int o = 1; o < 4; o <<= 1) {
        const float v2 = __shfl_xor_sync(0xffffffffu, bv[h], o);
        const int j2 = __shfl_xor_sync(0xffffffffu, bj[h], o);
        if (v2 > bv[h] || (v2 == bv[h] && j2 < bj[h])) { bv[h] = v2; bj[h] = j2; }
      }
      const int i = 16 * warp + qr + 8 * h;
      if (qc == 0 && i < nA) {
        best_b[i] = bj[h] == INT_MAX ? 0 : bj[h];
        best_s[i] = bv[h] == -INFINITY ? 0.f : bv[h] * invn[2 * i];
      }
    }
  }
  __syncthreads();

  // ---- the m most similar A rows merge (higher cosine first, lower row on ties): the
  //      rank of candidate i counted by two threads, each over half of the candidates
  //      (entries past nA hold -inf and never count)
  int* part = scan;                                       // free until the scan below
  {
    const int i = tid & 127, half = tid >> 7;
    const float st = best_s[i];
    const float4* bs4 = reinterpret_cast<const float4*>(best_s + 64 * half);
    int rank = 0;
#pragma unroll
    for (int q = 0; q < 16; ++q) {
      const float4 v = bs4[q];
      const int u = 64 * half + 4 * q;
      rank += (v.x > st || (v.x == st && u < i)) ? 1 : 0;
      rank += (v.y > st || (v.y == st && u + 1 < i)) ? 1 : 0;
      rank += (v.z > st || (v.z == st && u + 2 < i)) ? 1 : 0;
      rank += (v.w > st || (v.w == st && u + 3 < i)) ? 1 : 0;
    }
    part[tid] = rank;
  }
  __syncthreads();
  int* nm = reinterpret_cast<int*>(smem + SM::kNm);       // A rows merged into B row j
  if (tid < 128) {
    merged[tid] = (tid < nA && m > 0 && part[tid] + part[tid + 128] < m) ? 1 : 0;
    nm[tid] = 0;
  }
  __syncthreads();
  // per merged A row, how many merged A rows below it share its B row (its place among
  // them), and per B row the count: one warp walks the A rows in ascending order
  int* before = reinterpret_cast<int*>(best_s);           // best_s is no longer needed
  if (warp == 0) {
    for (int c = 0; c < 4; ++c) {
      const int a = 32 * c + lane;
      const bool mg = a < nA && merged[a];
      const int j = mg ? best_b[a] : -1 - lane;           // unmerged lanes: groups of one
      const unsigned same = __match_any_sync(0xffffffffu, j);
      const int below = __popc(same & ((1u << lane) - 1u));
      const int run = mg ? nm[j] : 0;
      __syncwarp();
      if (mg) {
        before[a] = run + below;
        if ((same >> lane) == 1u) nm[j] = run + below + 1;   // the group's highest lane
      }
      __syncwarp();
    }
  }
  __syncthreads();

  // ---- output places and the source list.  Every chunk row either is kept (an output
  //      row of its own) or is an A row merged into a kept B row.  The source list holds
  //      the chunk's rows grouped by output row, in output order: the kept row first,
  //      then the A rows merged into it in ascending order (the centroid's summation
  //      order).  One inclusive scan counts both: kept rows in the high half-word
  //      (output places), list entries in the low half-word (list places).
  auto kept = [&](int t) { return !((t & 1) == 0 && merged[t >> 1]); };
  const bool keep = tid < len && kept(tid);
  const int cnt = keep ? ((tid & 1) ? 1 + nm[tid >> 1] : 1) : 0;
  scan[tid] = (keep ? 1 << 16 : 0) | cnt;
  __syncthreads();
  for (int off = 1; off < kCsmMaxChunk; off <<= 1) {
    const int add = tid >= off ? scan[tid - off] : 0;
    __syncthreads();
    scan[tid] += add;
    __syncthreads();
  }
  // kept row t goes to output row base + (scan[t] >> 16) - 1; its list entries start at
  // (scan[t] & 0xffff) minus its own count
  int* src = reinterpret_cast<int*>(smem + SM::kSrc);
  if (keep) src[(scan[tid] & 0xffff) - cnt] = tid;
  if (tid < len && !keep) {
    const int a = tid >> 1, j = best_b[a];
    src[(scan[2 * j + 1] & 0xffff) - nm[j] + before[a]] = tid;   // after its B row
  }
  if (dst && tid < len) {
    const int own = keep ? tid : 2 * best_b[tid >> 1] + 1;
    dst[r0 + tid] = base + (scan[own] >> 16) - 1;
  }
  __syncthreads();

  // ---- write the kept rows: unmerged A rows as they are, B rows as centroids (B row
  //      times its degree, plus each merged A row times its degree in ascending order,
  //      over the summed degree, in fp32, rounded to bf16 once).  Warp w folds the
  //      list entries of the output rows that start in [w len / 8, (w + 1) len / 8), so
  //      every output row is one warp's; the value rows of eight entries are loaded
  //      from global memory together, so their latencies overlap.
  constexpr int DPL = D / 32;                     // channels per lane
  constexpr int kWarps = kCsmThreads / 32;
  constexpr int kBatch = 8;
  auto load_k = [&](int r, float (&x)[DPL]) {     // channels lane*DPL .. from shared
    const int d0 = lane * DPL;
    const uint8_t* srcp = smem + SM::kK + r * SM::kRowB + (((d0 >> 3) ^ (r & 7)) << 4) +
                          (d0 & 7) * 2;
    if constexpr (DPL == 4) {
      const uint2 w = *reinterpret_cast<const uint2*>(srcp);
      x[0] = bf16_lo(w.x); x[1] = bf16_hi(w.x); x[2] = bf16_lo(w.y); x[3] = bf16_hi(w.y);
    } else {
      const uint32_t w = *reinterpret_cast<const uint32_t*>(srcp);
      x[0] = bf16_lo(w); x[1] = bf16_hi(w);
    }
  };
  using VRaw = typename std::conditional<DPL == 4, uint2, uint32_t>::type;
  auto raw_v = [&](int r) -> VRaw {               // from global
    return *reinterpret_cast<const VRaw*>(vin + (int64_t)(r0 + r) * D + lane * DPL);
  };
  auto unpack = [&](VRaw w, float (&x)[DPL]) {
    if constexpr (DPL == 4) {
      x[0] = bf16_lo(w.x); x[1] = bf16_hi(w.x); x[2] = bf16_lo(w.y); x[3] = bf16_hi(w.y);
    } else {
      x[0] = bf16_lo(w); x[1] = bf16_hi(w);
    }
  };
  auto span_edge = [&](int e) {                   // first output-row start at or after e
    while (e < len && !kept(src[e])) ++e;
    return e;
  };
  const int lo = span_edge(min(len, (warp * len) / kWarps));
  const int hi = span_edge(min(len, ((warp + 1) * len) / kWarps));

  float ak[DPL], av[DPL];
  int cur = -1, ntot = 0;
  bool centroid = false;                          // a B row with merged A rows
  auto flush = [&]() {
    if (centroid) {
      const float inv = (float)ntot;
#pragma unroll
      for (int e = 0; e < DPL; ++e) { ak[e] = ak[e] / inv; av[e] = av[e] / inv; }
    }
    const int orow = base + (scan[cur] >> 16) - 1;
    __nv_bfloat16* ko = kout + (int64_t)orow * D + lane * DPL;
    __nv_bfloat16* vo = vout + (int64_t)orow * D + lane * DPL;
    if constexpr (DPL == 4) {
      *reinterpret_cast<uint2*>(ko) = make_uint2(pack_bf16x2(ak[0], ak[1]), pack_bf16x2(ak[2], ak[3]));
      *reinterpret_cast<uint2*>(vo) = make_uint2(pack_bf16x2(av[0], av[1]), pack_bf16x2(av[2], av[3]));
    } else {
      *reinterpret_cast<uint32_t*>(ko) = pack_bf16x2(ak[0], ak[1]);
      *reinterpret_cast<uint32_t*>(vo) = pack_bf16x2(av[0], av[1]);
    }
    if (lane == 0) dout[orow] = ntot;
  };
  for (int e0 = lo; e0 < hi; e0 += kBatch) {
    VRaw vr[kBatch];
#pragma unroll
    for (int b = 0; b < kBatch; ++b) vr[b] = raw_v(e0 + b < hi ? src[e0 + b] : src[lo]);
#pragma unroll
    for (int b = 0; b < kBatch; ++b) {
      if (e0 + b >= hi) break;
      const int t = src[e0 + b];                  // warp-uniform
      const int n = deg_s[t];
      float xk[DPL], xv[DPL];
      load_k(t, xk);
      unpack(vr[b], xv);
      if (kept(t)) {
        if (cur >= 0) flush();
        cur = t;
        ntot = n;
        // a row nothing merges into is copied as it is (n x / n is x exactly)
        centroid = (t & 1) && nm[t >> 1] > 0;
        const float nb = centroid ? (float)n : 1.f;
#pragma unroll
        for (int e = 0; e < DPL; ++e) { ak[e] = xk[e] * nb; av[e] = xv[e] * nb; }
      } else {
#pragma unroll
        for (int e = 0; e < DPL; ++e) {
          ak[e] = fmaf((float)n, xk[e], ak[e]);
          av[e] = fmaf((float)n, xv[e], av[e]);
        }
        ntot += n;
      }
    }
  }
  if (cur >= 0) flush();
}

int64_t csm_out_len(int64_t T, int n_sinks, int n_recent, int chunk, double r) {
  const int64_t mid = T - n_sinks - n_recent;
  int64_t n = n_sinks + n_recent;
  for (int64_t c0 = 0; c0 < mid; c0 += chunk) {
    const int64_t len = mid - c0 < chunk ? mid - c0 : chunk;
    // a one-row chunk has no B row: nothing merges
    n += len - (len >= 2 ? (int64_t)std::floor(r * (double)((len + 1) / 2)) : 0);
  }
  return n;
}

vc_status launch_csm(const void* k, const void* v, const int32_t* deg, int pairs, int D,
                     int64_t T, int64_t T_cap, int n_sinks, int n_recent, int chunk, double r,
                     void* k_out, void* v_out, int32_t* deg_out, int64_t T_cap_out,
                     int32_t* dest, cudaStream_t stream) {
  CsmParams p;
  p.k = static_cast<const __nv_bfloat16*>(k);
  p.v = static_cast<const __nv_bfloat16*>(v);
  p.deg = deg;
  p.k_out = static_cast<__nv_bfloat16*>(k_out);
  p.v_out = static_cast<__nv_bfloat16*>(v_out);
  p.deg_out = deg_out;
  p.dest = dest;
  p.T_cap = T_cap;
  p.T_cap_out = T_cap_out;
  p.T = (int)T;
  p.n_sinks = n_sinks;
  p.n_recent = n_recent;
  p.chunk = chunk;
  const int64_t mid = T - n_sinks - n_recent;
  p.n_chunks = (int)((mid + chunk - 1) / chunk);
  const int64_t last = mid - (int64_t)(p.n_chunks - 1) * chunk;
  p.m_full = (int)std::floor(r * (double)((chunk + 1) / 2));
  p.m_last = p.n_chunks > 0 && last >= 2 ? (int)std::floor(r * (double)((last + 1) / 2)) : 0;
  p.out_len = (int)csm_out_len(T, n_sinks, n_recent, chunk, r);
  const dim3 grid(p.n_chunks + 1, pairs);
  if (D == 128) {
    VC_CUDA(grant_smem((const void*)csm_kernel<128>, CsmSmem<128>::kTotal));
    VC_CUDA(launch_pdl(csm_kernel<128>, grid, dim3(kCsmThreads), CsmSmem<128>::kTotal, stream,
                       1, p));
  } else {
    VC_CUDA(grant_smem((const void*)csm_kernel<64>, CsmSmem<64>::kTotal));
    VC_CUDA(launch_pdl(csm_kernel<64>, grid, dim3(kCsmThreads), CsmSmem<64>::kTotal, stream, 1,
                       p));
  }
  VC_CUDA(cudaGetLastError());
  return VC_OK;
}

}  // namespace vc
