// Asymmetric 4-bit group quantisation of bf16 K/V rows into the int4 draft cache.
//
// Quantisation is one of the lossy compressors VeriCache plugs into its uniform
// compression interface ("Riepilogo Tecnico: VeriCache", section "Supporto
// Architetturale"; "Riassunto Tecnico: CentroidKV", section "Problematica", lists it
// among the known KV-cache reductions).  The format is the 128K-context workload's: keys
// per channel over groups of 32 consecutive tokens, values per token over groups of 32
// consecutive channels, each group with an fp16 scale and an fp16 zero point:
//     z = fp16(min G),  s = fp16((max G - min G) / 15)  (1 when that is 0),
//     n = clamp(rint((x - z) / s), 0, 15)  (round half to even),  x_hat = n s + z.
// The difference, the division and the rounding run in fp64 (every operand is a bf16 or
// fp16 value, so each step is one IEEE-rounded fp64 operation) and the fp16 conversions
// round once from fp64, so a block's bytes are a pure function of its 32 rows.  Values
// outside the fp16 range cannot be represented by the format.
//
// One CTA of 128 threads per (pair, 32-token block): the block's K and V rows are read
// once into shared memory (16-byte loads), nibbles are computed per group, then packed
// into the words of the documented layout (include/vericache.h) and written with the
// group scales and zeros.  The kernel is bound by its 8 KB (D = 64) or 16 KB (D = 128)
// of reads per block; it runs when 32 tokens leave the bf16 window, or once over a cache.
#include "vc_common.cuh"
#include "vc_internal.h"

namespace vc {

struct QuantParams {
  const __nv_bfloat16* k;   // [pairs, src_cap, D]
  const __nv_bfloat16* v;
  int64_t src_cap, src_t0;
  int n_blocks;
  uint32_t* kq;             // [pairs, blk_cap, 32, 4, D/32]
  __half* ks;               // [pairs, blk_cap, D]
  __half* kz;
  uint32_t* vq;             // [pairs, blk_cap, D, 4]
  __half* vs;               // [pairs, blk_cap, D/32, 32]
  __half* vz;
  int64_t blk_cap, blk0;
};

// One group: scale and zero (fp16) and the quantisation of one of its elements.
struct Group {
  __half s16, z16;
  double s, z;
  __device__ __forceinline__ Group(float mn, float mx) {
    z16 = __double2half((double)mn);
    s16 = __double2half(((double)mx - (double)mn) / 15.0);
    if (mx == mn || __half2float(s16) == 0.f) s16 = __float2half(1.f);
    s = (double)__half2float(s16);
    z = (double)__half2float(z16);
  }
  __device__ __forceinline__ uint32_t nib(float x) const {
    const double q = rint(((double)x - z) / s);
    return !(q > 0.0) ? 0u : q >= 15.0 ? 15u : (uint32_t)q;   // NaN maps to 0
  }
};

template <int D>
__global__ void __launch_bounds__(128) quantize_int4_kernel(const QuantParams p) {
  pdl_wait();
  pdl_trigger();
  constexpr int NW = D / 32;
  __shared__ __align__(16) __nv_bfloat16 sk[32][D];
  __shared__ __align__(16) __nv_bfloat16 sv[32][D];
  __shared__ uint8_t nk[32][D + 4];
  __shared__ uint8_t nv[32][D + 4];
  const int blk = blockIdx.x;
  const int64_t pair = blockIdx.y;
  const int tid = threadIdx.x;
  const int64_t row0 = pair * p.src_cap + p.src_t0 + 32 * (int64_t)blk;
  const uint4* ksrc = reinterpret_cast<const uint4*>(p.k + row0 * D);
  const uint4* vsrc = reinterpret_cast<const uint4*>(p.v + row0 * D);
  for (int c = tid; c < 32 * D / 8; c += 128) {
    reinterpret_cast<uint4*>(&sk[0][0])[c] = __ldg(ksrc + c);
    reinterpret_cast<uint4*>(&sv[0][0])[c] = __ldg(vsrc + c);
  }
  __syncthreads();
  const int64_t ob = pair * p.blk_cap + p.blk0 + blk;    // destination block
  // keys: one group per channel over the block's 32 tokens
  for (int d = tid; d < D; d += 128) {
    float mn = __bfloat162float(sk[0][d]), mx = mn;
    for (int t = 1; t < 32; ++t) {
      const float x = __bfloat162float(sk[t][d]);
      mn = fminf(mn, x);
      mx = fmaxf(mx, x);
    }
    const Group G(mn, mx);
    for (int t = 0; t < 32; ++t) nk[t][d] = (uint8_t)G.nib(__bfloat162float(sk[t][d]));
    p.ks[ob * D + d] = G.s16;
    p.kz[ob * D + d] = G.z16;
  }
  // values: one group per (token, 32 consecutive channels)
  for (int i = tid; i < 32 * NW; i += 128) {
    const int t = i / NW, g = i - t * NW;
    float mn = __bfloat162float(sv[t][32 * g]), mx = mn;
    for (int c = 1; c < 32; ++c) {
      const float x = __bfloat162float(sv[t][32 * g + c]);
      mn = fminf(mn, x);
      mx = fmaxf(mx, x);
    }
    const Group G(mn, mx);
    for (int c = 0; c < 32; ++c) nv[t][32 * g + c] = (uint8_t)G.nib(__bfloat162float(sv[t][32 * g + c]));
    p.vs[(ob * NW + g) * 32 + t] = G.s16;
    p.vz[(ob * NW + g) * 32 + t] = G.z16;
  }
  __syncthreads();
  // key words (token t, c, w): pair j holds channels e, e + 1 with
  // e = 2c + 32w + 16 (j / 2) + 8 (j % 2); first element in nibble j, second in j + 4
  uint32_t* kdst = p.kq + ob * (32 * 4 * NW);
  for (int wi = tid; wi < 32 * 4 * NW; wi += 128) {
    const int t = wi / (4 * NW), c = (wi / NW) & 3, w = wi % NW;
    uint32_t word = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int e = 2 * c + 32 * w + 16 * (j >> 1) + 8 * (j & 1);
      word |= (uint32_t)nk[t][e] << (4 * j);
      word |= (uint32_t)nk[t][e + 1] << (4 * (j + 4));
    }
    kdst[wi] = word;
  }
  // value words (channel d, c): pair j holds channel d of tokens 2c + 8j and 2c + 8j + 1
  uint32_t* vdst = p.vq + ob * (D * 4);
  for (int wi = tid; wi < D * 4; wi += 128) {
    const int d = wi >> 2, c = wi & 3;
    uint32_t word = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      word |= (uint32_t)nv[2 * c + 8 * j][d] << (4 * j);
      word |= (uint32_t)nv[2 * c + 8 * j + 1][d] << (4 * (j + 4));
    }
    vdst[wi] = word;
  }
}

vc_status launch_int4_quantize(const void* k, const void* v, int pairs, int D, int64_t src_cap,
                               int64_t src_t0, int n_blocks, uint32_t* kq, void* k_scale,
                               void* k_zero, uint32_t* vq, void* v_scale, void* v_zero,
                               int64_t blk_cap, int64_t blk0, cudaStream_t stream) {
  if (n_blocks == 0) return VC_OK;
  QuantParams p;
  p.k = static_cast<const __nv_bfloat16*>(k);
  p.v = static_cast<const __nv_bfloat16*>(v);
  p.src_cap = src_cap;
  p.src_t0 = src_t0;
  p.n_blocks = n_blocks;
  p.kq = kq;
  p.ks = static_cast<__half*>(k_scale);
  p.kz = static_cast<__half*>(k_zero);
  p.vq = vq;
  p.vs = static_cast<__half*>(v_scale);
  p.vz = static_cast<__half*>(v_zero);
  p.blk_cap = blk_cap;
  p.blk0 = blk0;
  const dim3 grid((unsigned)n_blocks, (unsigned)pairs);
  if (D == 128)
    VC_CUDA(launch_pdl(quantize_int4_kernel<128>, grid, dim3(128), 0, stream, 1, p));
  else
    VC_CUDA(launch_pdl(quantize_int4_kernel<64>, grid, dim3(128), 0, stream, 1, p));
  VC_CUDA(cudaGetLastError());
  return VC_OK;
}

}  // namespace vc
