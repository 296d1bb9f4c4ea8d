// The MoE block's neighbours on the residual stream ("Reflection releases Beam ...", section
// "Residual stream and numerical decisions"): the RMSNorm that turns the residual stream h
// into the layer input x (norms in FP32), and, in finalize_kernel, the weighted residual add
// of the layer output (the stream kept with weight sqrt((k-1)/k), the sublayer output added
// with weight 1/sqrt(k) at step k).
//
// x = bf16(fp32(fp32(h * r) * gamma)), r = fp32(1 / sqrt(mean(h^2) + eps)) with the mean, the
// root and the reciprocal in FP64 (every square of a BF16 value is exact in FP64).
#include "common.cuh"
#include "kernels.h"

namespace nvfp4moe {

namespace {
constexpr int kNormThreads = 256;

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  return (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(lo)) |
         ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(hi)) << 16);
}
}  // namespace

// One CTA per token row.  Pass 1: FP64 sum of squares (8 values per 16-byte load); pass 2
// (the row is re-read from L1/L2): the normalised, weighted, BF16-rounded layer input.
__global__ void __launch_bounds__(kNormThreads) rmsnorm_kernel(RmsNormArgs a) {
  __shared__ double s_part[kNormThreads / 32];
  __shared__ float s_r;
  const int64_t t = blockIdx.x;
  const uint4* row = reinterpret_cast<const uint4*>(a.h + t * a.H);
  const int n_vec = a.H / 8;
  double ss = 0.0;
  for (int v = threadIdx.x; v < n_vec; v += kNormThreads) {
    const uint4 q = __ldg(row + v);
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const double lo = bf16_lo(w[j]), hi = bf16_hi(w[j]);
      ss = __fma_rn(lo, lo, ss);
      ss = __fma_rn(hi, hi, ss);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss = __dadd_rn(ss, __shfl_xor_sync(0xffffffffu, ss, o));
  if ((threadIdx.x & 31) == 0) s_part[threadIdx.x >> 5] = ss;
  __syncthreads();
  if (threadIdx.x == 0) {
    double sum = 0.0;
    for (int i = 0; i < kNormThreads / 32; ++i) sum = __dadd_rn(sum, s_part[i]);
    const double ms = __ddiv_rn(sum, (double)a.H);
    const double r = __ddiv_rn(1.0, __dsqrt_rn(__dadd_rn(ms, (double)a.eps)));
    s_r = __double2float_rn(r);
  }
  __syncthreads();
  const float r = s_r;
  uint4* out = reinterpret_cast<uint4*>(a.x + t * a.H);
  const float4* g4 = reinterpret_cast<const float4*>(a.gamma);
  for (int v = threadIdx.x; v < n_vec; v += kNormThreads) {
    const uint4 q = __ldg(row + v);
    const float4 g0 = __ldg(g4 + 2 * v), g1 = __ldg(g4 + 2 * v + 1);
    const float g[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
    uint32_t o[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float lo = __fmul_rn(__fmul_rn(bf16_lo(w[j]), r), g[2 * j]);
      const float hi = __fmul_rn(__fmul_rn(bf16_hi(w[j]), r), g[2 * j + 1]);
      o[j] = pack_bf16x2(lo, hi);
    }
    out[v] = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

cudaError_t launch_rmsnorm(const RmsNormArgs& a, cudaStream_t stream) {
  rmsnorm_kernel<<<(unsigned)a.T, kNormThreads, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace nvfp4moe
