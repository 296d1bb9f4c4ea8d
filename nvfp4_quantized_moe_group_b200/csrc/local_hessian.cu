// Local-Hessian block-scale search for NVFP4 weight quantisation ("NVFP4 quantization",
// section "Quantization method": for each block, candidate scales are searched and the one
// with the smallest Hessian-weighted error dW^T H dW is kept).  Offline: it produces the codes
// and linear scales that nvfp4moe_experts_set takes.
//
// Per 16-value block of a weight row: S0 = the round-to-nearest scale of the quantisation rule,
// candidates S0, S0-1, S0+1, ..., S0-m, S0+m (E4M3 codes clamped to 1..0x7E; a zero block keeps
// 0); for each, the rule's codes with that scale, dW = E2M1(c) * d - w and e = dW^T H_b dW in
// FP32, H_b the block's 16x16 diagonal block of X^T X; a candidate replaces the best only when
// its error is strictly smaller.
#include "common.cuh"
#include "kernels.h"

namespace nvfp4moe {

namespace {
constexpr int kLhThreads = 256;

// Value of an E2M1 code (sign, 2 exponent bits with bias 1, 1 mantissa bit), built as FP32 bits:
// exponent field e > 0 gives (1 + m/2) 2^(e-1), e = 0 gives m/2.
__device__ __forceinline__ float e2m1_value(uint32_t nib) {
  const uint32_t e = (nib >> 1) & 3u, mb = nib & 1u;
  const uint32_t bits = e ? (((e + 126u) << 23) | (mb << 22)) : (mb ? 0x3F000000u : 0u);
  return __uint_as_float(bits | ((nib & 8u) << 28));
}

// Codes of the 16 values w with block-scale code S and global scale g (the quantisation rule).
__device__ __forceinline__ void block_codes(const float* w, uint32_t S, float g, uint32_t* c0, uint32_t* c1,
                                            float* d_out) {
  const float d = __fmul_rn(e4m3_to_f32(S), g);
  const float r_b = (d == 0.0f) ? 0.0f : __frcp_rn(d);
  float v[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __fmul_rn(w[i], r_b);
  *c0 = cvt_e2m1x8(v);
  *c1 = cvt_e2m1x8(v + 8);
  *d_out = d;
}

// dW^T H dW for the block with scale code S (FP32).
__device__ __forceinline__ float block_error(const float* w, uint32_t S, float g, const float (*H)[16]) {
  uint32_t c0, c1;
  float d;
  block_codes(w, S, g, &c0, &c1, &d);
  float dw[16];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    dw[i] = __fsub_rn(__fmul_rn(e2m1_value(c0 >> (4 * i)), d), w[i]);
    dw[8 + i] = __fsub_rn(__fmul_rn(e2m1_value(c1 >> (4 * i)), d), w[8 + i]);
  }
  float e = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    // every thread of the CTA reads the same H row: 16-byte broadcast loads
    const float4* hr = reinterpret_cast<const float4*>(H[i]);
    float y = 0.0f;
#pragma unroll
    for (int j4 = 0; j4 < 4; ++j4) {
      const float4 h = hr[j4];
      y = __fmaf_rn(h.x, dw[4 * j4], y);
      y = __fmaf_rn(h.y, dw[4 * j4 + 1], y);
      y = __fmaf_rn(h.z, dw[4 * j4 + 2], y);
      y = __fmaf_rn(h.w, dw[4 * j4 + 3], y);
    }
    e = __fmaf_rn(dw[i], y, e);
  }
  return e;
}
}  // namespace

// grid (ceil(rows / 256), cols / 16): thread = one row of one 16-column block; the block's
// H_b sits in shared memory for the 256 rows.
__global__ void __launch_bounds__(kLhThreads) lh_quantize_kernel(LhArgs a) {
  __shared__ __align__(16) float s_H[16][16];
  __shared__ float s_g;
  __shared__ int s_bad;
  const int tid = threadIdx.x;
  const int b = blockIdx.y;
  if (tid < 32) {
    uint32_t m = 0;
    for (int i = tid; i < a.n_partials; i += 32) m = max(m, a.partials[i]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (tid == 0) {
      s_bad = m >= 0x7F80u;
      s_g = global_scale_from_amax(__uint_as_float(m << 16));
      if (blockIdx.x == 0 && b == 0) {
        if (s_bad) raise_status(a.status, kStatusNonFinite);
        *a.g_out = s_g;
      }
    }
  }
  s_H[tid >> 4][tid & 15] = a.hess[(int64_t)b * 256 + tid];
  __syncthreads();
  const int64_t row = (int64_t)blockIdx.x * kLhThreads + tid;
  if (s_bad || row >= a.rows) return;
  const float g = s_g;
  const float r_t = __frcp_rn(__fmul_rn(6.0f, g));

  const uint4* src = reinterpret_cast<const uint4*>(a.w + row * a.cols + 16 * b);
  const uint4 q0 = __ldg(src), q1 = __ldg(src + 1);
  const uint32_t qw[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
  float w[16];
  uint32_t mag = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    w[2 * j] = __uint_as_float(qw[j] << 16);
    w[2 * j + 1] = __uint_as_float(qw[j] & 0xFFFF0000u);
    mag = max(mag, max(qw[j] & 0x7FFFu, (qw[j] >> 16) & 0x7FFFu));
  }
  const uint32_t S0 = cvt_e4m3(__fmul_rn(__uint_as_float(mag << 16), r_t));
  uint32_t best_S = S0;
  if (S0 != 0u) {
    float best_e = block_error(w, S0, g, s_H);
    for (int k = 1; k <= 2 * a.m; ++k) {
      const int off = (k & 1) ? -((k + 1) >> 1) : (k >> 1);
      int S = (int)S0 + off;
      S = S < 1 ? 1 : (S > 0x7E ? 0x7E : S);
      const float e = block_error(w, (uint32_t)S, g, s_H);
      if (e < best_e) {
        best_e = e;
        best_S = (uint32_t)S;
      }
    }
  }
  uint32_t c0, c1;
  float d;
  block_codes(w, best_S, g, &c0, &c1, &d);
  *reinterpret_cast<uint2*>(a.codes + row * (a.cols / 2) + 8 * b) = make_uint2(c0, c1);
  a.scales[row * (a.cols / 16) + b] = (uint8_t)best_S;
}

cudaError_t launch_lh_quantize(const LhArgs& a, cudaStream_t stream) {
  const dim3 grid((unsigned)((a.rows + kLhThreads - 1) / kLhThreads), (unsigned)(a.cols / 16));
  lh_quantize_kernel<<<grid, kLhThreads, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace nvfp4moe
