// Per-row FP8 E4M3 quantisation for the FP8 W8A8 variant ("FP8 quantization", section
// "Quantization scheme": weights with a fixed scale per output channel, activations with a
// scale computed per token at run time; section "Quantization method": round to nearest).
//
// Row scale s = fp32(amax / 448) (1 for an all-zero row), code = E4M3_rn_satfinite(fp32(v / s))
// with an IEEE division; the sign is kept.  One CTA per row.
#include "common.cuh"
#include "kernels.h"

namespace nvfp4moe {

namespace {
constexpr int kFp8Threads = 256;
constexpr float kE4M3Max = 448.0f;

// Two FP32 values -> two E4M3 bytes (lo in the low byte), round to nearest even, saturating.
__device__ __forceinline__ uint32_t cvt_e4m3x2(float lo, float hi) {
  uint16_t out;
  asm volatile("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(out) : "f"(hi), "f"(lo));
  return out;
}

// Block-wide max of non-negative FP32 values (as bit patterns, order-preserving for >= 0).
__device__ __forceinline__ uint32_t block_max_u32(uint32_t m) {
  __shared__ uint32_t s_red[kFp8Threads / 32];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = m;
  __syncthreads();
  m = 0;
  for (int i = 0; i < kFp8Threads / 32; ++i) m = max(m, s_red[i]);
  __syncthreads();
  return m;
}

__device__ __forceinline__ float row_scale(float amax) {
  return amax == 0.0f ? 1.0f : __fdiv_rn(amax, kE4M3Max);
}

// 8 values -> 8 E4M3 bytes
__device__ __forceinline__ uint2 encode8(const float* v, float s) {
  uint32_t b[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) b[j] = cvt_e4m3x2(__fdiv_rn(v[2 * j], s), __fdiv_rn(v[2 * j + 1], s));
  return make_uint2(b[0] | (b[1] << 16), b[2] | (b[3] << 16));
}

__device__ __forceinline__ void unpack_bf16x8(const uint4& q, float* v) {
  const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    v[2 * j] = __uint_as_float(w[j] << 16);
    v[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
  }
}
}  // namespace

// BF16 rows [rows][cols] -> E4M3 codes [rows][cols] + FP32 scales [rows].  Non-finite rows
// raise kStatusNonFinite (their outputs are left unwritten).
__global__ void __launch_bounds__(kFp8Threads) fp8_quantize_rows_kernel(Fp8RowsArgs a) {
  const int64_t r = blockIdx.x;
  const uint4* src = reinterpret_cast<const uint4*>(a.x + r * a.cols);
  const int n8 = (int)(a.cols / 8);
  uint32_t mag = 0;
  for (int v = threadIdx.x; v < n8; v += kFp8Threads) {
    const uint4 q = __ldg(src + v);
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) mag = max(mag, max(w[j] & 0x7FFFu, (w[j] >> 16) & 0x7FFFu));
  }
  mag = block_max_u32(mag);
  if (mag >= 0x7F80u) {
    if (threadIdx.x == 0) raise_status(a.status, kStatusNonFinite);
    return;
  }
  const float s = row_scale(__uint_as_float(mag << 16));
  if (threadIdx.x == 0) a.scales[r] = s;
  uint2* dst = reinterpret_cast<uint2*>(a.codes + r * a.cols);
  for (int v = threadIdx.x; v < n8; v += kFp8Threads) {
    float f[8];
    unpack_bf16x8(__ldg(src + v), f);
    dst[v] = encode8(f, s);
  }
}

// The layer input: token t's row quantised with its own scale and written to the expert-segment
// row of each of its topk pairs (codes [rows_cap][H], scale per segment row); the token's FP32
// accumulator row is zeroed; optionally the token-major codes and scales are kept.
__global__ void __launch_bounds__(kFp8Threads) fp8_quantize_scatter_kernel(Fp8ScatterArgs a) {
  __shared__ int64_t s_rows[8];
  const int64_t t = blockIdx.x;
  if (threadIdx.x < a.topk) {
    const int64_t p = t * a.topk + threadIdx.x;
    const int e = a.idx[p];
    s_rows[threadIdx.x] = (int64_t)a.mtile_prefix[e] * kBlockM + (a.inv[p] - a.offsets[e]);
  }
  const uint4* src = reinterpret_cast<const uint4*>(a.x + t * a.H);
  const int n8 = a.H / 8;
  uint32_t mag = 0;
  for (int v = threadIdx.x; v < n8; v += kFp8Threads) {
    const uint4 q = __ldg(src + v);
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) mag = max(mag, max(w[j] & 0x7FFFu, (w[j] >> 16) & 0x7FFFu));
    // the token's accumulator row
    float4* z = reinterpret_cast<float4*>(a.acc + t * a.H + 8 * v);
    z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
    z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  mag = block_max_u32(mag);          // also orders s_rows before their use
  if (mag >= 0x7F80u) {
    if (threadIdx.x == 0) raise_status(a.status, kStatusNonFinite);
    return;
  }
  const float s = row_scale(__uint_as_float(mag << 16));
  if (threadIdx.x < a.topk) a.seg_scale[s_rows[threadIdx.x]] = s;
  if (threadIdx.x == 0 && a.xq_scales != nullptr) a.xq_scales[t] = s;
  for (int v = threadIdx.x; v < n8; v += kFp8Threads) {
    float f[8];
    unpack_bf16x8(__ldg(src + v), f);
    const uint2 c = encode8(f, s);
    for (int j = 0; j < a.topk; ++j) reinterpret_cast<uint2*>(a.seg_codes + s_rows[j] * a.H)[v] = c;
    if (a.xq_codes != nullptr) reinterpret_cast<uint2*>(a.xq_codes + t * a.H)[v] = c;
  }
}

// The down projection's input: each segment row holding a pair has its FP32 SwiGLU product
// [I] quantised with its own scale (padding rows, and rows past the last segment, are skipped).
__global__ void __launch_bounds__(kFp8Threads) fp8_requant_rows_kernel(Fp8RequantArgs a) {
  const int64_t r = blockIdx.x;
  if (r >= (int64_t)__ldg(a.mtile_prefix + a.E) * kBlockM || a.row_pair[r] < 0) return;
  const float4* src = reinterpret_cast<const float4*>(a.h + r * a.I);
  const int n8 = a.I / 8;
  uint32_t mag = 0;
  for (int v = threadIdx.x; v < n8; v += kFp8Threads) {
    const float4 p = src[2 * v], q = src[2 * v + 1];
    const float f[8] = {p.x, p.y, p.z, p.w, q.x, q.y, q.z, q.w};
#pragma unroll
    for (int j = 0; j < 8; ++j) mag = max(mag, __float_as_uint(f[j]) & 0x7FFFFFFFu);
  }
  mag = block_max_u32(mag);
  if (mag >= 0x7F800000u) {
    if (threadIdx.x == 0) raise_status(a.status, kStatusNonFinite);
    return;
  }
  const float s = row_scale(__uint_as_float(mag));
  if (threadIdx.x == 0) a.scales[r] = s;
  uint2* dst = reinterpret_cast<uint2*>(a.codes + r * a.I);
  for (int v = threadIdx.x; v < n8; v += kFp8Threads) {
    const float4 p = src[2 * v], q = src[2 * v + 1];
    const float f[8] = {p.x, p.y, p.z, p.w, q.x, q.y, q.z, q.w};
    dst[v] = encode8(f, s);
  }
}

cudaError_t launch_fp8_quantize_rows(const Fp8RowsArgs& a, cudaStream_t stream) {
  fp8_quantize_rows_kernel<<<(unsigned)a.rows, kFp8Threads, 0, stream>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_fp8_quantize_scatter(const Fp8ScatterArgs& a, cudaStream_t stream) {
  fp8_quantize_scatter_kernel<<<(unsigned)a.T, kFp8Threads, 0, stream>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_fp8_requant_rows(const Fp8RequantArgs& a, cudaStream_t stream) {
  fp8_requant_rows_kernel<<<(unsigned)a.rows, kFp8Threads, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace nvfp4moe
