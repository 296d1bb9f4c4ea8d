// NVFP4 activation quantisation (quantize_nvfp4): global amax, per-16 block E4M3 scale,
// E2M1 codes with round-to-nearest-even, two codes per byte, linear or swizzled scales.
// Format: "NVFP4 quantization", section "Quantization scheme" (E2M1 values, one E4M3 scale
// per 16 values, one FP32 global scale per tensor); the scale rule is the library's reading
// stated in nvfp4moe.h.
#include "common.cuh"
#include "kernels.h"

namespace nvfp4moe {

// Per-block maximum of |x| as the BF16 magnitude bit pattern (bits & 0x7FFF).  Integer
// maxima are exact and order-free; a pattern >= 0x7F80 means Inf or NaN was seen.
__global__ void __launch_bounds__(256) amax_partial_kernel(const uint4* __restrict__ x, int64_t n_vec,
                                                           uint32_t* __restrict__ partials) {
  uint32_t m = 0;
  // four independent 16-byte loads in flight per thread and iteration
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n_vec; i += 4 * stride) {
    uint4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) v[u] = i + u * stride < n_vec ? __ldg(x + i + u * stride) : make_uint4(0, 0, 0, 0);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        m = max(m, w[j] & 0x7FFFu);
        m = max(m, (w[j] >> 16) & 0x7FFFu);
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
  __shared__ uint32_t red[8];
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x < 32) {
    m = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0u;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (threadIdx.x == 0) partials[blockIdx.x] = m;
  }
}

// The global scale from the amax partials (one warp): g = fp32(amax / 2688), 1 for amax 0;
// a non-finite amax raises kStatusNonFinite and stores NaN, which makes the quantiser skip.
__global__ void __launch_bounds__(32) global_scale_kernel(const uint32_t* partials, int n, float* g_out,
                                                          uint32_t* status) {
  uint32_t m = 0;
  for (int i = threadIdx.x; i < n; i += 32) m = max(m, partials[i]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (threadIdx.x == 0) {
    if (m >= 0x7F80u) {
      raise_status(status, kStatusNonFinite);
      *g_out = __uint_as_float(0x7FC00000u);
    } else {
      *g_out = global_scale_from_amax(__uint_as_float(m << 16));
    }
  }
}

// The tensor's amax as the BF16 magnitude bit pattern (one warp over the partials).
__global__ void __launch_bounds__(32) amax_reduce_kernel(const uint32_t* partials, int n, uint32_t* amax_bits) {
  uint32_t m = 0;
  for (int i = threadIdx.x; i < n; i += 32) m = max(m, partials[i]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (threadIdx.x == 0) *amax_bits = m;
}

// Per-halfword unsigned maximum of two packed pairs.
__device__ __forceinline__ uint32_t max_u16x2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.u16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// The E2M1 codes and E4M3 scale of one 16-value block held as 8 BF16 pairs in w: 8 code
// bytes in *c0, *c1, the scale byte returned.
__device__ __forceinline__ uint32_t quantize_block(const uint32_t* w, float r_t, float g, uint32_t* c0,
                                                   uint32_t* c1) {
  // block maximum of |x| on the BF16 magnitude bits, two halves per instruction (exact)
  uint32_t m2 = w[0] & 0x7FFF7FFFu;
#pragma unroll
  for (int j = 1; j < 8; ++j) m2 = max_u16x2(m2, w[j] & 0x7FFF7FFFu);
  const uint32_t mb = max(m2 & 0xFFFFu, m2 >> 16);
  float f[16];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    f[2 * j] = __uint_as_float(w[j] << 16);
    f[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
  }
  float r_b;
  const uint32_t s = block_scale(__uint_as_float(mb << 16), r_t, g, &r_b);
#pragma unroll
  for (int j = 0; j < 16; ++j) f[j] = __fmul_rn(f[j], r_b);
  *c0 = cvt_e2m1x8(f);
  *c1 = cvt_e2m1x8(f + 8);
  return s;
}

// One CTA per row (rows_padded CTAs), min(segments, 32) warps: each warp quantises the row's
// segments of 32 kBpl blocks (warp, warp + n_warps, ...), kBpl consecutive 16-value blocks per
// lane, so every load and store of the warp covers one contiguous span of the row.  Rows in
// [rows, rows_padded) only write zero scales (swizzled layout padding).  The global scale is
// read from g_in.  Two blocks per lane take fewer instructions per block (one 16-byte code
// store, one shuffle per scale word); one block per lane keeps twice the warps in flight for
// the forward's scatter into 8 segment rows and accumulator zeroing (measured faster there).
template <int kBpl>
__global__ void __launch_bounds__(1024) quantize_kernel(QuantizeArgs a) {
  static_assert(kBpl == 1 || kBpl == 2, "one or two blocks per lane");
  constexpr int kWordLanes = 4 / kBpl;          // lanes holding the 4 scales of one scale word
  const float g = __ldg(a.g_in);
  if (!(g > 0.0f && g < __uint_as_float(0x7F800000u))) return;   // non-finite input: skipped
  if (blockIdx.x == 0 && threadIdx.x == 0 && a.g_out != nullptr && a.g_out != a.g_in) *a.g_out = g;
  const float r_t = __frcp_rn(__fmul_rn(6.0f, g));

  const int blocks_per_row = (int)(a.cols >> 4);
  const int segs_per_row = (blocks_per_row + 32 * kBpl - 1) / (32 * kBpl);
  const int lane = threadIdx.x & 31;
  const int n_warps = blockDim.x >> 5;
  const int64_t r = blockIdx.x;
  // segment rows of the token's pairs (lane j < topk holds pair j's), found once per warp
  int64_t my_row = 0;
  if (a.seg_codes != nullptr && r < a.rows && lane < a.topk) {
    const int64_t p = r * a.topk + lane;
    const int e = a.idx[p];
    my_row = (int64_t)a.mtile_prefix[e] * kBlockM + (a.inv[p] - a.offsets[e]);
  }
  for (int seg = threadIdx.x >> 5; seg < segs_per_row; seg += n_warps) {
    const int b = seg * 32 * kBpl + kBpl * lane;    // first of the lane's blocks
    // lanes past the row's last block stay for the shuffles; the lanes of one scale word are
    // active or idle together (cols % 64 == 0)
    const bool active = b < blocks_per_row;
    const bool live = active && r < a.rows;

    if (a.zero_out != nullptr && live) {
      float4* z = reinterpret_cast<float4*>(a.zero_out + r * a.cols + (int64_t)b * 16);
      const float4 zero = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int i = 0; i < 4 * kBpl; ++i) z[i] = zero;
    }

    uint32_t sl = 0;                            // the lane's scale bytes
    uint32_t codes[2 * kBpl];
#pragma unroll
    for (int i = 0; i < 2 * kBpl; ++i) codes[i] = 0;
    if (live) {
      // every load of the lane in flight before the conversions (asm statements) start
      const uint4* src = reinterpret_cast<const uint4*>(a.x + r * a.cols + (int64_t)b * 16);
      uint4 v[2 * kBpl];
#pragma unroll
      for (int i = 0; i < 2 * kBpl; ++i) v[i] = __ldg(src + i);
#pragma unroll
      for (int k = 0; k < kBpl; ++k) {
        const uint32_t w[8] = {v[2 * k].x, v[2 * k].y, v[2 * k].z, v[2 * k].w,
                               v[2 * k + 1].x, v[2 * k + 1].y, v[2 * k + 1].z, v[2 * k + 1].w};
        sl |= quantize_block(w, r_t, g, &codes[2 * k], &codes[2 * k + 1]) << (8 * k);
      }
    }
    // the 32-bit scale word of this lane's group of 4 blocks (valid in lanes kWordLanes k)
    uint32_t sc = sl;
#pragma unroll
    for (int k = 1; k < kWordLanes; ++k) sc |= __shfl_down_sync(0xffffffffu, sl, k) << (8 * kBpl * k);
    const bool word_lane = active && (lane & (kWordLanes - 1)) == 0;

    auto store_codes = [&](uint8_t* row_base) {
      if constexpr (kBpl == 2) {
        reinterpret_cast<uint4*>(row_base)[b >> 1] = make_uint4(codes[0], codes[1], codes[2], codes[3]);
      } else {
        reinterpret_cast<uint2*>(row_base)[b] = make_uint2(codes[0], codes[1]);
      }
    };
    if (r < a.rows) {
      if (a.codes != nullptr && active) store_codes(a.codes + r * (a.cols >> 1));
      if (a.seg_codes != nullptr) {
        // every lane writes its blocks to all of the token's segment rows
        for (int j = 0; j < a.topk; ++j) {
          const int64_t row = __shfl_sync(0xffffffffu, my_row, j);
          if (active) store_codes(a.seg_codes + row * (a.cols >> 1));
          if (word_lane) *reinterpret_cast<uint32_t*>(a.seg_sf + swz_offset(row, b, a.n_col_tiles)) = sc;
        }
      }
    }
    if (a.scales != nullptr && word_lane) {
      uint32_t* sdst;
      if (a.swizzled) {
        sdst = reinterpret_cast<uint32_t*>(a.scales + swz_offset(r, b, a.n_col_tiles));
      } else {
        sdst = reinterpret_cast<uint32_t*>(a.scales + r * (a.cols >> 4) + b);
      }
      *sdst = sc;
    }
  }
}

int amax_partial_blocks(int64_t n_elems) {
  const int64_t n_vec = n_elems / 8;
  int64_t blocks = (n_vec + 255) / 256;
  if (blocks > kMaxAmaxPartials) blocks = kMaxAmaxPartials;
  if (blocks < 1) blocks = 1;
  return (int)blocks;
}

cudaError_t launch_amax_partial(const void* x, int64_t n_elems, uint32_t* partials, int blocks,
                                cudaStream_t stream) {
  amax_partial_kernel<<<blocks, 256, 0, stream>>>(reinterpret_cast<const uint4*>(x), n_elems / 8,
                                                  partials);
  return cudaGetLastError();
}

cudaError_t launch_quantize(QuantizeArgs a, cudaStream_t stream) {
  if (a.g_in == nullptr) {
    // dynamic scale: reduced once from the amax partials, then read by every CTA
    float* g = a.g_out != nullptr ? a.g_out : a.g_scratch;
    global_scale_kernel<<<1, 32, 0, stream>>>(a.partials, a.n_partials, g, a.status);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return err;
    a.g_in = g;
  }
  if (a.rows_padded == 0) {
    // no rows: only the scale used is reported
    if (a.g_out != nullptr && a.g_out != a.g_in)
      return cudaMemcpyAsync(a.g_out, a.g_in, sizeof(float), cudaMemcpyDeviceToDevice, stream);
    return cudaSuccess;
  }
  // the scatter into expert segments (the forward) keeps one block per lane
  if (a.seg_codes != nullptr || a.zero_out != nullptr) {
    const int segs = (int)(((a.cols >> 4) + 31) >> 5);
    quantize_kernel<1><<<(unsigned)a.rows_padded, 32 * (segs < 32 ? segs : 32), 0, stream>>>(a);
  } else {
    const int segs = (int)(((a.cols >> 4) + 63) >> 6);
    quantize_kernel<2><<<(unsigned)a.rows_padded, 32 * (segs < 32 ? segs : 32), 0, stream>>>(a);
  }
  return cudaGetLastError();
}

cudaError_t launch_global_scale(const uint32_t* partials, int n, float* g_out, uint32_t* status, cudaStream_t stream) {
  global_scale_kernel<<<1, 32, 0, stream>>>(partials, n, g_out, status);
  return cudaGetLastError();
}

cudaError_t launch_amax_reduce(const uint32_t* partials, int n, uint32_t* amax_bits, cudaStream_t stream) {
  amax_reduce_kernel<<<1, 32, 0, stream>>>(partials, n, amax_bits);
  return cudaGetLastError();
}

int quantize_launch_count(const QuantizeArgs& a) { return (a.g_in == nullptr ? 1 : 0) + (a.rows_padded > 0 ? 1 : 0); }

}  // namespace nvfp4moe
