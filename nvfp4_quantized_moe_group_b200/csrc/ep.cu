// Expert parallelism with an all-to-all exchange of quantised rows.
//
// The model's configuration places the experts on the devices, replicates the rest, and needs
// a device count that divides the 256 experts ("Reflection releases Beam ...", section "Tool
// calling and multi-node setups").  Rank d of G holds experts [d E/G, (d+1) E/G).  Each rank
// routes and quantises its own tokens (with the global scale of all ranks' tokens, so the
// codes equal those of the single-GPU layer on the concatenated batch), sends every
// (token, slot) pair's quantised row to the rank that holds the pair's expert, runs its
// experts on the rows it receives, returns the weighted FP32 output rows, and adds each
// token's returned rows in slot order.  The kernels here move the rows; routing, grouping,
// quantisation and the grouped GEMMs are the layer's own.
#include "common.cuh"
#include "kernels.h"

namespace nvfp4moe {

namespace {

constexpr int kEpThreads = 256;

// One warp per send position i (pairs in the stable expert-major order perm): the pair's token
// row (codes [H/2], linear scales [H/16]) copied to send row i, with the pair's destination-local
// expert, routing weight, and the position of pair p recorded in send_pos[p].
__global__ void __launch_bounds__(kEpThreads) ep_pack_kernel(EpPackArgs a) {
  const int64_t i = (int64_t)blockIdx.x * (kEpThreads / 32) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (i >= a.n_pairs) return;
  const int p = __ldg(a.perm + i);
  const int64_t t = p / a.topk;
  const int e = __ldg(a.idx + p);
  if (lane == 0) {
    a.send_expert[i] = e % a.experts_per_rank;
    a.send_w[i] = __ldg(a.wts + p);
    a.send_pos[p] = (int32_t)i;
  }
  const uint4* src = reinterpret_cast<const uint4*>(a.xq_codes + t * (a.H / 2));
  uint4* dst = reinterpret_cast<uint4*>(a.send_codes + i * (a.H / 2));
  for (int k = lane; k < a.H / 32; k += 32) dst[k] = __ldg(src + k);
  const uint32_t* ssrc = reinterpret_cast<const uint32_t*>(a.xq_scales + t * (a.H / 16));
  uint32_t* sdst = reinterpret_cast<uint32_t*>(a.send_scales + i * (a.H / 16));
  for (int k = lane; k < a.H / 64; k += 32) sdst[k] = __ldg(ssrc + k);
}

// Pairs per destination rank: the experts of rank d are d * epr .. (d + 1) * epr - 1.
__global__ void ep_rank_counts_kernel(const int32_t* counts, int E, int experts_per_rank, int32_t* rank_counts) {
  const int d = blockIdx.x * blockDim.x + threadIdx.x;
  if (d >= E / experts_per_rank) return;
  int32_t n = 0;
  for (int e = d * experts_per_rank; e < (d + 1) * experts_per_rank; ++e) n += counts[e];
  rank_counts[d] = n;
}

// One warp per received row i: its codes and scales copied into the padded expert-segment row
// of the grouping (segment row = tile prefix of its expert * 128 + its rank in the expert),
// scales into the swizzled 128 x 4 layout; its output row zeroed (the down GEMM adds into it).
__global__ void __launch_bounds__(kEpThreads) rows_to_segments_kernel(RowsToSegmentsArgs a) {
  const int64_t i = (int64_t)blockIdx.x * (kEpThreads / 32) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (i >= a.n_rows) return;
  const int e = __ldg(a.expert + i);
  const int64_t row = (int64_t)__ldg(a.mtile_prefix + e) * kBlockM + (__ldg(a.inv + i) - __ldg(a.offsets + e));
  const uint4* src = reinterpret_cast<const uint4*>(a.codes + i * (a.H / 2));
  uint4* dst = reinterpret_cast<uint4*>(a.seg_codes + row * (a.H / 2));
  for (int k = lane; k < a.H / 32; k += 32) dst[k] = __ldg(src + k);
  const uint32_t* ssrc = reinterpret_cast<const uint32_t*>(a.scales + i * (a.H / 16));
  for (int k = lane; k < a.H / 64; k += 32)
    *reinterpret_cast<uint32_t*>(a.seg_sf + swz_offset(row, 4 * k, a.n_col_tiles)) = __ldg(ssrc + k);
  float4* z = reinterpret_cast<float4*>(a.out_rows + i * a.H);
  const float4 zero = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int k = lane; k < a.H / 4; k += 32) z[k] = zero;
}

// out[t] = bf16(sum over slots j = 0 .. topk-1, in that order, of rows[send_pos[t topk + j]]):
// the FP32 sum of a token's weighted expert rows, one CTA per token, 8 values per thread step.
__global__ void __launch_bounds__(kEpThreads) ep_combine_kernel(const float* __restrict__ rows,
                                                                const int32_t* __restrict__ send_pos, int topk,
                                                                int H, uint16_t* __restrict__ out) {
  const int64_t t = blockIdx.x;
  __shared__ int32_t s_pos[8];
  if (threadIdx.x < topk) s_pos[threadIdx.x] = send_pos[t * topk + threadIdx.x];
  __syncthreads();
  for (int c = threadIdx.x * 8; c < H; c += kEpThreads * 8) {
    float acc[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) acc[k] = 0.0f;
    for (int j = 0; j < topk; ++j) {
      const float4* src = reinterpret_cast<const float4*>(rows + (int64_t)s_pos[j] * H + c);
      const float4 v0 = __ldg(src), v1 = __ldg(src + 1);
      acc[0] = __fadd_rn(acc[0], v0.x);
      acc[1] = __fadd_rn(acc[1], v0.y);
      acc[2] = __fadd_rn(acc[2], v0.z);
      acc[3] = __fadd_rn(acc[3], v0.w);
      acc[4] = __fadd_rn(acc[4], v1.x);
      acc[5] = __fadd_rn(acc[5], v1.y);
      acc[6] = __fadd_rn(acc[6], v1.z);
      acc[7] = __fadd_rn(acc[7], v1.w);
    }
    uint32_t w[4];
#pragma unroll
    for (int k = 0; k < 4; ++k)
      w[k] = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(acc[2 * k])) |
             ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(acc[2 * k + 1])) << 16);
    *reinterpret_cast<uint4*>(out + t * H + c) = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

// out[i] = idx[i] when 0 <= idx[i] < n, else 0 with kStatusBadInput raised.
__global__ void __launch_bounds__(kEpThreads) check_indices_kernel(const int32_t* idx, int64_t count, int n,
                                                                   int32_t* out, uint32_t* status) {
  const int64_t i = (int64_t)blockIdx.x * kEpThreads + threadIdx.x;
  if (i >= count) return;
  const int32_t v = idx[i];
  const bool ok = v >= 0 && v < n;
  out[i] = ok ? v : 0;
  if (!ok) raise_status(status, kStatusBadInput);
}

}  // namespace

cudaError_t launch_check_indices(const int32_t* idx, int64_t count, int n, int32_t* out, uint32_t* status,
                                 cudaStream_t stream) {
  if (count == 0) return cudaSuccess;
  check_indices_kernel<<<(unsigned)((count + kEpThreads - 1) / kEpThreads), kEpThreads, 0, stream>>>(idx, count, n,
                                                                                                        out, status);
  return cudaGetLastError();
}

cudaError_t launch_ep_pack(const EpPackArgs& a, cudaStream_t stream) {
  if (a.n_pairs > 0) {
    const int64_t blocks = (a.n_pairs + kEpThreads / 32 - 1) / (kEpThreads / 32);
    ep_pack_kernel<<<(unsigned)blocks, kEpThreads, 0, stream>>>(a);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return err;
  }
  const int ranks = a.E / a.experts_per_rank;
  ep_rank_counts_kernel<<<(ranks + 127) / 128, 128, 0, stream>>>(a.counts, a.E, a.experts_per_rank, a.rank_counts);
  return cudaGetLastError();
}

cudaError_t launch_rows_to_segments(const RowsToSegmentsArgs& a, cudaStream_t stream) {
  if (a.n_rows == 0) return cudaSuccess;
  const int64_t blocks = (a.n_rows + kEpThreads / 32 - 1) / (kEpThreads / 32);
  rows_to_segments_kernel<<<(unsigned)blocks, kEpThreads, 0, stream>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_ep_combine(const float* rows, const int32_t* send_pos, int64_t T, int topk, int H, uint16_t* out,
                              cudaStream_t stream) {
  if (T == 0) return cudaSuccess;
  ep_combine_kernel<<<(unsigned)T, kEpThreads, 0, stream>>>(rows, send_pos, topk, H, out);
  return cudaGetLastError();
}

}  // namespace nvfp4moe
