// Grouping of (token, slot) pairs by expert and the byte-moving kernels around the grouped
// GEMMs: stable counting sort into 128-row-padded expert segments, FP32 -> BF16 output,
// scale-layout conversions.
// Only the top-8 of 256 experts run per token ("Reflection releases Beam ...", section
// "Mixture-of-Experts details"), so the pairs are grouped by expert before the expert GEMMs.
#include "common.cuh"
#include "kernels.h"

namespace nvfp4moe {

// Per chunk of kPermChunkTokens tokens: how many of its pairs go to each expert.
__global__ void __launch_bounds__(256) perm_count_kernel(PermArgs a) {
  __shared__ int hist[256];
  for (int e = threadIdx.x; e < a.E; e += blockDim.x) hist[e] = 0;
  __syncthreads();
  const int64_t p0 = (int64_t)blockIdx.x * kPermChunkTokens * a.topk;
  const int64_t p1 = min(p0 + (int64_t)kPermChunkTokens * a.topk, a.T * a.topk);
  for (int64_t p = p0 + threadIdx.x; p < p1; p += blockDim.x) atomicAdd(&hist[a.idx[p]], 1);
  __syncthreads();
  for (int e = threadIdx.x; e < a.E; e += blockDim.x)
    a.chunk_counts[(int64_t)blockIdx.x * a.E + e] = hist[e];
}

// Per expert, the position of each chunk's first pair inside the expert's segment (exclusive
// prefix of the chunk counts over the chunks) and the expert's pair count.  One CTA per 32
// experts (lane = expert), its 8 warps splitting the chunks into 8 consecutive runs: each warp
// sums its run, the CTA turns the 8 sums into run bases, and each warp writes its run's
// prefixes.  The chunk counts are read in batches of independent loads.
__global__ void __launch_bounds__(256) perm_colscan_kernel(PermArgs a) {
  __shared__ int s_sum[8][32];
  constexpr int kBatch = 32;
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int e = blockIdx.x * 32 + lane;
  const bool on = e < a.E;
  const int per = (a.n_chunks + 7) / 8;
  const int c0 = warp * per;
  const int c1 = min(c0 + per, a.n_chunks);
  const int* __restrict__ cc = a.chunk_counts;
  int sum = 0;
  for (int b = c0; b < c1; b += kBatch) {
    int v[kBatch];
#pragma unroll
    for (int j = 0; j < kBatch; ++j) v[j] = on && b + j < c1 ? __ldg(cc + (int64_t)(b + j) * a.E + e) : 0;
#pragma unroll
    for (int j = 0; j < kBatch; ++j) sum += v[j];
  }
  s_sum[warp][lane] = sum;
  __syncthreads();
  int base = 0, total = 0;
#pragma unroll
  for (int w = 0; w < 8; ++w) {
    const int v = s_sum[w][lane];
    base += w < warp ? v : 0;
    total += v;
  }
  if (!on) return;
  if (warp == 0) a.counts[e] = total;
  for (int b = c0; b < c1; b += kBatch) {
    int v[kBatch];
#pragma unroll
    for (int j = 0; j < kBatch; ++j) v[j] = b + j < c1 ? __ldg(cc + (int64_t)(b + j) * a.E + e) : 0;
#pragma unroll
    for (int j = 0; j < kBatch; ++j) {
      if (b + j < c1) a.chunk_base[(int64_t)(b + j) * a.E + e] = base;
      base += v[j];
    }
  }
}

// One block, one thread per expert: offsets (exclusive scan of the counts), the 128-row tile
// prefix, and -1 in every padding row of every segment.
__global__ void __launch_bounds__(256) perm_scan_kernel(PermArgs a) {
  __shared__ int s_cnt[256];
  __shared__ int s_tiles[256];
  const int e = threadIdx.x;
  const int count = e < a.E ? a.counts[e] : 0;
  const int tiles = (count + kBlockM - 1) / kBlockM;
  s_cnt[e] = count;
  s_tiles[e] = tiles;
  __syncthreads();
  // inclusive scans (Hillis-Steele) of counts and tiles over the 256 threads
  for (int d = 1; d < 256; d <<= 1) {
    const int vc = e >= d ? s_cnt[e - d] : 0;
    const int vt = e >= d ? s_tiles[e - d] : 0;
    __syncthreads();
    s_cnt[e] += vc;
    s_tiles[e] += vt;
    __syncthreads();
  }
  if (e < a.E) {
    const int off = s_cnt[e] - count;         // exclusive
    const int tile0 = s_tiles[e] - tiles;
    a.offsets[e] = off;
    a.mtile_prefix[e] = tile0;
    if (e == a.E - 1) {
      a.offsets[a.E] = off + count;
      a.mtile_prefix[a.E] = tile0 + tiles;
    }
    const int64_t r0 = (int64_t)tile0 * kBlockM;
    const int64_t r1 = r0 + (int64_t)tiles * kBlockM;
    for (int64_t r = r0 + count; r < r1; ++r) a.row_pair[r] = -1;
  }
}

// One warp per chunk walks its pairs in order, so pairs of one expert keep ascending pair
// (and token) order: a stable counting sort.
__global__ void __launch_bounds__(32) perm_scatter_kernel(PermArgs a) {
  __shared__ int run[256];
  const int lane = threadIdx.x;
  const int c = blockIdx.x;
  for (int e = lane; e < a.E; e += 32) run[e] = a.offsets[e] + a.chunk_base[(int64_t)c * a.E + e];
  __syncwarp();
  const int64_t p0 = (int64_t)c * kPermChunkTokens * a.topk;
  const int64_t p1 = min(p0 + (int64_t)kPermChunkTokens * a.topk, a.T * a.topk);
  const uint32_t lt = (1u << lane) - 1u;
  for (int64_t base = p0; base < p1; base += 32) {
    const int64_t p = base + lane;
    const bool valid = p < p1;
    const int e = valid ? a.idx[p] : -1;
    const uint32_t peers = __match_any_sync(0xffffffffu, e);
    const int rank = __popc(peers & lt);
    if (valid) {
      const int pos = run[e] + rank;
      a.perm[pos] = (int32_t)p;
      a.inv[p] = pos;
      const int64_t row = (int64_t)a.mtile_prefix[e] * kBlockM + (pos - a.offsets[e]);
      a.row_pair[row] = (int32_t)p;
    }
    __syncwarp();
    if (valid && rank == 0) run[e] += __popc(peers);
    __syncwarp();
  }
}

// Small inputs: histogram, scan and the stable scatter in one block (the scatter walks the
// pairs in order with one warp, like perm_scatter_kernel does per chunk).
__global__ void __launch_bounds__(256) perm_small_kernel(PermArgs a) {
  __shared__ int s_cnt[256];
  __shared__ int s_tiles[256];
  __shared__ int run[256];
  const int e = threadIdx.x;
  s_cnt[e] = 0;
  __syncthreads();
  const int64_t n = a.T * a.topk;
  for (int64_t p = e; p < n; p += blockDim.x) atomicAdd(&s_cnt[a.idx[p]], 1);
  __syncthreads();
  const int count = e < a.E ? s_cnt[e] : 0;
  const int tiles = (count + kBlockM - 1) / kBlockM;
  s_tiles[e] = tiles;
  __syncthreads();
  for (int d = 1; d < 256; d <<= 1) {
    const int vc = e >= d ? s_cnt[e - d] : 0;
    const int vt = e >= d ? s_tiles[e - d] : 0;
    __syncthreads();
    s_cnt[e] += vc;
    s_tiles[e] += vt;
    __syncthreads();
  }
  if (e < a.E) {
    const int off = s_cnt[e] - count;
    const int tile0 = s_tiles[e] - tiles;
    a.offsets[e] = off;
    a.mtile_prefix[e] = tile0;
    a.counts[e] = count;
    run[e] = off;
    if (e == a.E - 1) {
      a.offsets[a.E] = off + count;
      a.mtile_prefix[a.E] = tile0 + tiles;
    }
    const int64_t r0 = (int64_t)tile0 * kBlockM;
    for (int64_t r = r0 + count; r < r0 + (int64_t)tiles * kBlockM; ++r) a.row_pair[r] = -1;
  }
  __syncthreads();
  if (e >= 32) return;
  const int lane = e;
  const uint32_t lt = (1u << lane) - 1u;
  for (int64_t base = 0; base < n; base += 32) {
    const int64_t p = base + lane;
    const bool valid = p < n;
    const int ex = valid ? a.idx[p] : -1;
    const uint32_t peers = __match_any_sync(0xffffffffu, ex);
    const int rank = __popc(peers & lt);
    if (valid) {
      const int pos = run[ex] + rank;
      a.perm[pos] = (int32_t)p;
      a.inv[p] = pos;
      a.row_pair[(int64_t)a.mtile_prefix[ex] * kBlockM + (pos - a.offsets[ex])] = (int32_t)p;
    }
    __syncwarp();
    if (valid && rank == 0) run[ex] += __popc(peers);
    __syncwarp();
  }
}

cudaError_t launch_permute(const PermArgs& a, cudaStream_t stream, int* launches) {
  if (a.T * a.topk <= kPermSmallPairs) {
    perm_small_kernel<<<1, 256, 0, stream>>>(a);
    *launches += 1;
    return cudaGetLastError();
  }
  *launches += 4;
  perm_count_kernel<<<a.n_chunks, 256, 0, stream>>>(a);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  perm_colscan_kernel<<<(a.E + 31) / 32, 256, 0, stream>>>(a);
  err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  perm_scan_kernel<<<1, 256, 0, stream>>>(a);
  err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  perm_scatter_kernel<<<a.n_chunks, 32, 0, stream>>>(a);
  return cudaGetLastError();
}

// out = bf16(acc), or with the residual stream bf16(fp32(a * res) + fp32(b * acc)) (the
// weighted residual add of "Reflection releases Beam ...", section "Residual stream and
// numerical decisions"); 8 values per thread.  res may alias out: each thread reads its 8
// residual values before it writes them.
__global__ void __launch_bounds__(256) finalize_kernel(FinalizeArgs a) {
  pdl_wait();   // launched programmatically after the down GEMM
  const int64_t i = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) * 8;
  if (i >= a.n) return;
  const float4 p = *reinterpret_cast<const float4*>(a.acc + i);
  const float4 q = *reinterpret_cast<const float4*>(a.acc + i + 4);
  float v[8] = {p.x, p.y, p.z, p.w, q.x, q.y, q.z, q.w};
  if (a.res != nullptr) {
    const uint4 r = *reinterpret_cast<const uint4*>(a.res + i);
    const uint32_t rw[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      v[2 * j] = __fadd_rn(__fmul_rn(a.a, __uint_as_float(rw[j] << 16)), __fmul_rn(a.b, v[2 * j]));
      v[2 * j + 1] = __fadd_rn(__fmul_rn(a.a, __uint_as_float(rw[j] & 0xFFFF0000u)), __fmul_rn(a.b, v[2 * j + 1]));
    }
  }
  uint32_t w[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t lo = __bfloat16_as_ushort(__float2bfloat16_rn(v[2 * j]));
    const uint32_t hi = __bfloat16_as_ushort(__float2bfloat16_rn(v[2 * j + 1]));
    w[j] = lo | (hi << 16);
  }
  *reinterpret_cast<uint4*>(a.out + i) = make_uint4(w[0], w[1], w[2], w[3]);
}

cudaError_t launch_finalize(const FinalizeArgs& a, cudaStream_t stream) {
  if (a.n == 0) return cudaSuccess;
  const int64_t threads = a.n / 8;
  return launch_pdl(finalize_kernel, dim3((unsigned)((threads + 255) / 256)), dim3(256), 0, stream, a);
}

// Linear [n_rows][cols16] scales from swizzled storage: row i of the output is row
// src_rows[i] (or i when src_rows is null) of the swizzled tensor.
__global__ void __launch_bounds__(256) unswizzle_rows_kernel(const uint8_t* sf, int64_t n_col_tiles,
                                                             const int32_t* src_rows, int64_t n_rows,
                                                             int cols16, uint8_t* out) {
  const int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (i >= n_rows * cols16) return;
  const int64_t r = i / cols16;
  const int c = (int)(i - r * cols16);
  const int64_t sr = src_rows ? src_rows[r] : r;
  out[i] = sf[swz_offset(sr, c, n_col_tiles)];
}

cudaError_t launch_unswizzle_rows(const uint8_t* sf, int64_t n_col_tiles, const int32_t* src_rows,
                                  int64_t n_rows, int cols16, uint8_t* out, cudaStream_t stream) {
  const int64_t n = n_rows * cols16;
  if (n == 0) return cudaSuccess;
  unswizzle_rows_kernel<<<(unsigned)((n + 255) / 256), 256, 0, stream>>>(sf, n_col_tiles, src_rows,
                                                                         n_rows, cols16, out);
  return cudaGetLastError();
}

// Debug export of the requantised SwiGLU intermediate: row pos of the output (perm order)
// is the padded segment row of pair perm[pos].
__global__ void __launch_bounds__(256) export_hq_kernel(const uint8_t* hq_codes, const uint8_t* hq_sf,
                                                        const int32_t* perm, const int32_t* idx,
                                                        const int32_t* offsets,
                                                        const int32_t* mtile_prefix, int64_t n_pairs,
                                                        int I, uint8_t* out_codes, uint8_t* out_sf) {
  const int64_t pos = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (pos >= n_pairs) return;
  const int e = idx[perm[pos]];
  const int64_t row = (int64_t)mtile_prefix[e] * kBlockM + (pos - offsets[e]);
  for (int j = lane; j < I / 2; j += 32) out_codes[pos * (I / 2) + j] = hq_codes[row * (I / 2) + j];
  for (int c = lane; c < I / 16; c += 32) out_sf[pos * (I / 16) + c] = hq_sf[swz_offset(row, c, I / 64)];
}

cudaError_t launch_export_hq(const uint8_t* hq_codes, const uint8_t* hq_sf, const int32_t* perm,
                             const int32_t* idx, const int32_t* offsets, const int32_t* mtile_prefix,
                             int64_t n_pairs, int I, uint8_t* out_codes, uint8_t* out_sf,
                             cudaStream_t stream) {
  if (n_pairs == 0) return cudaSuccess;
  export_hq_kernel<<<(unsigned)((n_pairs + 7) / 8), 256, 0, stream>>>(
      hq_codes, hq_sf, perm, idx, offsets, mtile_prefix, n_pairs, I, out_codes, out_sf);
  return cudaGetLastError();
}

// Linear [rows][cols16] weight scales -> swizzled operand storage.  Source row r goes to
// destination row (r / group) * group * mul + add * group + r % group (gate/up interleave:
// group 64, mul 2, add 0 for gate and 1 for up).
__global__ void __launch_bounds__(256) repack_sf_kernel(const uint8_t* linear, int rows, int cols16,
                                                        uint8_t* swz, int64_t n_col_tiles, int group, int mul,
                                                        int add) {
  const int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (i >= (int64_t)rows * cols16) return;
  const int r = (int)(i / cols16);
  const int c = (int)(i - (int64_t)r * cols16);
  const int64_t dr = (int64_t)(r / group) * group * mul + (int64_t)add * group + r % group;
  swz[swz_offset(dr, c, n_col_tiles)] = linear[i];
}

cudaError_t launch_repack_sf(const uint8_t* linear, int rows, int cols16, uint8_t* swz,
                             int64_t n_col_tiles, int group, int mul, int add, cudaStream_t stream) {
  const int64_t n = (int64_t)rows * cols16;
  repack_sf_kernel<<<(unsigned)((n + 255) / 256), 256, 0, stream>>>(linear, rows, cols16, swz, n_col_tiles,
                                                                    group, mul, add);
  return cudaGetLastError();
}

// One thread per 16-byte chunk of a weight row.
__global__ void __launch_bounds__(256) tile_weights_kernel(const uint8_t* src, int rows, int row_bytes,
                                                           uint8_t* dst, int group, int mul, int add) {
  const int chunks = row_bytes / 16;
  const int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (i >= (int64_t)rows * chunks) return;
  const int r = (int)(i / chunks);
  const int j = (int)(i - (int64_t)r * chunks);
  const int64_t pr = (int64_t)(r / group) * group * mul + (int64_t)add * group + r % group;
  const int64_t tile = pr >> 7;
  const int rr = (int)(pr & 127);
  const int kb_count = (row_bytes + 127) / 128;
  const int kb = j >> 3, c = j & 7;
  const int64_t off = ((tile * kb_count + kb) * 128 + rr) * 128 + ((c ^ (rr & 7)) << 4);
  *reinterpret_cast<uint4*>(dst + off) = *reinterpret_cast<const uint4*>(src + (int64_t)r * row_bytes + j * 16);
}

cudaError_t launch_tile_weights(const uint8_t* src, int rows, int row_bytes, uint8_t* dst, int group, int mul,
                                int add, cudaStream_t stream) {
  const int64_t n = (int64_t)rows * (row_bytes / 16);
  tile_weights_kernel<<<(unsigned)((n + 255) / 256), 256, 0, stream>>>(src, rows, row_bytes, dst, group, mul, add);
  return cudaGetLastError();
}

}  // namespace nvfp4moe
