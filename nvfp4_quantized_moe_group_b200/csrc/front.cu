// Fused front end of the layer for small token counts (decode): router logits, global amax
// of the input, group-limited top-k, grouping of the (token, slot) pairs by expert and the
// NVFP4 quantisation of x into the expert segments, in ONE cooperative launch with two
// grid-wide barriers.  At T <= 64 each of these steps moves a few hundred KB at most, so
// separate launches cost far more than the work; here each step is one round of loads.
//
// Same arithmetic as the separate kernels: logits as FP32 FMA chains of at most 32
// products summed in FP64 and rounded once ("Reflection releases Beam ...", sections
// "Mixture-of-Experts details" and "Residual stream and numerical decisions"); NVFP4 rule of
// "NVFP4 quantization", section "Quantization scheme", with the scale reading of nvfp4moe.h.
#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "route_topk.cuh"

namespace nvfp4moe {

namespace {
constexpr int kFrontThreads = kTopkThreads;
constexpr int kFrontTileE = 64;     // experts per CTA in the logits phase
constexpr int kFrontEpt = 4;        // experts per thread (one shared-memory load feeds 16 FMAs)
constexpr int kFrontKq = 8;         // threads per expert quad (each holds 1/8 of the K slice)
constexpr int kFrontTs = 2;         // token subsets (threads per expert quad and K eighth)
constexpr int kFrontMaxKq = 20;     // K values per thread and expert: an FMA chain of <= 20,
                                    // then 3 tree levels over the eighths: <= 23 roundings
constexpr size_t kFrontSmemCap = 64 * 1024;   // dynamic shared memory (the x slice) at most
constexpr int kFrontMaxGrid = 148;  // CTAs at most (one per SM of a B200)
constexpr int kFrontTokU = 4;       // tokens per group (x 4 experts = 16 interleaved chains)

__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Grid-wide barrier of a cooperative launch (all CTAs are resident).  *bar is 0 when the
// launch starts; every barrier adds 0x80000000 in total (CTA 0 adds 0x80000000 - (nb - 1),
// every other CTA 1), so the top bit takes the value `top` (0x80000000 after the first
// barrier, 0 after the second) exactly when the last CTA arrives, and the low bits are 0
// again.  The arrival is a release reduction (no round trip); the wait is bounded by limit_ns:
// on timeout kStatusTimeout is raised and false returned (the caller stops).  With
// arrive == false the CTA only waits (a test hook: the other CTAs' waits then run out too).
__device__ bool grid_barrier(uint32_t* bar, uint32_t top, uint32_t* status, uint64_t limit_ns, bool arrive = true) {
  __shared__ int s_ok;
  __syncthreads();
  if (threadIdx.x == 0) {
    const uint32_t nb = gridDim.x;
    const uint32_t add = blockIdx.x == 0 ? 0x80000000u - (nb - 1u) : 1u;
    if (arrive)
      asm volatile("fence.acq_rel.gpu;\n\tred.relaxed.gpu.global.add.u32 [%0], %1;" ::"l"(bar), "r"(add)
                   : "memory");
    int ok = 1;
    const uint64_t t0 = globaltimer_ns();
    uint32_t n = 0;
    while ((ld_acquire_u32(bar) & 0x80000000u) != top) {
      if ((++n & 63u) == 0u && globaltimer_ns() - t0 > limit_ns) {
        raise_status(status, kStatusTimeout);
        ok = 0;
        break;
      }
    }
    s_ok = ok;
  }
  __syncthreads();
  return s_ok != 0;
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }
}  // namespace

// Dynamic shared memory: the CTA's x slice, [T][k_slice] FP32.
__global__ void __launch_bounds__(kFrontThreads, 1) front_kernel(FrontArgs a) {
  extern __shared__ __align__(16) uint8_t dsm[];
  __shared__ float s_sc[256];
  __shared__ unsigned long long s_mask[256];
  __shared__ int s_off[256];
  __shared__ int s_tile0[256];
  __shared__ int s_wsum[8][2];
  __shared__ int s_row[kFrontMaxT * 8];
  __shared__ int s_idx[kFrontMaxT * 8];
  __shared__ uint32_t s_red[kFrontThreads / 32];
  __shared__ int s_bad;

  const int tid = threadIdx.x;
  const int nb = gridDim.x;
  const int T = (int)a.T, E = a.E, H = a.H, topk = a.topk;
  // the gate/up GEMM that follows may take the SMs this grid leaves free and set up there
  pdl_trigger();

  // ---------------------------------------------------------------- phase 1: logits --
  // CTA b: experts [64 * (b % n_etiles), +64), K slice b / n_etiles.  Thread (ts, eq, kq):
  // experts 4 eq .. 4 eq + 3 of the tile, the kq-th eighth of the K slice (<= 20 values per
  // expert, in registers), token groups g = ts, ts + 2, ... of 4 tokens.  Each of the 16
  // (token, expert) values is an FP32 FMA chain; the eight eighths are then added by a
  // butterfly over adjacent lanes (3 FP32 levels), so every product passes through at most
  // 23 FP32 roundings before the FP64 sum over the K slices.
  {
    const int n_etiles = (E + kFrontTileE - 1) / kFrontTileE;
    const int etile = blockIdx.x % n_etiles;
    const int ks = blockIdx.x / n_etiles;
    const int kslice = a.k_slice;
    const int kq_len = kslice / kFrontKq;
    const int64_t k_begin = (int64_t)ks * kslice;
    float* xs = reinterpret_cast<float*>(dsm);

    // x slice -> shared as FP32 (one conversion per value, shared by the CTA's 64 experts),
    // with the running max of |x| (BF16 magnitude bits)
    uint32_t mag = 0;
    const int vec_per_row = kslice >> 3;
    for (int v = tid; v < T * vec_per_row; v += kFrontThreads) {
      const int t = v / vec_per_row, c = v - t * vec_per_row;
      const uint4 q = __ldg(reinterpret_cast<const uint4*>(a.x + (int64_t)t * H + k_begin) + c);
      const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) mag = max(mag, max(w[j] & 0x7FFFu, (w[j] >> 16) & 0x7FFFu));
      float4* dst = reinterpret_cast<float4*>(xs + (int64_t)t * kslice + 8 * c);
      dst[0] = make_float4(bf16_lo(q.x), bf16_hi(q.x), bf16_lo(q.y), bf16_hi(q.y));
      dst[1] = make_float4(bf16_lo(q.z), bf16_hi(q.z), bf16_lo(q.w), bf16_hi(q.w));
    }
    const int kq = tid % kFrontKq;
    const int eq = (tid / kFrontKq) % (kFrontTileE / kFrontEpt);
    const int ts = tid / (kFrontKq * (kFrontTileE / kFrontEpt));
    const int e_base = etile * kFrontTileE + eq * kFrontEpt;
    float wr[kFrontEpt][kFrontMaxKq];
#pragma unroll
    for (int i = 0; i < kFrontEpt; ++i) {
      const int e = e_base + i;
      const float4* src =
          reinterpret_cast<const float4*>(a.w + (int64_t)(e < E ? e : 0) * H + k_begin + kq * kq_len);
#pragma unroll
      for (int j = 0; j < kFrontMaxKq / 4; ++j) {
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (4 * j < kq_len && e < E) v = __ldg(src + j);
        wr[i][4 * j] = v.x; wr[i][4 * j + 1] = v.y; wr[i][4 * j + 2] = v.z; wr[i][4 * j + 3] = v.w;
      }
    }
    // the layer accumulator is zeroed while the loads are in flight
    {
      float4* z = reinterpret_cast<float4*>(a.acc);
      const int64_t n4 = (int64_t)T * H / 4;
      for (int64_t i = blockIdx.x * (int64_t)kFrontThreads + tid; i < n4; i += (int64_t)nb * kFrontThreads)
        z[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    if (etile == 0) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mag = max(mag, __shfl_xor_sync(0xffffffffu, mag, o));
      if ((tid & 31) == 0) s_red[tid >> 5] = mag;
    }
    __syncthreads();
    if (etile == 0 && tid < 32) {
      mag = tid < kFrontThreads / 32 ? s_red[tid] : 0u;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mag = max(mag, __shfl_xor_sync(0xffffffffu, mag, o));
      if (tid == 0) a.amax_partials[ks] = mag;
    }
    double* out = a.parts + (int64_t)ks * T * E;
    const float* xq = xs + kq * kq_len;
    for (int g = ts; g * kFrontTokU < T; g += kFrontTs) {
      const int t0 = g * kFrontTokU;
      float v[kFrontTokU * kFrontEpt];   // v[u * 4 + i]: token t0 + u, expert e_base + i
#pragma unroll
      for (int n = 0; n < kFrontTokU * kFrontEpt; ++n) v[n] = 0.f;
#pragma unroll
      for (int j = 0; j < kFrontMaxKq / 4; ++j) {
        if (4 * j < kq_len) {
#pragma unroll
          for (int u = 0; u < kFrontTokU; ++u) {
            const int t = min(t0 + u, T - 1);   // rows past T are computed, not stored
            const float4 xv = *reinterpret_cast<const float4*>(xq + t * kslice + 4 * j);
#pragma unroll
            for (int i = 0; i < kFrontEpt; ++i) {
              float& p = v[u * kFrontEpt + i];
              p = __fmaf_rn(xv.x, wr[i][4 * j + 0], p);
              p = __fmaf_rn(xv.y, wr[i][4 * j + 1], p);
              p = __fmaf_rn(xv.z, wr[i][4 * j + 2], p);
              p = __fmaf_rn(xv.w, wr[i][4 * j + 3], p);
            }
          }
        }
      }
      // butterfly reduce-scatter over the 8 K-eighths: after the levels xor 4, 2, 1 lane kq
      // holds the full sums of values 2 * kq' and 2 * kq' + 1, kq' = its bit-reversed index
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        const bool hi = kq & 4;
        const float send = hi ? v[m] : v[m + 8];
        const float keep = hi ? v[m + 8] : v[m];
        v[m] = __fadd_rn(keep, __shfl_xor_sync(0xffffffffu, send, 4));
      }
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const bool hi = kq & 2;
        const float send = hi ? v[m] : v[m + 4];
        const float keep = hi ? v[m + 4] : v[m];
        v[m] = __fadd_rn(keep, __shfl_xor_sync(0xffffffffu, send, 2));
      }
#pragma unroll
      for (int m = 0; m < 2; ++m) {
        const bool hi = kq & 1;
        const float send = hi ? v[m] : v[m + 2];
        const float keep = hi ? v[m + 2] : v[m];
        v[m] = __fadd_rn(keep, __shfl_xor_sync(0xffffffffu, send, 1));
      }
      const int base = ((kq & 4) ? 8 : 0) + ((kq & 2) ? 4 : 0) + ((kq & 1) ? 2 : 0);
#pragma unroll
      for (int m = 0; m < 2; ++m) {
        const int n = base + m;
        const int t = t0 + n / kFrontEpt, e = e_base + n % kFrontEpt;
        if (t < T && e < E) out[(int64_t)t * E + e] = (double)v[m];
      }
    }
  }
  const uint64_t wait_ns = wait_limit(a.wait_ns);
  if (!grid_barrier(a.barrier, 0x80000000u, a.status, wait_ns, (int)blockIdx.x + 1 != a.skip_arrive)) return;

  // ------------------------------------------------------------ phase 2: top-k ---------
  for (int t = blockIdx.x; t < T; t += nb) {
    for (int e = tid; e < E; e += kFrontThreads) {
      const double* src = a.parts + (int64_t)t * E + e;
      const int64_t step = (int64_t)T * E;
      double acc = 0.0;
      int ks = 0;
      for (; ks + 32 <= a.ksplit; ks += 32) {   // 32 loads in flight
        double v[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = __ldcg(src + (int64_t)(ks + j) * step);
#pragma unroll
        for (int j = 0; j < 32; ++j) acc = __dadd_rn(acc, v[j]);
      }
      for (; ks < a.ksplit; ++ks) acc = __dadd_rn(acc, __ldcg(src + (int64_t)ks * step));
      if (a.bias != nullptr) acc = __dadd_rn(acc, (double)a.bias[e]);
      const float l = __double2float_rn(acc);
      if (a.logits_out != nullptr) a.logits_out[(int64_t)t * E + e] = l;
      s_sc[e] = router_sigmoid(l);
    }
    __syncthreads();
    route_topk_block(s_sc, E, a.n_groups, a.topk_groups, topk, a.routed_scale, a.idx + (int64_t)t * topk,
                     a.wts + (int64_t)t * topk, a.status);
  }
  if (!grid_barrier(a.barrier, 0u, a.status, wait_ns)) return;

  // ------------------------------------------- phase 3: grouping + quantise-scatter --
  // Every CTA rebuilds the grouping from idx (at most 512 pairs) in shared memory; CTA 0
  // publishes it.  Rank of pair (t, j) in its expert = earlier tokens that chose the same
  // expert (the topk experts of a token are distinct), so the sort is stable in pair order.
  const int n_pairs = T * topk;
  const int blocks_per_row = H >> 4;
  const int n_units = T * blocks_per_row;
  const int u0 = blockIdx.x * kFrontThreads + tid;
  // loads that do not depend on the grouping are issued first
  uint4 xv0 = make_uint4(0, 0, 0, 0), xv1 = xv0;
  if (u0 < n_units) {
    const int t = u0 / blocks_per_row, c = u0 - t * blocks_per_row;
    const uint4* src = reinterpret_cast<const uint4*>(a.x + (int64_t)t * H + 16 * c);
    xv0 = __ldg(src);
    xv1 = __ldg(src + 1);
  }
  uint32_t amax_bits = 0;
  if (tid < 32)
    for (int i = tid; i < a.ksplit; i += 32) amax_bits = max(amax_bits, __ldcg(a.amax_partials + i));
  for (int p = tid; p < n_pairs; p += kFrontThreads) s_idx[p] = __ldcg(a.idx + p);
  if (tid == 0) s_bad = 0;
  for (int e = tid; e < 256; e += kFrontThreads) s_mask[e] = 0ull;
  __syncthreads();
  for (int p = tid; p < n_pairs; p += kFrontThreads) {
    const int e = s_idx[p];
    if ((unsigned)e >= (unsigned)E) {
      s_bad = 1;
    } else {
      atomicOr(&s_mask[e], 1ull << (p / topk));
    }
  }
  __syncthreads();
  if (s_bad) {
    if (blockIdx.x == 0 && tid == 0) raise_status(a.status, kStatusNonFinite);
    return;
  }
  {
    // exclusive scans of counts and 128-row tiles over the experts (threads 0..255, one
    // expert each: warp prefix sums, then the sums of the earlier warps)
    const int e = tid;
    const int cnt = e < E ? __popcll(s_mask[e]) : 0;
    const int tiles = (cnt + kBlockM - 1) / kBlockM;
    int ic = cnt, it = tiles;
    if (tid < 256) {
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int vc = __shfl_up_sync(0xffffffffu, ic, o);
        const int vt = __shfl_up_sync(0xffffffffu, it, o);
        if ((tid & 31) >= o) { ic += vc; it += vt; }
      }
      if ((tid & 31) == 31) { s_wsum[tid >> 5][0] = ic; s_wsum[tid >> 5][1] = it; }
    }
    __syncthreads();
    if (tid < 256) {
      int bc = 0, bt = 0;
      for (int w = 0; w < (tid >> 5); ++w) { bc += s_wsum[w][0]; bt += s_wsum[w][1]; }
      const int off = bc + ic - cnt, tile0 = bt + it - tiles;
      s_off[e] = off;
      s_tile0[e] = tile0;
      if (blockIdx.x == 0 && e < E) {
        a.counts[e] = cnt;
        a.offsets[e] = off;
        a.mtile_prefix[e] = tile0;
        if (e == E - 1) {
          a.offsets[E] = off + cnt;
          a.mtile_prefix[E] = tile0 + tiles;
        }
      }
      // padding rows of this expert's segment: -1 (spread over the CTAs by expert)
      if (e < E && cnt > 0) {
        const int64_t r0 = (int64_t)tile0 * kBlockM;
        const int n_pad = tiles * kBlockM - cnt;
        for (int i = blockIdx.x; i < n_pad; i += nb) a.row_pair[r0 + cnt + i] = -1;
      }
    }
  }
  __syncthreads();
  for (int p = tid; p < n_pairs; p += kFrontThreads) {
    const int t = p / topk;
    const int e = s_idx[p];
    const int rank = __popcll(s_mask[e] & ((1ull << t) - 1ull));
    const int row = s_tile0[e] * kBlockM + rank;
    s_row[p] = row;
    if (blockIdx.x == 0) {
      const int pos = s_off[e] + rank;
      a.perm[pos] = p;
      a.inv[p] = pos;
      a.row_pair[row] = p;
    }
  }
  // without segment buffers (the FP8 variant quantises in its own kernel) the grouping ends it
  if (a.seg_codes == nullptr) return;
  // global scale of x from the per-slice maxima
  __shared__ float s_g;
  __shared__ int s_nonfinite;
  if (tid < 32) {
    uint32_t m = amax_bits;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (tid == 0) {
      s_nonfinite = m >= 0x7F80u;
      s_g = global_scale_from_amax(__uint_as_float(m << 16));
      if (blockIdx.x == 0) {
        if (s_nonfinite) raise_status(a.status, kStatusNonFinite);
        *a.g_out = s_g;
      }
    }
  }
  __syncthreads();
  if (s_nonfinite) return;
  const float g = s_g;
  const float r_t = __frcp_rn(__fmul_rn(6.0f, g));
  // one thread per (token, 16-value block): 8 code bytes + 1 scale byte to each of the
  // token's topk segment rows (and to the token-major copy when it is asked for)
  for (int u = u0; u < n_units; u += nb * kFrontThreads) {
    const int t = u / blocks_per_row, c = u - t * blocks_per_row;
    uint4 v0 = xv0, v1 = xv1;
    if (u != u0) {
      const uint4* src = reinterpret_cast<const uint4*>(a.x + (int64_t)t * H + 16 * c);
      v0 = __ldg(src);
      v1 = __ldg(src + 1);
    }
    const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
    float f[16];
    uint32_t mb = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      f[2 * j] = bf16_lo(w[j]);
      f[2 * j + 1] = bf16_hi(w[j]);
      mb = max(mb, max(w[j] & 0x7FFFu, (w[j] >> 16) & 0x7FFFu));
    }
    float r_b;
    const uint32_t s = block_scale(__uint_as_float(mb << 16), r_t, g, &r_b);
#pragma unroll
    for (int j = 0; j < 16; ++j) f[j] = __fmul_rn(f[j], r_b);
    const uint2 code = make_uint2(cvt_e2m1x8(f), cvt_e2m1x8(f + 8));
    for (int j = 0; j < topk; ++j) {
      const int64_t row = s_row[t * topk + j];
      *reinterpret_cast<uint2*>(a.seg_codes + row * (H >> 1) + 8 * c) = code;
      a.seg_sf[swz_offset(row, c, a.n_col_tiles)] = (uint8_t)s;
    }
    if (a.xq_codes != nullptr) {
      *reinterpret_cast<uint2*>(a.xq_codes + (int64_t)t * (H >> 1) + 8 * c) = code;
      a.xq_sf[swz_offset(t, c, a.n_col_tiles)] = (uint8_t)s;
    }
  }
}

namespace {
struct FrontDeviceInfo {
  int sms = 0;
  int blocks_per_sm = -1;
};
}  // namespace

// K split of the front kernel: the largest divisor of H / 32 whose grid (expert tiles x
// splits) stays within kFrontMaxGrid CTAs and whose slice eighth fits the registers
// (<= kFrontMaxKq values); 0 when there is none.
int front_ksplit(int E, int H) {
  const int n_etiles = (E + kFrontTileE - 1) / kFrontTileE;
  const int chunks = H / 32;
  int best = 0;
  for (int d = 1; d <= chunks; ++d) {
    if (chunks % d != 0) continue;
    const int kslice = H / d;
    if (kslice / kFrontKq > kFrontMaxKq || n_etiles * d > kFrontMaxGrid) continue;
    best = d;
  }
  return best;
}

size_t front_smem_bytes(int64_t T, int H, int ksplit) {
  return (size_t)T * (size_t)(H / ksplit) * sizeof(float);
}

bool front_supported(int64_t T, int E, int H) {
  if (T < 1 || T > kFrontMaxT) return false;
  const int ks = front_ksplit(E, H);
  if (ks == 0) return false;
  if (front_smem_bytes(T, H, ks) > kFrontSmemCap) return false;
  static FrontDeviceInfo info[64];
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
  std::lock_guard<std::mutex> lock(mu);
  if (info[dev].blocks_per_sm < 0) {
    int n = 0;
    if (cudaFuncSetAttribute(front_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kFrontSmemCap) !=
            cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, front_kernel, kFrontThreads, kFrontSmemCap) != cudaSuccess)
      n = 0;
    info[dev].blocks_per_sm = n;
    info[dev].sms = num_sms();
  }
  const int n_etiles = (E + kFrontTileE - 1) / kFrontTileE;
  return info[dev].blocks_per_sm >= 1 && n_etiles * ks <= info[dev].blocks_per_sm * info[dev].sms;
}

cudaError_t launch_front(FrontArgs a, cudaStream_t stream) {
  a.ksplit = front_ksplit(a.E, a.H);
  a.k_slice = a.H / a.ksplit;
  const int n_etiles = (a.E + kFrontTileE - 1) / kFrontTileE;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3((unsigned)(n_etiles * a.ksplit));
  cfg.blockDim = dim3(kFrontThreads);
  cfg.dynamicSmemBytes = front_smem_bytes(a.T, a.H, a.ksplit);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, front_kernel, a);
}

}  // namespace nvfp4moe
