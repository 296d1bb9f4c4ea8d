// Group-limited sigmoid router ("Reflection releases Beam ...", section "Mixture-of-Experts
// details"): FP32 logits x.W_r^T, sigmoid scores, group score = sum of the two best scores of
// each group, keep the best topk_groups groups, pick the topk best experts inside them,
// weights = routed_scale * s / sum(selected s).  FP32 throughout (section "Residual stream and
// numerical decisions").
//
// This file holds the FP32 logits kernels (CUDA cores) and the top-k kernel.  The FP32
// kernels serve T <= 64 when the fused front end cannot run, and every T in the
// allocation-free router; with workspace for the digit planes, T > 64 takes the integer
// tensor-core logits of route_tc.cu.
#include "common.cuh"
#include "kernels.h"
#include "route_topk.cuh"

namespace nvfp4moe {

namespace {
constexpr int kTM = 64;   // tokens per CTA tile (small-T kernel)
constexpr int kTN = 64;   // experts per CTA tile
constexpr int kTK = 32;   // K chunk; each chunk is summed into a fresh partial
constexpr int kBigTM = 128;        // tokens per CTA tile (large-T FP32 kernel)
constexpr int kBigMinT = 65;       // the large-T FP32 kernel runs from this many tokens on
}  // namespace

// Split-K logits: parts[ks][t][e] = sum over this CTA's K slice of x[t][k] * W[e][k].
// Each 32-product chunk is an FP32 FMA chain into a fresh register; the chunk sums are
// added in FP64 (and so are the split-K parts and the bias), and the logit is rounded to
// FP32 once.  The error is then at most 32 * 2^-24 * sum|x W| + 2^-24 |logit| (plus FP64
// terms), independent of H.
__global__ void __launch_bounds__(256) router_logits_kernel(RouterArgs a) {
  __shared__ __align__(16) float xs[kTK][kTM + 4];
  __shared__ __align__(16) float ws[kTK][kTN + 4];
  const int tid = threadIdx.x;
  const int tx = tid & 15;  // expert quad
  const int ty = tid >> 4;  // token quad
  const int64_t t0 = (int64_t)blockIdx.x * kTM;
  const int e0 = blockIdx.y * kTN;
  const int64_t k_begin = (int64_t)blockIdx.z * a.k_slice;
  const int64_t k_end = k_begin + a.k_slice;

  double acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.0;

  // global -> shared mapping: x tile 64 rows x 32 bf16 (4 threads per row, 8 bf16 each);
  // W tile 64 rows x 32 fp32 (4 threads per row, 8 floats each).
  const int lr = tid >> 2;
  const int lc = (tid & 3) * 8;
  uint32_t mag = 0;  // max BF16 magnitude bits of the x elements this thread loads
  for (int64_t k0 = k_begin; k0 < k_end; k0 += kTK) {
    {
      const int64_t t = t0 + lr;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (t < a.T) v = __ldg(reinterpret_cast<const uint4*>(a.x + t * a.H + k0 + lc));
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        xs[lc + 2 * j][lr] = __uint_as_float(w[j] << 16);
        xs[lc + 2 * j + 1][lr] = __uint_as_float(w[j] & 0xFFFF0000u);
        mag = max(mag, max(w[j] & 0x7FFFu, (w[j] >> 16) & 0x7FFFu));
      }
      const int e = e0 + lr;
      float4 p = make_float4(0.f, 0.f, 0.f, 0.f), q = p;
      if (e < a.E) {
        const float4* src = reinterpret_cast<const float4*>(a.w + (int64_t)e * a.H + k0 + lc);
        p = __ldg(src);
        q = __ldg(src + 1);
      }
      ws[lc + 0][lr] = p.x; ws[lc + 1][lr] = p.y; ws[lc + 2][lr] = p.z; ws[lc + 3][lr] = p.w;
      ws[lc + 4][lr] = q.x; ws[lc + 5][lr] = q.y; ws[lc + 6][lr] = q.z; ws[lc + 7][lr] = q.w;
    }
    __syncthreads();
    float part[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) part[i][j] = 0.f;
#pragma unroll 8
    for (int k = 0; k < kTK; ++k) {
      const float4 xv = *reinterpret_cast<const float4*>(&xs[k][ty * 4]);
      const float4 wv = *reinterpret_cast<const float4*>(&ws[k][tx * 4]);
      const float xa[4] = {xv.x, xv.y, xv.z, xv.w};
      const float wa[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) part[i][j] = __fmaf_rn(xa[i], wa[j], part[i][j]);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] = __dadd_rn(acc[i][j], (double)part[i][j]);
    __syncthreads();
  }
  // the CTAs of the first expert tile together load every x element exactly once: they
  // also produce the per-block maxima of |x| for the global activation scale
  if (a.amax_partials != nullptr && blockIdx.y == 0) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mag = max(mag, __shfl_xor_sync(0xffffffffu, mag, o));
    __shared__ uint32_t red[8];
    if ((tid & 31) == 0) red[tid >> 5] = mag;
    __syncthreads();
    if (tid < 32) {
      mag = tid < 8 ? red[tid] : 0u;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mag = max(mag, __shfl_xor_sync(0xffffffffu, mag, o));
      if (tid == 0) a.amax_partials[blockIdx.z * gridDim.x + blockIdx.x] = mag;
    }
  }
  double* out = a.parts + (int64_t)blockIdx.z * a.T * a.E;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t t = t0 + ty * 4 + i;
    if (t >= a.T) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int e = e0 + tx * 4 + j;
      if (e < a.E) out[t * a.E + e] = acc[i][j];
    }
  }
}

// Large-T logits: 128 tokens x 64 experts per CTA, 256 threads, 8 x 4 outputs per thread,
// K in chunks of 32 through double-buffered shared memory (the next chunk's loads are in
// flight while the current one is multiplied).  Same arithmetic as router_logits_kernel: each
// 32-product chunk is an FP32 FMA chain into a fresh register, chunk sums and split-K parts
// are added in FP64.
__global__ void __launch_bounds__(256) router_logits_big_kernel(RouterArgs a) {
  __shared__ __align__(16) float xs[2][kTK][kBigTM];
  __shared__ __align__(16) float ws[2][kTK][kTN];
  const int tid = threadIdx.x;
  const int tx = tid & 15;   // expert quad: experts 4tx..4tx+3
  const int ty = tid >> 4;   // token octet: tokens 8ty..8ty+7
  const int64_t t0 = (int64_t)blockIdx.x * kBigTM;
  const int e0 = blockIdx.y * kTN;
  const int64_t k_begin = (int64_t)blockIdx.z * a.k_slice;
  const int n_chunks = a.k_slice / kTK;

  // loaders: x tile 128 rows x 32 bf16 = 2 threads per row (16 bf16 each);
  //          W tile 64 rows x 32 fp32 = 4 threads per row (8 floats each)
  const int xr = tid >> 1, xc = (tid & 1) * 16;
  const int wr = tid >> 2, wc = (tid & 3) * 8;
  uint4 xv0, xv1;
  float4 wv0, wv1;
  uint32_t mag = 0;
  auto load = [&](int chunk) {
    const int64_t k0 = k_begin + (int64_t)chunk * kTK;
    const int64_t t = t0 + xr;
    xv0 = xv1 = make_uint4(0, 0, 0, 0);
    if (t < a.T) {
      const uint4* src = reinterpret_cast<const uint4*>(a.x + t * a.H + k0 + xc);
      xv0 = __ldg(src);
      xv1 = __ldg(src + 1);
    }
    const int e = e0 + wr;
    wv0 = wv1 = make_float4(0.f, 0.f, 0.f, 0.f);
    if (e < a.E) {
      const float4* src = reinterpret_cast<const float4*>(a.w + (int64_t)e * a.H + k0 + wc);
      wv0 = __ldg(src);
      wv1 = __ldg(src + 1);
    }
  };
  auto store = [&](int buf) {
    const uint32_t w[8] = {xv0.x, xv0.y, xv0.z, xv0.w, xv1.x, xv1.y, xv1.z, xv1.w};
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      xs[buf][xc + 2 * j][xr] = __uint_as_float(w[j] << 16);
      xs[buf][xc + 2 * j + 1][xr] = __uint_as_float(w[j] & 0xFFFF0000u);
      mag = max(mag, max(w[j] & 0x7FFFu, (w[j] >> 16) & 0x7FFFu));
    }
    const float wf[8] = {wv0.x, wv0.y, wv0.z, wv0.w, wv1.x, wv1.y, wv1.z, wv1.w};
#pragma unroll
    for (int j = 0; j < 8; ++j) ws[buf][wc + j][wr] = wf[j];
  };

  double acc[8][4];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.0;

  load(0);
  store(0);
  __syncthreads();
  for (int c = 0; c < n_chunks; ++c) {
    const int buf = c & 1;
    if (c + 1 < n_chunks) load(c + 1);
    float part[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) part[i][j] = 0.f;
#pragma unroll 8
    for (int k = 0; k < kTK; ++k) {
      const float4 xa = *reinterpret_cast<const float4*>(&xs[buf][k][ty * 8]);
      const float4 xb = *reinterpret_cast<const float4*>(&xs[buf][k][ty * 8 + 4]);
      const float4 wv = *reinterpret_cast<const float4*>(&ws[buf][k][tx * 4]);
      const float xv[8] = {xa.x, xa.y, xa.z, xa.w, xb.x, xb.y, xb.z, xb.w};
      const float wa[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) part[i][j] = __fmaf_rn(xv[i], wa[j], part[i][j]);
    }
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] = __dadd_rn(acc[i][j], (double)part[i][j]);
    if (c + 1 < n_chunks) store(buf ^ 1);
    __syncthreads();
  }
  if (a.amax_partials != nullptr && blockIdx.y == 0) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mag = max(mag, __shfl_xor_sync(0xffffffffu, mag, o));
    uint32_t* red = reinterpret_cast<uint32_t*>(&xs[0][0][0]);  // tiles are no longer read
    if ((tid & 31) == 0) red[tid >> 5] = mag;
    __syncthreads();
    if (tid < 32) {
      mag = tid < 8 ? red[tid] : 0u;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mag = max(mag, __shfl_xor_sync(0xffffffffu, mag, o));
      if (tid == 0) a.amax_partials[blockIdx.z * gridDim.x + blockIdx.x] = mag;
    }
  }
  double* out = a.parts + (int64_t)blockIdx.z * a.T * a.E;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int64_t t = t0 + ty * 8 + i;
    if (t >= a.T) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int e = e0 + tx * 4 + j;
      if (e < a.E) out[t * a.E + e] = acc[i][j];
    }
  }
}

// One token per block.  Phase 1: thread e sums expert e's split-K parts in FP64 (the
// loads of consecutive experts are coalesced and independent across parts), adds the bias,
// rounds the logit to FP32 once and takes the sigmoid.  Phase 2: the block does the
// group-limited top-k.  Equal scores go to the lower index (groups and experts).
__global__ void __launch_bounds__(kTopkThreads) router_topk_kernel(RouterArgs a) {
  __shared__ float s_sc[256];
  const int E = a.E;
  const int64_t t = blockIdx.x;
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    const double* src = a.parts + t * E + e;
    const int64_t step = a.T * E;
    double acc = 0.0;
    int ks = 0;
    for (; ks + 8 <= a.ksplit; ks += 8) {
      double v[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) v[j] = src[(int64_t)(ks + j) * step];
#pragma unroll
      for (int j = 0; j < 8; ++j) acc = __dadd_rn(acc, v[j]);
    }
    for (; ks < a.ksplit; ++ks) acc = __dadd_rn(acc, src[(int64_t)ks * step]);
    if (a.bias != nullptr) acc = __dadd_rn(acc, (double)a.bias[e]);
    const float l = __double2float_rn(acc);
    if (a.logits_out != nullptr) a.logits_out[t * E + e] = l;
    s_sc[e] = router_sigmoid(l);
  }
  __syncthreads();
  route_topk_block(s_sc, E, a.n_groups, a.topk_groups, a.topk, a.routed_scale, a.idx + t * a.topk,
                   a.wts + t * a.topk, a.status);
}

static int tile_tokens(int64_t T) { return T >= kBigMinT ? kBigTM : kTM; }

// K split: doubled while the grid stays within about two CTAs per SM; the cap is chosen so
// that, whenever the K dimension is split, splits * tile tokens * 64 <= 296 * 64 * 64, which
// bounds the split-K partials by max(T * E, 296 * 64 * 64) for either kernel.
int router_ksplit(int64_t T, int E, int H) {
  const int tm = tile_tokens(T);
  const int64_t tiles = ((T + tm - 1) / tm) * ((E + kTN - 1) / kTN);
  const int64_t cap = 296 * kTM / tm;
  int ks = 1;
  while (ks < 32 && tiles * ks * 2 <= cap && (H / kTK) % (ks * 2) == 0) ks *= 2;
  return ks;
}

size_t router_parts_elems(int64_t T_max, int E, int H) {
  size_t best = 0;
  // ksplit depends on T only through the number of token tiles (64 or 128 tokens); the
  // tensor-core path splits 128-token tiles
  for (int64_t c = 1; c <= (T_max + kTM - 1) / kTM; ++c) {
    const int64_t T = c * kTM < T_max ? c * kTM : T_max;
    size_t n = (size_t)router_ksplit(T, E, H) * (size_t)T * (size_t)E;
    if (T >= kRouterTcMinT) {
      const size_t n_tc = (size_t)router_tc_ksplit(T, E, H) * (size_t)T * (size_t)E;
      if (n_tc > n) n = n_tc;
    }
    if (n > best) best = n;
  }
  return best;
}

size_t router_fp32_parts_elems(int64_t T_max, int E, int H) {
  size_t best = 0;
  for (int64_t c = 1; c <= (T_max + kTM - 1) / kTM; ++c) {
    const int64_t T = c * kTM < T_max ? c * kTM : T_max;
    const size_t n = (size_t)router_ksplit(T, E, H) * (size_t)T * (size_t)E;
    if (n > best) best = n;
  }
  return best;
}

int router_amax_partials(int64_t T, int E, int H) {
  if (T >= kRouterTcMinT) return router_tc_amax_partials(T);
  const int tm = tile_tokens(T);
  return (int)((T + tm - 1) / tm) * router_ksplit(T, E, H);
}

int router_launch_count(const RouterArgs& a) {
  return (a.T >= kRouterTcMinT && a.x_digits != nullptr) ? 4 : 2;
}

cudaError_t launch_router(RouterArgs a, cudaStream_t stream) {
  if (a.T >= kRouterTcMinT && a.x_digits != nullptr) return launch_router_tc(a, stream);
  a.ksplit = router_ksplit(a.T, a.E, a.H);
  a.k_slice = a.H / a.ksplit;
  const int tm = tile_tokens(a.T);
  dim3 grid((unsigned)((a.T + tm - 1) / tm), (unsigned)((a.E + kTN - 1) / kTN), (unsigned)a.ksplit);
  if (tm == kBigTM)
    router_logits_big_kernel<<<grid, 256, 0, stream>>>(a);
  else
    router_logits_kernel<<<grid, 256, 0, stream>>>(a);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  return launch_router_topk(a, stream);
}

cudaError_t launch_router_topk(const RouterArgs& a, cudaStream_t stream) {
  router_topk_kernel<<<(unsigned)a.T, kTopkThreads, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace nvfp4moe
