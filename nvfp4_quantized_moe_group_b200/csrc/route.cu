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

constexpr int kTopkWarpTokens = 8;   // tokens per CTA of the warp-per-token top-k

// The group-limited top-k of one token per warp, for layouts whose groups are 1, 2 or 4 whole
// lanes (group size 8, 16 or 32, E <= 256): lane l holds experts 8l .. 8l + 7.
// The arithmetic and the tie rules are route_topk_block's: the logit is the FP64 sum of the
// split-K parts in split order (plus the bias) rounded to FP32, the score its sigmoid, a NaN
// score becomes -1 (raising kStatusNonFinite), a group's score is fp32(top1 + top2) of its
// scores, equal values go to the lower group / expert index, the selected experts are listed
// by score, and the weights divide routed_scale * s by the sum of the selected scores in slot
// order.  No shared memory and no block barrier: 8 tokens per 256-thread CTA.
__global__ void __launch_bounds__(256) router_topk_warp_kernel(RouterArgs a) {
  const int lane = threadIdx.x & 31;
  const int64_t t = (int64_t)blockIdx.x * kTopkWarpTokens + (threadIdx.x >> 5);
  if (t >= a.T) return;
  const int E = a.E, G = a.n_groups, gs = E / G, L = gs / 8;   // lanes per group
  const int e0 = lane * 8;
  const bool valid = e0 < E;
  float v[8];
  bool nan = false;
  {
    double acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.0;
    if (valid) {
      const int64_t step = a.T * E;
      const double2* src = reinterpret_cast<const double2*>(a.parts + t * E + e0);
      for (int ks = 0; ks < a.ksplit; ++ks) {
        const double2* q = src + (int64_t)ks * (step / 2);
        const double2 q0 = __ldcg(q), q1 = __ldcg(q + 1), q2 = __ldcg(q + 2), q3 = __ldcg(q + 3);
        acc[0] = __dadd_rn(acc[0], q0.x);
        acc[1] = __dadd_rn(acc[1], q0.y);
        acc[2] = __dadd_rn(acc[2], q1.x);
        acc[3] = __dadd_rn(acc[3], q1.y);
        acc[4] = __dadd_rn(acc[4], q2.x);
        acc[5] = __dadd_rn(acc[5], q2.y);
        acc[6] = __dadd_rn(acc[6], q3.x);
        acc[7] = __dadd_rn(acc[7], q3.y);
      }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      v[i] = -3.0f;
      if (valid) {
        double d = acc[i];
        if (a.bias != nullptr) d = __dadd_rn(d, (double)a.bias[e0 + i]);
        const float l = __double2float_rn(d);
        if (a.logits_out != nullptr) a.logits_out[t * E + e0 + i] = l;
        float sc = router_sigmoid(l);
        if (sc != sc) {
          sc = -1.0f;
          nan = true;
        }
        v[i] = sc;
      }
    }
  }
  if (__any_sync(0xffffffffu, nan) && lane == 0 && a.status != nullptr) raise_status(a.status, kStatusNonFinite);
  // the two best scores of the lane, then of its group (values only: equal values count twice)
  float t1 = v[0], t2 = -4.0f;
#pragma unroll
  for (int i = 1; i < 8; ++i) {
    if (v[i] > t1) {
      t2 = t1;
      t1 = v[i];
    } else if (v[i] > t2) {
      t2 = v[i];
    }
  }
#pragma unroll
  for (int off = 1; off < 4; off <<= 1) {
    const float o1 = __shfl_xor_sync(0xffffffffu, t1, off);
    const float o2 = __shfl_xor_sync(0xffffffffu, t2, off);
    if (off < L) {
      const float n2 = fmaxf(fminf(t1, o1), fmaxf(t2, o2));
      t1 = fmaxf(t1, o1);
      t2 = n2;
    }
  }
  const int g = e0 / gs;
  const float gscore = __fadd_rn(t1, t2);
  // rank of the lane's group among the G groups (lane h L holds group h's score)
  int grank = 0;
#pragma unroll
  for (int h = 0; h < 32; ++h) {
    const float o = __shfl_sync(0xffffffffu, gscore, (h * L) & 31);
    grank += (int)((h < G) & ((o > gscore) | ((o == gscore) & (h < g))));
  }
  const bool keep = valid && g < G && grank < a.topk_groups;
  // the topk best experts of the kept groups, one per round (max score, then lower index)
  uint32_t cand = keep ? 0xFFu : 0u;
  float sum = 0.0f, my_s = 0.0f;
  int my_e = 0;
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    if (r < a.topk) {
      float bv = -5.0f;
      int be = 0x7FFFFFFF;
#pragma unroll
      for (int i = 0; i < 8; ++i)
        if (((cand >> i) & 1u) && v[i] > bv) {
          bv = v[i];
          be = e0 + i;
        }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
        const int oe = __shfl_xor_sync(0xffffffffu, be, off);
        if (ov > bv || (ov == bv && oe < be)) {
          bv = ov;
          be = oe;
        }
      }
      if ((be >> 3) == lane) cand &= ~(1u << (be & 7));
      sum = __fadd_rn(sum, bv);
      if (lane == r) {
        my_s = bv;
        my_e = be;
      }
    }
  }
  if (lane < a.topk) {
    a.idx[t * a.topk + lane] = my_e;
    a.wts[t * a.topk + lane] = __fdiv_rn(__fmul_rn(a.routed_scale, my_s), sum);
  }
}

// The warp-per-token top-k handles layouts whose groups are 1, 2 or 4 whole lanes (the
// group's top-2 merge is an xor butterfly inside aligned lane groups).
static bool topk_warp_layout(const RouterArgs& a) {
  const int gs = a.E / a.n_groups;
  return a.E <= 256 && (gs == 8 || gs == 16 || gs == 32);
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
  if (topk_warp_layout(a)) {
    router_topk_warp_kernel<<<(unsigned)((a.T + kTopkWarpTokens - 1) / kTopkWarpTokens), 32 * kTopkWarpTokens, 0,
                              stream>>>(a);
  } else {
    router_topk_kernel<<<(unsigned)a.T, kTopkThreads, 0, stream>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace nvfp4moe
