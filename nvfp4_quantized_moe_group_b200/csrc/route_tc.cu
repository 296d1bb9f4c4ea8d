// Router logits for T > 64 on the tensor cores, in integer arithmetic ("Reflection releases
// Beam ...", section "Mixture-of-Experts details": every token scores all 256 experts; section
// "Residual stream and numerical decisions": the router runs in FP32, and these logits are
// more accurate than an FP32 accumulation).
//
// Each token row x_t (BF16) is scaled by a power of two to 22-bit fixed point and each expert
// row W_e (FP32) to 30-bit fixed point: with e the binary exponent of the row's largest
// magnitude (max |v| < 2^e), X = RNE(x 2^(22 - e_x)), W = RNE(w 2^(30 - e_W)).  A BF16 value
// has 8 significant bits, so X is exact for every element within 2^14 of the row's largest.
// X is split into three balanced base-256 digits, X = a0 2^16 + a1 2^8 + a2, W into four,
// W = b0 2^24 + b1 2^16 + b2 2^8 + b3 (digits in [-128, 127], |a0|, |b0| <= 64).  Then
//     X . W = sum_{i,j} (a_i . b_j) 2^(8 (5 - i - j)),
// and the 9 digit pairs with i + j <= 3 are multiplied by tcgen05 kind::i8 MMAs: int8 x int8
// products accumulated in int32, which is exact (|class sum| < 3 * 2^14 * K < 2^31 for the
// K <= 26,112 columns of one split).  One tensor-memory accumulator per class c = i + j (4 x 128
// columns: 128 experts per CTA); the epilogue combines the classes in FP64 and scales by
// 2^(e_x + e_W - 52).  Error against the exact logit, before the FP32 rounding of the sum with
// the bias:
//     sum_h |x_h - X_h 2^(e_x-22)| |W_eh| + sum_h |x_h| |W_eh - W_h 2^(e_W-30)|     (rounding)
//       <= 2^(e_x - 23) sum|W_e| + 2^(e_W - 31) sum|x_t| + H 2^(e_x + e_W - 54)
//   + H (2^23 + 2^14) 2^(e_x + e_W - 52)                                 (pairs i + j > 3)
//   + FP64 roundings of the combination and of the split-K sum (< H 2^(e_x + e_W - 50)),
// in all at most 2^(e_x - 23) sum|W_e| + 2^(e_W - 31) sum|x_t| + H 2^(e_x + e_W - 28).
// A row with a non-finite element gets the exponent kExpNonFinite and NaN logits.
#include "common.cuh"
#include "kernels.h"

namespace nvfp4moe {

namespace {
constexpr int kSliceThreads = 256;
constexpr int kSliceMaxCtas = 1024;       // amax partials of the token rows
constexpr int kTcM = 128;                 // tokens per tile
constexpr int kTcN = 128;                 // experts per tile
constexpr int kTcStages = 2;
constexpr int kXDigits = kRouterXDigits;  // 3: 22-bit token rows
constexpr int kWDigits = kRouterWDigits;  // 4: 30-bit expert rows
constexpr int kClasses = 4;               // digit-pair classes c = i + j <= 3
constexpr int kTcThreads = 192;           // producer, MMA issuer, 4 epilogue warps
constexpr uint32_t kTcTmemCols = 512;     // 4 x 128 columns
constexpr int kAPlaneBytes = kTcM * 128;  // one digit plane of the token tile, 128-byte K block
constexpr int kBPlaneBytes = kTcN * 128;

struct __align__(1024) TcSmem {
  uint8_t a[kTcStages][kXDigits][kAPlaneBytes];
  uint8_t b[kTcStages][kWDigits][kBPlaneBytes];
  uint64_t full[kTcStages];
  uint64_t empty[kTcStages];
  uint64_t acc_full;
  uint32_t tmem_base;
  int abort_flag;
};

__device__ __forceinline__ void tc_set_abort(int* flag, uint32_t* status) {
  raise_status(status, kStatusTimeout);
  *reinterpret_cast<volatile int*>(flag) = 1;
}

__device__ __forceinline__ bool tc_aborted(const int* flag) {
  return *reinterpret_cast<const volatile int*>(flag) != 0;
}

// tcgen05.mma kind::i8: s8 x s8 -> s32, K = 32 (both operands K-major).
__device__ __forceinline__ void mma_i8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Instruction descriptor of kind::i8: S32 accumulator (bits 4-5 = 2), A and B signed 8-bit
// (bits 7-9, 10-12 = 1), both K-major, N / 8 at bit 17, M / 16 at bit 24.
__host__ __device__ constexpr uint32_t idesc_i8(uint32_t m, uint32_t n) {
  return (2u << 4) | (1u << 7) | (1u << 10) | ((n >> 3) << 17) | ((m >> 4) << 24);
}

// Binary exponent e with max|v| < 2^e from the magnitude's biased exponent field (subnormal
// and zero rows take the smallest normal exponent).
__device__ __forceinline__ int row_exponent(uint32_t biased) { return (int)(biased > 1u ? biased : 1u) - 126; }

// Three balanced base-256 digits of RNE(v 2^(s1 + s2)) for a BF16 value v with
// |v 2^(s1 + s2)| < 2^22, the scaling applied as two FP32 multiplications by 2^s1 and 2^s2
// (s1, s2 of the same sign, each within the normal range): exact, since an upward scaling
// cannot overflow and a downward one only underflows values that round to 0 anyway.  Packed
// into one byte each of the three words' byte lane `lane`.
__device__ __forceinline__ void digits3(float v, float scale1, float scale2, uint32_t lane, uint32_t* d) {
  int X = __float2int_rn(__fmul_rn(__fmul_rn(v, scale1), scale2));
  const int d2 = ((X + 128) & 255) - 128;
  X = (X - d2) >> 8;
  const int d1 = ((X + 128) & 255) - 128;
  const int d0 = (X - d1) >> 8;
  d[0] |= ((uint32_t)d0 & 255u) << (8 * lane);
  d[1] |= ((uint32_t)d1 & 255u) << (8 * lane);
  d[2] |= ((uint32_t)d2 & 255u) << (8 * lane);
}

// Four balanced base-256 digits of v * 2^shift (exact power-of-two scaling in FP64, then
// round to nearest even), packed into one byte each of the four words' byte lane `lane`.
__device__ __forceinline__ void digits4(double v, double scale, uint32_t lane, uint32_t* d) {
  int X = __double2int_rn(v * scale);
  const int d3 = ((X + 128) & 255) - 128;
  X = (X - d3) >> 8;
  const int d2 = ((X + 128) & 255) - 128;
  X = (X - d2) >> 8;
  const int d1 = ((X + 128) & 255) - 128;
  const int d0 = (X - d1) >> 8;
  d[0] |= ((uint32_t)d0 & 255u) << (8 * lane);
  d[1] |= ((uint32_t)d1 & 255u) << (8 * lane);
  d[2] |= ((uint32_t)d2 & 255u) << (8 * lane);
  d[3] |= ((uint32_t)d3 & 255u) << (8 * lane);
}

__device__ __forceinline__ uint32_t block_max(uint32_t m, uint32_t* s_red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = m;
  __syncthreads();
  m = 0;
#pragma unroll
  for (int i = 0; i < kSliceThreads / 32; ++i) m = max(m, s_red[i]);
  __syncthreads();
  return m;
}
}  // namespace

// Token rows: BF16 x [T][H] -> digit planes [3][T][H], exponents [T]; CTA b also writes the
// max |x| of its rows (BF16 magnitude bits) to amax_partials[b] for the quantiser's global scale.
__global__ void __launch_bounds__(kSliceThreads) slice_x_kernel(RouterArgs a) {
  __shared__ uint32_t s_red[kSliceThreads / 32];
  const int n8 = a.H / 8;
  uint32_t cta_mag = 0;
  for (int64_t t = blockIdx.x; t < a.T; t += gridDim.x) {
    const uint4* src = reinterpret_cast<const uint4*>(a.x + t * a.H);
    uint32_t mag = 0;
    for (int v = threadIdx.x; v < n8; v += kSliceThreads) {
      const uint4 q = __ldg(src + v);
      const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) mag = max(mag, max(w[j] & 0x7FFFu, (w[j] >> 16) & 0x7FFFu));
    }
    mag = block_max(mag, s_red);
    cta_mag = max(cta_mag, mag);
    const uint32_t be = mag >> 7;
    if (be == 255u) {
      if (threadIdx.x == 0) a.x_exp[t] = kExpNonFinite;
      continue;
    }
    const int e = row_exponent(be);
    if (threadIdx.x == 0) a.x_exp[t] = e;
    // 2^(22 - e) as 2^k1 * 2^k2, e in [-125, 128]: k1, k2 in [-53, 74]
    const int k = 22 - e, k1 = k / 2, k2 = k - k1;
    const float scale1 = __uint_as_float((uint32_t)(127 + k1) << 23);
    const float scale2 = __uint_as_float((uint32_t)(127 + k2) << 23);
    for (int v = threadIdx.x; v < n8; v += kSliceThreads) {
      const uint4 q = __ldg(src + v);
      const uint32_t w[4] = {q.x, q.y, q.z, q.w};
      uint32_t lo[3] = {0, 0, 0}, hi[3] = {0, 0, 0};
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        digits3(__uint_as_float(w[j] << 16), scale1, scale2, 2 * j, lo);
        digits3(__uint_as_float(w[j] & 0xFFFF0000u), scale1, scale2, 2 * j + 1, lo);
        digits3(__uint_as_float(w[j + 2] << 16), scale1, scale2, 2 * j, hi);
        digits3(__uint_as_float(w[j + 2] & 0xFFFF0000u), scale1, scale2, 2 * j + 1, hi);
      }
#pragma unroll
      for (int p = 0; p < kXDigits; ++p)
        reinterpret_cast<uint2*>(a.x_digits + ((int64_t)p * a.T + t) * a.H)[v] = make_uint2(lo[p], hi[p]);
    }
  }
  if (threadIdx.x == 0 && a.amax_partials != nullptr) a.amax_partials[blockIdx.x] = cta_mag;
}

// Expert rows: FP32 W [E][H] -> digit planes [4][E][H], exponents [E].  One CTA per row.
__global__ void __launch_bounds__(kSliceThreads) slice_w_kernel(RouterArgs a) {
  __shared__ uint32_t s_red[kSliceThreads / 32];
  const int e_row = blockIdx.x;
  const float4* src = reinterpret_cast<const float4*>(a.w + (int64_t)e_row * a.H);
  const int n8 = a.H / 8;
  uint32_t mag = 0;
  for (int v = threadIdx.x; v < n8; v += kSliceThreads) {
    const float4 p = __ldg(src + 2 * v), q = __ldg(src + 2 * v + 1);
    const float f[8] = {p.x, p.y, p.z, p.w, q.x, q.y, q.z, q.w};
#pragma unroll
    for (int j = 0; j < 8; ++j) mag = max(mag, __float_as_uint(f[j]) & 0x7FFFFFFFu);
  }
  mag = block_max(mag, s_red);
  const uint32_t be = mag >> 23;
  if (be == 255u) {
    if (threadIdx.x == 0) a.w_exp[e_row] = kExpNonFinite;
    return;
  }
  const int e = row_exponent(be);
  if (threadIdx.x == 0) a.w_exp[e_row] = e;
  const double scale = ldexp(1.0, 30 - e);
  for (int v = threadIdx.x; v < n8; v += kSliceThreads) {
    const float4 p = __ldg(src + 2 * v), q = __ldg(src + 2 * v + 1);
    const float f[8] = {p.x, p.y, p.z, p.w, q.x, q.y, q.z, q.w};
    uint32_t lo[4] = {0, 0, 0, 0}, hi[4] = {0, 0, 0, 0};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      digits4((double)f[j], scale, j, lo);
      digits4((double)f[4 + j], scale, j, hi);
    }
#pragma unroll
    for (int p2 = 0; p2 < kWDigits; ++p2)
      reinterpret_cast<uint2*>(a.w_digits + ((int64_t)p2 * a.E + e_row) * a.H)[v] = make_uint2(lo[p2], hi[p2]);
  }
}

// One (token tile, expert tile, K split) per CTA.  Warp 0 loads the three token and four
// expert digit planes of each 128-byte K block (2 stages of 112 KB), warp 1 issues the 9
// digit-pair MMAs per K step into the four class accumulators, warps 2-5 combine the classes
// of their 32 token rows in FP64 and write the split's partial logits.
__global__ void __launch_bounds__(kTcThreads, 1)
router_i8_kernel(const __grid_constant__ CUtensorMap tma_x, const __grid_constant__ CUtensorMap tma_w,
                 const RouterArgs a) {
  extern __shared__ uint8_t smem_raw[];
  TcSmem& s = *reinterpret_cast<TcSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // expert tiles vary fastest, so the CTAs that share a token tile run together and read its
  // digit planes from L2
  const int e0 = blockIdx.x * kTcN;
  const int t0 = blockIdx.y * kTcM;
  const int kb_total = a.H / 128;
  const int kb0 = (int)((int64_t)blockIdx.z * kb_total / gridDim.z);
  const int kb1 = (int)((int64_t)(blockIdx.z + 1) * kb_total / gridDim.z);

  if (threadIdx.x == 0) {
    for (int st = 0; st < kTcStages; ++st) {
      mbar_init(&s.full[st], 1);
      mbar_init(&s.empty[st], 1);
    }
    mbar_init(&s.acc_full, 1);
    s.abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tma_x);
    prefetch_tmap(&tma_w);
  }
  if (warp == 1) {
    tmem_alloc(&s.tmem_base, kTcTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s.tmem_base;
  const uint64_t wait_ns = wait_limit(a.wait_ns);

  if (warp == 0) {
    // ------------------------------------------------------------ producer ----
    __syncwarp();
    if (elect_one()) {
      const uint64_t pol = policy_evict_last();
      uint32_t stage = 0, phase = 0, issued = 0, issued_par = 0;
      for (int kb = kb0; kb < kb1; ++kb) {
        if (tc_aborted(&s.abort_flag) || !mbar_wait(&s.empty[stage], phase ^ 1u, wait_ns)) {
          tc_set_abort(&s.abort_flag, a.status);
          break;
        }
        mbar_arrive_expect_tx(&s.full[stage], kXDigits * kAPlaneBytes + kWDigits * kBPlaneBytes);
#pragma unroll
        for (int p = 0; p < kXDigits; ++p)
          tma_load_2d(s.a[stage][p], &tma_x, &s.full[stage], kb * 128, (int)(p * a.T) + t0, pol);
#pragma unroll
        for (int p = 0; p < kWDigits; ++p)
          tma_load_2d(s.b[stage][p], &tma_w, &s.full[stage], kb * 128, p * a.E + e0, pol);
        issued |= 1u << stage;
        issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
        if (++stage == kTcStages) { stage = 0; phase ^= 1u; }
      }
      for (int st = 0; st < kTcStages; ++st)
        if ((issued >> st) & 1u)
          if (!mbar_wait(&s.full[st], (issued_par >> st) & 1u, wait_ns)) tc_set_abort(&s.abort_flag, a.status);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer ----
    __syncwarp();
    if (elect_one()) {
      constexpr uint32_t idesc = idesc_i8(kTcM, kTcN);
      uint32_t stage = 0, phase = 0;
      uint32_t started = 0;   // bit c: class c has its first product
      for (int kb = kb0; kb < kb1; ++kb) {
        if (tc_aborted(&s.abort_flag) || !mbar_wait(&s.full[stage], phase, wait_ns)) {
          tc_set_abort(&s.abort_flag, a.status);
          break;
        }
        tc_fence_after();
        for (int k = 0; k < 4; ++k) {
#pragma unroll
          for (int c = 0; c < kClasses; ++c) {
#pragma unroll
            for (int i = 0; i < kXDigits; ++i) {
              const int j = c - i;
              if (j < 0 || j >= kWDigits) continue;
              mma_i8(tmem + kTcN * c, desc_k_sw128(smem_u32(s.a[stage][i]) + 32 * k),
                     desc_k_sw128(smem_u32(s.b[stage][j]) + 32 * k), idesc, (started >> c) & 1u);
              started |= 1u << c;
            }
          }
        }
        tc_commit(&s.empty[stage]);
        if (++stage == kTcStages) { stage = 0; phase ^= 1u; }
      }
      // also marks the end of every MMA this thread issued (tensor memory may then be freed)
      tc_commit(&s.acc_full);
    }
  } else {
    // ------------------------------------------------------------ epilogue ----
    const int q = warp & 3;                       // tensor-memory lane quarter of this warp
    const int64_t t = t0 + q * 32 + lane;
    const bool got = mbar_wait(&s.acc_full, 0, wait_ns);
    if (__any_sync(0xffffffffu, !got)) {
      tc_set_abort(&s.abort_flag, a.status);
    } else if (!tc_aborted(&s.abort_flag)) {
      tc_fence_after();
      const int ex = t < a.T ? a.x_exp[t] : 0;
      double* out = a.parts + (int64_t)blockIdx.z * a.T * a.E + t * a.E;
      for (int ch = 0; ch < kTcN / 16; ++ch) {
        uint32_t C[kClasses][16];
#pragma unroll
        for (int c = 0; c < kClasses; ++c)
          tmem_ld_32x32b_x16(tmem + ((uint32_t)(q * 32) << 16) + kTcN * c + 16 * ch, C[c]);
        tmem_ld_wait();
        if (t >= a.T) continue;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int e = e0 + 16 * ch + j;
          if (e >= a.E) continue;
          const int ew = __ldg(a.w_exp + e);
          double v;
          if (ex == kExpNonFinite || ew == kExpNonFinite) {
            v = __longlong_as_double(0x7FF8000000000000ll);
          } else {
            v = (double)(int)C[3][j];
            v = __dadd_rn(v, (double)(int)C[2][j] * 256.0);
            v = __dadd_rn(v, (double)(int)C[1][j] * 65536.0);
            v = __dadd_rn(v, (double)(int)C[0][j] * 16777216.0);
            v = ldexp(v, ex + ew - 52 + 16);   // class c carries 2^(8 (5 - c)) = 2^(8 (3 - c)) 2^16
          }
          out[e] = v;
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTcTmemCols);
  }
}

static int tc_tiles(int64_t T, int E) { return (int)(((T + kTcM - 1) / kTcM) * ((E + kTcN - 1) / kTcN)); }

// K split: doubled while the grid stays within one CTA per SM and every split keeps at least
// two K blocks; also large enough that a split's class sums stay below 2^31 (at most 26,112
// columns of K per split: 3 * 2^14 * 26,112 < 2^31).
int router_tc_ksplit(int64_t T, int E, int H) {
  const int tiles = tc_tiles(T, E);
  const int kb_total = H / 128;
  int ks = 1;
  while (ks < 16 && tiles * ks * 2 <= 148 && kb_total >= ks * 2 * 2) ks *= 2;
  while ((kb_total + ks - 1) / ks * 128 > 26112) ks *= 2;
  return ks;
}

int router_tc_amax_partials(int64_t T) { return (int)(T < kSliceMaxCtas ? T : kSliceMaxCtas); }

cudaError_t launch_router_tc(RouterArgs a, cudaStream_t stream) {
  a.ksplit = router_tc_ksplit(a.T, a.E, a.H);
  a.k_slice = a.H / a.ksplit;
  CUtensorMap tma_x, tma_w;
  if (make_tma_2d(&tma_x, a.x_digits, (uint64_t)a.H, (uint64_t)kXDigits * a.T, kTcM) != 0 ||
      make_tma_2d(&tma_w, a.w_digits, (uint64_t)a.H, (uint64_t)kWDigits * a.E, kTcN) != 0)
    return cudaErrorInvalidValue;
  slice_x_kernel<<<(unsigned)router_tc_amax_partials(a.T), kSliceThreads, 0, stream>>>(a);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  slice_w_kernel<<<(unsigned)a.E, kSliceThreads, 0, stream>>>(a);
  err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  const size_t smem = sizeof(TcSmem) + 1024;
  err = cudaFuncSetAttribute(router_i8_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  const dim3 grid((unsigned)((a.E + kTcN - 1) / kTcN), (unsigned)((a.T + kTcM - 1) / kTcM), (unsigned)a.ksplit);
  router_i8_kernel<<<grid, kTcThreads, smem, stream>>>(tma_x, tma_w, a);
  err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  return launch_router_topk(a, stream);
}

static_assert(sizeof(TcSmem) + 1024 <= 232448, "router shared memory exceeds the per-block limit");

}  // namespace nvfp4moe
