// Grouped block-scaled NVFP4 GEMMs of the expert MLPs on the 5th-generation tensor cores.
//
// Each expert's token rows form a segment padded to 128 rows; a work item is one
// (expert, 128-column tile, 128-row tile).  One persistent CTA per SM walks work items
// (expert-major, then column tile, then row tile, so row tiles of one expert that share a
// weight tile run at the same time and the second read of that tile comes from L2).
//
// Per CTA: warp 0 fills a shared-memory ring: the A tile by a TMA load with 128-byte
// swizzle (a 32-row box when at most 32 rows of the tile hold pairs, as at decode: the
// other rows only feed accumulator rows that are never read), the B (weight) tile by one
// contiguous bulk copy from the pre-tiled, pre-swizzled weight layout, the block scales by
// bulk copies; warp 1 copies the block scales into tensor memory
// (tcgen05.cp) and issues tcgen05.mma kind::mxf4nvf4 (E2M1 x E2M1, UE4M3 scale per 16
// values) into one of two 128 x 128 FP32 accumulators in tensor memory, so the epilogue of
// one work item overlaps the main loop of the next; warps 2-9 read the accumulator
// (tcgen05.ld; warp w reads lanes 32 * (w % 4) .. +31, and the two warps of a lane quarter
// split the columns) and run the epilogue:
//   gate/up:  the tile's 64 gate and 64 up columns give h = silu(g_x g_gate acc_gate) *
//             (g_x g_up acc_up) in FP32, requantised to NVFP4 with the expert's static
//             scale g_h (the down GEMM's A operand);
//   down:     acc_out[token] += w * g_h * g_down * acc, staged through shared memory so each
//             warp issues FP32 vector reductions over contiguous 512-byte row pieces.
// Every wait is bounded; a wait that runs out sets the timeout bit of the status word and
// the CTA winds down (waits for its own copies and tensor-core work, frees tensor memory).
//
// Expert MLP: "Reflection releases Beam ...", section "Mixture-of-Experts details" (SwiGLU
// experts, weighted combine of the 8 routed experts); operand format: "NVFP4 quantization",
// section "Quantization scheme".
#include "common.cuh"
#include "kernels.h"

namespace nvfp4moe {

namespace {

constexpr int kThreads = 320;                 // producer, MMA issuer, 8 epilogue warps
constexpr int kEpiWarps = 8;
constexpr int kABytes = kBlockM * 128;        // 128 rows x 256 E2M1
constexpr int kBBytes = kBlockN * 128;        // 128 rows x 256 E2M1
constexpr int kSfBytes = 4 * 512;             // 4 K-steps x (128 rows x 4 scales), per operand
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSfCol0 = 2 * kBlockN;     // two accumulators use columns 0..255
constexpr uint32_t kSfColsPerStage = 32;      // 16 for A scales + 16 for B scales

template <int kStages, bool kStaging>
struct __align__(1024) Smem {
  uint8_t a[kStages][kABytes];
  uint8_t b[kStages][kBBytes];
  uint8_t sfa[kStages][kSfBytes];
  uint8_t sfb[kStages][kSfBytes];
  float stage_out[kStaging ? kEpiWarps : 1][32][33];  // per epilogue warp: 32 rows x 32 columns
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
  int prefix[257];
  int counts[256];
};

struct Work {
  int e;          // expert
  int mtile;      // global 128-row tile (row = mtile * 128 + r)
  int mt_local;   // tile index inside the expert's segment
  int nt;         // 128-column tile
  int rows_valid; // rows of this tile that hold a pair
};

__device__ __forceinline__ Work decode_work(const int* prefix, int w, int E, int ntn, const int* counts) {
  int lo = 0, hi = E;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (prefix[mid] * ntn <= w) lo = mid; else hi = mid;
  }
  Work k;
  k.e = lo;
  const int mt_e = prefix[lo + 1] - prefix[lo];
  const int local = w - prefix[lo] * ntn;
  k.nt = local / mt_e;
  k.mt_local = local - k.nt * mt_e;
  k.mtile = prefix[lo] + k.mt_local;
  const int left = counts[lo] - k.mt_local * kBlockM;
  k.rows_valid = left < kBlockM ? left : kBlockM;
  return k;
}

__device__ __forceinline__ void set_abort(int* flag, uint32_t* status) {
  raise_status(status, kStatusTimeout);
  *reinterpret_cast<volatile int*>(flag) = 1;
}

__device__ __forceinline__ bool aborted(const int* flag) {
  return *reinterpret_cast<const volatile int*>(flag) != 0;
}

template <bool kGateUp>
struct Cfg {
  static constexpr int kStages = kGateUp ? 6 : 5;
  static constexpr bool kStaging = !kGateUp;
  using S = Smem<kStages, kStaging>;
};

template <bool kGateUp>
__global__ void __launch_bounds__(kThreads, 1)
moe_gemm_kernel(const __grid_constant__ CUtensorMap tma_a, const __grid_constant__ CUtensorMap tma_a32,
                const GemmArgs p) {
  constexpr int kStages = Cfg<kGateUp>::kStages;
  using S = typename Cfg<kGateUp>::S;
  extern __shared__ uint8_t smem_raw[];
  S& s = *reinterpret_cast<S*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  for (int i = threadIdx.x; i <= p.E; i += kThreads) {
    s.prefix[i] = p.mtile_prefix[i];
    if (i < p.E) s.counts[i] = p.counts[i];
  }
  if (threadIdx.x == 0) {
    for (int st = 0; st < kStages; ++st) {
      mbar_init(&s.full[st], 1);
      mbar_init(&s.empty[st], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s.acc_full[b], 1);
      mbar_init(&s.acc_empty[b], kEpiWarps);
    }
    mbar_init(&s.drain, 1);
    s.abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tma_a);
    prefetch_tmap(&tma_a32);
  }
  if (warp == 1) {
    tmem_alloc(&s.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  const uint32_t tmem = s.tmem_base;
  const int ntn = p.n_total / kBlockN;
  const int total = s.prefix[p.E] * ntn;
  const int kb_count = (p.K + kBlockK - 1) / kBlockK;
  const int k64 = p.K / 64;  // scale-column tiles of A and B

  if (warp == 0) {
    // ------------------------------------------------------------ producer ----
    __syncwarp();
    if (elect_one()) {
      uint32_t stage = 0, phase = 0, issued = 0, issued_par = 0;
      const uint64_t pol_w = policy_evict_first();
      const uint64_t pol_a = policy_evict_last();
      bool ok = true;
      for (int w = blockIdx.x; ok && w < total; w += gridDim.x) {
        const Work wk = decode_work(s.prefix, w, p.E, ntn, s.counts);
        const int arow = wk.mtile * kBlockM;
        const bool a_small = wk.rows_valid <= 32;
        const uint32_t a_bytes = a_small ? 32u * 128u : (uint32_t)kABytes;
        const uint8_t* btile = p.b_tiles + ((int64_t)wk.e * ntn + wk.nt) * kb_count * (int64_t)kBBytes;
        const uint8_t* sfa = p.sfa + (int64_t)wk.mtile * k64 * 512;
        const uint8_t* sfb = p.sfb + ((int64_t)wk.e * (p.n_total / 128) + wk.nt) * k64 * 512;
        for (int kb = 0; kb < kb_count; ++kb) {
          if (aborted(&s.abort_flag) || !mbar_wait(&s.empty[stage], phase ^ 1u)) {
            set_abort(&s.abort_flag, p.status);
            ok = false;
            break;
          }
          const int left = (p.K - kb * kBlockK) / 64;
          const uint32_t sf_bytes = (uint32_t)(left < 4 ? left : 4) * 512u;
          mbar_arrive_expect_tx(&s.full[stage], a_bytes + kBBytes + 2u * sf_bytes);
          tma_load_2d(s.a[stage], a_small ? (const void*)&tma_a32 : (const void*)&tma_a, &s.full[stage],
                      kb * 128, arow, pol_a);
          bulk_load(s.b[stage], btile + (int64_t)kb * kBBytes, kBBytes, &s.full[stage], pol_w);
          bulk_load(s.sfa[stage], sfa + kb * 2048, sf_bytes, &s.full[stage], pol_a);
          bulk_load(s.sfb[stage], sfb + kb * 2048, sf_bytes, &s.full[stage], pol_w);
          issued |= 1u << stage;
          issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
      }
      // wait for every copy this thread started before the CTA can exit
      for (int st = 0; st < kStages; ++st)
        if ((issued >> st) & 1u)
          if (!mbar_wait(&s.full[st], (issued_par >> st) & 1u)) set_abort(&s.abort_flag, p.status);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer ----
    __syncwarp();
    if (elect_one()) {
      uint32_t stage = 0, phase = 0;
      const uint32_t idesc = idesc_nvf4(kBlockN);
      bool ok = true;
      int it = 0;
      for (int w = blockIdx.x; ok && w < total; w += gridDim.x, ++it) {
        const int buf = it & 1;
        const uint32_t acc_par = ((uint32_t)it >> 1) & 1u;
        if (aborted(&s.abort_flag) || !mbar_wait(&s.acc_empty[buf], acc_par ^ 1u)) {
          set_abort(&s.abort_flag, p.status);
          break;
        }
        tc_fence_after();
        const uint32_t acc = tmem + (uint32_t)(buf * kBlockN);
        for (int kb = 0; kb < kb_count; ++kb) {
          if (aborted(&s.abort_flag) || !mbar_wait(&s.full[stage], phase)) {
            set_abort(&s.abort_flag, p.status);
            ok = false;
            break;
          }
          tc_fence_after();
          const int left = (p.K - kb * kBlockK) / 64;
          const int ksteps = left < 4 ? left : 4;
          const uint32_t sfa_t = tmem + kSfCol0 + stage * kSfColsPerStage;
          const uint32_t sfb_t = sfa_t + 16;
          const uint32_t sa = smem_u32(s.sfa[stage]);
          const uint32_t sb = smem_u32(s.sfb[stage]);
          for (int k = 0; k < ksteps; ++k) {
            tc_cp_32x128b_x4(sfa_t + 4 * k, desc_sf_block(sa + 512 * k));
            tc_cp_32x128b_x4(sfb_t + 4 * k, desc_sf_block(sb + 512 * k));
          }
          const uint32_t a0 = smem_u32(s.a[stage]);
          const uint32_t b0 = smem_u32(s.b[stage]);
          for (int k = 0; k < ksteps; ++k) {
            mma_nvf4(acc, desc_k_sw128(a0 + 32 * k), desc_k_sw128(b0 + 32 * k), idesc, sfa_t + 4 * k,
                     sfb_t + 4 * k, (kb | k) != 0 ? 1u : 0u);
          }
          tc_commit(&s.empty[stage]);
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        tc_commit(&s.acc_full[buf]);
      }
      // every tensor-core operation of this thread is done before the memory is freed
      tc_commit(&s.drain);
      if (!mbar_wait(&s.drain, 0)) set_abort(&s.abort_flag, p.status);
    }
  } else {
    // ------------------------------------------------------------ epilogue ----
    const int q = warp & 3;              // tensor-memory lane quarter this warp may read
    const int half = (warp - 2) >> 2;    // which half of the tile's columns it handles
    const int row_l = q * 32 + lane;
    int it = 0;
    for (int w = blockIdx.x; w < total; w += gridDim.x, ++it) {
      const Work wk = decode_work(s.prefix, w, p.E, ntn, s.counts);
      const int buf = it & 1;
      const uint32_t acc_par = ((uint32_t)it >> 1) & 1u;
      const int64_t row = (int64_t)wk.mtile * kBlockM + row_l;
      const bool valid = row_l < wk.rows_valid;
      // rows of this warp that hold a pair (rows are filled from the top of the tile)
      const bool warp_live = q * 32 < wk.rows_valid;
      // per-expert / per-row constants, loaded before the accumulator is ready
      float c0s = 0.f, c1s = 0.f, c2s = 0.f;
      int token = -1;
      if (warp_live) {
        if constexpr (kGateUp) {
          const float gx = *p.g_x;
          c0s = __fmul_rn(gx, p.g_gate[wk.e]);
          c1s = __fmul_rn(gx, p.g_up[wk.e]);
          c2s = p.g_h[wk.e];
        } else {
          const int pair = valid ? p.row_pair[row] : -1;
          if (pair >= 0) {
            c0s = __fmul_rn(p.alpha_down[wk.e], p.wts[pair]);
            token = pair / p.topk;
          }
        }
      }
      const bool got = !aborted(&s.abort_flag) && mbar_wait(&s.acc_full[buf], acc_par);
      if (__any_sync(0xffffffffu, !got)) {
        set_abort(&s.abort_flag, p.status);
        break;
      }
      __syncwarp();
      tc_fence_after();
      const uint32_t t_row = tmem + (uint32_t)(buf * kBlockN) + ((uint32_t)(q * 32) << 16);
      if constexpr (kGateUp) {
        if (warp_live) {
          // this warp: features [half * 32, half * 32 + 32) of the tile's 64
          const float sg = c0s, su = c1s, gh = c2s;
          const float r_t = __frcp_rn(__fmul_rn(6.0f, gh));
          const int64_t n_ct = p.I / 64;
          const int c0 = half * 32;
          uint32_t G[32], U[32];
          tmem_ld_32x32b_x32(t_row + c0, G);
          tmem_ld_32x32b_x32(t_row + kBlockN / 2 + c0, U);
          tmem_ld_wait();
          float h[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float g = __fmul_rn(__uint_as_float(G[i]), sg);
            const float u = __fmul_rn(__uint_as_float(U[i]), su);
            // silu(g) * u = g * u / (1 + exp(-g)), FP32 with an approximate reciprocal
            h[i] = __fmul_rn(__fmul_rn(g, u), rcp_approx(__fadd_rn(1.0f, __expf(-g))));
          }
          uint32_t codes[4];
          uint32_t sfp = 0;
#pragma unroll
          for (int b = 0; b < 2; ++b) {
            float amax = 0.0f;
#pragma unroll
            for (int j = 0; j < 16; ++j) amax = fmaxf(amax, fabsf(h[16 * b + j]));
            float r_b;
            sfp |= block_scale(amax, r_t, gh, &r_b) << (8 * b);
            float v[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) v[j] = __fmul_rn(h[16 * b + j], r_b);
            codes[2 * b] = cvt_e2m1x8(v);
            codes[2 * b + 1] = cvt_e2m1x8(v + 8);
          }
          if (valid) {
            const int f0 = wk.nt * (kBlockN / 2) + c0;
            *reinterpret_cast<uint4*>(p.hq_codes + row * (p.I / 2) + f0 / 2) =
                make_uint4(codes[0], codes[1], codes[2], codes[3]);
            *reinterpret_cast<uint16_t*>(p.hq_sf + swz_offset(row, f0 / 16, n_ct)) = (uint16_t)sfp;
          }
        }
      } else {
        if (warp_live) {
          const float scale = c0s;
          float (*st)[33] = s.stage_out[warp - 2];
          const int sub = lane >> 3;        // which of the 4 rows this lane writes per pass
          const int col = (lane & 7) * 4;   // its 4 columns inside the 32-column chunk
#pragma unroll 1
          for (int c0 = half * (kBlockN / 2); c0 < (half + 1) * (kBlockN / 2); c0 += 32) {
            uint32_t Y[32];
            tmem_ld_32x32b_x32(t_row + c0, Y);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 32; ++j) st[lane][j] = __fmul_rn(__uint_as_float(Y[j]), scale);
            __syncwarp();
#pragma unroll
            for (int pass = 0; pass < 8; ++pass) {
              const int r = pass * 4 + sub;
              const int tok = __shfl_sync(0xffffffffu, token, r);
              if (tok >= 0) {
                float* dst = p.acc + (int64_t)tok * p.H + wk.nt * kBlockN + c0 + col;
                red_add_v4(dst, st[r][col], st[r][col + 1], st[r][col + 2], st[r][col + 3]);
              }
            }
            __syncwarp();
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s.acc_empty[buf]);
    }
  }

  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <bool kGateUp>
cudaError_t launch_gemm(const CUtensorMap& tma_a, const CUtensorMap& tma_a32, const GemmArgs& a, int grid,
                        cudaStream_t stream) {
  const size_t smem = sizeof(typename Cfg<kGateUp>::S) + 1024;
  cudaError_t err = cudaFuncSetAttribute(moe_gemm_kernel<kGateUp>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  moe_gemm_kernel<kGateUp><<<grid, kThreads, smem, stream>>>(tma_a, tma_a32, a);
  return cudaGetLastError();
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                   CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                   CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

}  // namespace

static_assert(sizeof(Cfg<true>::S) + 1024 <= 232448, "gate/up GEMM shared memory exceeds the per-block limit");
static_assert(sizeof(Cfg<false>::S) + 1024 <= 232448, "down GEMM shared memory exceeds the per-block limit");
static_assert(kSfCol0 + 6 * kSfColsPerStage <= kTmemCols, "tensor memory columns");

cudaError_t launch_gemm_gateup(const CUtensorMap& tma_a, const CUtensorMap& tma_a32, const GemmArgs& a,
                               int grid, cudaStream_t stream) {
  return launch_gemm<true>(tma_a, tma_a32, a, grid, stream);
}

cudaError_t launch_gemm_down(const CUtensorMap& tma_a, const CUtensorMap& tma_a32, const GemmArgs& a,
                             int grid, cudaStream_t stream) {
  return launch_gemm<false>(tma_a, tma_a32, a, grid, stream);
}

int make_tma_2d(CUtensorMap* map, const void* base, uint64_t row_bytes, uint64_t rows, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return -1;
  const cuuint64_t dims[2] = {row_bytes, rows};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {128, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box,
                        estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? 0 : (int)r;
}

int num_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 148;
  return n;
}

}  // namespace nvfp4moe
