// Grouped block-scaled NVFP4 GEMMs of the expert MLPs on the 5th-generation tensor cores.
//
// Each expert's token rows form a segment padded to 128 rows; a work item is one
// (expert, 128-row tile, 256-column tile).  One persistent CTA per SM walks work items
// (expert-major, then column tile, then row tile, so row tiles of one expert that share a
// weight tile run at the same time and the second read of that tile comes from L2).
//
// Per CTA: warp 0 issues TMA loads (A and B tiles with 128-byte swizzle, block scales by
// bulk copy) into a 4-stage shared-memory ring; warp 1 copies the block scales into tensor
// memory (tcgen05.cp) and issues tcgen05.mma kind::mxf4nvf4 (E2M1 x E2M1, UE4M3 scale per
// 16 values, FP32 accumulator of 128 x 256 in tensor memory); warps 2-5 read the
// accumulator (tcgen05.ld) and run the epilogue:
//   gate/up:  h = silu(g_x g_gate acc_gate) * (g_x g_up acc_up) in FP32, then NVFP4
//             requantisation of h with the expert's static scale g_h (the down GEMM's A).
//   down:     acc_out[token] += w * g_h * g_down * acc, FP32 vector reductions.
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

constexpr int kStages = 4;
constexpr int kThreads = 192;
constexpr int kABytes = kBlockM * 128;        // 128 rows x 256 E2M1
constexpr int kBBytes = kBlockN * 128;        // 256 rows x 256 E2M1
constexpr int kSfaBytes = 4 * 512;            // 4 K-steps x (128 rows x 4 scales)
constexpr int kSfbBytes = 2 * 4 * 512;        // 2 row blocks x 4 K-steps
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSfCol0 = 256;             // accumulator uses columns 0..255
constexpr uint32_t kSfColsPerStage = 48;      // 16 for A scales + 32 for B scales

struct __align__(1024) Smem {
  uint8_t a[kStages][kABytes];
  uint8_t b[kStages][kBBytes];
  uint8_t sfa[kStages][kSfaBytes];
  uint8_t sfb[kStages][kSfbBytes];
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t acc_full;
  uint64_t acc_empty;
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
  int prefix[257];
};

struct Work {
  int e;          // expert
  int mtile;      // global 128-row tile (row = mtile * 128 + r)
  int mt_local;   // tile index inside the expert's segment
  int nt;         // 256-column tile
  int rows_valid; // rows of this tile that hold a pair
};

__device__ __forceinline__ Work decode_work(const Smem& s, int w, int E, int ntn,
                                            const int32_t* __restrict__ counts) {
  int lo = 0, hi = E;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (s.prefix[mid] * ntn <= w) lo = mid; else hi = mid;
  }
  Work k;
  k.e = lo;
  const int mt_e = s.prefix[lo + 1] - s.prefix[lo];
  const int local = w - s.prefix[lo] * ntn;
  k.nt = local / mt_e;
  k.mt_local = local - k.nt * mt_e;
  k.mtile = s.prefix[lo] + k.mt_local;
  const int left = counts[lo] - k.mt_local * kBlockM;
  k.rows_valid = left < kBlockM ? left : kBlockM;
  return k;
}

__device__ __forceinline__ void set_abort(Smem& s, uint32_t* status) {
  raise_status(status, kStatusTimeout);
  *reinterpret_cast<volatile int*>(&s.abort_flag) = 1;
}

__device__ __forceinline__ bool aborted(const Smem& s) {
  return *reinterpret_cast<const volatile int*>(&s.abort_flag) != 0;
}

template <bool kGateUp>
__global__ void __launch_bounds__(kThreads, 1)
moe_gemm_kernel(const __grid_constant__ CUtensorMap tma_a, const __grid_constant__ CUtensorMap tma_b,
                const GemmArgs p) {
  extern __shared__ uint8_t smem_raw[];
  Smem& s = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                     ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  for (int i = threadIdx.x; i <= p.E; i += kThreads) s.prefix[i] = p.mtile_prefix[i];
  if (threadIdx.x == 0) {
    for (int st = 0; st < kStages; ++st) {
      mbar_init(&s.full[st], 1);
      mbar_init(&s.empty[st], 1);
    }
    mbar_init(&s.acc_full, 1);
    mbar_init(&s.acc_empty, 4);
    mbar_init(&s.drain, 1);
    s.abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tma_a);
    prefetch_tmap(&tma_b);
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
        const Work wk = decode_work(s, w, p.E, ntn, p.counts);
        const int arow = wk.mtile * kBlockM;
        const int brow = wk.e * p.n_total + wk.nt * kBlockN;
        const uint8_t* sfa = p.sfa + (int64_t)wk.mtile * k64 * 512;
        const uint8_t* sfb0 = p.sfb + ((int64_t)wk.e * (p.n_total / 128) + wk.nt * 2) * k64 * 512;
        for (int kb = 0; kb < kb_count; ++kb) {
          if (aborted(s) || !mbar_wait(&s.empty[stage], phase ^ 1u)) {
            set_abort(s, p.status);
            ok = false;
            break;
          }
          const int left = (p.K - kb * kBlockK) / 64;
          const uint32_t sf_bytes = (uint32_t)(left < 4 ? left : 4) * 512u;
          mbar_arrive_expect_tx(&s.full[stage], kABytes + kBBytes + 3u * sf_bytes);
          tma_load_2d(s.a[stage], &tma_a, &s.full[stage], kb * 128, arow, pol_a);
          tma_load_2d(s.b[stage], &tma_b, &s.full[stage], kb * 128, brow, pol_w);
          bulk_load(s.sfa[stage], sfa + kb * 2048, sf_bytes, &s.full[stage], pol_a);
          bulk_load(s.sfb[stage], sfb0 + kb * 2048, sf_bytes, &s.full[stage], pol_w);
          bulk_load(s.sfb[stage] + 2048, sfb0 + (int64_t)k64 * 512 + kb * 2048, sf_bytes,
                    &s.full[stage], pol_w);
          issued |= 1u << stage;
          issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
      }
      // wait for every copy this thread started before the CTA can exit
      for (int st = 0; st < kStages; ++st)
        if ((issued >> st) & 1u)
          if (!mbar_wait(&s.full[st], (issued_par >> st) & 1u)) set_abort(s, p.status);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer ----
    __syncwarp();
    if (elect_one()) {
      uint32_t stage = 0, phase = 0, acc_phase = 0;
      const uint32_t idesc = idesc_nvf4(kBlockN);
      bool ok = true;
      for (int w = blockIdx.x; ok && w < total; w += gridDim.x) {
        if (aborted(s) || !mbar_wait(&s.acc_empty, acc_phase ^ 1u)) {
          set_abort(s, p.status);
          break;
        }
        tc_fence_after();
        for (int kb = 0; kb < kb_count; ++kb) {
          if (aborted(s) || !mbar_wait(&s.full[stage], phase)) {
            set_abort(s, p.status);
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
            tc_cp_32x128b_x4(sfb_t + 8 * k, desc_sf_block(sb + 512 * k));
            tc_cp_32x128b_x4(sfb_t + 8 * k + 4, desc_sf_block(sb + 2048 + 512 * k));
          }
          const uint32_t a0 = smem_u32(s.a[stage]);
          const uint32_t b0 = smem_u32(s.b[stage]);
          for (int k = 0; k < ksteps; ++k) {
            mma_nvf4(tmem, desc_k_sw128(a0 + 32 * k), desc_k_sw128(b0 + 32 * k), idesc,
                     sfa_t + 4 * k, sfb_t + 8 * k, (kb | k) != 0 ? 1u : 0u);
          }
          tc_commit(&s.empty[stage]);
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        tc_commit(&s.acc_full);
        acc_phase ^= 1u;
      }
      // every tensor-core operation of this thread is done before the memory is freed
      tc_commit(&s.drain);
      if (!mbar_wait(&s.drain, 0)) set_abort(s, p.status);
    }
  } else {
    // ------------------------------------------------------------ epilogue ----
    const int q = warp & 3;  // tensor-memory lane quadrant this warp may read
    const int row_l = q * 32 + lane;
    const uint32_t t_row = tmem + ((uint32_t)(q * 32) << 16);
    uint32_t acc_phase = 0;
    for (int w = blockIdx.x; w < total; w += gridDim.x) {
      const Work wk = decode_work(s, w, p.E, ntn, p.counts);
      const bool got = !aborted(s) && mbar_wait(&s.acc_full, acc_phase);
      if (__any_sync(0xffffffffu, !got)) {
        set_abort(s, p.status);
        break;
      }
      __syncwarp();
      tc_fence_after();
      const int64_t row = (int64_t)wk.mtile * kBlockM + row_l;
      const bool valid = row_l < wk.rows_valid;
      if constexpr (kGateUp) {
        const float gx = *p.g_x;
        const float sg = __fmul_rn(gx, p.g_gate[wk.e]);
        const float su = __fmul_rn(gx, p.g_up[wk.e]);
        const float gh = p.g_h[wk.e];
        const float r_t = __frcp_rn(__fmul_rn(6.0f, gh));
        const int64_t n_ct = p.I / 64;
#pragma unroll 1
        for (int c0 = 0; c0 < 128; c0 += 32) {
          uint32_t G[32], U[32];
          tmem_ld_32x32b_x32(t_row + c0, G);
          tmem_ld_32x32b_x32(t_row + 128 + c0, U);
          tmem_ld_wait();
          float h[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float g = __fmul_rn(__uint_as_float(G[i]), sg);
            const float u = __fmul_rn(__uint_as_float(U[i]), su);
            h[i] = __fmul_rn(__fdiv_rn(g, __fadd_rn(1.0f, expf(-g))), u);
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
        const float alpha = p.alpha_down[wk.e];
        const int pair = valid ? p.row_pair[row] : -1;
        float wgt = 0.0f;
        int64_t token = 0;
        if (pair >= 0) {
          wgt = p.wts[pair];
          token = pair / p.topk;
        }
        float* dst = p.acc + token * p.H + wk.nt * kBlockN;
#pragma unroll 1
        for (int c0 = 0; c0 < kBlockN; c0 += 32) {
          uint32_t Y[32];
          tmem_ld_32x32b_x32(t_row + c0, Y);
          tmem_ld_wait();
          if (pair >= 0) {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              float v[4];
#pragma unroll
              for (int j = 0; j < 4; ++j)
                v[j] = __fmul_rn(__fmul_rn(__uint_as_float(Y[4 * i + j]), alpha), wgt);
              red_add_v4(dst + c0 + 4 * i, v[0], v[1], v[2], v[3]);
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s.acc_empty);
      acc_phase ^= 1u;
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
cudaError_t launch_gemm(const CUtensorMap& tma_a, const CUtensorMap& tma_b, const GemmArgs& a, int grid,
                        cudaStream_t stream) {
  const size_t smem = sizeof(Smem) + 1024;
  cudaError_t err = cudaFuncSetAttribute(moe_gemm_kernel<kGateUp>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  moe_gemm_kernel<kGateUp><<<grid, kThreads, smem, stream>>>(tma_a, tma_b, a);
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

static_assert(sizeof(Smem) + 1024 <= 232448, "GEMM shared memory exceeds the per-block limit");

cudaError_t launch_gemm_gateup(const CUtensorMap& tma_a, const CUtensorMap& tma_b, const GemmArgs& a,
                               int grid, cudaStream_t stream) {
  return launch_gemm<true>(tma_a, tma_b, a, grid, stream);
}

cudaError_t launch_gemm_down(const CUtensorMap& tma_a, const CUtensorMap& tma_b, const GemmArgs& a,
                             int grid, cudaStream_t stream) {
  return launch_gemm<false>(tma_a, tma_b, a, grid, stream);
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
