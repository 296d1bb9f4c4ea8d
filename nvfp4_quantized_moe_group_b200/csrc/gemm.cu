// Grouped block-scaled NVFP4 GEMMs of the expert MLPs on the 5th-generation tensor cores.
//
// Each expert's token rows form a segment padded to 128 rows; a work item is one
// (expert, 256-column tile, 128-row tile).  One persistent CTA per SM takes work items in
// index order (expert-major, then column tile, then row tile, so row tiles of one expert that
// share a weight tile run at the same time and the second read of that tile comes from L2):
// its first item is its own CTA index, the following ones are claimed from a grid-wide
// counter, so faster CTAs take more items.
//
// Per CTA: warp 0 fills a shared-memory ring: the A tile by a TMA load with 128-byte
// swizzle (a 32-row box when at most 32 rows of the tile hold pairs, as at decode: the
// other rows only feed accumulator rows that are never read), the B (weight) tile by two
// contiguous bulk copies from the pre-tiled, pre-swizzled weight layout, the block scales by
// bulk copies; warp 1 copies the block scales into tensor memory (tcgen05.cp) and issues
// tcgen05.mma kind::mxf4nvf4 (E2M1 x E2M1, UE4M3 scale per 16 values, M = 128, N = 256)
// into a 128 x 256 FP32 accumulator in tensor memory; warps 2-9 read the accumulator
// (tcgen05.ld; warp w reads lanes 32 * (w % 4) .. +31, and the two warps of a lane quarter
// split the columns), free it for the next item's MMAs, and run the epilogue:
//   gate/up:  each 128-column half holds 64 gate and 64 up columns of the same features:
//             h = silu(g_x g_gate acc_gate) * (g_x g_up acc_up) in FP32, requantised to
//             NVFP4 with the expert's static scale g_h (the down GEMM's A operand);
//   down:     acc_out[token] += w * g_h * g_down * acc, FP32 additions into the token's row
//             (given a table of the ranks' accumulators, the row in the owning rank's one):
//             with full segments half the lanes at a time stage their row's 64-column piece in
//             shared memory and add it with one bulk reduction (cp.reduce.async.bulk .add.f32,
//             256 bytes);
//             when segments hold few rows, vector reductions straight from the 16x256b register
//             layout.
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
constexpr int kWorkRing = 4;                  // items the producer may run ahead of the epilogue
constexpr int kABytes = kBlockM * 128;        // 128 rows x 256 E2M1
constexpr int kTileBytes = 128 * 128;         // one 128-row weight tile x 256 K values
constexpr int kAtomBytes = 512;               // one 128-row block-scale atom (one 64-deep K step)
constexpr uint32_t kTmemCols = 512;

// Work items are 256 output columns wide (two 128-row weight tiles), with one 256-column
// FP32 accumulator in tensor memory: the epilogue copies it to registers and frees it before
// the rest of its arithmetic.  At 128 columns the main loop was bound by the block-scale
// copies into tensor memory (each 128-row scale atom written to all four lane quarters);
// 256-wide items give each A-scale atom twice the MMA work.
constexpr int kN = 256;
constexpr int kNT = kN / 128;                       // 128-row weight tiles per item

// kMode: which GEMM the launch runs.  kModeFused runs both in one persistent launch (used
// with short segments): the gate/up items and the down items share the work counter, and a
// down item waits until every gate/up item of its 128-row tile has stored its part of h
// (per-tile counters), so no CTA idles at a boundary between two launches.
enum : int { kModeDown = 0, kModeGateUp = 1, kModeFused = 2 };

// kDecode: segments average fewer than 32 rows.  The down epilogue then reduces straight from
// the 16x256b register layout, and the down GEMM keeps 4 stages; with full segments it stages
// row pieces in shared memory for bulk reductions (3 stages), measured faster there.  The
// gate/up epilogue reads its whole share of the accumulator before any arithmetic in both
// regimes (the accumulator is free for the next item's MMAs as early as possible).
// The fused launch keeps 4 stages and reduces from registers in both regimes.
//
// kFp8: the FP8 W8A8 variant (E4M3 x E4M3 with FP32 accumulation, kind::f8f6f4): a 128-byte
// K block holds 128 values instead of 256, there are no block scales (per-row activation and
// per-channel weight scales are applied in the epilogue), and gate/up writes h in FP32 for
// the per-row requantisation that follows.
template <int kMode, bool kDecode, bool kFp8>
struct Cfg {
  static constexpr int kStages = (kMode != kModeDown || kDecode) ? 4 : 3;
  static constexpr bool kStaging = kMode == kModeDown && !kDecode;
  static constexpr uint32_t kSfCol0 = kN;                        // the accumulator first
  static constexpr uint32_t kSfColsA = kFp8 ? 0 : 16;            // 4 K steps x 4 columns
  static constexpr uint32_t kSfColsPerStage = kFp8 ? 0 : kSfColsA + 16 * kNT;
  static constexpr int kSfaBytes = kFp8 ? 16 : 4 * kAtomBytes;
  static constexpr int kSfbBytes = kFp8 ? 16 : kNT * 4 * kAtomBytes;
  static_assert(kSfCol0 + kStages * kSfColsPerStage <= kTmemCols, "tensor memory columns");
};

template <int kMode, bool kDecode, bool kFp8>
struct __align__(1024) Smem {
  using C = Cfg<kMode, kDecode, kFp8>;
  uint8_t a[C::kStages][kABytes];
  uint8_t b[C::kStages][kNT * kTileBytes];
  uint8_t sfa[C::kStages][C::kSfaBytes];
  uint8_t sfb[C::kStages][C::kSfbBytes];
  // down, full segments: per epilogue warp, 16 staged row pieces of 64 FP32 values, 272 bytes
  // apart (32 pieces of 32 values, 144 bytes apart, for FP8; 16-byte aligned for the bulk
  // reductions, and the float4 stores of consecutive lanes fall in different bank groups)
  alignas(16) float stage_rows[C::kStaging ? kEpiWarps : 1][32 * 36];
  uint64_t full[C::kStages];
  uint64_t empty[C::kStages];
  uint64_t acc_full;
  uint64_t acc_empty;
  uint64_t drain;
  uint64_t work_full[kWorkRing];    // the producer published the item of this slot
  uint64_t work_empty[kWorkRing];   // the MMA issuer and the epilogue warps have read it
  int work[kWorkRing];              // item index, -1: no more items
  uint32_t tmem_base;
  int abort_flag;
};

// 16 lanes x 128 columns of FP32 from tensor memory (16x256b shape, 16 repetitions along the
// columns): thread i receives, for k = 0..15, lane (i / 4) columns 8k + 2 (i % 4) + {0, 1} in
// r[4k], r[4k + 1] and lane (i / 4 + 8) at the same columns in r[4k + 2], r[4k + 3].
__device__ __forceinline__ void tmem_ld_16x256b_x16(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.16x256b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, "
      "%32, %33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, "
      "%48, %49, %50, %51, %52, %53, %54, %55, %56, %57, %58, %59, %60, %61, %62, %63}, [%64];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]),
        "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]),
        "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]),
        "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]),
        "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
      : "r"(taddr));
}

// tcgen05.mma kind::f8f6f4, E4M3 x E4M3 -> FP32, K = 32 (both operands K-major).
__device__ __forceinline__ void mma_f8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Instruction descriptor of kind::f8f6f4: FP32 accumulator (bits 4-5 = 1), A and B formats
// E4M3 (bits 7-9, 10-12 = 0), both K-major, N / 8 at bit 17, M / 16 (128) at bit 24.
__host__ __device__ constexpr uint32_t idesc_f8(uint32_t n) {
  return (1u << 4) | (0u << 7) | (0u << 10) | ((n >> 3) << 17) | ((128u >> 4) << 24);
}

__device__ __forceinline__ void red_add_v2(float* addr, float a, float b) {
  asm volatile("red.global.add.v2.f32 [%0], {%1, %2};" ::"l"(addr), "f"(a), "f"(b) : "memory");
}

// Orders this thread's earlier shared-memory writes before its later bulk (async-proxy) reads.
__device__ __forceinline__ void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// gdst[i] += ssrc[i] for bytes / 4 FP32 values (both 16-byte aligned, bytes a multiple of 16),
// performed by the bulk-copy unit; completion tracked in this thread's bulk group.
__device__ __forceinline__ void bulk_reduce_add_f32(float* gdst, const float* ssrc, uint32_t bytes) {
  asm volatile("cp.reduce.async.bulk.global.shared::cta.bulk_group.add.f32 [%0], [%1], %2;" ::"l"(gdst),
               "r"(smem_u32(ssrc)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Waits until this thread's committed bulk operations have read their shared-memory sources.
__device__ __forceinline__ void bulk_wait_read0() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// Waits until they have completed (their global writes done).
__device__ __forceinline__ void bulk_wait_all0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

struct Work {
  int e;          // expert
  int mtile;      // global 128-row tile (row = mtile * 128 + r)
  int mt_local;   // tile index inside the expert's segment
  int nt;         // kN-column tile
  int rows_valid; // rows of this tile that hold a pair
};

// prefix / counts are read through the read-only cache (1-2 KB, written by an earlier kernel).
__device__ __forceinline__ Work decode_work(const int* prefix, int w, int E, int ntn, const int* counts) {
  int lo = 0, hi = E;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (__ldg(prefix + mid) * ntn <= w) lo = mid; else hi = mid;
  }
  Work k;
  k.e = lo;
  const int p_lo = __ldg(prefix + lo);
  const int mt_e = __ldg(prefix + lo + 1) - p_lo;
  const int local = w - p_lo * ntn;
  k.nt = local / mt_e;
  k.mt_local = local - k.nt * mt_e;
  k.mtile = p_lo + k.mt_local;
  const int left = __ldg(counts + lo) - k.mt_local * kBlockM;
  k.rows_valid = left < kBlockM ? left : kBlockM;
  return k;
}

// The fused schedule.  The gate/up items keep their order (expert-major, then column tile,
// then row tile); expert e's down items (same order) follow as one block after the first
// min(G(e + 1) + lag, NG) gate/up items, G(e) counting the gate/up items of the experts before
// e and NG all of them.  Every gate/up item of an expert thus precedes its down items by at
// least lag claims (except for the last experts, whose down items close the list), so the
// dependency waits stay rare.  (Spreading the down items evenly among the gate/up items
// measured 6 % slower at decode.)
struct Sched {
  int base;      // global tile number of the launch's first row tile
  int ntn_g;     // gate/up items per row tile
  int ntn_d;     // down items per row tile
  int NG;        // gate/up items
  int lag;
  int E;
};

__device__ __forceinline__ Work decode_fused(const int* prefix, const int* counts, const Sched& sc, int w,
                                             bool* gu) {
  // start of expert e's down block: min(G(e + 1) + lag, NG) + D(e)
  auto start = [&](int e) {
    const int g1 = (__ldg(prefix + e + 1) - sc.base) * sc.ntn_g + sc.lag;
    return (g1 < sc.NG ? g1 : sc.NG) + (__ldg(prefix + e) - sc.base) * sc.ntn_d;
  };
  int lo = -1, hi = sc.E;     // start(lo) <= w < start(hi); lo = -1: before every down block
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (start(mid) <= w) lo = mid; else hi = mid;
  }
  int g = w;
  if (lo >= 0) {
    const int s0 = start(lo);
    const int p_lo = __ldg(prefix + lo);
    const int mt_e = __ldg(prefix + lo + 1) - p_lo;
    if (w < s0 + mt_e * sc.ntn_d) {
      *gu = false;
      return decode_work(prefix, (p_lo - sc.base) * sc.ntn_d + (w - s0) + sc.base * sc.ntn_d, sc.E, sc.ntn_d,
                         counts);
    }
    g = w - (p_lo + mt_e - sc.base) * sc.ntn_d;   // the down items before w: experts 0 .. lo
  }
  *gu = true;
  return decode_work(prefix, g + sc.base * sc.ntn_g, sc.E, sc.ntn_g, counts);
}

__device__ __forceinline__ int ld_acquire_gpu(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Orders this thread's generic-proxy global accesses with its async-proxy (TMA, bulk copy) ones.
__device__ __forceinline__ void fence_proxy_async_global() { asm volatile("fence.proxy.async.global;" ::: "memory"); }

// The FP32 accumulator row of a token: the launch's own accumulator, or the row in the owning
// rank's accumulator (expert parallelism with the combine into peer memory).
__device__ __forceinline__ float* acc_row(const GemmArgs& p, int token) {
  if (p.acc_peers != nullptr)
    return p.acc_peers[token / p.rows_per_peer] + (int64_t)(token % p.rows_per_peer) * p.H;
  return p.acc + (int64_t)token * p.H;
}

__device__ __forceinline__ void set_abort(int* flag, uint32_t* status) {
  raise_status(status, kStatusTimeout);
  *reinterpret_cast<volatile int*>(flag) = 1;
}

__device__ __forceinline__ bool aborted(const int* flag) {
  return *reinterpret_cast<const volatile int*>(flag) != 0;
}

// SwiGLU of 32 features of one token row (this lane's): h = silu(sg acc_g) * (su acc_u), FP32
// with an approximate reciprocal.
__device__ __forceinline__ void swiglu32(const uint32_t* G, const uint32_t* U, float sg, float su, float* h) {
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const float g = __fmul_rn(__uint_as_float(G[i]), sg);
    const float u = __fmul_rn(__uint_as_float(U[i]), su);
    // silu(g) * u = g * u / (1 + exp(-g))
    h[i] = __fmul_rn(__fmul_rn(g, u), rcp_approx(__fadd_rn(1.0f, __expf(-g))));
  }
}

// Debug export of 32 features of one pair's FP32 h (feature f0 on).
__device__ __forceinline__ void store_h_dbg(const GemmArgs& p, const Work& wk, int row_l, int f0, const float* h) {
  const int64_t pos = (int64_t)__ldg(p.dbg_offsets + wk.e) + (int64_t)wk.mt_local * kBlockM + row_l;
  float4* dst = reinterpret_cast<float4*>(p.h_dbg + pos * p.I + f0);
#pragma unroll
  for (int i = 0; i < 8; ++i) dst[i] = make_float4(h[4 * i], h[4 * i + 1], h[4 * i + 2], h[4 * i + 3]);
}

// NVFP4 requantisation of 32 features with the expert's static scale gh: 16 code bytes and
// 2 scale bytes stored at feature f0 of the row.
__device__ __forceinline__ void quant_store32(const float* h, float gh, float r_t, bool valid, int64_t row, int f0,
                                              const GemmArgs& p, int64_t n_ct) {
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
    *reinterpret_cast<uint4*>(p.hq_codes + row * (p.I / 2) + f0 / 2) =
        make_uint4(codes[0], codes[1], codes[2], codes[3]);
    *reinterpret_cast<uint16_t*>(p.hq_sf + swz_offset(row, f0 / 16, n_ct)) = (uint16_t)sfp;
  }
}

template <int kMode, bool kDecode, bool kFp8>
__global__ void __launch_bounds__(kThreads, 1)
moe_gemm_kernel(const __grid_constant__ CUtensorMap tma_a, const __grid_constant__ CUtensorMap tma_a32,
                const __grid_constant__ CUtensorMap tma_h, const __grid_constant__ CUtensorMap tma_h32,
                const __grid_constant__ GemmArgs pg, const __grid_constant__ GemmArgs pd, int* dep, int lag) {
  using C = Cfg<kMode, kDecode, kFp8>;
  constexpr int kStages = C::kStages;
  using S = Smem<kMode, kDecode, kFp8>;
  extern __shared__ uint8_t smem_raw[];
  S& s = *reinterpret_cast<S*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // the fields every item shares (status, grouping tables, work counter)
  const GemmArgs& P0 = kMode == kModeDown ? pd : pg;

  if (threadIdx.x == 0) {
    for (int st = 0; st < kStages; ++st) {
      mbar_init(&s.full[st], 1);
      mbar_init(&s.empty[st], 1);
    }
    mbar_init(&s.acc_full, 1);
    mbar_init(&s.acc_empty, kEpiWarps);
    mbar_init(&s.drain, 1);
    for (int i = 0; i < kWorkRing; ++i) {
      mbar_init(&s.work_full[i], 1);
      mbar_init(&s.work_empty[i], kEpiWarps + 1);
    }
    s.abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    if (kMode != kModeDown) {
      prefetch_tmap(&tma_a);
      prefetch_tmap(&tma_a32);
    }
    if (kMode != kModeGateUp) {
      prefetch_tmap(&tma_h);
      prefetch_tmap(&tma_h32);
    }
  }
  if (warp == 1) {
    tmem_alloc(&s.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // launched programmatically: everything above overlapped the previous kernel's tail; the
  // routing tables and the A operand are read only after it has completed.  The next kernel
  // may then be scheduled onto SMs as this grid's CTAs exit.
  pdl_wait();
  pdl_trigger();

  const uint64_t wait_ns = wait_limit(P0.wait_ns);
  const uint32_t tmem = s.tmem_base;
  // P0.mtile_prefix may start at a later expert (a handle with one rank's share of the experts):
  // its tiles are numbered from the first entry on.  When an earlier kernel of the call has
  // timed out, the grouping tables may be incomplete: no work items then.
  const bool upstream_timeout = (*reinterpret_cast<const volatile uint32_t*>(P0.status) & kStatusTimeout) != 0;
  const int tile_base = upstream_timeout ? 0 : __ldg(P0.mtile_prefix);
  const int m_total = upstream_timeout ? 0 : __ldg(P0.mtile_prefix + P0.E) - tile_base;
  const int ntn_g = pg.n_total / kN;        // 256-wide items per row tile: gate/up
  const int ntn_d = pd.n_total / kN;        // and down
  const Sched sc{tile_base, ntn_g, ntn_d, m_total * ntn_g, lag, P0.E};
  const int total = kMode == kModeFused ? m_total * (ntn_g + ntn_d) : m_total * (kMode == kModeGateUp ? ntn_g : ntn_d);
  // item w of the schedule; *gu: a gate/up item (else down)
  auto item = [&](int w, bool* gu) -> Work {
    if constexpr (kMode == kModeFused) {
      return decode_fused(P0.mtile_prefix, P0.counts, sc, w, gu);
    } else {
      *gu = kMode == kModeGateUp;
      const int ntn = kMode == kModeGateUp ? ntn_g : ntn_d;
      return decode_work(P0.mtile_prefix, w + tile_base * ntn, P0.E, ntn, P0.counts);
    }
  };
  auto k_blocks = [](int K) { return kFp8 ? (K + 127) / 128 : (K + kBlockK - 1) / kBlockK; };   // 128-byte K blocks

  if (warp == 0) {
    // ------------------------------------------------------------ producer ----
    __syncwarp();
    if (elect_one()) {
      uint32_t stage = 0, phase = 0, issued = 0, issued_par = 0;
      const uint64_t pol_w = policy_evict_first();
      const uint64_t pol_a = policy_evict_last();
      bool ok = true;
      for (int it = 0; ok; ++it) {
        // items are handed out dynamically: the first is the CTA's own index, the next ones
        // come from a counter shared by the grid, so CTAs that run faster take more items
        const int slot = it & (kWorkRing - 1);
        if (aborted(&s.abort_flag) || !mbar_wait(&s.work_empty[slot], ((uint32_t)(it / kWorkRing) & 1u) ^ 1u, wait_ns)) {
          set_abort(&s.abort_flag, P0.status);
          break;
        }
        int w = it == 0 ? (int)blockIdx.x : atomicAdd(P0.work_counter, 1) + (int)gridDim.x;
        if (w >= total) w = -1;
        s.work[slot] = w;
        mbar_arrive(&s.work_full[slot]);      // releases the index to the MMA issuer and the epilogue
        if (w < 0) break;
        bool gu;
        const Work wk = item(w, &gu);
        const GemmArgs& P = gu ? pg : pd;
        if constexpr (kMode == kModeFused) {
          if (!gu) {
            // h of this row tile is complete once all gate/up items of the tile have signalled
            const int* d = dep + (wk.mtile - tile_base);
            const int need = kEpiWarps * ntn_g;
            if (ld_acquire_gpu(d) < need) {
              const uint64_t t_start = globaltimer_ns();
              while (ld_acquire_gpu(d) < need) {
                if (aborted(&s.abort_flag) || globaltimer_ns() - t_start > wait_ns) {
                  ok = false;
                  break;
                }
                __nanosleep(256);
              }
              if (!ok) {
                set_abort(&s.abort_flag, P0.status);
                break;
              }
            }
            fence_proxy_async_global();
          }
        }
        const int kb_count = k_blocks(P.K);
        const int k64 = P.K / 64;               // scale-column tiles of A and B
        const int ntn128 = P.n_total / 128;     // 128-row weight tiles per expert
        const int arow = wk.mtile * kBlockM;
        const bool a_small = wk.rows_valid <= 32;
        const uint32_t a_bytes = a_small ? 32u * 128u : (uint32_t)kABytes;
        const void* amap = gu ? (a_small ? (const void*)&tma_a32 : (const void*)&tma_a)
                              : (a_small ? (const void*)&tma_h32 : (const void*)&tma_h);
        const int t0 = wk.nt * kNT;           // first 128-row weight tile of the item
        const uint8_t* btile = P.b_tiles + ((int64_t)wk.e * ntn128 + t0) * kb_count * (int64_t)kTileBytes;
        const uint8_t* sfa = P.sfa + (int64_t)wk.mtile * k64 * kAtomBytes;
        const uint8_t* sfb = P.sfb + ((int64_t)wk.e * ntn128 + t0) * k64 * kAtomBytes;
        for (int kb = 0; kb < kb_count; ++kb) {
          if (aborted(&s.abort_flag) || !mbar_wait(&s.empty[stage], phase ^ 1u, wait_ns)) {
            set_abort(&s.abort_flag, P0.status);
            ok = false;
            break;
          }
          const int left = (P.K - kb * kBlockK) / 64;
          const uint32_t sf_bytes = kFp8 ? 0u : (uint32_t)(left < 4 ? left : 4) * kAtomBytes;
          mbar_arrive_expect_tx(&s.full[stage], a_bytes + kNT * (kTileBytes + sf_bytes) + sf_bytes);
          tma_load_2d(s.a[stage], amap, &s.full[stage], kb * 128, arow, pol_a);
          if constexpr (!kFp8) bulk_load(s.sfa[stage], sfa + kb * 4 * kAtomBytes, sf_bytes, &s.full[stage], pol_a);
#pragma unroll
          for (int j = 0; j < kNT; ++j) {
            bulk_load(s.b[stage] + j * kTileBytes, btile + ((int64_t)j * kb_count + kb) * kTileBytes, kTileBytes,
                      &s.full[stage], pol_w);
            if constexpr (!kFp8)
              bulk_load(s.sfb[stage] + j * 4 * kAtomBytes, sfb + ((int64_t)j * k64 + kb * 4) * kAtomBytes, sf_bytes,
                        &s.full[stage], pol_w);
          }
          issued |= 1u << stage;
          issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
      }
      // wait for every copy this thread started before the CTA can exit
      for (int st = 0; st < kStages; ++st)
        if ((issued >> st) & 1u)
          if (!mbar_wait(&s.full[st], (issued_par >> st) & 1u, wait_ns)) set_abort(&s.abort_flag, P0.status);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer ----
    __syncwarp();
    if (elect_one()) {
      uint32_t stage = 0, phase = 0;
      const uint32_t idesc = kFp8 ? idesc_f8(kN) : idesc_nvf4(kN);
      bool ok = true;
      for (int it = 0; ok; ++it) {
        const int slot = it & (kWorkRing - 1);
        if (aborted(&s.abort_flag) || !mbar_wait(&s.work_full[slot], (uint32_t)(it / kWorkRing) & 1u, wait_ns)) {
          set_abort(&s.abort_flag, P0.status);
          break;
        }
        const int w = *reinterpret_cast<volatile int*>(&s.work[slot]);
        mbar_arrive(&s.work_empty[slot]);
        if (w < 0) break;
        bool gu = kMode == kModeGateUp;
        if constexpr (kMode == kModeFused) item(w, &gu);
        const int K = gu ? pg.K : pd.K;
        const int kb_count = k_blocks(K);
        const uint32_t acc_par = (uint32_t)it & 1u;
        const uint32_t acc = tmem;
        for (int kb = 0; kb < kb_count; ++kb) {
          if (aborted(&s.abort_flag) || !mbar_wait(&s.full[stage], phase, wait_ns)) {
            set_abort(&s.abort_flag, P0.status);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(s.a[stage]);
          const uint32_t b0 = smem_u32(s.b[stage]);
          if constexpr (kFp8) {
            if (kb == 0) {
              if (aborted(&s.abort_flag) || !mbar_wait(&s.acc_empty, acc_par ^ 1u, wait_ns)) {
                set_abort(&s.abort_flag, P0.status);
                ok = false;
                break;
              }
              tc_fence_after();
            }
            // four K = 32 instructions per 128-byte K block (32 bytes apart, like the FP4 steps)
            for (int k = 0; k < 4; ++k)
              mma_f8(acc, desc_k_sw128(a0 + 32 * k), desc_k_sw128(b0 + 32 * k), idesc, (kb | k) != 0 ? 1u : 0u);
            tc_commit(&s.empty[stage]);
            if (++stage == kStages) { stage = 0; phase ^= 1u; }
            continue;
          }
          const int left = (K - kb * kBlockK) / 64;
          const int ksteps = left < 4 ? left : 4;
          // scale atoms: A at sfa_t + 4k; B (row n at lane n % 32, column n / 32) at
          // sfb_t + 4 (kNT k + j) for its 128-row tile j
          const uint32_t sfa_t = tmem + C::kSfCol0 + stage * C::kSfColsPerStage;
          const uint32_t sfb_t = sfa_t + C::kSfColsA;
          const uint32_t sa = smem_u32(s.sfa[stage]);
          const uint32_t sb = smem_u32(s.sfb[stage]);
          for (int k = 0; k < ksteps; ++k) {
            tc_cp_32x128b_x4(sfa_t + 4 * k, desc_sf_block(sa + kAtomBytes * k));
#pragma unroll
            for (int j = 0; j < kNT; ++j)
              tc_cp_32x128b_x4(sfb_t + 4 * (kNT * k + j), desc_sf_block(sb + (j * 4 + k) * kAtomBytes));
          }
          // the first K block's scale copies go out before the wait for the accumulator (they
          // write only this stage's scale columns), so they overlap the previous item's
          // accumulator read-out
          if (kb == 0) {
            if (aborted(&s.abort_flag) || !mbar_wait(&s.acc_empty, acc_par ^ 1u, wait_ns)) {
              set_abort(&s.abort_flag, P0.status);
              ok = false;
              break;
            }
            tc_fence_after();
          }
          for (int k = 0; k < ksteps; ++k) {
            mma_nvf4(acc, desc_k_sw128(a0 + 32 * k), desc_k_sw128(b0 + 32 * k), idesc, sfa_t + 4 * k,
                     sfb_t + 4 * kNT * k, (kb | k) != 0 ? 1u : 0u);
          }
          tc_commit(&s.empty[stage]);
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        tc_commit(&s.acc_full);
      }
      // every tensor-core operation of this thread is done before the memory is freed
      tc_commit(&s.drain);
      if (!mbar_wait(&s.drain, 0, wait_ns)) set_abort(&s.abort_flag, P0.status);
    }
  } else {
    // ------------------------------------------------------------ epilogue ----
    const int q = warp & 3;              // tensor-memory lane quarter this warp may read
    const int half = (warp - 2) >> 2;    // which half of the tile's columns it handles
    const int row_l = q * 32 + lane;
    for (int it = 0;; ++it) {
      const int slot = it & (kWorkRing - 1);
      const bool got_work = !aborted(&s.abort_flag) && mbar_wait(&s.work_full[slot], (uint32_t)(it / kWorkRing) & 1u, wait_ns);
      if (__any_sync(0xffffffffu, !got_work)) {
        set_abort(&s.abort_flag, P0.status);
        break;
      }
      const int w = *reinterpret_cast<volatile int*>(&s.work[slot]);
      __syncwarp();
      if (lane == 0) mbar_arrive(&s.work_empty[slot]);
      if (w < 0) break;
      bool gu;
      const Work wk = item(w, &gu);
      const GemmArgs& P = gu ? pg : pd;
      if constexpr (kMode == kModeGateUp) {
        // the launch's share of zeroing the down GEMM's accumulator, item w's slice, while the
        // tensor cores work on the item
        if (P.zero_acc != nullptr) {
          const int64_t n = P.zero_acc_elems;
          const int64_t per = ((n + total - 1) / total + 3) & ~(int64_t)3;
          const int64_t z1 = min((int64_t)(w + 1) * per, n);
          const float4 zero = make_float4(0.f, 0.f, 0.f, 0.f);
          for (int64_t i = (int64_t)w * per + 4 * ((warp - 2) * 32 + lane); i < z1; i += 4 * 32 * kEpiWarps)
            *reinterpret_cast<float4*>(P.zero_acc + i) = zero;
        }
      }
      const uint32_t acc_par = (uint32_t)it & 1u;
      const int64_t row = (int64_t)wk.mtile * kBlockM + row_l;
      const bool valid = row_l < wk.rows_valid;
      // rows of this warp that hold a pair (rows are filled from the top of the tile)
      const bool warp_live = q * 32 < wk.rows_valid;
      // per-expert / per-row constants, loaded before the accumulator is ready
      float c0s = 0.f, c1s = 0.f, c2s = 0.f;
      int token = -1;
      if (warp_live) {
        if (gu) {
          if constexpr (kFp8) {
            c0s = P.a_scale[row];                     // the token's activation scale
          } else {
            const float gx = *P.g_x;
            c0s = __fmul_rn(gx, P.g_gate[wk.e]);
            c1s = __fmul_rn(gx, P.g_up[wk.e]);
            c2s = P.g_h[wk.e];
          }
        } else {
          const int pair = valid ? P.row_pair[row] : -1;
          if (pair >= 0) {
            c0s = kFp8 ? __fmul_rn(P.wts[pair], P.h_scale[row]) : __fmul_rn(P.alpha_down[wk.e], P.wts[pair]);
            token = pair / P.topk;
          }
        }
      }
      const bool got = !aborted(&s.abort_flag) && mbar_wait(&s.acc_full, acc_par, wait_ns);
      if (__any_sync(0xffffffffu, !got)) {
        set_abort(&s.abort_flag, P0.status);
        break;
      }
      __syncwarp();
      tc_fence_after();
      const uint32_t t_row = tmem + ((uint32_t)(q * 32) << 16);
      // the accumulator is released as soon as this warp's last columns are in registers
      auto release = [&]() {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s.acc_empty);
      };
      if (!warp_live) {
        release();
      } else if (gu) {
        if constexpr (kFp8) {
          // h = silu(acc_g * sx * wg) * (acc_u * sx * wu) per feature, stored in FP32
          const int t = wk.nt * kNT + half;           // weight tile of this warp's 64 features
          const int tcol = half * 128;
          const float* wsc = P.w_scale + (int64_t)wk.e * P.n_total + wk.nt * kN + tcol;
          const float sx = c0s;
#pragma unroll
          for (int pr = 0; pr < 2; ++pr) {
            uint32_t G[32], U[32];
            tmem_ld_32x32b_x32(t_row + tcol + 32 * pr, G);
            tmem_ld_32x32b_x32(t_row + tcol + 64 + 32 * pr, U);
            tmem_ld_wait();
            if (pr == 1) release();
            float h[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const float gv = __fmul_rn(__fmul_rn(__uint_as_float(G[i]), sx), __ldg(wsc + 32 * pr + i));
              const float uv = __fmul_rn(__fmul_rn(__uint_as_float(U[i]), sx), __ldg(wsc + 64 + 32 * pr + i));
              h[i] = __fmul_rn(__fmul_rn(gv, uv), rcp_approx(__fadd_rn(1.0f, __expf(-gv))));
            }
            if (valid) {
              float4* dst = reinterpret_cast<float4*>(P.h32 + row * P.I + t * 64 + 32 * pr);
#pragma unroll
              for (int i = 0; i < 8; ++i) dst[i] = make_float4(h[4 * i], h[4 * i + 1], h[4 * i + 2], h[4 * i + 3]);
            }
          }
        } else {
          const float sg = c0s, su = c1s, gh = c2s;
          const float r_t = __frcp_rn(__fmul_rn(6.0f, gh));
          const int64_t n_ct = P.I / 64;
          // weight tile t = 2 nt + half holds this warp's 64 features: accumulator columns
          // [128 half, +64) are their gate, [128 half + 64, +64) their up projections
          const int t = wk.nt * kNT + half;
          const int tcol = half * 128;
          // all four 32-column chunks into registers first, then the accumulator is released
          uint32_t G0[32], U0[32], G1[32], U1[32];
          tmem_ld_32x32b_x32(t_row + tcol, G0);
          tmem_ld_32x32b_x32(t_row + tcol + 64, U0);
          tmem_ld_32x32b_x32(t_row + tcol + 32, G1);
          tmem_ld_32x32b_x32(t_row + tcol + 96, U1);
          tmem_ld_wait();
          release();
          float h[32];
          swiglu32(G0, U0, sg, su, h);
          if (P.h_dbg != nullptr && valid) store_h_dbg(P, wk, row_l, t * 64, h);
          quant_store32(h, gh, r_t, valid, row, t * 64, P, n_ct);
          swiglu32(G1, U1, sg, su, h);
          if (P.h_dbg != nullptr && valid) store_h_dbg(P, wk, row_l, t * 64 + 32, h);
          quant_store32(h, gh, r_t, valid, row, t * 64 + 32, P, n_ct);
        }
      } else if constexpr (!C::kStaging) {
        // two 16-lane blocks of this warp's rows, 128 columns each, in the 16x256b layout:
        // four consecutive threads hold one row's 8 consecutive columns, so every reduction
        // instruction adds whole 32-byte sectors of 8 token rows
        uint32_t V[2][64];
        tmem_ld_16x256b_x16(t_row + half * (kN / 2), V[0]);
        tmem_ld_16x256b_x16(t_row + (16u << 16) + half * (kN / 2), V[1]);
        tmem_ld_wait();
        release();
        const int cq = 2 * (lane & 3);   // this thread's column pair inside each 8-column group
#pragma unroll
        for (int lh = 0; lh < 2; ++lh) {
#pragma unroll
          for (int rr = 0; rr < 2; ++rr) {
            const int r = 16 * lh + 8 * rr + (lane >> 2);   // row inside the warp's 32
            const int tok = __shfl_sync(0xffffffffu, token, r);
            const float sc = __shfl_sync(0xffffffffu, c0s, r);
            if (tok >= 0) {
              float* dst = acc_row(P, tok) + wk.nt * kN + half * (kN / 2) + cq;
              const float* wsc = kFp8 ? P.w_scale + (int64_t)wk.e * P.n_total + wk.nt * kN + half * (kN / 2) + cq
                                      : nullptr;
#pragma unroll
              for (int k = 0; k < 16; ++k) {
                float v0 = __fmul_rn(__uint_as_float(V[lh][4 * k + 2 * rr]), sc);
                float v1 = __fmul_rn(__uint_as_float(V[lh][4 * k + 2 * rr + 1]), sc);
                if constexpr (kFp8) {
                  v0 = __fmul_rn(v0, __ldg(wsc + 8 * k));
                  v1 = __fmul_rn(v1, __ldg(wsc + 8 * k + 1));
                }
                red_add_v2(dst + 8 * k, v0, v1);
              }
            }
          }
        }
      } else {
        uint32_t R[4][32];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld_32x32b_x32(t_row + half * (kN / 2) + c * 32, R[c]);
        tmem_ld_wait();
        release();
        // row pieces staged in shared memory and added to the tokens' accumulator rows by bulk
        // reductions (async proxy)
        const float scale = c0s;
        if constexpr (kFp8) {
          // FP8: each lane's 32-column piece (128 bytes), one reduction per piece
          float* mine = s.stage_rows[warp - 2] + lane * 36;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const int c0 = half * (kN / 2) + c * 32;
            if (c > 0) bulk_wait_read0();
            const float* wsc = P.w_scale + (int64_t)wk.e * P.n_total + wk.nt * kN + c0;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const float4 w4 = __ldg(reinterpret_cast<const float4*>(wsc) + i);
              *reinterpret_cast<float4*>(mine + 4 * i) =
                  make_float4(__fmul_rn(__fmul_rn(__uint_as_float(R[c][4 * i]), scale), w4.x),
                              __fmul_rn(__fmul_rn(__uint_as_float(R[c][4 * i + 1]), scale), w4.y),
                              __fmul_rn(__fmul_rn(__uint_as_float(R[c][4 * i + 2]), scale), w4.z),
                              __fmul_rn(__fmul_rn(__uint_as_float(R[c][4 * i + 3]), scale), w4.w));
            }
            if (token >= 0) {
              fence_proxy_async_smem();
              bulk_reduce_add_f32(acc_row(P, token) + wk.nt * kN + c0, mine, 128u);
              bulk_commit();
            }
          }
        } else {
          // 16 lanes at a time stage their row's 64 columns (256 bytes) and add each with one
          // bulk reduction: the L2 takes bulk reductions at a rate per operation, so 256-byte
          // operations move twice the bytes of 128-byte ones (T = 32768: 2.96 -> 2.73 ms)
          float* slot = s.stage_rows[warp - 2] + (lane & 15) * 68;
#pragma unroll
          for (int c2 = 0; c2 < 2; ++c2) {
            const int c0 = half * (kN / 2) + c2 * 64;
#pragma unroll
            for (int rd = 0; rd < 2; ++rd) {
              if ((lane >> 4) == rd) {
#pragma unroll
                for (int cc = 0; cc < 2; ++cc)
#pragma unroll
                  for (int i = 0; i < 8; ++i)
                    *reinterpret_cast<float4*>(slot + 32 * cc + 4 * i) =
                        make_float4(__fmul_rn(__uint_as_float(R[2 * c2 + cc][4 * i]), scale), __fmul_rn(__uint_as_float(R[2 * c2 + cc][4 * i + 1]), scale),
                                    __fmul_rn(__uint_as_float(R[2 * c2 + cc][4 * i + 2]), scale), __fmul_rn(__uint_as_float(R[2 * c2 + cc][4 * i + 3]), scale));
                if (token >= 0) {
                  fence_proxy_async_smem();
                  bulk_reduce_add_f32(acc_row(P, token) + wk.nt * kN + c0, slot, 256u);
                  bulk_commit();
                  bulk_wait_read0();
                }
              }
              __syncwarp();
            }
          }
        }
        bulk_wait_read0();
      }
      if constexpr (kMode == kModeFused) {
        if (gu) {
          // this warp's share of the tile's h is stored: make it visible to the TMA and bulk
          // loads of the down items, then count it
          fence_proxy_async_global();
          __threadfence();
          __syncwarp();
          if (lane == 0) atomicAdd(dep + (wk.mtile - tile_base), 1);
        }
      }
    }
    bulk_wait_all0();
  }

  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int kMode, bool kDecode, bool kFp8 = false>
cudaError_t launch_gemm(const CUtensorMap& tma_a, const CUtensorMap& tma_a32, const CUtensorMap& tma_h,
                        const CUtensorMap& tma_h32, const GemmArgs& pg, const GemmArgs& pd, int* dep, int lag,
                        int grid, cudaStream_t stream) {
  const size_t smem = sizeof(Smem<kMode, kDecode, kFp8>) + 1024;
  cudaError_t err = cudaFuncSetAttribute(moe_gemm_kernel<kMode, kDecode, kFp8>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  return launch_pdl(moe_gemm_kernel<kMode, kDecode, kFp8>, dim3(grid), dim3(kThreads), smem, stream, tma_a,
                    tma_a32, tma_h, tma_h32, pg, pd, dep, lag);
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

static_assert(sizeof(Smem<kModeGateUp, true, false>) + 1024 <= 232448, "GEMM shared memory exceeds the per-block limit");
static_assert(sizeof(Smem<kModeGateUp, false, false>) + 1024 <= 232448, "GEMM shared memory exceeds the per-block limit");
static_assert(sizeof(Smem<kModeDown, true, false>) + 1024 <= 232448, "GEMM shared memory exceeds the per-block limit");
static_assert(sizeof(Smem<kModeDown, false, false>) + 1024 <= 232448, "GEMM shared memory exceeds the per-block limit");
static_assert(sizeof(Smem<kModeFused, true, false>) + 1024 <= 232448, "GEMM shared memory exceeds the per-block limit");
static_assert(sizeof(Smem<kModeGateUp, true, true>) + 1024 <= 232448, "GEMM shared memory exceeds the per-block limit");
static_assert(sizeof(Smem<kModeGateUp, false, true>) + 1024 <= 232448, "GEMM shared memory exceeds the per-block limit");
static_assert(sizeof(Smem<kModeDown, true, true>) + 1024 <= 232448, "GEMM shared memory exceeds the per-block limit");
static_assert(sizeof(Smem<kModeDown, false, true>) + 1024 <= 232448, "GEMM shared memory exceeds the per-block limit");

cudaError_t launch_gemm_gateup(const CUtensorMap& tma_a, const CUtensorMap& tma_a32, const GemmArgs& a,
                               int grid, bool decode, cudaStream_t stream) {
  return decode ? launch_gemm<kModeGateUp, true>(tma_a, tma_a32, tma_a, tma_a32, a, a, nullptr, 0, grid, stream)
                : launch_gemm<kModeGateUp, false>(tma_a, tma_a32, tma_a, tma_a32, a, a, nullptr, 0, grid, stream);
}

cudaError_t launch_gemm_down(const CUtensorMap& tma_a, const CUtensorMap& tma_a32, const GemmArgs& a,
                             int grid, bool decode, cudaStream_t stream) {
  return decode ? launch_gemm<kModeDown, true>(tma_a, tma_a32, tma_a, tma_a32, a, a, nullptr, 0, grid, stream)
                : launch_gemm<kModeDown, false>(tma_a, tma_a32, tma_a, tma_a32, a, a, nullptr, 0, grid, stream);
}

cudaError_t launch_gemm_fused(const CUtensorMap& tma_a, const CUtensorMap& tma_a32, const CUtensorMap& tma_h,
                              const CUtensorMap& tma_h32, const GemmArgs& gate_up, const GemmArgs& down, int* dep,
                              int lag, int grid, cudaStream_t stream) {
  return launch_gemm<kModeFused, true>(tma_a, tma_a32, tma_h, tma_h32, gate_up, down, dep, lag, grid, stream);
}

cudaError_t launch_gemm_gateup_fp8(const CUtensorMap& tma_a, const CUtensorMap& tma_a32, const GemmArgs& a,
                                   int grid, bool decode, cudaStream_t stream) {
  return decode ? launch_gemm<kModeGateUp, true, true>(tma_a, tma_a32, tma_a, tma_a32, a, a, nullptr, 0, grid, stream)
                : launch_gemm<kModeGateUp, false, true>(tma_a, tma_a32, tma_a, tma_a32, a, a, nullptr, 0, grid, stream);
}

cudaError_t launch_gemm_down_fp8(const CUtensorMap& tma_a, const CUtensorMap& tma_a32, const GemmArgs& a,
                                 int grid, bool decode, cudaStream_t stream) {
  return decode ? launch_gemm<kModeDown, true, true>(tma_a, tma_a32, tma_a, tma_a32, a, a, nullptr, 0, grid, stream)
                : launch_gemm<kModeDown, false, true>(tma_a, tma_a32, tma_a, tma_a32, a, a, nullptr, 0, grid, stream);
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
