// Internal kernel interfaces of libnvfp4moe (not part of the C ABI).
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "gemm.h"
#include "nvfp4moe.h"

namespace nvfp4moe {

constexpr int kMaxAmaxPartials = 1024;   // blocks of the amax pass
constexpr int kPermChunkTokens = 32;     // tokens per chunk of the grouping kernels

struct QuantizeArgs {
  const uint16_t* x;       // [rows][cols] bf16
  int64_t rows;
  int64_t rows_padded;     // rows rounded up to 128 in the swizzled layout, else rows
  int64_t cols;
  const float* g_in;       // static scale or nullptr
  const uint32_t* partials;
  int n_partials;
  uint8_t* codes;
  uint8_t* scales;
  int swizzled;
  int64_t n_col_tiles;     // ceil(cols/16/4)
  float* g_out;            // the global scale used (may be nullptr)
  float* g_scratch;        // dynamic scale with g_out == nullptr: where the scale is kept
  float* zero_out;         // optional [rows][cols] fp32 zeroed alongside (layer accumulator)
  uint32_t* status;
  // optional scatter into expert segments: row t also goes to the padded segment row of
  // each of its pairs (t*topk + j), codes [seg rows][cols/2], swizzled scales
  const int32_t* idx;
  const int32_t* inv;
  const int32_t* offsets;
  const int32_t* mtile_prefix;
  int topk;
  uint8_t* seg_codes;
  uint8_t* seg_sf;
};

struct RouterArgs {
  const uint16_t* x;       // [T][H] bf16
  const float* w;          // [E][H]
  const float* bias;       // [E] or nullptr
  double* parts;           // [ksplit][T][E]
  int32_t* idx;            // [T][topk]
  float* wts;              // [T][topk]
  int64_t T;
  int H, E, n_groups, topk_groups, topk;
  float routed_scale;
  int ksplit, k_slice;
  uint32_t* amax_partials;  // optional: per-CTA max |x| (BF16 magnitude bits) for the global scale
  float* logits_out;        // optional [T][E]: the FP32 logits (bias included) the top-k used
  uint32_t* status;         // kStatusNonFinite is raised here for a NaN logit (may be nullptr)
  uint64_t wait_ns;         // limit of each bounded wait of the tensor-core logits (0: kWaitLimitNs)
  // integer tensor-core logits (T >= kRouterTcMinT, when given; route_tc.cu)
  uint8_t* x_digits;        // [kRouterXDigits][T][H] int8 digit planes of the token rows
  uint8_t* w_digits;        // [kRouterWDigits][E][H] int8 digit planes of the expert rows
  int32_t* x_exp;           // [T] row exponents (kExpNonFinite: the row has a non-finite value)
  int32_t* w_exp;           // [E]
};
constexpr int kRouterTcMinT = 65;
constexpr int kRouterXDigits = 3;   // int8 digit planes of a token row (22-bit fixed point)
constexpr int kRouterWDigits = 4;   // and of an expert row (30-bit)
constexpr int32_t kExpNonFinite = 0x7FFFFFFF;

struct PermArgs {
  const int32_t* idx;      // [T][topk]
  int64_t T;
  int topk, E;
  int n_chunks;
  int32_t* chunk_counts;   // [n_chunks][E]
  int32_t* chunk_base;     // [n_chunks][E] first position of the chunk's pairs in the expert's segment
  int32_t* counts;         // [E]
  int32_t* offsets;        // [E+1]
  int32_t* mtile_prefix;   // [E+1] cumulative 128-row tiles
  int32_t* perm;           // [T*topk]
  int32_t* inv;            // [T*topk]
  int32_t* row_pair;       // [rows_cap] pair id of each padded row, -1 for padding
};


// Fused front end for T <= kFrontMaxT (front.cu).
constexpr int kFrontMaxT = 64;
struct FrontArgs {
  const uint16_t* x;        // [T][H] bf16
  const float* w;           // router weight [E][H]
  const float* bias;        // [E] or nullptr
  int64_t T;
  int H, E, n_groups, topk_groups, topk;
  float routed_scale;
  int ksplit, k_slice;      // set by launch_front
  double* parts;            // [ksplit][T][E]
  uint32_t* amax_partials;  // [ksplit]
  int32_t* idx;             // [T][topk]
  float* wts;               // [T][topk]
  float* logits_out;        // optional [T][E]
  int32_t* counts;          // [E]
  int32_t* offsets;         // [E+1]
  int32_t* mtile_prefix;    // [E+1]
  int32_t* perm;            // [T*topk]
  int32_t* inv;             // [T*topk]
  int32_t* row_pair;        // [rows_cap]
  uint8_t* seg_codes;       // [rows_cap][H/2]; nullptr: routing and grouping only (no quantisation)
  uint8_t* seg_sf;          // swizzled [rows_cap][H/16]
  int64_t n_col_tiles;      // H / 64
  uint8_t* xq_codes;        // optional token-major copy [T][H/2]
  uint8_t* xq_sf;           // swizzled, with xq_codes
  float* g_out;             // global scale of x
  float* acc;               // [T][H] FP32, zeroed
  uint32_t* status;
  uint32_t* barrier;        // zero at launch
  uint64_t wait_ns;         // limit of each grid-barrier wait (0: kWaitLimitNs)
  int skip_arrive;          // test hook: CTA skip_arrive - 1 does not arrive at the first grid
                            // barrier (0: every CTA arrives)
};

struct FinalizeArgs {
  const float* acc;
  uint16_t* out;
  int64_t n;  // elements, multiple of 8
  // optional weighted residual add: out = bf16(fp32(a * res) + fp32(b * acc)); res may be out
  const uint16_t* res;
  float a, b;
};

// RMSNorm of the residual stream into the layer input (residual.cu).
struct RmsNormArgs {
  const uint16_t* h;       // [T][H] bf16 residual stream
  const float* gamma;      // [H]
  float eps;
  int64_t T;
  int H;                   // multiple of 8
  uint16_t* x;             // [T][H] bf16 out
};

// quantize.cu
int amax_partial_blocks(int64_t n_elems);
cudaError_t launch_amax_partial(const void* x, int64_t n_elems, uint32_t* partials, int blocks,
                                cudaStream_t stream);
// Dynamic scale (g_in == nullptr): a one-warp kernel reduces the amax partials first.
cudaError_t launch_quantize(QuantizeArgs a, cudaStream_t stream);
// g = A / 2688 (1 for A = 0) from BF16 magnitude-bit partials; NaN and kStatusNonFinite for a
// non-finite amax (the kernel the dynamic quantisation runs first).
cudaError_t launch_global_scale(const uint32_t* partials, int n, float* g_out, uint32_t* status, cudaStream_t stream);
// The maximum of n amax partials (BF16 magnitude bits) into *amax_bits.
cudaError_t launch_amax_reduce(const uint32_t* partials, int n, uint32_t* amax_bits, cudaStream_t stream);
int quantize_launch_count(const QuantizeArgs& a);

// route.cu
int router_ksplit(int64_t T, int E, int H);
// Kernels launch_router enqueues for these arguments.
int router_launch_count(const RouterArgs& a);
size_t router_parts_elems(int64_t T_max, int E, int H);
// The same bound for the FP32 logits kernels alone (what launch_router uses when it is given
// no digit-plane buffers, as the allocation-free router is).
size_t router_fp32_parts_elems(int64_t T_max, int E, int H);
// Number of amax partials the logits kernel writes for T tokens (grid x * split-K).
int router_amax_partials(int64_t T, int E, int H);
cudaError_t launch_router(RouterArgs a, cudaStream_t stream);
// The top-k stage alone (sums a.ksplit split-K parts of a.parts).
cudaError_t launch_router_topk(const RouterArgs& a, cudaStream_t stream);

// route_tc.cu: logits in exact integer arithmetic on the tensor cores (digit planes, int8 MMAs)
int router_tc_ksplit(int64_t T, int E, int H);
int router_tc_amax_partials(int64_t T);
cudaError_t launch_router_tc(RouterArgs a, cudaStream_t stream);



// ep.cu: expert parallelism with an all-to-all exchange of quantised rows
struct EpPackArgs {
  const int32_t* perm;       // [n_pairs] pair ids in stable expert-major order
  const int32_t* idx;        // [T][topk] experts (global indices)
  const float* wts;          // [T][topk] routing weights
  const uint8_t* xq_codes;   // [T][H/2] the tokens' codes (quantised with the global scale)
  const uint8_t* xq_scales;  // [T][H/16] their block scales, linear
  const int32_t* counts;     // [E] pairs per expert
  int64_t n_pairs;           // T * topk
  int topk, H, E, experts_per_rank;
  uint8_t* send_codes;       // [n_pairs][H/2]
  uint8_t* send_scales;      // [n_pairs][H/16]
  int32_t* send_expert;      // [n_pairs] expert index local to the destination rank
  float* send_w;             // [n_pairs]
  int32_t* send_pos;         // [n_pairs] position of pair p in the send order
  int32_t* rank_counts;      // [E / experts_per_rank] pairs sent to each rank
};
cudaError_t launch_ep_pack(const EpPackArgs& a, cudaStream_t stream);

struct RowsToSegmentsArgs {
  const uint8_t* codes;      // [n_rows][H/2]
  const uint8_t* scales;     // [n_rows][H/16] linear
  const int32_t* expert;     // [n_rows] local expert of each row
  const int32_t* inv;        // [n_rows] position of row i in the grouping (topk = 1)
  const int32_t* offsets;    // [E_local + 1]
  const int32_t* mtile_prefix;  // [E_local + 1]
  int64_t n_rows;
  int H;
  int64_t n_col_tiles;       // H / 64
  uint8_t* seg_codes;        // [rows_cap][H/2]
  uint8_t* seg_sf;           // swizzled
  float* out_rows;           // [n_rows][H] FP32, zeroed
};
cudaError_t launch_rows_to_segments(const RowsToSegmentsArgs& a, cudaStream_t stream);
// out[i] = idx[i] if 0 <= idx[i] < n, else 0 and kStatusBadInput raised (indices from another rank).
cudaError_t launch_check_indices(const int32_t* idx, int64_t count, int n, int32_t* out, uint32_t* status,
                                 cudaStream_t stream);
// out[t] = bf16(sum_j rows[send_pos[t topk + j]]), slots in order.
cudaError_t launch_ep_combine(const float* rows, const int32_t* send_pos, int64_t T, int topk, int H, uint16_t* out,
                              cudaStream_t stream);

// front.cu
// True when the fused front end runs for T tokens on the current device (T <= kFrontMaxT and
// its cooperative grid fits).
bool front_supported(int64_t T, int E, int H);
// Split-K partials the front kernel writes: ksplit * T * E doubles.
int front_ksplit(int E, int H);
cudaError_t launch_front(FrontArgs a, cudaStream_t stream);

// residual.cu
cudaError_t launch_rmsnorm(const RmsNormArgs& a, cudaStream_t stream);

// local_hessian.cu: block-scale search for weight quantisation.
struct LhArgs {
  const uint16_t* w;       // [rows][cols] bf16
  int64_t rows;
  int64_t cols;            // multiple of 16
  const float* hess;       // [cols/16][16][16] local Hessian blocks
  int m;                   // candidates S0 - m .. S0 + m
  const uint32_t* partials;
  int n_partials;
  uint8_t* codes;          // [rows][cols/2]
  uint8_t* scales;         // [rows][cols/16] linear
  float* g_out;
  uint32_t* status;
};
cudaError_t launch_lh_quantize(const LhArgs& a, cudaStream_t stream);

// fp8.cu: per-row E4M3 quantisation for the FP8 W8A8 variant.
struct Fp8RowsArgs {
  const uint16_t* x;       // [rows][cols] bf16, cols % 8 == 0
  int64_t rows, cols;
  uint8_t* codes;          // [rows][cols]
  float* scales;           // [rows]
  uint32_t* status;
};
struct Fp8ScatterArgs {
  const uint16_t* x;       // [T][H] bf16
  int64_t T;
  int H, topk;
  const int32_t* idx;
  const int32_t* inv;
  const int32_t* offsets;
  const int32_t* mtile_prefix;
  uint8_t* seg_codes;      // [rows_cap][H]
  float* seg_scale;        // [rows_cap]
  float* acc;              // [T][H], zeroed
  uint8_t* xq_codes;       // optional [T][H]
  float* xq_scales;        // optional [T]
  uint32_t* status;
};
struct Fp8RequantArgs {
  const float* h;          // [rows][I] FP32
  int64_t rows;            // capacity of the buffers (grid size)
  int I;
  const int32_t* row_pair; // rows with a pair (>= 0) are quantised
  const int32_t* mtile_prefix;  // [E+1]: rows past mtile_prefix[E] * 128 hold no segment
  int E;
  uint8_t* codes;          // [rows][I]
  float* scales;           // [rows]
  uint32_t* status;
};
cudaError_t launch_fp8_quantize_rows(const Fp8RowsArgs& a, cudaStream_t stream);
cudaError_t launch_fp8_quantize_scatter(const Fp8ScatterArgs& a, cudaStream_t stream);
cudaError_t launch_fp8_requant_rows(const Fp8RequantArgs& a, cudaStream_t stream);

// permute.cu
// Grouping kernels: one kernel when T * topk <= kPermSmallPairs, else three.
constexpr int kPermSmallPairs = 4096;
cudaError_t launch_permute(const PermArgs& a, cudaStream_t stream, int* launches);
cudaError_t launch_finalize(const FinalizeArgs& a, cudaStream_t stream);
cudaError_t launch_unswizzle_rows(const uint8_t* sf, int64_t n_col_tiles, const int32_t* src_rows,
                                  int64_t n_rows, int cols16, uint8_t* out, cudaStream_t stream);
cudaError_t launch_export_hq(const uint8_t* hq_codes, const uint8_t* hq_sf, const int32_t* perm,
                             const int32_t* idx, const int32_t* offsets, const int32_t* mtile_prefix,
                             int64_t n_pairs, int I, uint8_t* out_codes, uint8_t* out_sf,
                             cudaStream_t stream);
// Source row r goes to destination row (r / group) * group * mul + add * group + r % group.
cudaError_t launch_repack_sf(const uint8_t* linear, int rows, int cols16, uint8_t* swz,
                             int64_t n_col_tiles, int group, int mul, int add, cudaStream_t stream);

int num_sms();

// Zeroes the first `words` 32-bit words of a call's status header on the stream and records
// the status word as this host thread's latest (read by nvfp4moe_last_device_status).
cudaError_t reset_status(void* header, int words, cudaStream_t stream);

// A failed runtime call (an allocation, an IPC mapping, a copy) stays the host thread's last
// CUDA error, and the launch checks of the next call read that word: every entry point that
// returns NVFP4MOE_ERR_CUDA goes through here, so the next call does not report it again.
inline int cuda_failed() {
  (void)cudaGetLastError();
  return NVFP4MOE_ERR_CUDA;
}

}  // namespace nvfp4moe
