/*
 * nvfp4moe — NVFP4 (W4A4) group-limited mixture-of-experts layer for NVIDIA B200 (sm_100a).
 *
 * C ABI of libnvfp4moe.so.  The layer it computes:
 *
 *   * Router ("Reflection releases Beam ...", section "Mixture-of-Experts details"):
 *     sigmoid scores s = 1/(1+exp(-x.W_r^T)) over E experts; experts split into
 *     n_groups contiguous groups; keep the topk_groups groups with the largest sum of
 *     their two best scores; select the topk best experts inside the kept groups;
 *     weights w = routed_scale * s / sum(selected s).  Computed in FP32 (section
 *     "Residual stream and numerical decisions").
 *   * Experts: SwiGLU MLPs, y = W_down (silu(W_gate x) * (W_up x)), whose weights and
 *     input activations are NVFP4 ("NVFP4 quantization", section "Quantization
 *     scheme"): 4-bit E2M1 values, one FP8 E4M3 scale per 16 consecutive values along a
 *     row, one FP32 global scale per tensor; a value decodes to E2M1 * E4M3 * global.
 *   * Output: out[t] = sum over the token's selected experts of w * y, as BF16.
 *
 * Quantisation rule (the pages give the format, not the rule; this is the library's
 * reading, with every FP32 step one IEEE round-to-nearest-even operation):
 *     g   = A / 2688 (A = max|x| of the tensor; A == 0 -> g = 1)
 *     r_t = 1 / (6 g)
 *     S_b = E4M3_rn_satfinite(amax_b * r_t)      (block of 16 values, unsigned)
 *     d_b = E4M3(S_b) * g,  r_b = (d_b == 0) ? 0 : 1 / d_b
 *     c_i = E2M1_rn_satfinite(x_i * r_b)         (sign kept, also for zero)
 *     byte j of a row holds c_{2j} in its low nibble and c_{2j+1} in its high nibble.
 *   The layer input is quantised with a dynamic global scale (its own amax, all tokens of
 *   the call); the SwiGLU intermediate h (FP32) with a static per-expert global scale g_h
 *   supplied with the weights.
 *
 * Conventions for every call:
 *   * Tensor pointers are DEVICE pointers owned by the caller unless stated otherwise;
 *     row-major, densely packed.  BF16 is the IEEE bfloat16 bit pattern (uint16).
 *   * Calls run on the calling thread's current CUDA device: device pointers are memory
 *     of that device (or, for nvfp4moe_forward_partial_peer's table, memory mapped into
 *     it) and `stream` is a stream of that device.
 *   * `stream` is a cudaStream_t (NULL = legacy default stream).  Calls are asynchronous
 *     on it and allocate nothing; they return after enqueueing work.
 *   * Argument and shape errors are reported synchronously by the return code and
 *     nothing is enqueued.  Errors found on the device (non-finite input, a bounded
 *     wait that ran out) are OR-ed into a status word at the start of the caller's
 *     workspace; nvfp4moe_status_read() (or nvfp4moe_last_device_status() for the
 *     thread's latest call) returns it once the stream has finished.
 *   * Workspaces are caller-allocated device memory, 256-byte aligned, of at least the
 *     size the matching *_workspace_bytes() function returns.  A workspace must not be
 *     used by two calls that can run at the same time.
 *   * Scale layouts: NVFP4MOE_SCALES_LINEAR is [rows][cols/16] bytes.
 *     NVFP4MOE_SCALES_SWIZZLED is the 128x4 tile layout of block-scaled tensor-core
 *     operands: rows padded to a multiple of 128 and scale columns to a multiple of 4
 *     (padding written as zero), 512-byte tiles of 128 rows x 4 scale columns ordered
 *     row-tile-major then column tile, scale (r, c) at byte
 *     (r % 32) * 16 + ((r % 128) / 32) * 4 + c % 4 inside its tile.
 */
#ifndef NVFP4MOE_H
#define NVFP4MOE_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define NVFP4MOE_API __attribute__((visibility("default")))
#else
#define NVFP4MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Return codes. */
typedef enum {
  NVFP4MOE_OK = 0,
  NVFP4MOE_ERR_ARG = -1,        /* NULL pointer, misaligned pointer, bad enum value */
  NVFP4MOE_ERR_SHAPE = -2,      /* shape outside the supported limits */
  NVFP4MOE_ERR_CUDA = -3,       /* a CUDA runtime/driver call failed */
  NVFP4MOE_ERR_WORKSPACE = -4,  /* workspace smaller than required */
  NVFP4MOE_ERR_NONFINITE = -5,  /* device status: the input held NaN or Inf */
  NVFP4MOE_ERR_TIMEOUT = -6,    /* device status: a bounded wait inside a kernel ran out */
  NVFP4MOE_ERR_DEVICE = -7      /* current device is not compute capability 10.0 */
} nvfp4moe_status;

enum { NVFP4MOE_SCALES_LINEAR = 0, NVFP4MOE_SCALES_SWIZZLED = 1 };

/* Layer configuration.  Defaults (nvfp4moe_cfg_default) are the Beam layer:
 * E=256, n_groups=8, topk_groups=4, topk=8, H=5120, I=2560, routed_scale=2.5
 * ("Reflection releases Beam ...", sections "Model architecture and attention" and
 * "Mixture-of-Experts details").
 * Limits: H % 256 == 0, I % 128 == 0, 1 <= E <= 256, E % n_groups == 0,
 * E / n_groups <= 32, 1 <= topk_groups <= n_groups <= 32, 1 <= topk <= 8,
 * topk <= topk_groups * (E / n_groups). */
typedef struct {
  int32_t E;
  int32_t n_groups;
  int32_t topk_groups;
  int32_t topk;
  int32_t H;
  int32_t I;
  float routed_scale;
} nvfp4moe_cfg;

/* Fills *cfg with the Beam defaults.  Returns NVFP4MOE_ERR_ARG if cfg is NULL. */
NVFP4MOE_API int nvfp4moe_cfg_default(nvfp4moe_cfg* cfg);

/* Checks *cfg against the limits above: NVFP4MOE_OK or NVFP4MOE_ERR_SHAPE / _ARG. */
NVFP4MOE_API int nvfp4moe_cfg_check(const nvfp4moe_cfg* cfg);

/* ---------------------------------------------------------------- quantize ----
 * quantize_nvfp4(x) -> codes + block scales + global scale
 * ("NVFP4 quantization", section "Quantization scheme"; rule in the file header).
 *
 *   x_bf16   [rows][cols] BF16, cols % 64 == 0, rows >= 0.
 *   g_in     NULL: the global scale is computed from max|x| (dynamic).  Otherwise a
 *            device pointer to one FP32 global scale used as given (static).
 *   codes    out, [rows][cols/2] bytes (even element in the low nibble).
 *   scales   out, E4M3 block scales in `scale_layout` (linear: rows*cols/16 bytes;
 *            swizzled: nvfp4moe_swizzled_scale_bytes(rows, cols/16) bytes).
 *   g_out    out, device pointer to one FP32: the global scale used (may be NULL).
 *   ws       workspace of nvfp4moe_quantize_workspace_bytes(rows, cols) bytes.
 * A non-finite max|x| (dynamic scale) sets NVFP4MOE_ERR_NONFINITE in the status word;
 * codes, scales and g_out are then unspecified.  Limits: rows < 2^31 - 128, cols < 2^31,
 * rows * cols < 2^40; outside them NVFP4MOE_ERR_SHAPE. */
NVFP4MOE_API size_t nvfp4moe_quantize_workspace_bytes(int64_t rows, int64_t cols);
NVFP4MOE_API size_t nvfp4moe_swizzled_scale_bytes(int64_t rows, int64_t cols16);
NVFP4MOE_API int nvfp4moe_quantize(const void* x_bf16, int64_t rows, int64_t cols, const float* g_in,
                      uint8_t* codes, uint8_t* scales, int32_t scale_layout, float* g_out,
                      void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------- weights, local-Hessian scales ----
 * Weight quantisation with the block-scale search of "NVFP4 quantization", section
 * "Quantization method": for each 16-value block, candidate scales are tried and the one
 * minimising the Hessian-weighted error dW^T H dW is kept.
 *
 *   w_bf16 [rows][cols] BF16 weight matrix (1 <= rows < 2^31, cols % 16 == 0, cols / 16 <=
 *       65535, rows * cols < 2^40, 16-byte aligned);
 *   hess_blocks [cols/16][16][16] FP32: for each 16-column block, the 16x16 diagonal block of
 *       H = X^T X over calibration inputs X of this projection (shared by all rows);
 *   m  0..16: candidates are the E4M3 scale codes S0-m .. S0+m (clamped to 1..0x7E) around the
 *       round-to-nearest code S0 of nvfp4moe_quantize's rule; a zero block keeps scale 0;
 *       m = 0 gives exactly nvfp4moe_quantize with linear scales;
 *   codes out [rows][cols/2] (8-byte aligned), scales out [rows][cols/16] linear, g_out out
 *       device scalar: the global scale fp32(amax / 2688) of the matrix.
 * For each candidate the codes follow the quantisation rule with that block scale, and the
 * error is computed in FP32; a candidate replaces the best only when its error is strictly
 * smaller, in the visiting order S0, S0-1, S0+1, ..., S0-m, S0+m.  The outputs feed
 * nvfp4moe_experts_set.  Workspace: nvfp4moe_quantize_workspace_bytes.  A non-finite weight
 * raises NVFP4MOE_ERR_NONFINITE in the status word (nvfp4moe_status_read). */
NVFP4MOE_API int nvfp4moe_quantize_weights_lh(const void* w_bf16, int64_t rows, int64_t cols,
                                              const float* hess_blocks, int32_t m, uint8_t* codes,
                                              uint8_t* scales, float* g_out, void* ws, size_t ws_bytes,
                                              void* stream);

/* ------------------------------------------------------------------- route ----
 * route(hidden, W_router) -> top-k experts and weights
 * ("Reflection releases Beam ...", section "Mixture-of-Experts details").
 *
 *   hidden_bf16 [T][H] BF16;  w_router [E][H] FP32;  logit_bias [E] FP32 or NULL
 *   (added to the logits before the sigmoid; the Beam router has none).
 *   idx  out [T][topk] int32: selected experts by score descending, equal scores by
 *        lower expert index (the same rule picks the groups).
 *   w    out [T][topk] FP32: routed_scale * s / sum(selected s).
 * Logits, T <= 64: FP32 products accumulated in FP32 so that every product passes through
 * at most 32 FP32 roundings (FMA chains of at most 32 products, or of at most 20 products
 * added by a 3-level FP32 tree); these partial sums, the split-K parts and the bias are
 * added in FP64 and the logit is rounded to FP32 once, so
 *   |logit - exact| <= 32 * 2^-24 * sum_h |x_h W_eh| + 2^-24 |logit| (+ FP64 rounding).
 * Logits, T > 64: integer arithmetic on the tensor cores.  Token row x_t is scaled by a
 * power of two to 22-bit fixed point and expert row W_e to 30-bit fixed point (e_x, e_W: the
 * binary exponents with max|x_t| < 2^e_x, max|W_e| < 2^e_W) and rounded to integers (a BF16
 * element within 2^14 of its row's largest is exact), split into three and four int8 digits,
 * and the 9 most significant digit-pair products are summed in int32 (exact); the classes,
 * split-K parts and bias are added in FP64 and the logit is rounded to FP32 once, so
 *   |logit - exact| <= 2^-24 |logit| + sum_h |x_h - x'_h| |W_eh| + sum_h |x_h| |W_eh - W'_eh|
 *                      + H 2^(e_x + e_W - 28)
 * where x', W' are the fixed-point values (the two sums are at most 2^(e_x - 23) sum_h |W_eh|
 * and 2^(e_W - 31) sum_h |x_h|; the last term covers the dropped digit pairs, the product of
 * the two roundings and the FP64 additions); for Beam's shapes this is below the FP32 bound.
 * A token or expert row with a non-finite element makes its logits NaN.
 * Scores are 1 / (1 + expf(-logit)) in FP32.  nvfp4moe_forward uses the same arithmetic
 * and bounds (for T <= 64 in its fused front-end kernel).  A NaN logit raises
 * NVFP4MOE_ERR_NONFINITE in the status word and ranks below every finite score. */
NVFP4MOE_API size_t nvfp4moe_route_workspace_bytes(const nvfp4moe_cfg* cfg, int64_t T);
NVFP4MOE_API int nvfp4moe_route(const nvfp4moe_cfg* cfg, const void* hidden_bf16, int64_t T,
                   const float* w_router, const float* logit_bias, int32_t* idx, float* w,
                   void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------ route, no allocation ----
 * The pages have no counterpart of this call; it exists for callers that cannot allocate
 * device memory: a host runtime that passes the library only its input and output buffers
 * and allows no device allocation after start-up, or a host framework that owns every
 * device allocation and gives the libraries it embeds no allocator.  Such a caller has no
 * workspace to pass to nvfp4moe_route.
 *
 * Same arguments and results as nvfp4moe_route, minus the workspace; for T > 64 it computes
 * the logits with the FP32 kernel and bound of the T <= 64 path (the integer path's digit
 * planes would not fit the fixed scratch), so idx can differ from nvfp4moe_route's where two
 * scores lie within that bound.  The router's scratch is a fixed array of 9,699,584 bytes of device memory
 * declared by the library; every GPU that loads the library holds it until the process
 * exits.  Limit: the split-K partial sums must fit, which holds whenever T * E <= 1,212,416
 * (T <= 4736 for 256 experts); larger calls return NVFP4MOE_ERR_WORKSPACE and enqueue
 * nothing.  The call allocates nothing.
 *   * The first call on a device looks up that device's address of the array (once per
 *     device, with the device current); make that first call before any stream capture.
 *   * All calls share the one array, which keeps the contents of the last call.  Calls whose
 *     work can overlap on the GPU (different streams, or different host threads, on the
 *     same device) race on it; serialise them. */
NVFP4MOE_API int nvfp4moe_route_noalloc(const nvfp4moe_cfg* cfg, const void* hidden_bf16, int64_t T,
                                        const float* w_router, const float* logit_bias, int32_t* idx,
                                        float* w, void* stream);

/* ----------------------------------------------------------------- experts ----
 * Library-owned, repacked copy of the E experts' NVFP4 weights (the operand layout of
 * the grouped GEMMs).  nvfp4moe_experts_create allocates it (device memory of the
 * current device, about E * 3 * H * I * 0.5625 bytes) and is the only allocating call;
 * nvfp4moe_experts_destroy frees it. */
typedef struct nvfp4moe_experts nvfp4moe_experts;

/* One expert's tensors, as nvfp4moe_quantize produces them with linear scales.
 * Device pointers: gate/up codes [I][H/2], scales [I][H/16]; down codes [H][I/2],
 * scales [H][I/16]; the three code pointers 16-byte aligned (else NVFP4MOE_ERR_ARG).
 * Global scales are host values.  g_h is the static global scale of the SwiGLU
 * intermediate (input of the down projection). */
typedef struct {
  const uint8_t* gate_codes;
  const uint8_t* gate_scales;
  const uint8_t* up_codes;
  const uint8_t* up_scales;
  const uint8_t* down_codes;
  const uint8_t* down_scales;
  float g_gate;
  float g_up;
  float g_down;
  float g_h;
} nvfp4moe_expert_tensors;

NVFP4MOE_API int nvfp4moe_experts_create(const nvfp4moe_cfg* cfg, nvfp4moe_experts** out);
/* Copies expert e (0 <= e < E) into the handle, on `stream`.  The caller's buffers may be
 * reused once the stream has passed this call. */
NVFP4MOE_API int nvfp4moe_experts_set(nvfp4moe_experts* experts, int32_t e, const nvfp4moe_expert_tensors* t,
                         void* stream);
NVFP4MOE_API void nvfp4moe_experts_destroy(nvfp4moe_experts* experts);
/* The handle's configuration (copied out). */
NVFP4MOE_API int nvfp4moe_experts_cfg(const nvfp4moe_experts* experts, nvfp4moe_cfg* cfg);

/* A handle that holds only experts e_begin .. e_begin + e_count - 1 of the layer (one rank's
 * share under expert parallelism: the deployment on the pages spreads the experts over the
 * GPUs of a node).  cfg describes the whole layer; 0 <= e_begin, e_begin + e_count <= E.
 * nvfp4moe_experts_set takes the global expert index, which must lie in the range; the
 * handle's device memory is e_count / E of a full one.  nvfp4moe_experts_create(cfg) is
 * nvfp4moe_experts_create_local(cfg, 0, E). */
NVFP4MOE_API int nvfp4moe_experts_create_local(const nvfp4moe_cfg* cfg, int32_t e_begin, int32_t e_count,
                                               nvfp4moe_experts** out);
NVFP4MOE_API int nvfp4moe_experts_range(const nvfp4moe_experts* experts, int32_t* e_begin, int32_t* e_count);

/* ----------------------------------------------------------------- forward ----
 * moe_forward(hidden, experts) -> out: the whole layer (route, quantise x, group the
 * token/expert pairs by expert, gate/up GEMM + SwiGLU + requantisation of h, down GEMM
 * + weighted combine, BF16 output).
 *
 *   hidden_bf16 [T][H] BF16, 1 <= T <= T_max of the workspace;  w_router [E][H] FP32;
 *   logit_bias [E] FP32 or NULL;  out_bf16 [T][H] BF16 (out).
 *   dbg  NULL on the hot path.  Otherwise every non-NULL member receives a copy of that
 *        intermediate (sizes below), for checking the layer step by step.
 *   ws   workspace of nvfp4moe_forward_workspace_bytes(cfg, T_max) bytes.
 * The grouped GEMMs and finalize are launched with programmatic stream serialization: each may
 * be scheduled onto SMs its predecessor has left and waits on the device for that kernel's
 * results, so a kernel's set-up overlaps the previous one's tail.  Stream order is kept:
 * work enqueued after the call sees the finished output. */
/* Stages of nvfp4moe_forward (for nvfp4moe_debug.events).  Launch order: ROUTE, PERMUTE,
 * QUANTIZE, GATEUP, DOWN, FINALIZE.  The input's global amax is computed inside ROUTE and
 * the rows are written into the expert segments inside QUANTIZE, so the AMAX and GATHER
 * events are recorded back to back (zero time).  For T <= 64 (when the device can hold the
 * cooperative grid) ROUTE is one fused launch that also groups the pairs and quantises x,
 * and the PERMUTE and QUANTIZE events are recorded back to back after it. */
enum {
  NVFP4MOE_STAGE_AMAX = 0,      /* global amax of the input (inside ROUTE) */
  NVFP4MOE_STAGE_ROUTE = 1,     /* router logits (+ amax partials) + group-limited top-k */
  NVFP4MOE_STAGE_QUANTIZE = 2,  /* NVFP4 quantisation of the input into the expert segments
                                   (+ accumulator zeroing) */
  NVFP4MOE_STAGE_PERMUTE = 3,   /* grouping of pairs by expert */
  NVFP4MOE_STAGE_GATHER = 4,    /* (inside QUANTIZE) */
  NVFP4MOE_STAGE_GATEUP = 5,    /* gate/up grouped GEMM + SwiGLU + requantisation */
  NVFP4MOE_STAGE_DOWN = 6,      /* down grouped GEMM + weighted combine */
  NVFP4MOE_STAGE_FINALIZE = 7,  /* FP32 accumulator -> BF16 output */
  NVFP4MOE_NUM_STAGES = 8
};

typedef struct {
  int32_t* idx;        /* [T][topk] selected experts */
  float* w;            /* [T][topk] routing weights */
  float* g_x;          /* [1] global scale of the quantised layer input */
  uint8_t* xq_codes;   /* [T][H/2] quantised layer input */
  uint8_t* xq_scales;  /* [T][H/16] its block scales, linear */
  int32_t* counts;     /* [E] pairs per expert */
  int32_t* offsets;    /* [E+1] exclusive scan of counts */
  int32_t* perm;       /* [T*topk] pair ids (t*topk + j) grouped by expert, tokens ascending */
  uint8_t* hq_codes;   /* [T*topk][I/2] quantised SwiGLU intermediate, rows in perm order */
  uint8_t* hq_scales;  /* [T*topk][I/16] its block scales, linear */
  void* const* events; /* NULL, or 2 * NVFP4MOE_NUM_STAGES cudaEvent_t created by the caller:
                          events[2s] / events[2s+1] are recorded on the stream right before /
                          after stage s (timing of the stages inside a forward); NULL entries
                          are skipped */
  float* logits;       /* [T][E] FP32 router logits (bias included) the selection used */
  uint16_t* x_norm;    /* [T][H] BF16 layer input computed by nvfp4moe_forward_residual */
  uint8_t* xq8_codes;  /* [T][H] E4M3 layer input of nvfp4moe_forward_fp8 */
  float* xq8_scales;   /* [T] its per-token scales */
  float* acc;          /* [T][H] FP32 sums of the weighted expert rows, the values the BF16 output
                          rounds (to nearest, ties to even); nvfp4moe_forward and _residual */
  float* h_f32;        /* [T*topk][I] FP32 SwiGLU product of every pair, rows in perm order, as
                          the gate/up epilogue computes it before requantising it (NVFP4 forward
                          calls); pairs of experts a local handle does not hold are not written */
  /* Failure detection (nvfp4moe_forward, nvfp4moe_forward_residual, nvfp4moe_forward_partial;
   * the other calls ignore these two fields).  Every wait of the call's kernels on another
   * CTA or on the tensor cores is bounded: when one runs out, the kernel raises
   * NVFP4MOE_ERR_TIMEOUT in the status word and returns, and the later kernels of the call
   * (the grouped GEMMs) find the timeout in the status word and do no work, so the call ends
   * with its outputs unspecified but finite work, no access outside its buffers, and the
   * device context usable. */
  uint32_t wait_limit_us;      /* limit of each bounded wait in microseconds; 0: 1.5 s */
  int32_t inject_skip_arrive;  /* test hook, 0 in normal use: c > 0 makes CTA c - 1 of the fused
                                  front-end kernel (T <= 64) skip its arrival at the first grid
                                  barrier, so every CTA's wait there runs out (a timeout that
                                  needs no fault); NVFP4MOE_ERR_ARG when the call does not take
                                  the fused front end, or c < 0 */
  int32_t separate_gemms;      /* 0 (normal use): when the expert segments average fewer than
                                  32 rows (T * topk < 32 * E), the NVFP4 forward calls run the
                                  gate/up and the down GEMM in one persistent launch (each down
                                  tile starts once the gate/up tiles of its rows are done),
                                  bracketed by the GATEUP stage events, DOWN empty; otherwise
                                  two launches.  Nonzero: always two launches, which the GATEUP
                                  and DOWN events time apart */
} nvfp4moe_debug;

NVFP4MOE_API size_t nvfp4moe_forward_workspace_bytes(const nvfp4moe_cfg* cfg, int64_t T_max);
NVFP4MOE_API int nvfp4moe_forward(const nvfp4moe_experts* experts, const void* hidden_bf16, int64_t T,
                     const float* w_router, const float* logit_bias, void* out_bf16,
                     const nvfp4moe_debug* dbg, void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------- forward, expert parallel ----
 * One rank's part of the layer under expert parallelism.  Every rank holds the router and a
 * share of the experts (nvfp4moe_experts_create_local); the ranks gather their tokens (the
 * same hidden_all on every rank), each runs
 *   nvfp4moe_forward_partial(its experts, hidden_all, T_all, ...) -> acc_out [T_all][H] FP32,
 * the acc_out arrays are summed across ranks with a reduce-scatter that leaves each rank the
 * rows of its own tokens, and nvfp4moe_finalize rounds those rows to BF16.  Routing and the
 * input's global scale are computed from hidden_all, so every rank takes the same decisions
 * and the ranks' sums add up to the single-GPU layer (up to the order of FP32 additions).
 *
 *   acc_out  [T][H] FP32 (16-byte aligned, out): the sum over the token's selected slots whose
 *            expert the handle holds of w * y (zero for a token with none), written in full.
 *   hidden_bf16, T, w_router, logit_bias, dbg, ws as for nvfp4moe_forward (same workspace
 *   size); dbg->hq_codes / hq_scales are meaningful only for pairs of the handle's experts.
 * With a full handle, acc_out is the FP32 sum nvfp4moe_forward rounds to BF16.
 *
 * nvfp4moe_finalize: out_bf16[i] = bf16(acc[i]) for n values (n % 8 == 0, n < 2^40, both
 * 16-byte aligned), the layer's output rounding. */
NVFP4MOE_API int nvfp4moe_forward_partial(const nvfp4moe_experts* experts, const void* hidden_bf16, int64_t T,
                                          const float* w_router, const float* logit_bias, float* acc_out,
                                          const nvfp4moe_debug* dbg, void* ws, size_t ws_bytes, void* stream);
NVFP4MOE_API int nvfp4moe_finalize(const float* acc, int64_t n, void* out_bf16, void* stream);

/* ------------------------------------ expert parallel, combine into peer memory ----
 * nvfp4moe_forward_partial with the cross-rank sum folded into the down GEMM: instead of
 * writing [T_all][H] FP32 sums for a reduce-scatter, the down GEMM's epilogue adds each pair's
 * weighted row straight into the accumulator of the rank that owns the token, over NVLink (or
 * into local memory for the caller's own rows), with the same FP32 reductions it uses for a
 * local accumulator: the exchange overlaps the MMAs tile by tile and no reduce-scatter runs.
 *
 *   acc_peers      device array of n_peers pointers (8-byte aligned; pointers 16-byte
 *                  aligned): rank d's FP32 accumulator [rows_per_peer][H], in this process's
 *                  address space (its own allocation, or another GPU's memory mapped with
 *                  nvfp4moe_ipc_open); token t of hidden_all is row t % rows_per_peer of rank
 *                  t / rows_per_peer.  n_peers * rows_per_peer must equal T.
 *   the other arguments as for nvfp4moe_forward_partial.
 * Every owner's accumulator must hold zeros (or the values to add to) before any rank's call
 * starts adding into it, and an owner reads its rows (nvfp4moe_finalize) only after every
 * rank's call has completed: the caller orders both (a barrier between the ranks' streams).
 * The ranks' additions into one row run in no fixed order, so the sums equal the single-GPU
 * layer's up to the order of FP32 additions.  The call writes nothing else in the peers'
 * memory, and reads none of it.  ERR_SHAPE when n_peers * rows_per_peer != T or n_peers < 1.
 *
 * nvfp4moe_ipc_get_handle / _open / _close: CUDA inter-process handles of device memory, for
 * mapping the other ranks' accumulators.  get_handle: the handle (NVFP4MOE_IPC_HANDLE_BYTES
 * opaque bytes) of the device allocation that contains dev_ptr, and dev_ptr's byte offset from
 * that allocation's start.  open (in another process): maps that allocation and returns its
 * start, to which the importer adds the offset.  close unmaps an address that open returned.
 * Errors: ERR_ARG for a null argument or an address that is not device memory; ERR_CUDA when
 * CUDA refuses the handle or the mapping (inter-process handles cover memory from cudaMalloc,
 * not from the virtual-memory calls); ERR_DEVICE off a B200. */
#define NVFP4MOE_IPC_HANDLE_BYTES 64
NVFP4MOE_API int nvfp4moe_forward_partial_peer(const nvfp4moe_experts* experts, const void* hidden_bf16, int64_t T,
                                               const float* w_router, const float* logit_bias,
                                               float* const* acc_peers, int32_t n_peers, int64_t rows_per_peer,
                                               const nvfp4moe_debug* dbg, void* ws, size_t ws_bytes, void* stream);
NVFP4MOE_API int nvfp4moe_ipc_get_handle(const void* dev_ptr, void* handle_out, int64_t* offset_out);
NVFP4MOE_API int nvfp4moe_ipc_open(const void* handle, void** dev_ptr_out);
NVFP4MOE_API int nvfp4moe_ipc_close(void* dev_ptr);

/* ------------------------------- expert parallelism, all-to-all exchange of quantised rows ----
 * The exchange of the experts' placement across devices ("Reflection releases Beam ...",
 * section "Tool calling and multi-node setups": experts on the devices, a device count that
 * divides the 256 experts) in which each token's pairs travel to the experts, for batches where
 * gathering every rank's tokens costs more than sending the pairs.  Rank d of G (G divides E)
 * holds experts d E/G .. (d+1) E/G - 1 (nvfp4moe_experts_create_local) and the whole router;
 * every rank passes the same T.  One step on rank d:
 *   1. nvfp4moe_amax(x_d) -> amax_d; the ranks' values are combined with a maximum (an
 *      all-reduce over int32, the values being below 2^15).
 *   2. nvfp4moe_ep_dispatch(x_d, amax): routes the rank's tokens, groups their T*topk pairs by
 *      expert (stable: expert, then token, then slot), quantises the tokens with the global
 *      scale g = A / 2688 of the combined amax A (so every code and scale equals the
 *      single-GPU layer's on the concatenated batch), and writes the pairs in that order:
 *      send_codes [P][H/2], send_scales [P][H/16] (linear), send_expert [P] (the expert's index
 *      on its rank), send_w [P] (routing weight), send_pos [T*topk] (position of pair t*topk+j
 *      in the send order) and rank_counts [G] (pairs for each rank, in rank order), P = T*topk.
 *   3. the caller's all-to-all sends rank_counts[e] consecutive rows (and their expert and
 *      weight entries) to rank e.
 *   4. nvfp4moe_ep_experts(local handle, received rows) -> out_rows [n][H] FP32: row i is
 *      w_i * (the expert's SwiGLU MLP of the row), through the layer's grouped GEMMs.
 *   5. the caller's all-to-all returns those rows (the reverse split).
 *   6. nvfp4moe_ep_combine(returned rows, send_pos) -> out [T][H] BF16: for each token the
 *      FP32 sum of its topk rows in slot order, rounded to nearest even.
 * The result equals nvfp4moe_forward on the concatenated batch up to the order of the FP32
 * additions of a token's rows (fixed here, atomic there).
 *
 * nvfp4moe_amax: amax_bits[0] = max over the rows x cols BF16 values of (bits & 0x7FFF) (the
 *   magnitude's bit pattern: 0x7F80 and above mean Inf or NaN; 0 for no rows).  cols % 8 == 0;
 *   workspace nvfp4moe_quantize_workspace_bytes(rows, cols).  amax_bits: device, 4-byte aligned.
 * nvfp4moe_ep_dispatch: cfg of the whole layer; n_ranks divides cfg->E; amax_bits (device) the
 *   combined amax; send buffers device, send_codes 16-byte and send_scales 4-byte aligned;
 *   rank_counts device [n_ranks].  A non-finite amax raises NVFP4MOE_ERR_NONFINITE in the
 *   status word and leaves the codes unwritten.
 * nvfp4moe_ep_experts: the rank's handle; codes [n][H/2] (16-byte aligned), scales [n][H/16]
 *   (4-byte aligned), expert [n] (0 <= expert < the handle's count), w [n] (device), amax_bits
 *   as for dispatch; out_rows [n][H] FP32 (16-byte aligned, written in full).  n from 0 to
 *   2^23; the workspace of nvfp4moe_ep_experts_workspace_bytes(cfg, handle's count, n).  The
 *   expert indices arrive from other ranks and are checked on the device: one out of range is
 *   replaced by 0 (so every access stays inside the buffers) and the status word reports
 *   NVFP4MOE_ERR_ARG.
 * nvfp4moe_ep_combine: rows [T*topk][H] FP32 in send order (16-byte aligned), send_pos from
 *   dispatch, out_bf16 [T][H] (16-byte aligned); topk <= 8, H % 64 == 0.
 * All arguments on the device are owned by the caller; all calls are asynchronous on `stream`. */
NVFP4MOE_API int nvfp4moe_amax(const void* x_bf16, int64_t rows, int64_t cols, uint32_t* amax_bits, void* ws,
                               size_t ws_bytes, void* stream);
NVFP4MOE_API size_t nvfp4moe_ep_dispatch_workspace_bytes(const nvfp4moe_cfg* cfg, int64_t T);
NVFP4MOE_API int nvfp4moe_ep_dispatch(const nvfp4moe_cfg* cfg, int32_t n_ranks, const void* hidden_bf16, int64_t T,
                                      const float* w_router, const float* logit_bias, const uint32_t* amax_bits,
                                      uint8_t* send_codes, uint8_t* send_scales, int32_t* send_expert, float* send_w,
                                      int32_t* send_pos, int32_t* rank_counts, void* ws, size_t ws_bytes,
                                      void* stream);
NVFP4MOE_API size_t nvfp4moe_ep_experts_workspace_bytes(const nvfp4moe_cfg* cfg, int32_t e_count, int64_t n_rows_max);
NVFP4MOE_API int nvfp4moe_ep_experts(const nvfp4moe_experts* experts, const uint8_t* codes, const uint8_t* scales,
                                     const int32_t* expert, const float* w, int64_t n_rows,
                                     const uint32_t* amax_bits, float* out_rows, void* ws, size_t ws_bytes,
                                     void* stream);
NVFP4MOE_API int nvfp4moe_ep_combine(const float* rows, const int32_t* send_pos, int64_t T, int32_t topk, int32_t H,
                                     void* out_bf16, void* stream);

/* ------------------------------------------------------------------ status ----
 * Waits for `stream`, then returns the device-side status of the last call that used
 * workspace `ws` (NVFP4MOE_OK, _ERR_NONFINITE, _ERR_TIMEOUT, or _ERR_ARG for an argument the
 * device found out of range; _ERR_CUDA if the wait or the read failed). */
NVFP4MOE_API int nvfp4moe_status_read(const void* ws, void* stream);
NVFP4MOE_API const char* nvfp4moe_status_string(int status);

/* Waits for `stream`, then returns the device-side status of the last call on this host
 * thread that enqueued work with a status word: the quantize, route, forward and FP8 calls
 * (their workspace's word) and nvfp4moe_route_noalloc (the word of the library's fixed
 * scratch, which only this call can read).  Same results as nvfp4moe_status_read; also
 * NVFP4MOE_ERR_ARG when no such call has been made on this thread.  The workspace that call
 * used must still be allocated. */
NVFP4MOE_API int nvfp4moe_last_device_status(void* stream);

/* Workspace bytes of nvfp4moe_forward for up to T_max tokens (the value of
 * nvfp4moe_forward_workspace_bytes; 0 for an invalid cfg or T_max < 1). */
NVFP4MOE_API size_t nvfp4moe_workspace_bytes(const nvfp4moe_cfg* cfg, int64_t T_max);

/* ------------------------------------------------------- forward, residual ----
 * The layer with its neighbours on the residual stream fused in ("Reflection releases Beam
 * ...", section "Residual stream and numerical decisions": at step k a sublayer output is
 * added with weight 1/sqrt(k) and the stream kept with weight sqrt((k-1)/k); norms in FP32):
 *
 *   x  = bf16(fp32(fp32(h * r) * gamma)),  r = fp32(1 / sqrt(mean_j h[t][j]^2 + eps))
 *        (mean, root and reciprocal in FP64; the RMSNorm of the residual stream)
 *   h' = bf16(fp32(a * h) + fp32(b * moe(x))),  a = fp32(sqrt((k-1)/k)), b = fp32(1/sqrt(k))
 *        (moe(x) is the FP32 accumulator nvfp4moe_forward rounds to BF16; here it goes into
 *        the residual add without that rounding)
 *
 *   h_bf16 [T][H] BF16 residual stream;  gamma [H] FP32 norm weight (16-byte aligned);
 *   eps >= 0;  step_k >= 1 (k = 1 keeps only the layer output);  h_out_bf16 [T][H] BF16
 *   (out), may be h_bf16 itself (in-place update of the stream).  w_router, logit_bias,
 *   dbg, ws as for nvfp4moe_forward (same workspace size); dbg->x_norm receives x.
 * One more launch than nvfp4moe_forward (the norm); the residual add is part of finalize. */
NVFP4MOE_API int nvfp4moe_forward_residual(const nvfp4moe_experts* experts, const void* h_bf16, int64_t T,
                                           const float* gamma, float eps, int32_t step_k,
                                           const float* w_router, const float* logit_bias, void* h_out_bf16,
                                           const nvfp4moe_debug* dbg, void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------- FP8 W8A8 variant ----
 * The same layer with FP8 experts ("FP8 quantization", section "Quantization scheme": E4M3
 * weights with a fixed scale per output channel, E4M3 input activations with a scale per
 * token computed at run time; the router stays in high precision; section "Quantization
 * method": round to nearest).  Rule for one row v (a weight output channel, a token's input
 * row, or a pair's SwiGLU product):
 *   s = fp32(max|v| / 448)  (s = 1 when max|v| = 0),  code = E4M3_rn_satfinite(fp32(v / s))
 * (IEEE division, sign kept).  The down projection's input is the SwiGLU product h in FP32,
 * quantised per (token, slot) row.  The GEMMs multiply E4M3 codes with FP32 accumulation and
 * apply the row scales in the epilogue; routing, grouping and the weighted combine are the
 * NVFP4 layer's.
 *
 * nvfp4moe_quantize_fp8: x_bf16 [rows][cols] BF16 (16-byte aligned, cols % 16 == 0) ->
 *   codes [rows][cols] (8-byte aligned) and scales [rows] FP32.  Limits: 1 <= rows < 2^31,
 *   cols < 2^31, rows * cols < 2^40; outside them NVFP4MOE_ERR_SHAPE.  Workspace:
 *   nvfp4moe_quantize_workspace_bytes.  A non-finite row raises NVFP4MOE_ERR_NONFINITE in the
 *   status word and leaves that row's outputs unwritten. */
NVFP4MOE_API int nvfp4moe_quantize_fp8(const void* x_bf16, int64_t rows, int64_t cols, uint8_t* codes,
                                       float* scales, void* ws, size_t ws_bytes, void* stream);

/* Library-owned FP8 experts (about E * 3 * H * I bytes of device memory), laid out for the
 * FP8 grouped GEMMs; same life cycle as nvfp4moe_experts. */
typedef struct nvfp4moe_fp8_experts nvfp4moe_fp8_experts;

/* One expert's FP8 tensors, as nvfp4moe_quantize_fp8 produces them.  Device pointers:
 * gate/up codes [I][H] (16-byte aligned), scales [I] FP32; down codes [H][I] (16-byte
 * aligned), scales [H] FP32. */
typedef struct {
  const uint8_t* gate_codes;
  const float* gate_scales;
  const uint8_t* up_codes;
  const float* up_scales;
  const uint8_t* down_codes;
  const float* down_scales;
} nvfp4moe_fp8_expert_tensors;

NVFP4MOE_API int nvfp4moe_fp8_experts_create(const nvfp4moe_cfg* cfg, nvfp4moe_fp8_experts** out);
/* Copies expert e into the handle on `stream` (experts never set hold zero weights). */
NVFP4MOE_API int nvfp4moe_fp8_experts_set(nvfp4moe_fp8_experts* experts, int32_t e,
                                          const nvfp4moe_fp8_expert_tensors* t, void* stream);
NVFP4MOE_API void nvfp4moe_fp8_experts_destroy(nvfp4moe_fp8_experts* experts);

/* The FP8 layer: arguments as nvfp4moe_forward, with its own workspace size.  dbg: idx, w,
 * counts, offsets, perm, logits, xq8_codes and xq8_scales are filled; the NVFP4-specific
 * members and events are ignored.  Launches: routing and grouping (T <= 64: the fused
 * front-end launch of nvfp4moe_forward without its NVFP4 quantisation; above: router 2 or 4,
 * grouping 1 or 3), quantise-scatter, gate/up GEMM, requantisation of h, down GEMM,
 * finalize. */
NVFP4MOE_API size_t nvfp4moe_forward_fp8_workspace_bytes(const nvfp4moe_cfg* cfg, int64_t T_max);
NVFP4MOE_API int nvfp4moe_forward_fp8(const nvfp4moe_fp8_experts* experts, const void* hidden_bf16, int64_t T,
                                      const float* w_router, const float* logit_bias, void* out_bf16,
                                      const nvfp4moe_debug* dbg, void* ws, size_t ws_bytes, void* stream);

/* Number of kernels enqueued by the last call on this host thread that enqueues work
 * (the quantize, route, experts_set, forward and finalize families; nvfp4moe_route_noalloc
 * leaves the count unchanged), for launch accounting in benchmarks.  A call that returns an
 * error before enqueuing anything reports 0. */
NVFP4MOE_API int32_t nvfp4moe_last_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* NVFP4MOE_H */
