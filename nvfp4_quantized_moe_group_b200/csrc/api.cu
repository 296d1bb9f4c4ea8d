// C ABI of libnvfp4moe: argument checking, workspace layout and the launch sequences of the
// quantize / route / forward calls.  Declarations and contracts are in nvfp4moe.h.
#include <cmath>
#include <cstring>
#include <vector>

#include "common.cuh"
#include "kernels.h"

using namespace nvfp4moe;

struct nvfp4moe_experts {
  nvfp4moe_cfg cfg;
  int device;
  int e_begin, e_count;  // the experts this handle holds (all E, or one rank's share)
  uint8_t* w13_codes;   // tiled (see launch_tile_weights), gate/up rows interleaved per 64-row group
  uint8_t* w13_sf;      // swizzled, [E][2I/128 row tiles][H/64 column tiles][512]
  uint8_t* wd_codes;    // tiled, [E][H/128][ceil(I/256)][128][128]
  uint8_t* wd_sf;       // swizzled, [E][H/128][I/64][512]
  float* g_gate;        // [E] device
  float* g_up;
  float* g_h;
  float* alpha_down;    // [E] g_h * g_down
};

// FP8 W8A8 experts ("FP8 quantization", section "Quantization scheme").
struct nvfp4moe_fp8_experts {
  nvfp4moe_cfg cfg;
  int device;
  uint8_t* w13_codes;   // tiled like the NVFP4 codes with 128-value K blocks, gate/up interleaved per 64 rows
  float* w13_scale;     // [E][2I] channel scales in the same interleaved order
  uint8_t* wd_codes;    // tiled, [E][H/128][I/128][128][128]
  float* wd_scale;      // [E][H]
};

namespace {

thread_local int32_t g_launches = 0;
thread_local const void* g_last_status = nullptr;   // status word of this thread's latest call

constexpr size_t kAlign = 256;
// Fused GEMM launch: gate/up items claimed between an expert's last gate/up item and its first
// down item, per SM of the grid (about the items a CTA has in flight, so that the down items
// rarely wait for h).
constexpr int kFusedLagPerSm = 4;

size_t align_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }


int check_device() {
  int dev = 0, major = 0, minor = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cuda_failed();
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
    return cuda_failed();
  return (major == 10 && minor == 0) ? NVFP4MOE_OK : NVFP4MOE_ERR_DEVICE;
}

// Carves a workspace into 256-byte aligned pieces.
struct Carver {
  uint8_t* base;
  size_t off = 0;
  explicit Carver(void* b) : base(static_cast<uint8_t*>(b)) {}
  template <typename T>
  T* take(size_t count) {
    T* p = base ? reinterpret_cast<T*>(base + off) : nullptr;
    off += align_up(count * sizeof(T));
    return p;
  }
};

int64_t round128(int64_t v) { return (v + 127) / 128 * 128; }

struct QuantWs {
  WsHeader* hdr;
  uint32_t* partials;
  float* g;                // the dynamic global scale when the caller asks for none back
  size_t bytes;
};

QuantWs carve_quant(void* ws) {
  Carver c(ws);
  QuantWs q;
  q.hdr = c.take<WsHeader>(1);
  q.partials = c.take<uint32_t>(kMaxAmaxPartials);
  q.g = c.take<float>(1);
  q.bytes = c.off;
  return q;
}

// Scratch of the integer tensor-core router (T >= kRouterTcMinT): digit planes of the expert
// rows and the row exponents.  The token rows' planes (3 T H bytes) go to a buffer the caller
// names when it is large enough (in the forward, the expert-segment input buffer, which is
// written only afterwards), else to their own.
struct RouterTcWs {
  uint8_t* w_digits = nullptr;
  uint8_t* x_digits = nullptr;   // own planes, when the caller's buffer is too small
  int32_t* x_exp = nullptr;
  int32_t* w_exp = nullptr;
};

RouterTcWs carve_router_tc(Carver& c, const nvfp4moe_cfg& cfg, int64_t T, size_t shared_bytes) {
  RouterTcWs r;
  if (T < kRouterTcMinT) return r;
  r.w_digits = c.take<uint8_t>((size_t)kRouterWDigits * cfg.E * cfg.H);
  if (shared_bytes < (size_t)kRouterXDigits * T * cfg.H)
    r.x_digits = c.take<uint8_t>((size_t)kRouterXDigits * T * cfg.H);
  r.x_exp = c.take<int32_t>(T);
  r.w_exp = c.take<int32_t>(cfg.E);
  return r;
}

void set_router_tc(RouterArgs& r, const RouterTcWs& w, uint8_t* shared) {
  r.x_digits = w.w_digits == nullptr ? nullptr : (w.x_digits != nullptr ? w.x_digits : shared);
  r.w_digits = w.w_digits;
  r.x_exp = w.x_exp;
  r.w_exp = w.w_exp;
}

struct RouteWs {
  WsHeader* hdr;
  double* parts;
  uint8_t* x_digits;
  RouterTcWs tc;
  size_t bytes;
};

RouteWs carve_route(void* ws, const nvfp4moe_cfg& cfg, int64_t T) {
  Carver c(ws);
  RouteWs r;
  r.hdr = c.take<WsHeader>(1);
  r.parts = c.take<double>(router_parts_elems(T, cfg.E, cfg.H));
  r.x_digits = T >= kRouterTcMinT ? c.take<uint8_t>((size_t)kRouterXDigits * T * cfg.H) : nullptr;
  r.tc = carve_router_tc(c, cfg, T, T >= kRouterTcMinT ? (size_t)kRouterXDigits * T * cfg.H : 0);
  r.bytes = c.off;
  return r;
}

int64_t rows_capacity(const nvfp4moe_cfg& cfg, int64_t T) {
  const int64_t pairs = T * cfg.topk;
  const int64_t pad = 127 * (pairs < cfg.E ? pairs : cfg.E);
  return round128(pairs + pad);
}

struct ForwardWs {
  WsHeader* hdr;
  int32_t* dep;            // per 128-row tile: gate/up epilogue warps done (fused GEMM launch)
  uint32_t* partials;
  float* g_x;
  double* parts;
  int32_t* idx;
  float* wts;
  uint8_t* xq_codes;
  uint8_t* xq_sf;
  float* acc;
  int32_t* chunk_counts;
  int32_t* chunk_base;
  int32_t* counts;
  int32_t* offsets;
  int32_t* mtile_prefix;
  int32_t* perm;
  int32_t* inv;
  int32_t* row_pair;
  uint8_t* a_codes;
  uint8_t* a_sf;
  uint8_t* hq_codes;
  uint8_t* hq_sf;
  uint16_t* x_norm;        // residual forward: the normalised layer input
  RouterTcWs tc;           // token-row digit planes alias a_codes (when rows_cap H / 2 >= 3 T H)
  int64_t rows_cap;
  size_t bytes;
};

ForwardWs carve_forward(void* ws, const nvfp4moe_cfg& cfg, int64_t T) {
  Carver c(ws);
  ForwardWs f;
  const int64_t pairs = T * cfg.topk;
  const int64_t n_chunks = (T + kPermChunkTokens - 1) / kPermChunkTokens;
  f.rows_cap = rows_capacity(cfg, T);
  f.hdr = c.take<WsHeader>(1);
  f.dep = c.take<int32_t>(f.rows_cap / kBlockM);   // right after the header: zeroed with it
  const int n_part = router_amax_partials(T, cfg.E, cfg.H);
  f.partials = c.take<uint32_t>(n_part > kMaxAmaxPartials ? n_part : kMaxAmaxPartials);
  f.g_x = c.take<float>(1);
  size_t n_parts = router_parts_elems(T, cfg.E, cfg.H);
  if (T <= kFrontMaxT) {
    const size_t nf = (size_t)front_ksplit(cfg.E, cfg.H) * (size_t)T * (size_t)cfg.E;
    if (nf > n_parts) n_parts = nf;
  }
  f.parts = c.take<double>(n_parts);
  f.idx = c.take<int32_t>(pairs);
  f.wts = c.take<float>(pairs);
  f.xq_codes = c.take<uint8_t>(T * cfg.H / 2);
  f.xq_sf = c.take<uint8_t>(round128(T) * cfg.H / 16);
  f.acc = c.take<float>(T * cfg.H);
  f.chunk_counts = c.take<int32_t>(n_chunks * cfg.E);
  f.chunk_base = c.take<int32_t>(n_chunks * cfg.E);
  f.counts = c.take<int32_t>(cfg.E);
  f.offsets = c.take<int32_t>(cfg.E + 1);
  f.mtile_prefix = c.take<int32_t>(cfg.E + 1);
  f.perm = c.take<int32_t>(pairs);
  f.inv = c.take<int32_t>(pairs);
  f.row_pair = c.take<int32_t>(f.rows_cap);
  f.a_codes = c.take<uint8_t>(f.rows_cap * cfg.H / 2);
  f.a_sf = c.take<uint8_t>(f.rows_cap * cfg.H / 16);
  f.hq_codes = c.take<uint8_t>(f.rows_cap * cfg.I / 2);
  f.hq_sf = c.take<uint8_t>(f.rows_cap * cfg.I / 16);
  f.x_norm = c.take<uint16_t>(T * cfg.H);
  f.tc = carve_router_tc(c, cfg, T, (size_t)f.rows_cap * cfg.H / 2);
  f.bytes = c.off;
  return f;
}

struct ForwardFp8Ws {
  WsHeader* hdr;
  uint32_t* partials;
  double* parts;
  int32_t* idx;
  float* wts;
  float* acc;
  int32_t* chunk_counts;
  int32_t* chunk_base;
  int32_t* counts;
  int32_t* offsets;
  int32_t* mtile_prefix;
  int32_t* perm;
  int32_t* inv;
  int32_t* row_pair;
  uint8_t* a_codes;     // [rows_cap][H] E4M3
  float* a_scale;       // [rows_cap]
  float* h32;           // [rows_cap][I]
  uint8_t* hq;          // [rows_cap][I] E4M3
  float* h_scale;       // [rows_cap]
  RouterTcWs tc;        // token-row digit planes alias a_codes (when rows_cap H >= 3 T H)
  int64_t rows_cap;
  size_t bytes;
};

ForwardFp8Ws carve_forward_fp8(void* ws, const nvfp4moe_cfg& cfg, int64_t T) {
  Carver c(ws);
  ForwardFp8Ws f;
  const int64_t pairs = T * cfg.topk;
  const int64_t n_chunks = (T + kPermChunkTokens - 1) / kPermChunkTokens;
  f.rows_cap = rows_capacity(cfg, T);
  f.hdr = c.take<WsHeader>(1);
  const int n_part = router_amax_partials(T, cfg.E, cfg.H);
  f.partials = c.take<uint32_t>(n_part > kMaxAmaxPartials ? n_part : kMaxAmaxPartials);
  size_t n_parts = router_parts_elems(T, cfg.E, cfg.H);
  if (T <= kFrontMaxT) {
    const size_t nf = (size_t)front_ksplit(cfg.E, cfg.H) * (size_t)T * (size_t)cfg.E;
    if (nf > n_parts) n_parts = nf;
  }
  f.parts = c.take<double>(n_parts);
  f.idx = c.take<int32_t>(pairs);
  f.wts = c.take<float>(pairs);
  f.acc = c.take<float>(T * cfg.H);
  f.chunk_counts = c.take<int32_t>(n_chunks * cfg.E);
  f.chunk_base = c.take<int32_t>(n_chunks * cfg.E);
  f.counts = c.take<int32_t>(cfg.E);
  f.offsets = c.take<int32_t>(cfg.E + 1);
  f.mtile_prefix = c.take<int32_t>(cfg.E + 1);
  f.perm = c.take<int32_t>(pairs);
  f.inv = c.take<int32_t>(pairs);
  f.row_pair = c.take<int32_t>(f.rows_cap);
  f.a_codes = c.take<uint8_t>(f.rows_cap * cfg.H);
  f.a_scale = c.take<float>(f.rows_cap);
  f.h32 = c.take<float>(f.rows_cap * cfg.I);
  f.hq = c.take<uint8_t>(f.rows_cap * cfg.I);
  f.h_scale = c.take<float>(f.rows_cap);
  f.tc = carve_router_tc(c, cfg, T, (size_t)f.rows_cap * cfg.H);
  f.bytes = c.off;
  return f;
}

// Expert parallelism, all-to-all exchange: the dispatching rank's scratch (routing of its own
// tokens, their grouping by expert, the global scale, the tokens quantised token-major).
struct EpDispatchWs {
  WsHeader* hdr;
  double* parts;
  RouterTcWs tc;
  int32_t* idx;
  float* wts;
  int32_t* chunk_counts;
  int32_t* chunk_base;
  int32_t* counts;
  int32_t* offsets;
  int32_t* mtile_prefix;
  int32_t* perm;
  int32_t* inv;
  int32_t* row_pair;
  float* g;
  uint8_t* xq_codes;
  uint8_t* xq_scales;
  size_t bytes;
};

EpDispatchWs carve_ep_dispatch(void* ws, const nvfp4moe_cfg& cfg, int64_t T) {
  Carver c(ws);
  EpDispatchWs d;
  const int64_t pairs = T * cfg.topk;
  const int64_t n_chunks = (T + kPermChunkTokens - 1) / kPermChunkTokens;
  d.hdr = c.take<WsHeader>(1);
  d.parts = c.take<double>(router_parts_elems(T, cfg.E, cfg.H));
  d.tc = carve_router_tc(c, cfg, T, 0);
  d.idx = c.take<int32_t>(pairs);
  d.wts = c.take<float>(pairs);
  d.chunk_counts = c.take<int32_t>(n_chunks * cfg.E);
  d.chunk_base = c.take<int32_t>(n_chunks * cfg.E);
  d.counts = c.take<int32_t>(cfg.E);
  d.offsets = c.take<int32_t>(cfg.E + 1);
  d.mtile_prefix = c.take<int32_t>(cfg.E + 1);
  d.perm = c.take<int32_t>(pairs);
  d.inv = c.take<int32_t>(pairs);
  d.row_pair = c.take<int32_t>(rows_capacity(cfg, T));
  d.g = c.take<float>(1);
  d.xq_codes = c.take<uint8_t>(T * cfg.H / 2);
  d.xq_scales = c.take<uint8_t>(T * cfg.H / 16);
  d.bytes = c.off;
  return d;
}

// The receiving rank's scratch: the grouping of the received rows by local expert (one slot
// per row), the global scale, the rows in padded expert segments and the requantised h.
struct EpExpertsWs {
  WsHeader* hdr;
  float* g_x;
  int32_t* chunk_counts;
  int32_t* chunk_base;
  int32_t* counts;
  int32_t* offsets;
  int32_t* mtile_prefix;
  int32_t* perm;
  int32_t* inv;
  int32_t* row_pair;
  int32_t* expert;         // the received rows' expert indices, checked
  uint8_t* a_codes;
  uint8_t* a_sf;
  uint8_t* hq_codes;
  uint8_t* hq_sf;
  int64_t rows_cap;
  size_t bytes;
};

// cfg_local: the layer's cfg with E = the handle's expert count and topk = 1.
EpExpertsWs carve_ep_experts(void* ws, const nvfp4moe_cfg& cfg_local, int64_t n) {
  Carver c(ws);
  EpExpertsWs f;
  const int64_t n_chunks = (n + kPermChunkTokens - 1) / kPermChunkTokens;
  f.rows_cap = rows_capacity(cfg_local, n);
  f.hdr = c.take<WsHeader>(1);
  f.g_x = c.take<float>(1);
  f.chunk_counts = c.take<int32_t>(n_chunks * cfg_local.E);
  f.chunk_base = c.take<int32_t>(n_chunks * cfg_local.E);
  f.counts = c.take<int32_t>(cfg_local.E);
  f.offsets = c.take<int32_t>(cfg_local.E + 1);
  f.mtile_prefix = c.take<int32_t>(cfg_local.E + 1);
  f.perm = c.take<int32_t>(n);
  f.inv = c.take<int32_t>(n);
  f.row_pair = c.take<int32_t>(f.rows_cap);
  f.expert = c.take<int32_t>(n);
  f.a_codes = c.take<uint8_t>(f.rows_cap * cfg_local.H / 2);
  f.a_sf = c.take<uint8_t>(f.rows_cap * cfg_local.H / 16);
  f.hq_codes = c.take<uint8_t>(f.rows_cap * cfg_local.I / 2);
  f.hq_sf = c.take<uint8_t>(f.rows_cap * cfg_local.I / 16);
  f.bytes = c.off;
  return f;
}

__global__ void set_expert_scalars_kernel(float* g_gate, float* g_up, float* g_h, float* alpha, int e,
                                          float gg, float gu, float gh, float gd) {
  g_gate[e] = gg;
  g_up[e] = gu;
  g_h[e] = gh;
  alpha[e] = __fmul_rn(gh, gd);
}

// Weighted residual add fused into finalize: out = bf16(a * h + b * layer output).
struct Residual {
  const uint16_t* h;
  float a, b;
};

struct StageEvents {
  void* const* ev;
  cudaStream_t s;
  void mark(int stage, int which) const {
    if (ev != nullptr && ev[2 * stage + which] != nullptr)
      cudaEventRecord(static_cast<cudaEvent_t>(ev[2 * stage + which]), s);
  }
};

}  // namespace

cudaError_t nvfp4moe::reset_status(void* header, int words, cudaStream_t stream) {
  g_last_status = header;
  return cudaMemsetAsync(header, 0, (size_t)words * sizeof(uint32_t), stream);
}

extern "C" {

int nvfp4moe_cfg_default(nvfp4moe_cfg* cfg) {
  if (cfg == nullptr) return NVFP4MOE_ERR_ARG;
  cfg->E = 256;
  cfg->n_groups = 8;
  cfg->topk_groups = 4;
  cfg->topk = 8;
  cfg->H = 5120;
  cfg->I = 2560;
  cfg->routed_scale = 2.5f;
  return NVFP4MOE_OK;
}

int nvfp4moe_cfg_check(const nvfp4moe_cfg* c) {
  if (c == nullptr) return NVFP4MOE_ERR_ARG;
  if (c->H <= 0 || c->I <= 0 || c->H % 256 != 0 || c->I % 128 != 0) return NVFP4MOE_ERR_SHAPE;
  if (c->E < 1 || c->E > 256 || c->n_groups < 1 || c->n_groups > 32 || c->E % c->n_groups != 0)
    return NVFP4MOE_ERR_SHAPE;
  if (c->E / c->n_groups > 32) return NVFP4MOE_ERR_SHAPE;
  if (c->topk_groups < 1 || c->topk_groups > c->n_groups) return NVFP4MOE_ERR_SHAPE;
  if (c->topk < 1 || c->topk > 8 || c->topk > c->topk_groups * (c->E / c->n_groups))
    return NVFP4MOE_ERR_SHAPE;
  if (!(c->routed_scale == c->routed_scale)) return NVFP4MOE_ERR_ARG;
  return NVFP4MOE_OK;
}

size_t nvfp4moe_swizzled_scale_bytes(int64_t rows, int64_t cols16) {
  if (rows < 0 || cols16 < 0) return 0;
  return (size_t)round128(rows) * (size_t)((cols16 + 3) / 4 * 4);
}

size_t nvfp4moe_quantize_workspace_bytes(int64_t rows, int64_t cols) {
  (void)rows;
  (void)cols;
  return carve_quant(nullptr).bytes;
}

int nvfp4moe_quantize(const void* x_bf16, int64_t rows, int64_t cols, const float* g_in, uint8_t* codes,
                      uint8_t* scales, int32_t scale_layout, float* g_out, void* ws, size_t ws_bytes,
                      void* stream) {
  g_launches = 0;
  // rows and cols bounded first so that rows * cols cannot overflow
  if (rows < 0 || cols <= 0 || cols % 64 != 0 || cols >= ((int64_t)1 << 31)) return NVFP4MOE_ERR_SHAPE;
  if (rows >= ((int64_t)1 << 31) - 128) return NVFP4MOE_ERR_SHAPE;   // one CTA per (padded) row
  if (rows * cols >= ((int64_t)1 << 40)) return NVFP4MOE_ERR_SHAPE;
  if (scale_layout != NVFP4MOE_SCALES_LINEAR && scale_layout != NVFP4MOE_SCALES_SWIZZLED)
    return NVFP4MOE_ERR_ARG;
  if (ws == nullptr || !aligned(ws, kAlign)) return NVFP4MOE_ERR_ARG;
  if (rows > 0 && (scales == nullptr || !aligned(scales, 4))) return NVFP4MOE_ERR_ARG;
  if (rows > 0 && (x_bf16 == nullptr || codes == nullptr || !aligned(x_bf16, 16) || !aligned(codes, 16)))
    return NVFP4MOE_ERR_ARG;
  const QuantWs q = carve_quant(ws);
  if (ws_bytes < q.bytes) return NVFP4MOE_ERR_WORKSPACE;
  int st = check_device();
  if (st != NVFP4MOE_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (reset_status(q.hdr, 1, s) != cudaSuccess) return cuda_failed();
  int blocks = 0;
  if (g_in == nullptr) {
    blocks = amax_partial_blocks(rows * cols);
    if (launch_amax_partial(x_bf16, rows * cols, q.partials, blocks, s) != cudaSuccess)
      return cuda_failed();
    ++g_launches;
  }
  QuantizeArgs a{};
  a.x = static_cast<const uint16_t*>(x_bf16);
  a.rows = rows;
  a.rows_padded = scale_layout == NVFP4MOE_SCALES_SWIZZLED ? round128(rows) : rows;
  a.cols = cols;
  a.g_in = g_in;
  a.partials = q.partials;
  a.n_partials = blocks;
  a.codes = codes;
  a.scales = scales;
  a.swizzled = scale_layout == NVFP4MOE_SCALES_SWIZZLED;
  a.n_col_tiles = cols / 64;
  a.g_out = g_out;
  a.g_scratch = q.g;
  a.zero_out = nullptr;
  a.status = &q.hdr->status;
  if (launch_quantize(a, s) != cudaSuccess) return cuda_failed();
  g_launches += quantize_launch_count(a);
  return NVFP4MOE_OK;
}

int nvfp4moe_quantize_weights_lh(const void* w_bf16, int64_t rows, int64_t cols, const float* hess_blocks,
                                 int32_t m, uint8_t* codes, uint8_t* scales, float* g_out, void* ws,
                                 size_t ws_bytes, void* stream) {
  g_launches = 0;
  if (rows < 1 || cols <= 0 || cols % 16 != 0 || cols / 16 > 65535) return NVFP4MOE_ERR_SHAPE;
  if (rows >= ((int64_t)1 << 31) || rows * cols >= ((int64_t)1 << 40)) return NVFP4MOE_ERR_SHAPE;
  if (m < 0 || m > 16) return NVFP4MOE_ERR_ARG;
  if (w_bf16 == nullptr || hess_blocks == nullptr || codes == nullptr || scales == nullptr || g_out == nullptr ||
      ws == nullptr)
    return NVFP4MOE_ERR_ARG;
  if (!aligned(w_bf16, 16) || !aligned(hess_blocks, 4) || !aligned(codes, 8) || !aligned(g_out, 4) ||
      !aligned(ws, kAlign))
    return NVFP4MOE_ERR_ARG;
  const QuantWs q = carve_quant(ws);
  if (ws_bytes < q.bytes) return NVFP4MOE_ERR_WORKSPACE;
  int st = check_device();
  if (st != NVFP4MOE_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (reset_status(q.hdr, 1, s) != cudaSuccess) return cuda_failed();
  const int blocks = amax_partial_blocks(rows * cols);
  if (launch_amax_partial(w_bf16, rows * cols, q.partials, blocks, s) != cudaSuccess) return cuda_failed();
  LhArgs la{static_cast<const uint16_t*>(w_bf16), rows, cols, hess_blocks, m, q.partials, blocks, codes, scales,
            g_out, &q.hdr->status};
  if (launch_lh_quantize(la, s) != cudaSuccess) return cuda_failed();
  g_launches = 2;
  return NVFP4MOE_OK;
}

size_t nvfp4moe_route_workspace_bytes(const nvfp4moe_cfg* cfg, int64_t T) {
  if (nvfp4moe_cfg_check(cfg) != NVFP4MOE_OK || T < 0) return 0;
  return carve_route(nullptr, *cfg, T > 0 ? T : 1).bytes;
}

int nvfp4moe_route(const nvfp4moe_cfg* cfg, const void* hidden_bf16, int64_t T, const float* w_router,
                   const float* logit_bias, int32_t* idx, float* w, void* ws, size_t ws_bytes,
                   void* stream) {
  g_launches = 0;
  int st = nvfp4moe_cfg_check(cfg);
  if (st != NVFP4MOE_OK) return st;
  if (T < 0 || T > (1 << 24)) return NVFP4MOE_ERR_SHAPE;
  if (ws == nullptr || !aligned(ws, kAlign)) return NVFP4MOE_ERR_ARG;
  if (T > 0 && (hidden_bf16 == nullptr || w_router == nullptr || idx == nullptr || w == nullptr ||
                !aligned(hidden_bf16, 16) || !aligned(w_router, 16)))
    return NVFP4MOE_ERR_ARG;
  const RouteWs r = carve_route(ws, *cfg, T > 0 ? T : 1);
  if (ws_bytes < r.bytes) return NVFP4MOE_ERR_WORKSPACE;
  st = check_device();
  if (st != NVFP4MOE_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (reset_status(r.hdr, 1, s) != cudaSuccess) return cuda_failed();
  if (T == 0) return NVFP4MOE_OK;
  RouterArgs a{};
  a.x = static_cast<const uint16_t*>(hidden_bf16);
  a.w = w_router;
  a.bias = logit_bias;
  a.parts = r.parts;
  a.idx = idx;
  a.wts = w;
  a.T = T;
  a.H = cfg->H;
  a.E = cfg->E;
  a.n_groups = cfg->n_groups;
  a.topk_groups = cfg->topk_groups;
  a.topk = cfg->topk;
  a.routed_scale = cfg->routed_scale;
  a.status = &r.hdr->status;
  set_router_tc(a, r.tc, r.x_digits);
  if (launch_router(a, s) != cudaSuccess) return cuda_failed();
  g_launches += router_launch_count(a);
  return NVFP4MOE_OK;
}

int nvfp4moe_experts_create_local(const nvfp4moe_cfg* cfg, int32_t e_begin, int32_t e_count,
                                  nvfp4moe_experts** out) {
  if (out == nullptr) return NVFP4MOE_ERR_ARG;
  *out = nullptr;
  int st = nvfp4moe_cfg_check(cfg);
  if (st != NVFP4MOE_OK) return st;
  if (e_begin < 0 || e_count < 1 || e_begin + e_count > cfg->E) return NVFP4MOE_ERR_ARG;
  st = check_device();
  if (st != NVFP4MOE_OK) return st;
  nvfp4moe_experts* x = new nvfp4moe_experts();
  std::memset(x, 0, sizeof(*x));
  x->cfg = *cfg;
  x->e_begin = e_begin;
  x->e_count = e_count;
  cudaGetDevice(&x->device);
  const int64_t E = e_count, H = cfg->H, I = cfg->I;
  // tiled codes: K padded to a multiple of 256 values (128 bytes)
  const size_t w13 = (size_t)E * 2 * I * ((H + 255) / 256 * 128), w13sf = (size_t)E * 2 * I * H / 16;
  const size_t wd = (size_t)E * H * ((I + 255) / 256 * 128), wdsf = (size_t)E * H * I / 16;
  bool ok = cudaMalloc(&x->w13_codes, w13) == cudaSuccess && cudaMalloc(&x->w13_sf, w13sf) == cudaSuccess &&
            cudaMalloc(&x->wd_codes, wd) == cudaSuccess && cudaMalloc(&x->wd_sf, wdsf) == cudaSuccess &&
            cudaMalloc(&x->g_gate, E * sizeof(float)) == cudaSuccess &&
            cudaMalloc(&x->g_up, E * sizeof(float)) == cudaSuccess &&
            cudaMalloc(&x->g_h, E * sizeof(float)) == cudaSuccess &&
            cudaMalloc(&x->alpha_down, E * sizeof(float)) == cudaSuccess;
  ok = ok && cudaMemset(x->w13_codes, 0, w13) == cudaSuccess && cudaMemset(x->wd_codes, 0, wd) == cudaSuccess;
  if (!ok) {
    nvfp4moe_experts_destroy(x);
    return cuda_failed();
  }
  *out = x;
  return NVFP4MOE_OK;
}

int nvfp4moe_experts_create(const nvfp4moe_cfg* cfg, nvfp4moe_experts** out) {
  if (cfg == nullptr) return NVFP4MOE_ERR_ARG;
  return nvfp4moe_experts_create_local(cfg, 0, cfg->E, out);
}

int nvfp4moe_experts_range(const nvfp4moe_experts* x, int32_t* e_begin, int32_t* e_count) {
  if (x == nullptr || e_begin == nullptr || e_count == nullptr) return NVFP4MOE_ERR_ARG;
  *e_begin = x->e_begin;
  *e_count = x->e_count;
  return NVFP4MOE_OK;
}

int nvfp4moe_experts_set(nvfp4moe_experts* x, int32_t e_global, const nvfp4moe_expert_tensors* t, void* stream) {
  g_launches = 0;
  if (x == nullptr || t == nullptr) return NVFP4MOE_ERR_ARG;
  const nvfp4moe_cfg& c = x->cfg;
  if (e_global < x->e_begin || e_global >= x->e_begin + x->e_count) return NVFP4MOE_ERR_ARG;
  const int32_t e = e_global - x->e_begin;   // slot in this handle
  if (!t->gate_codes || !t->gate_scales || !t->up_codes || !t->up_scales || !t->down_codes || !t->down_scales)
    return NVFP4MOE_ERR_ARG;
  // the code rows are copied 16 bytes at a time
  if (!aligned(t->gate_codes, 16) || !aligned(t->up_codes, 16) || !aligned(t->down_codes, 16))
    return NVFP4MOE_ERR_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t H = c.H, I = c.I;
  // gate/up rows are interleaved in groups of half a GEMM column tile: packed group 2j holds
  // gate rows [64j, 64j+64), group 2j+1 the up rows of the same features
  constexpr int kG = kWeightTileRows / 2;
  const size_t w13_expert = (size_t)2 * I * ((H + 255) / 256 * 128);
  const size_t wd_expert = (size_t)H * ((I + 255) / 256 * 128);
  uint8_t* w13 = x->w13_codes + (size_t)e * w13_expert;
  if (launch_tile_weights(t->gate_codes, (int)I, (int)(H / 2), w13, kG, 2, 0, s) != cudaSuccess ||
      launch_tile_weights(t->up_codes, (int)I, (int)(H / 2), w13, kG, 2, 1, s) != cudaSuccess ||
      launch_tile_weights(t->down_codes, (int)H, (int)(I / 2), x->wd_codes + (size_t)e * wd_expert, (int)H, 1, 0,
                          s) != cudaSuccess)
    return cuda_failed();
  uint8_t* w13sf = x->w13_sf + (size_t)e * 2 * I * H / 16;
  if (launch_repack_sf(t->gate_scales, (int)I, (int)(H / 16), w13sf, H / 64, kG, 2, 0, s) != cudaSuccess ||
      launch_repack_sf(t->up_scales, (int)I, (int)(H / 16), w13sf, H / 64, kG, 2, 1, s) != cudaSuccess ||
      launch_repack_sf(t->down_scales, (int)H, (int)(I / 16), x->wd_sf + (size_t)e * H * I / 16, I / 64, (int)H,
                       1, 0, s) != cudaSuccess)
    return cuda_failed();
  set_expert_scalars_kernel<<<1, 1, 0, s>>>(x->g_gate, x->g_up, x->g_h, x->alpha_down, e, t->g_gate, t->g_up,
                                            t->g_h, t->g_down);
  if (cudaGetLastError() != cudaSuccess) return cuda_failed();
  g_launches += 7;
  return NVFP4MOE_OK;
}

void nvfp4moe_experts_destroy(nvfp4moe_experts* x) {
  if (x == nullptr) return;
  cudaFree(x->w13_codes);
  cudaFree(x->w13_sf);
  cudaFree(x->wd_codes);
  cudaFree(x->wd_sf);
  cudaFree(x->g_gate);
  cudaFree(x->g_up);
  cudaFree(x->g_h);
  cudaFree(x->alpha_down);
  delete x;
}

int nvfp4moe_experts_cfg(const nvfp4moe_experts* x, nvfp4moe_cfg* cfg) {
  if (x == nullptr || cfg == nullptr) return NVFP4MOE_ERR_ARG;
  *cfg = x->cfg;
  return NVFP4MOE_OK;
}

size_t nvfp4moe_forward_workspace_bytes(const nvfp4moe_cfg* cfg, int64_t T_max) {
  if (nvfp4moe_cfg_check(cfg) != NVFP4MOE_OK || T_max < 1) return 0;
  return carve_forward(nullptr, *cfg, T_max).bytes;
}

// The layer; with res, finalize adds the output into the residual stream.
// acc_out: NULL for the whole layer (BF16 out_bf16); otherwise the FP32 sums of the handle's
// experts' contributions are left in acc_out [T][H] and there is no finalize.
// acc_peers: the down GEMM adds each token's rows into the owning rank's accumulator instead
// (the workspace's own accumulator is then unused), rows_per_peer tokens per rank.
static int forward_core(const nvfp4moe_experts* x, const void* hidden_bf16, int64_t T, const float* w_router,
                        const float* logit_bias, void* out_bf16, const Residual* res, const nvfp4moe_debug* dbg,
                        void* ws, size_t ws_bytes, void* stream, float* acc_out = nullptr,
                        float* const* acc_peers = nullptr, int64_t rows_per_peer = 0) {
  g_launches = 0;
  if (x == nullptr) return NVFP4MOE_ERR_ARG;
  const nvfp4moe_cfg& c = x->cfg;
  if (T < 1 || T > (1 << 20)) return NVFP4MOE_ERR_SHAPE;
  if (hidden_bf16 == nullptr || w_router == nullptr ||
      (out_bf16 == nullptr && acc_out == nullptr && acc_peers == nullptr) || ws == nullptr)
    return NVFP4MOE_ERR_ARG;
  if (!aligned(hidden_bf16, 16) || !aligned(w_router, 16) || !aligned(out_bf16, 16) || !aligned(acc_out, 16) ||
      !aligned(ws, kAlign))
    return NVFP4MOE_ERR_ARG;
  ForwardWs f = carve_forward(ws, c, T);
  if (acc_out != nullptr) f.acc = acc_out;
  if (ws_bytes < f.bytes) return NVFP4MOE_ERR_WORKSPACE;
  // the bounded waits' limit and the front-end test hook (nvfp4moe_debug)
  const uint64_t wait_ns = dbg != nullptr ? (uint64_t)dbg->wait_limit_us * 1000ull : 0ull;
  const int32_t skip_arrive = dbg != nullptr ? dbg->inject_skip_arrive : 0;
  if (skip_arrive < 0 || (skip_arrive > 0 && !front_supported(T, c.E, c.H))) return NVFP4MOE_ERR_ARG;
  int st = check_device();
  if (st != NVFP4MOE_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t pairs = T * c.topk;

  CUtensorMap tma_a, tma_a32, tma_h, tma_h32;
  if (make_tma_2d(&tma_a, f.a_codes, c.H / 2, f.rows_cap, kBlockM) != 0 ||
      make_tma_2d(&tma_a32, f.a_codes, c.H / 2, f.rows_cap, 32) != 0 ||
      make_tma_2d(&tma_h, f.hq_codes, c.I / 2, f.rows_cap, kBlockM) != 0 ||
      make_tma_2d(&tma_h32, f.hq_codes, c.I / 2, f.rows_cap, 32) != 0)
    return cuda_failed();

  const StageEvents ev{dbg != nullptr ? dbg->events : nullptr, s};
  // status word, front-end barrier, the GEMM work counters and the row-tile counters that follow
  // the header
  if (reset_status(f.hdr, (int)(sizeof(WsHeader) / 4 + f.rows_cap / kBlockM), s) != cudaSuccess)
    return cuda_failed();
  const bool keep_xq = dbg != nullptr && (dbg->xq_codes != nullptr || dbg->xq_scales != nullptr);
  const bool decode_cfg = T * c.topk < 32 * c.E;   // segments average fewer than 32 rows
  // two GEMM launches (else one for both, see below); the gate/up launch then zeroes the FP32
  // accumulator beside its work (its HBM traffic leaves room at large T), else the quantiser
  // or the front end does
  const bool separate = !decode_cfg || (dbg != nullptr && dbg->separate_gemms != 0);

  if (front_supported(T, c.E, c.H)) {
    // small T: route, amax, grouping and quantise-scatter in one cooperative launch
    FrontArgs fa{};
    fa.x = static_cast<const uint16_t*>(hidden_bf16);
    fa.w = w_router;
    fa.bias = logit_bias;
    fa.T = T;
    fa.H = c.H;
    fa.E = c.E;
    fa.n_groups = c.n_groups;
    fa.topk_groups = c.topk_groups;
    fa.topk = c.topk;
    fa.routed_scale = c.routed_scale;
    fa.parts = f.parts;
    fa.amax_partials = f.partials;
    fa.idx = f.idx;
    fa.wts = f.wts;
    fa.logits_out = dbg != nullptr ? dbg->logits : nullptr;
    fa.counts = f.counts;
    fa.offsets = f.offsets;
    fa.mtile_prefix = f.mtile_prefix;
    fa.perm = f.perm;
    fa.inv = f.inv;
    fa.row_pair = f.row_pair;
    fa.seg_codes = f.a_codes;
    fa.seg_sf = f.a_sf;
    fa.n_col_tiles = c.H / 64;
    fa.xq_codes = keep_xq ? f.xq_codes : nullptr;
    fa.xq_sf = keep_xq ? f.xq_sf : nullptr;
    fa.g_out = f.g_x;
    fa.acc = f.acc;
    fa.status = &f.hdr->status;
    fa.barrier = &f.hdr->barrier;
    fa.wait_ns = wait_ns;
    fa.skip_arrive = skip_arrive;
    ev.mark(NVFP4MOE_STAGE_AMAX, 0);
    ev.mark(NVFP4MOE_STAGE_AMAX, 1);
    ev.mark(NVFP4MOE_STAGE_ROUTE, 0);
    if (launch_front(fa, s) != cudaSuccess) return cuda_failed();
    ev.mark(NVFP4MOE_STAGE_ROUTE, 1);
    for (int stage : {NVFP4MOE_STAGE_PERMUTE, NVFP4MOE_STAGE_QUANTIZE, NVFP4MOE_STAGE_GATHER}) {
      ev.mark(stage, 0);
      ev.mark(stage, 1);
    }
    ++g_launches;
  } else {

    // route: logits (with the per-block maxima of |x| for the global scale) + top-k
    RouterArgs r{};
    r.x = static_cast<const uint16_t*>(hidden_bf16);
    r.w = w_router;
    r.bias = logit_bias;
    r.parts = f.parts;
    r.idx = f.idx;
    r.wts = f.wts;
    r.T = T;
    r.H = c.H;
    r.E = c.E;
    r.n_groups = c.n_groups;
    r.topk_groups = c.topk_groups;
    r.topk = c.topk;
    r.routed_scale = c.routed_scale;
    r.logits_out = dbg != nullptr ? dbg->logits : nullptr;
    r.amax_partials = f.partials;
    r.status = &f.hdr->status;
    r.wait_ns = wait_ns;
    set_router_tc(r, f.tc, f.a_codes);
    const int n_partials = router_amax_partials(T, c.E, c.H);
    ev.mark(NVFP4MOE_STAGE_AMAX, 0);
    ev.mark(NVFP4MOE_STAGE_AMAX, 1);
    ev.mark(NVFP4MOE_STAGE_ROUTE, 0);
    if (launch_router(r, s) != cudaSuccess) return cuda_failed();
    ev.mark(NVFP4MOE_STAGE_ROUTE, 1);
    g_launches += router_launch_count(r);

    // group the (token, slot) pairs by expert
    PermArgs pa{};
    pa.idx = f.idx;
    pa.T = T;
    pa.topk = c.topk;
    pa.E = c.E;
    pa.n_chunks = (int)((T + kPermChunkTokens - 1) / kPermChunkTokens);
    pa.chunk_counts = f.chunk_counts;
    pa.chunk_base = f.chunk_base;
    pa.counts = f.counts;
    pa.offsets = f.offsets;
    pa.mtile_prefix = f.mtile_prefix;
    pa.perm = f.perm;
    pa.inv = f.inv;
    pa.row_pair = f.row_pair;
    ev.mark(NVFP4MOE_STAGE_PERMUTE, 0);
    if (launch_permute(pa, s, &g_launches) != cudaSuccess) return cuda_failed();
    ev.mark(NVFP4MOE_STAGE_PERMUTE, 1);

    // quantise x and write each token's row into its expert-segment rows (zeroes the
    // accumulator alongside when one launch runs both GEMMs); the token-major copy is only
    // kept for the debug export
    QuantizeArgs q{};
    q.x = static_cast<const uint16_t*>(hidden_bf16);
    q.rows = T;
    q.rows_padded = keep_xq ? round128(T) : T;
    q.cols = c.H;
    q.g_in = nullptr;
    q.partials = f.partials;
    q.n_partials = n_partials;
    q.codes = keep_xq ? f.xq_codes : nullptr;
    q.scales = keep_xq ? f.xq_sf : nullptr;
    q.swizzled = 1;
    q.n_col_tiles = c.H / 64;
    q.g_out = f.g_x;
    q.zero_out = separate ? nullptr : f.acc;
    q.status = &f.hdr->status;
    q.idx = f.idx;
    q.inv = f.inv;
    q.offsets = f.offsets;
    q.mtile_prefix = f.mtile_prefix;
    q.topk = c.topk;
    q.seg_codes = f.a_codes;
    q.seg_sf = f.a_sf;
    ev.mark(NVFP4MOE_STAGE_QUANTIZE, 0);
    if (launch_quantize(q, s) != cudaSuccess) return cuda_failed();
    ev.mark(NVFP4MOE_STAGE_QUANTIZE, 1);
    ev.mark(NVFP4MOE_STAGE_GATHER, 0);
    ev.mark(NVFP4MOE_STAGE_GATHER, 1);
    g_launches += quantize_launch_count(q);
  }

  const int grid = num_sms();
  GemmArgs g{};
  g.b_tiles = x->w13_codes;
  g.sfa = f.a_sf;
  g.sfb = x->w13_sf;
  // the handle's experts only (all of them unless it holds one rank's share): tiles of
  // experts e_begin .. e_begin + e_count - 1, weights indexed from the handle's first expert
  g.mtile_prefix = f.mtile_prefix + x->e_begin;
  g.counts = f.counts + x->e_begin;
  g.E = x->e_count;
  g.K = c.H;
  g.n_total = 2 * c.I;
  g.status = &f.hdr->status;
  g.hq_codes = f.hq_codes;
  g.hq_sf = f.hq_sf;
  g.g_x = f.g_x;
  g.g_gate = x->g_gate;
  g.g_up = x->g_up;
  g.g_h = x->g_h;
  g.I = c.I;
  g.wait_ns = wait_ns;
  g.h_dbg = dbg != nullptr ? dbg->h_f32 : nullptr;
  g.dbg_offsets = f.offsets + x->e_begin;
  g.acc = f.acc;
  g.row_pair = f.row_pair;
  g.wts = f.wts;
  g.alpha_down = x->alpha_down;
  g.topk = c.topk;
  g.H = c.H;
  g.work_counter = &f.hdr->work[0];
  GemmArgs gd = g;
  gd.b_tiles = x->wd_codes;
  gd.sfa = f.hq_sf;
  gd.sfb = x->wd_sf;
  gd.K = c.I;
  gd.n_total = c.H;
  gd.h_dbg = nullptr;
  gd.acc_peers = acc_peers;
  gd.rows_per_peer = rows_per_peer;
  // one launch for both GEMMs when segments are short (weight streaming dominates and the
  // boundary between two launches costs a few per cent); with full segments the down GEMM's
  // FP32 reductions, bound by the L2's reduction rate, slow the gate/up loads they would run
  // beside, and two launches are faster
  if (separate) {
    ev.mark(NVFP4MOE_STAGE_GATEUP, 0);
    GemmArgs gz = g;
    if (!front_supported(T, c.E, c.H)) {
      gz.zero_acc = f.acc;
      gz.zero_acc_elems = T * c.H;
    }
    if (launch_gemm_gateup(tma_a, tma_a32, gz, grid, decode_cfg, s) != cudaSuccess) return cuda_failed();
    ev.mark(NVFP4MOE_STAGE_GATEUP, 1);
    ++g_launches;
    ev.mark(NVFP4MOE_STAGE_DOWN, 0);
    gd.work_counter = &f.hdr->work[1];
    if (launch_gemm_down(tma_h, tma_h32, gd, grid, decode_cfg, s) != cudaSuccess) return cuda_failed();
    ev.mark(NVFP4MOE_STAGE_DOWN, 1);
    ++g_launches;
  } else {
    // both GEMMs in one launch: an expert's down items are claimed kFusedLagPerSm * grid
    // gate/up items after its last gate/up item
    ev.mark(NVFP4MOE_STAGE_GATEUP, 0);
    if (launch_gemm_fused(tma_a, tma_a32, tma_h, tma_h32, g, gd, f.dep, kFusedLagPerSm * grid, grid, s) !=
        cudaSuccess)
      return cuda_failed();
    ev.mark(NVFP4MOE_STAGE_GATEUP, 1);
    ev.mark(NVFP4MOE_STAGE_DOWN, 0);
    ev.mark(NVFP4MOE_STAGE_DOWN, 1);
    ++g_launches;
  }

  if (acc_out == nullptr && acc_peers == nullptr) {
    FinalizeArgs fa{f.acc, static_cast<uint16_t*>(out_bf16), T * c.H, res != nullptr ? res->h : nullptr,
                    res != nullptr ? res->a : 0.0f, res != nullptr ? res->b : 0.0f};
    ev.mark(NVFP4MOE_STAGE_FINALIZE, 0);
    if (launch_finalize(fa, s) != cudaSuccess) return cuda_failed();
    ev.mark(NVFP4MOE_STAGE_FINALIZE, 1);
    ++g_launches;
  }

  if (dbg != nullptr) {
    bool ok = true;
    if (dbg->idx) ok &= cudaMemcpyAsync(dbg->idx, f.idx, pairs * 4, cudaMemcpyDeviceToDevice, s) == cudaSuccess;
    if (dbg->w) ok &= cudaMemcpyAsync(dbg->w, f.wts, pairs * 4, cudaMemcpyDeviceToDevice, s) == cudaSuccess;
    if (dbg->g_x) ok &= cudaMemcpyAsync(dbg->g_x, f.g_x, 4, cudaMemcpyDeviceToDevice, s) == cudaSuccess;
    if (dbg->xq_codes)
      ok &= cudaMemcpyAsync(dbg->xq_codes, f.xq_codes, T * c.H / 2, cudaMemcpyDeviceToDevice, s) == cudaSuccess;
    if (dbg->xq_scales)
      ok &= launch_unswizzle_rows(f.xq_sf, c.H / 64, nullptr, T, c.H / 16, dbg->xq_scales, s) == cudaSuccess;
    if (dbg->counts) ok &= cudaMemcpyAsync(dbg->counts, f.counts, c.E * 4, cudaMemcpyDeviceToDevice, s) == cudaSuccess;
    if (dbg->offsets)
      ok &= cudaMemcpyAsync(dbg->offsets, f.offsets, (c.E + 1) * 4, cudaMemcpyDeviceToDevice, s) == cudaSuccess;
    if (dbg->perm) ok &= cudaMemcpyAsync(dbg->perm, f.perm, pairs * 4, cudaMemcpyDeviceToDevice, s) == cudaSuccess;
    if (dbg->hq_codes && dbg->hq_scales)
      ok &= launch_export_hq(f.hq_codes, f.hq_sf, f.perm, f.idx, f.offsets, f.mtile_prefix, pairs, c.I,
                             dbg->hq_codes, dbg->hq_scales, s) == cudaSuccess;
    if (dbg->acc && dbg->acc != f.acc)
      ok &= cudaMemcpyAsync(dbg->acc, f.acc, T * c.H * 4, cudaMemcpyDeviceToDevice, s) == cudaSuccess;
    if (!ok) return cuda_failed();
  }
  return NVFP4MOE_OK;
}

int nvfp4moe_forward(const nvfp4moe_experts* x, const void* hidden_bf16, int64_t T, const float* w_router,
                     const float* logit_bias, void* out_bf16, const nvfp4moe_debug* dbg, void* ws,
                     size_t ws_bytes, void* stream) {
  return forward_core(x, hidden_bf16, T, w_router, logit_bias, out_bf16, nullptr, dbg, ws, ws_bytes, stream);
}

int nvfp4moe_forward_partial(const nvfp4moe_experts* x, const void* hidden_bf16, int64_t T, const float* w_router,
                             const float* logit_bias, float* acc_out, const nvfp4moe_debug* dbg, void* ws,
                             size_t ws_bytes, void* stream) {
  g_launches = 0;
  if (acc_out == nullptr) return NVFP4MOE_ERR_ARG;
  return forward_core(x, hidden_bf16, T, w_router, logit_bias, nullptr, nullptr, dbg, ws, ws_bytes, stream, acc_out);
}

int nvfp4moe_forward_partial_peer(const nvfp4moe_experts* x, const void* hidden_bf16, int64_t T,
                                  const float* w_router, const float* logit_bias, float* const* acc_peers,
                                  int32_t n_peers, int64_t rows_per_peer, const nvfp4moe_debug* dbg, void* ws,
                                  size_t ws_bytes, void* stream) {
  g_launches = 0;
  if (acc_peers == nullptr || !aligned(acc_peers, 8)) return NVFP4MOE_ERR_ARG;
  if (n_peers < 1 || rows_per_peer < 1 || (int64_t)n_peers * rows_per_peer != T) return NVFP4MOE_ERR_SHAPE;
  if (dbg != nullptr && dbg->acc != nullptr) return NVFP4MOE_ERR_ARG;   // the sums are in the peers
  return forward_core(x, hidden_bf16, T, w_router, logit_bias, nullptr, nullptr, dbg, ws, ws_bytes, stream, nullptr,
                      acc_peers, rows_per_peer);
}

namespace {
using AddressRangeFn = CUresult (*)(CUdeviceptr*, size_t*, CUdeviceptr);
AddressRangeFn address_range_fn() {
  static AddressRangeFn fn = nullptr;
  if (fn == nullptr) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuMemGetAddressRange", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<AddressRangeFn>(ptr);
  }
  return fn;
}
}  // namespace

int nvfp4moe_ipc_get_handle(const void* dev_ptr, void* handle_out, int64_t* offset_out) {
  static_assert(sizeof(cudaIpcMemHandle_t) == NVFP4MOE_IPC_HANDLE_BYTES, "IPC handle size");
  if (dev_ptr == nullptr || handle_out == nullptr || offset_out == nullptr) return NVFP4MOE_ERR_ARG;
  int st = check_device();
  if (st != NVFP4MOE_OK) return st;
  AddressRangeFn range = address_range_fn();
  CUdeviceptr base = 0;
  size_t size = 0;
  if (range == nullptr || range(&base, &size, reinterpret_cast<CUdeviceptr>(dev_ptr)) != CUDA_SUCCESS)
    return NVFP4MOE_ERR_ARG;                                      // not device memory
  cudaIpcMemHandle_t h;
  if (cudaIpcGetMemHandle(&h, reinterpret_cast<void*>(base)) != cudaSuccess) return cuda_failed();
  std::memcpy(handle_out, &h, sizeof(h));
  *offset_out = (int64_t)(reinterpret_cast<CUdeviceptr>(dev_ptr) - base);
  return NVFP4MOE_OK;
}

int nvfp4moe_ipc_open(const void* handle, void** dev_ptr_out) {
  if (handle == nullptr || dev_ptr_out == nullptr) return NVFP4MOE_ERR_ARG;
  int st = check_device();
  if (st != NVFP4MOE_OK) return st;
  cudaIpcMemHandle_t h;
  std::memcpy(&h, handle, sizeof(h));
  if (cudaIpcOpenMemHandle(dev_ptr_out, h, cudaIpcMemLazyEnablePeerAccess) != cudaSuccess) return cuda_failed();
  return NVFP4MOE_OK;
}

int nvfp4moe_ipc_close(void* dev_ptr) {
  if (dev_ptr == nullptr) return NVFP4MOE_ERR_ARG;
  int st = check_device();
  if (st != NVFP4MOE_OK) return st;
  return cudaIpcCloseMemHandle(dev_ptr) == cudaSuccess ? NVFP4MOE_OK : cuda_failed();
}

int nvfp4moe_finalize(const float* acc, int64_t n, void* out_bf16, void* stream) {
  g_launches = 0;
  if (n < 0 || n % 8 != 0 || n >= ((int64_t)1 << 40)) return NVFP4MOE_ERR_SHAPE;
  if (n == 0) return NVFP4MOE_OK;
  if (acc == nullptr || out_bf16 == nullptr || !aligned(acc, 16) || !aligned(out_bf16, 16)) return NVFP4MOE_ERR_ARG;
  int st = check_device();
  if (st != NVFP4MOE_OK) return st;
  FinalizeArgs fa{acc, static_cast<uint16_t*>(out_bf16), n, nullptr, 0.0f, 0.0f};
  if (launch_finalize(fa, static_cast<cudaStream_t>(stream)) != cudaSuccess) return cuda_failed();
  g_launches = 1;
  return NVFP4MOE_OK;
}

int nvfp4moe_forward_residual(const nvfp4moe_experts* x, const void* h_bf16, int64_t T, const float* gamma,
                              float eps, int32_t step_k, const float* w_router, const float* logit_bias,
                              void* h_out_bf16, const nvfp4moe_debug* dbg, void* ws, size_t ws_bytes,
                              void* stream) {
  g_launches = 0;
  if (x == nullptr) return NVFP4MOE_ERR_ARG;
  const nvfp4moe_cfg& c = x->cfg;
  if (T < 1 || T > (1 << 20)) return NVFP4MOE_ERR_SHAPE;
  if (h_bf16 == nullptr || gamma == nullptr || w_router == nullptr || h_out_bf16 == nullptr || ws == nullptr)
    return NVFP4MOE_ERR_ARG;
  if (!aligned(h_bf16, 16) || !aligned(gamma, 16) || !aligned(h_out_bf16, 16) || !aligned(ws, kAlign))
    return NVFP4MOE_ERR_ARG;
  if (step_k < 1 || !(eps >= 0.0f) || eps > 3.0e38f) return NVFP4MOE_ERR_ARG;
  const ForwardWs f = carve_forward(ws, c, T);
  if (ws_bytes < f.bytes) return NVFP4MOE_ERR_WORKSPACE;
  int st = check_device();
  if (st != NVFP4MOE_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // the status word is reset by the forward that follows; the norm raises nothing
  RmsNormArgs na{static_cast<const uint16_t*>(h_bf16), gamma, eps, T, c.H, f.x_norm};
  if (launch_rmsnorm(na, s) != cudaSuccess) return cuda_failed();
  const Residual r{static_cast<const uint16_t*>(h_bf16), (float)std::sqrt((double)(step_k - 1) / (double)step_k),
                   (float)(1.0 / std::sqrt((double)step_k))};
  st = forward_core(x, f.x_norm, T, w_router, logit_bias, h_out_bf16, &r, dbg, ws, ws_bytes, stream);
  g_launches += 1;
  if (st == NVFP4MOE_OK && dbg != nullptr && dbg->x_norm != nullptr &&
      cudaMemcpyAsync(dbg->x_norm, f.x_norm, (size_t)T * c.H * 2, cudaMemcpyDeviceToDevice, s) != cudaSuccess)
    return cuda_failed();
  return st;
}

int nvfp4moe_quantize_fp8(const void* x_bf16, int64_t rows, int64_t cols, uint8_t* codes, float* scales, void* ws,
                          size_t ws_bytes, void* stream) {
  g_launches = 0;
  if (rows < 1 || cols <= 0 || cols % 16 != 0 || cols >= ((int64_t)1 << 31)) return NVFP4MOE_ERR_SHAPE;
  if (rows >= ((int64_t)1 << 31) || rows * cols >= ((int64_t)1 << 40)) return NVFP4MOE_ERR_SHAPE;
  if (x_bf16 == nullptr || codes == nullptr || scales == nullptr || ws == nullptr) return NVFP4MOE_ERR_ARG;
  if (!aligned(x_bf16, 16) || !aligned(codes, 8) || !aligned(scales, 4) || !aligned(ws, kAlign))
    return NVFP4MOE_ERR_ARG;
  const QuantWs q = carve_quant(ws);
  if (ws_bytes < q.bytes) return NVFP4MOE_ERR_WORKSPACE;
  int st = check_device();
  if (st != NVFP4MOE_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (reset_status(q.hdr, 1, s) != cudaSuccess) return cuda_failed();
  Fp8RowsArgs fa{static_cast<const uint16_t*>(x_bf16), rows, cols, codes, scales, &q.hdr->status};
  if (launch_fp8_quantize_rows(fa, s) != cudaSuccess) return cuda_failed();
  g_launches = 1;
  return NVFP4MOE_OK;
}

int nvfp4moe_fp8_experts_create(const nvfp4moe_cfg* cfg, nvfp4moe_fp8_experts** out) {
  if (out == nullptr) return NVFP4MOE_ERR_ARG;
  *out = nullptr;
  int st = nvfp4moe_cfg_check(cfg);
  if (st != NVFP4MOE_OK) return st;
  st = check_device();
  if (st != NVFP4MOE_OK) return st;
  nvfp4moe_fp8_experts* x = new nvfp4moe_fp8_experts();
  std::memset(x, 0, sizeof(*x));
  x->cfg = *cfg;
  cudaGetDevice(&x->device);
  const int64_t E = cfg->E, H = cfg->H, I = cfg->I;
  const size_t w13 = (size_t)E * 2 * I * H, wd = (size_t)E * H * I;
  const bool ok = cudaMalloc(&x->w13_codes, w13) == cudaSuccess && cudaMalloc(&x->wd_codes, wd) == cudaSuccess &&
                  cudaMalloc(&x->w13_scale, (size_t)E * 2 * I * sizeof(float)) == cudaSuccess &&
                  cudaMalloc(&x->wd_scale, (size_t)E * H * sizeof(float)) == cudaSuccess &&
                  cudaMemset(x->w13_codes, 0, w13) == cudaSuccess && cudaMemset(x->wd_codes, 0, wd) == cudaSuccess &&
                  cudaMemset(x->w13_scale, 0, (size_t)E * 2 * I * sizeof(float)) == cudaSuccess &&
                  cudaMemset(x->wd_scale, 0, (size_t)E * H * sizeof(float)) == cudaSuccess;
  if (!ok) {
    nvfp4moe_fp8_experts_destroy(x);
    return cuda_failed();
  }
  *out = x;
  return NVFP4MOE_OK;
}

int nvfp4moe_fp8_experts_set(nvfp4moe_fp8_experts* x, int32_t e, const nvfp4moe_fp8_expert_tensors* t,
                             void* stream) {
  g_launches = 0;
  if (x == nullptr || t == nullptr) return NVFP4MOE_ERR_ARG;
  const nvfp4moe_cfg& c = x->cfg;
  if (e < 0 || e >= c.E) return NVFP4MOE_ERR_ARG;
  if (!t->gate_codes || !t->gate_scales || !t->up_codes || !t->up_scales || !t->down_codes || !t->down_scales)
    return NVFP4MOE_ERR_ARG;
  if (!aligned(t->gate_codes, 16) || !aligned(t->up_codes, 16) || !aligned(t->down_codes, 16))
    return NVFP4MOE_ERR_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t H = c.H, I = c.I;
  constexpr int kG = kWeightTileRows / 2;
  uint8_t* w13 = x->w13_codes + (size_t)e * 2 * I * H;
  // gate/up rows interleaved in groups of 64 (packed group 2j: gate rows [64j, 64j+64), 2j+1: up rows)
  if (launch_tile_weights(t->gate_codes, (int)I, (int)H, w13, kG, 2, 0, s) != cudaSuccess ||
      launch_tile_weights(t->up_codes, (int)I, (int)H, w13, kG, 2, 1, s) != cudaSuccess ||
      launch_tile_weights(t->down_codes, (int)H, (int)I, x->wd_codes + (size_t)e * H * I, (int)H, 1, 0, s) !=
          cudaSuccess)
    return cuda_failed();
  float* sc = x->w13_scale + (size_t)e * 2 * I;
  const size_t gb = kG * sizeof(float);
  if (cudaMemcpy2DAsync(sc, 2 * gb, t->gate_scales, gb, gb, I / kG, cudaMemcpyDeviceToDevice, s) != cudaSuccess ||
      cudaMemcpy2DAsync(sc + kG, 2 * gb, t->up_scales, gb, gb, I / kG, cudaMemcpyDeviceToDevice, s) != cudaSuccess ||
      cudaMemcpyAsync(x->wd_scale + (size_t)e * H, t->down_scales, H * sizeof(float), cudaMemcpyDeviceToDevice,
                      s) != cudaSuccess)
    return cuda_failed();
  g_launches = 3;
  return NVFP4MOE_OK;
}

void nvfp4moe_fp8_experts_destroy(nvfp4moe_fp8_experts* x) {
  if (x == nullptr) return;
  cudaFree(x->w13_codes);
  cudaFree(x->w13_scale);
  cudaFree(x->wd_codes);
  cudaFree(x->wd_scale);
  delete x;
}

size_t nvfp4moe_forward_fp8_workspace_bytes(const nvfp4moe_cfg* cfg, int64_t T_max) {
  if (nvfp4moe_cfg_check(cfg) != NVFP4MOE_OK || T_max < 1) return 0;
  return carve_forward_fp8(nullptr, *cfg, T_max).bytes;
}

int nvfp4moe_forward_fp8(const nvfp4moe_fp8_experts* x, const void* hidden_bf16, int64_t T, const float* w_router,
                         const float* logit_bias, void* out_bf16, const nvfp4moe_debug* dbg, void* ws,
                         size_t ws_bytes, void* stream) {
  g_launches = 0;
  if (x == nullptr) return NVFP4MOE_ERR_ARG;
  const nvfp4moe_cfg& c = x->cfg;
  if (T < 1 || T > (1 << 20)) return NVFP4MOE_ERR_SHAPE;
  if (hidden_bf16 == nullptr || w_router == nullptr || out_bf16 == nullptr || ws == nullptr)
    return NVFP4MOE_ERR_ARG;
  if (!aligned(hidden_bf16, 16) || !aligned(w_router, 16) || !aligned(out_bf16, 16) || !aligned(ws, kAlign))
    return NVFP4MOE_ERR_ARG;
  const ForwardFp8Ws f = carve_forward_fp8(ws, c, T);
  if (ws_bytes < f.bytes) return NVFP4MOE_ERR_WORKSPACE;
  int st = check_device();
  if (st != NVFP4MOE_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t pairs = T * c.topk;
  CUtensorMap tma_a, tma_a32, tma_h, tma_h32;
  if (make_tma_2d(&tma_a, f.a_codes, c.H, f.rows_cap, kBlockM) != 0 ||
      make_tma_2d(&tma_a32, f.a_codes, c.H, f.rows_cap, 32) != 0 ||
      make_tma_2d(&tma_h, f.hq, c.I, f.rows_cap, kBlockM) != 0 ||
      make_tma_2d(&tma_h32, f.hq, c.I, f.rows_cap, 32) != 0)
    return cuda_failed();
  // status word, front-end barrier and the two GEMM work counters
  if (reset_status(f.hdr, 4, s) != cudaSuccess) return cuda_failed();

  if (front_supported(T, c.E, c.H)) {
    // small T: routing and grouping in the fused front-end launch (its NVFP4 quantisation
    // is skipped: no segment buffers)
    FrontArgs fa{};
    fa.x = static_cast<const uint16_t*>(hidden_bf16);
    fa.w = w_router;
    fa.bias = logit_bias;
    fa.T = T;
    fa.H = c.H;
    fa.E = c.E;
    fa.n_groups = c.n_groups;
    fa.topk_groups = c.topk_groups;
    fa.topk = c.topk;
    fa.routed_scale = c.routed_scale;
    fa.parts = f.parts;
    fa.amax_partials = f.partials;
    fa.idx = f.idx;
    fa.wts = f.wts;
    fa.logits_out = dbg != nullptr ? dbg->logits : nullptr;
    fa.counts = f.counts;
    fa.offsets = f.offsets;
    fa.mtile_prefix = f.mtile_prefix;
    fa.perm = f.perm;
    fa.inv = f.inv;
    fa.row_pair = f.row_pair;
    fa.n_col_tiles = c.H / 64;
    fa.acc = f.acc;
    fa.status = &f.hdr->status;
    fa.barrier = &f.hdr->barrier;
    if (launch_front(fa, s) != cudaSuccess) return cuda_failed();
    ++g_launches;
  } else {
    RouterArgs r{};
    r.x = static_cast<const uint16_t*>(hidden_bf16);
    r.w = w_router;
    r.bias = logit_bias;
    r.parts = f.parts;
    r.idx = f.idx;
    r.wts = f.wts;
    r.T = T;
    r.H = c.H;
    r.E = c.E;
    r.n_groups = c.n_groups;
    r.topk_groups = c.topk_groups;
    r.topk = c.topk;
    r.routed_scale = c.routed_scale;
    r.logits_out = dbg != nullptr ? dbg->logits : nullptr;
    r.amax_partials = f.partials;
    r.status = &f.hdr->status;
    set_router_tc(r, f.tc, f.a_codes);
    if (launch_router(r, s) != cudaSuccess) return cuda_failed();
    g_launches += router_launch_count(r);

    PermArgs pa{};
    pa.idx = f.idx;
    pa.T = T;
    pa.topk = c.topk;
    pa.E = c.E;
    pa.n_chunks = (int)((T + kPermChunkTokens - 1) / kPermChunkTokens);
    pa.chunk_counts = f.chunk_counts;
    pa.chunk_base = f.chunk_base;
    pa.counts = f.counts;
    pa.offsets = f.offsets;
    pa.mtile_prefix = f.mtile_prefix;
    pa.perm = f.perm;
    pa.inv = f.inv;
    pa.row_pair = f.row_pair;
    if (launch_permute(pa, s, &g_launches) != cudaSuccess) return cuda_failed();
  }

  Fp8ScatterArgs qa{static_cast<const uint16_t*>(hidden_bf16), T, c.H, c.topk, f.idx, f.inv, f.offsets,
                    f.mtile_prefix, f.a_codes, f.a_scale, f.acc,
                    dbg != nullptr ? dbg->xq8_codes : nullptr, dbg != nullptr ? dbg->xq8_scales : nullptr,
                    &f.hdr->status};
  if (launch_fp8_quantize_scatter(qa, s) != cudaSuccess) return cuda_failed();
  ++g_launches;

  const int grid = num_sms();
  const bool decode_cfg = T * c.topk < 32 * c.E;
  GemmArgs g{};
  g.b_tiles = x->w13_codes;
  g.mtile_prefix = f.mtile_prefix;
  g.counts = f.counts;
  g.E = c.E;
  g.K = c.H;
  g.n_total = 2 * c.I;
  g.status = &f.hdr->status;
  g.I = c.I;
  g.acc = f.acc;
  g.row_pair = f.row_pair;
  g.wts = f.wts;
  g.topk = c.topk;
  g.H = c.H;
  g.a_scale = f.a_scale;
  g.w_scale = x->w13_scale;
  g.h32 = f.h32;
  g.work_counter = &f.hdr->work[0];
  if (launch_gemm_gateup_fp8(tma_a, tma_a32, g, grid, decode_cfg, s) != cudaSuccess) return cuda_failed();
  Fp8RequantArgs ra{f.h32, f.rows_cap, c.I, f.row_pair, f.mtile_prefix, c.E, f.hq, f.h_scale, &f.hdr->status};
  if (launch_fp8_requant_rows(ra, s) != cudaSuccess) return cuda_failed();
  g.b_tiles = x->wd_codes;
  g.K = c.I;
  g.n_total = c.H;
  g.w_scale = x->wd_scale;
  g.h_scale = f.h_scale;
  g.work_counter = &f.hdr->work[1];
  if (launch_gemm_down_fp8(tma_h, tma_h32, g, grid, decode_cfg, s) != cudaSuccess) return cuda_failed();
  FinalizeArgs fa{f.acc, static_cast<uint16_t*>(out_bf16), T * c.H, nullptr, 0.0f, 0.0f};
  if (launch_finalize(fa, s) != cudaSuccess) return cuda_failed();
  g_launches += 4;

  if (dbg != nullptr) {
    bool ok = true;
    if (dbg->idx) ok &= cudaMemcpyAsync(dbg->idx, f.idx, pairs * 4, cudaMemcpyDeviceToDevice, s) == cudaSuccess;
    if (dbg->w) ok &= cudaMemcpyAsync(dbg->w, f.wts, pairs * 4, cudaMemcpyDeviceToDevice, s) == cudaSuccess;
    if (dbg->counts) ok &= cudaMemcpyAsync(dbg->counts, f.counts, c.E * 4, cudaMemcpyDeviceToDevice, s) == cudaSuccess;
    if (dbg->offsets)
      ok &= cudaMemcpyAsync(dbg->offsets, f.offsets, (c.E + 1) * 4, cudaMemcpyDeviceToDevice, s) == cudaSuccess;
    if (dbg->perm) ok &= cudaMemcpyAsync(dbg->perm, f.perm, pairs * 4, cudaMemcpyDeviceToDevice, s) == cudaSuccess;
    if (!ok) return cuda_failed();
  }
  return NVFP4MOE_OK;
}

int nvfp4moe_status_read(const void* ws, void* stream) {
  if (ws == nullptr) return NVFP4MOE_ERR_ARG;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return cuda_failed();
  uint32_t v = 0;
  if (cudaMemcpy(&v, ws, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return cuda_failed();
  if (v & kStatusTimeout) return NVFP4MOE_ERR_TIMEOUT;
  if (v & kStatusBadInput) return NVFP4MOE_ERR_ARG;
  if (v & kStatusNonFinite) return NVFP4MOE_ERR_NONFINITE;
  return NVFP4MOE_OK;
}

int nvfp4moe_last_device_status(void* stream) {
  if (g_last_status == nullptr) return NVFP4MOE_ERR_ARG;
  return nvfp4moe_status_read(g_last_status, stream);
}

size_t nvfp4moe_workspace_bytes(const nvfp4moe_cfg* cfg, int64_t T_max) {
  return nvfp4moe_forward_workspace_bytes(cfg, T_max);
}

const char* nvfp4moe_status_string(int status) {
  switch (status) {
    case NVFP4MOE_OK: return "ok";
    case NVFP4MOE_ERR_ARG: return "invalid argument";
    case NVFP4MOE_ERR_SHAPE: return "unsupported shape";
    case NVFP4MOE_ERR_CUDA: return "CUDA call failed";
    case NVFP4MOE_ERR_WORKSPACE: return "workspace too small";
    case NVFP4MOE_ERR_NONFINITE: return "non-finite input";
    case NVFP4MOE_ERR_TIMEOUT: return "bounded device wait ran out";
    case NVFP4MOE_ERR_DEVICE: return "device is not compute capability 10.0 (B200)";
    default: return "unknown status";
  }
}

/* ------------------------------------------ expert parallelism, all-to-all exchange ---- */

int nvfp4moe_amax(const void* x_bf16, int64_t rows, int64_t cols, uint32_t* amax_bits, void* ws, size_t ws_bytes,
                  void* stream) {
  g_launches = 0;
  if (rows < 0 || cols <= 0 || cols % 8 != 0 || rows * cols >= ((int64_t)1 << 40)) return NVFP4MOE_ERR_SHAPE;
  if (amax_bits == nullptr || ws == nullptr || !aligned(ws, kAlign) || !aligned(amax_bits, 4)) return NVFP4MOE_ERR_ARG;
  if (rows > 0 && (x_bf16 == nullptr || !aligned(x_bf16, 16))) return NVFP4MOE_ERR_ARG;
  const QuantWs q = carve_quant(ws);
  if (ws_bytes < q.bytes) return NVFP4MOE_ERR_WORKSPACE;
  int st = check_device();
  if (st != NVFP4MOE_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (rows == 0) return cudaMemsetAsync(amax_bits, 0, 4, s) == cudaSuccess ? NVFP4MOE_OK : cuda_failed();
  const int blocks = amax_partial_blocks(rows * cols);
  if (launch_amax_partial(x_bf16, rows * cols, q.partials, blocks, s) != cudaSuccess) return cuda_failed();
  if (launch_amax_reduce(q.partials, blocks, amax_bits, s) != cudaSuccess) return cuda_failed();
  g_launches = 2;
  return NVFP4MOE_OK;
}

size_t nvfp4moe_ep_dispatch_workspace_bytes(const nvfp4moe_cfg* cfg, int64_t T) {
  if (nvfp4moe_cfg_check(cfg) != NVFP4MOE_OK || T < 1) return 0;
  return carve_ep_dispatch(nullptr, *cfg, T).bytes;
}

int nvfp4moe_ep_dispatch(const nvfp4moe_cfg* cfg, int32_t n_ranks, const void* hidden_bf16, int64_t T,
                         const float* w_router, const float* logit_bias, const uint32_t* amax_bits,
                         uint8_t* send_codes, uint8_t* send_scales, int32_t* send_expert, float* send_w,
                         int32_t* send_pos, int32_t* rank_counts, void* ws, size_t ws_bytes, void* stream) {
  g_launches = 0;
  int st = nvfp4moe_cfg_check(cfg);
  if (st != NVFP4MOE_OK) return st;
  if (n_ranks < 1 || cfg->E % n_ranks != 0) return NVFP4MOE_ERR_ARG;
  if (T < 1 || T > (1 << 20)) return NVFP4MOE_ERR_SHAPE;
  if (hidden_bf16 == nullptr || w_router == nullptr || amax_bits == nullptr || send_codes == nullptr ||
      send_scales == nullptr || send_expert == nullptr || send_w == nullptr || send_pos == nullptr ||
      rank_counts == nullptr || ws == nullptr)
    return NVFP4MOE_ERR_ARG;
  if (!aligned(hidden_bf16, 16) || !aligned(w_router, 16) || !aligned(send_codes, 16) || !aligned(send_scales, 4) ||
      !aligned(ws, kAlign))
    return NVFP4MOE_ERR_ARG;
  const nvfp4moe_cfg& c = *cfg;
  const EpDispatchWs d = carve_ep_dispatch(ws, c, T);
  if (ws_bytes < d.bytes) return NVFP4MOE_ERR_WORKSPACE;
  st = check_device();
  if (st != NVFP4MOE_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (reset_status(d.hdr, 1, s) != cudaSuccess) return cuda_failed();
  // route this rank's tokens
  RouterArgs r{};
  r.x = static_cast<const uint16_t*>(hidden_bf16);
  r.w = w_router;
  r.bias = logit_bias;
  r.parts = d.parts;
  r.idx = d.idx;
  r.wts = d.wts;
  r.T = T;
  r.H = c.H;
  r.E = c.E;
  r.n_groups = c.n_groups;
  r.topk_groups = c.topk_groups;
  r.topk = c.topk;
  r.routed_scale = c.routed_scale;
  r.status = &d.hdr->status;
  set_router_tc(r, d.tc, nullptr);
  if (launch_router(r, s) != cudaSuccess) return cuda_failed();
  g_launches += router_launch_count(r);
  // group its pairs by expert: the stable expert-major order is also destination-rank order
  PermArgs pa{};
  pa.idx = d.idx;
  pa.T = T;
  pa.topk = c.topk;
  pa.E = c.E;
  pa.n_chunks = (int)((T + kPermChunkTokens - 1) / kPermChunkTokens);
  pa.chunk_counts = d.chunk_counts;
  pa.chunk_base = d.chunk_base;
  pa.counts = d.counts;
  pa.offsets = d.offsets;
  pa.mtile_prefix = d.mtile_prefix;
  pa.perm = d.perm;
  pa.inv = d.inv;
  pa.row_pair = d.row_pair;
  if (launch_permute(pa, s, &g_launches) != cudaSuccess) return cuda_failed();
  // quantise the tokens with the global scale of all ranks' tokens (from their amax)
  QuantizeArgs q{};
  q.x = static_cast<const uint16_t*>(hidden_bf16);
  q.rows = T;
  q.rows_padded = T;
  q.cols = c.H;
  q.g_in = nullptr;
  q.partials = amax_bits;
  q.n_partials = 1;
  q.codes = d.xq_codes;
  q.scales = d.xq_scales;
  q.swizzled = 0;
  q.n_col_tiles = c.H / 64;
  q.g_out = d.g;
  q.status = &d.hdr->status;
  if (launch_quantize(q, s) != cudaSuccess) return cuda_failed();
  g_launches += quantize_launch_count(q);
  // pack the pairs' rows in send order, with their metadata and the per-rank counts
  EpPackArgs pk{};
  pk.perm = d.perm;
  pk.idx = d.idx;
  pk.wts = d.wts;
  pk.xq_codes = d.xq_codes;
  pk.xq_scales = d.xq_scales;
  pk.counts = d.counts;
  pk.n_pairs = T * c.topk;
  pk.topk = c.topk;
  pk.H = c.H;
  pk.E = c.E;
  pk.experts_per_rank = c.E / n_ranks;
  pk.send_codes = send_codes;
  pk.send_scales = send_scales;
  pk.send_expert = send_expert;
  pk.send_w = send_w;
  pk.send_pos = send_pos;
  pk.rank_counts = rank_counts;
  if (launch_ep_pack(pk, s) != cudaSuccess) return cuda_failed();
  g_launches += 2;
  return NVFP4MOE_OK;
}

size_t nvfp4moe_ep_experts_workspace_bytes(const nvfp4moe_cfg* cfg, int32_t e_count, int64_t n_rows_max) {
  if (nvfp4moe_cfg_check(cfg) != NVFP4MOE_OK || e_count < 1 || e_count > cfg->E || n_rows_max < 1) return 0;
  nvfp4moe_cfg cl = *cfg;
  cl.E = e_count;
  cl.topk = 1;
  return carve_ep_experts(nullptr, cl, n_rows_max).bytes;
}

int nvfp4moe_ep_experts(const nvfp4moe_experts* x, const uint8_t* codes, const uint8_t* scales,
                        const int32_t* expert, const float* w, int64_t n_rows, const uint32_t* amax_bits,
                        float* out_rows, void* ws, size_t ws_bytes, void* stream) {
  g_launches = 0;
  if (x == nullptr) return NVFP4MOE_ERR_ARG;
  if (n_rows < 0 || n_rows > ((int64_t)1 << 23)) return NVFP4MOE_ERR_SHAPE;
  if (amax_bits == nullptr || ws == nullptr || !aligned(ws, kAlign)) return NVFP4MOE_ERR_ARG;
  if (n_rows > 0 && (codes == nullptr || scales == nullptr || expert == nullptr || w == nullptr ||
                     out_rows == nullptr || !aligned(codes, 16) || !aligned(scales, 4) || !aligned(out_rows, 16)))
    return NVFP4MOE_ERR_ARG;
  nvfp4moe_cfg cl = x->cfg;
  cl.E = x->e_count;
  cl.topk = 1;
  const EpExpertsWs f = carve_ep_experts(ws, cl, n_rows > 0 ? n_rows : 1);
  if (ws_bytes < f.bytes) return NVFP4MOE_ERR_WORKSPACE;
  int st = check_device();
  if (st != NVFP4MOE_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (reset_status(f.hdr, 4, s) != cudaSuccess) return cuda_failed();
  if (n_rows == 0) return NVFP4MOE_OK;
  CUtensorMap tma_a, tma_a32, tma_h, tma_h32;
  if (make_tma_2d(&tma_a, f.a_codes, cl.H / 2, f.rows_cap, kBlockM) != 0 ||
      make_tma_2d(&tma_a32, f.a_codes, cl.H / 2, f.rows_cap, 32) != 0 ||
      make_tma_2d(&tma_h, f.hq_codes, cl.I / 2, f.rows_cap, kBlockM) != 0 ||
      make_tma_2d(&tma_h32, f.hq_codes, cl.I / 2, f.rows_cap, 32) != 0)
    return cuda_failed();
  // the expert indices come from other ranks: checked on the device (an index outside the
  // handle's experts is replaced by 0 and raises NVFP4MOE_ERR_ARG in the status word)
  if (launch_check_indices(expert, n_rows, cl.E, f.expert, &f.hdr->status, s) != cudaSuccess)
    return cuda_failed();
  ++g_launches;
  // group the received rows by local expert (stable: source rank, then its order)
  PermArgs pa{};
  pa.idx = f.expert;
  pa.T = n_rows;
  pa.topk = 1;
  pa.E = cl.E;
  pa.n_chunks = (int)((n_rows + kPermChunkTokens - 1) / kPermChunkTokens);
  pa.chunk_counts = f.chunk_counts;
  pa.chunk_base = f.chunk_base;
  pa.counts = f.counts;
  pa.offsets = f.offsets;
  pa.mtile_prefix = f.mtile_prefix;
  pa.perm = f.perm;
  pa.inv = f.inv;
  pa.row_pair = f.row_pair;
  if (launch_permute(pa, s, &g_launches) != cudaSuccess) return cuda_failed();
  if (launch_global_scale(amax_bits, 1, f.g_x, &f.hdr->status, s) != cudaSuccess) return cuda_failed();
  ++g_launches;
  RowsToSegmentsArgs ra{codes, scales, f.expert, f.inv, f.offsets, f.mtile_prefix, n_rows, cl.H, cl.H / 64,
                        f.a_codes, f.a_sf, out_rows};
  if (launch_rows_to_segments(ra, s) != cudaSuccess) return cuda_failed();
  ++g_launches;
  const int grid = num_sms();
  const bool decode_cfg = n_rows < 32 * (int64_t)cl.E;
  GemmArgs g{};
  g.b_tiles = x->w13_codes;
  g.sfa = f.a_sf;
  g.sfb = x->w13_sf;
  g.mtile_prefix = f.mtile_prefix;
  g.counts = f.counts;
  g.E = cl.E;
  g.K = cl.H;
  g.n_total = 2 * cl.I;
  g.status = &f.hdr->status;
  g.hq_codes = f.hq_codes;
  g.hq_sf = f.hq_sf;
  g.g_x = f.g_x;
  g.g_gate = x->g_gate;
  g.g_up = x->g_up;
  g.g_h = x->g_h;
  g.I = cl.I;
  g.acc = out_rows;          // one received row per slot: the reduction writes it once
  g.row_pair = f.row_pair;
  g.wts = w;
  g.alpha_down = x->alpha_down;
  g.topk = 1;
  g.H = cl.H;
  g.work_counter = &f.hdr->work[0];
  if (launch_gemm_gateup(tma_a, tma_a32, g, grid, decode_cfg, s) != cudaSuccess) return cuda_failed();
  ++g_launches;
  g.b_tiles = x->wd_codes;
  g.sfa = f.hq_sf;
  g.sfb = x->wd_sf;
  g.K = cl.I;
  g.n_total = cl.H;
  g.work_counter = &f.hdr->work[1];
  if (launch_gemm_down(tma_h, tma_h32, g, grid, decode_cfg, s) != cudaSuccess) return cuda_failed();
  ++g_launches;
  return NVFP4MOE_OK;
}

int nvfp4moe_ep_combine(const float* rows, const int32_t* send_pos, int64_t T, int32_t topk, int32_t H, void* out_bf16,
                        void* stream) {
  g_launches = 0;
  if (T < 0 || T > (1 << 20) || topk < 1 || topk > 8 || H < 64 || H % 64 != 0) return NVFP4MOE_ERR_SHAPE;
  if (T == 0) return NVFP4MOE_OK;
  if (rows == nullptr || send_pos == nullptr || out_bf16 == nullptr || !aligned(rows, 16) || !aligned(out_bf16, 16))
    return NVFP4MOE_ERR_ARG;
  int st = check_device();
  if (st != NVFP4MOE_OK) return st;
  if (launch_ep_combine(rows, send_pos, T, topk, H, static_cast<uint16_t*>(out_bf16), static_cast<cudaStream_t>(stream)) !=
      cudaSuccess)
    return cuda_failed();
  g_launches = 1;
  return NVFP4MOE_OK;
}

int32_t nvfp4moe_last_launch_count(void) { return g_launches; }

}  // extern "C"
