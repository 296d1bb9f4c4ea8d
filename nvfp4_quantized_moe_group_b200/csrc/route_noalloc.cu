// nvfp4moe_route_noalloc: the router for callers that cannot allocate device memory.
//
// Some callers have no way to obtain a workspace: a host runtime that hands this library
// only its input and output buffers and does not allow device allocation once it has
// started (its memory budget is fixed up front), or a host framework that owns every
// device allocation and exposes no allocator to the libraries it embeds.  For them this
// entry point runs exactly the kernels of nvfp4moe_route, with the router's scratch (the
// split-K logit partial sums and a status word) in a fixed array of device memory that the
// library itself declares below.  Every GPU that loads the library holds that array until
// the process exits.
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace nvfp4moe {
namespace {

// Capacity: the header, then the split-K partial sums.  The router chooses its K split so
// that splits * 64-token tiles * 64-expert tiles <= 296 whenever it splits at all, so the
// partials never exceed 296 * 64 * 64 doubles unless T * E itself is larger; T * E up to
// kNoAllocParts (T <= 4736 for 256 experts) always fits.
constexpr size_t kNoAllocParts = 296u * 64u * 64u;
constexpr size_t kNoAllocBytes = sizeof(WsHeader) + kNoAllocParts * sizeof(double);

static __device__ __align__(256) uint8_t g_route_scratch[kNoAllocBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_route_scratch on the current device (looked up once per device; in
// host code the symbol itself is only a host-side stand-in for that address).
int scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cuda_failed();
  if (dev < 0 || dev >= kMaxDevices) return NVFP4MOE_ERR_DEVICE;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_route_scratch) != cudaSuccess || p == nullptr) return cuda_failed();
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return NVFP4MOE_OK;
}

}  // namespace
}  // namespace nvfp4moe

using namespace nvfp4moe;

extern "C" {

int nvfp4moe_route_noalloc(const nvfp4moe_cfg* cfg, const void* hidden_bf16, int64_t T, const float* w_router,
                           const float* logit_bias, int32_t* idx, float* w, void* stream) {
  int st = nvfp4moe_cfg_check(cfg);
  if (st != NVFP4MOE_OK) return st;
  if (T < 0 || T > (1 << 24)) return NVFP4MOE_ERR_SHAPE;
  if (T > 0 && (hidden_bf16 == nullptr || w_router == nullptr || idx == nullptr || w == nullptr ||
                reinterpret_cast<uintptr_t>(hidden_bf16) % 16 != 0 ||
                reinterpret_cast<uintptr_t>(w_router) % 16 != 0))
    return NVFP4MOE_ERR_ARG;
  // this call runs the FP32 logits kernels only (no digit-plane buffers), so only their
  // split-K partials have to fit
  if (T > 0 && router_fp32_parts_elems(T, cfg->E, cfg->H) > kNoAllocParts) return NVFP4MOE_ERR_WORKSPACE;
  int dev = 0, major = 0, minor = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
    return cuda_failed();
  if (major != 10 || minor != 0) return NVFP4MOE_ERR_DEVICE;
  void* scratch = nullptr;
  st = scratch_address(&scratch);
  if (st != NVFP4MOE_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  WsHeader* hdr = static_cast<WsHeader*>(scratch);
  // the array keeps the previous call's contents: the status word starts at zero; the
  // partial sums are overwritten before they are read
  if (reset_status(hdr, 1, s) != cudaSuccess) return cuda_failed();
  if (T == 0) return NVFP4MOE_OK;
  RouterArgs a{};
  a.x = static_cast<const uint16_t*>(hidden_bf16);
  a.w = w_router;
  a.bias = logit_bias;
  a.parts = reinterpret_cast<double*>(static_cast<uint8_t*>(scratch) + sizeof(WsHeader));
  a.idx = idx;
  a.wts = w;
  a.T = T;
  a.H = cfg->H;
  a.E = cfg->E;
  a.n_groups = cfg->n_groups;
  a.topk_groups = cfg->topk_groups;
  a.topk = cfg->topk;
  a.routed_scale = cfg->routed_scale;
  a.status = &hdr->status;
  return launch_router(a, s) == cudaSuccess ? NVFP4MOE_OK : cuda_failed();
}

}  // extern "C"
