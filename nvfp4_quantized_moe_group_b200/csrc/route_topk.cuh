// Group-limited top-k selection of one token, shared by the router kernels.
// "Reflection releases Beam ...", section "Mixture-of-Experts details": the score of a group is
// the sum of its two best sigmoid scores, the best topk_groups groups are kept, and the topk
// best experts inside the kept groups are routed to with weights
// routed_scale * s / sum(selected s).  Equal scores go to the lower index (groups and experts).
#pragma once

#include "common.cuh"

namespace nvfp4moe {

constexpr int kTopkThreads = 256;

// Sigmoid of an FP32 logit, IEEE-rounded division.
__device__ __forceinline__ float router_sigmoid(float l) {
  return __fdiv_rn(1.0f, __fadd_rn(1.0f, expf(-l)));
}

// Called by all kTopkThreads threads of a CTA (it synchronises the CTA).  sc[0..E) holds the
// token's sigmoid scores in shared memory; a NaN score (a non-finite logit) is replaced by -1
// in place, raises kStatusNonFinite, and so ranks below every finite score (the selected
// indices are always distinct and inside [0, E)).
// E <= 256, E / n_groups <= 32, topk <= 8 and topk <= topk_groups * (E / n_groups).
//
// Every step is a rank count, so all threads work at once: rank of a value = number of
// values above it plus equal values at lower expert indices.  Group score = (rank 0) +
// (rank 1) of the group; kept groups = group rank < topk_groups; an expert can only be
// selected if it is among the topk best of its group, so those (at most topk per kept group)
// are the candidates, and a candidate's rank among them is its selection slot.  The weight
// sum adds the selected scores in slot order.  Within a group of a power-of-two size, and
// among at most 32 candidates, the values are exchanged with warp shuffles.
__device__ __forceinline__ void route_topk_block(float* sc, int E, int n_groups, int topk_groups, int topk,
                                                 float routed_scale, int32_t* idx_out, float* w_out,
                                                 uint32_t* status) {
  __shared__ float s_top1[32], s_top2[32], s_gsc[32];
  __shared__ int s_keep[32];
  __shared__ float s_cv[256];        // candidates' scores
  __shared__ int s_ce[256];          // their expert indices
  __shared__ float s_sel_s[8];
  __shared__ int s_sel_e[8];
  const int tid = threadIdx.x;
  const int G = n_groups, gs = E / n_groups;

  bool nan = false;
  float v = -3.0f;
  if (tid < E) {
    v = sc[tid];
    nan = (v != v);
    if (nan) {
      v = -1.0f;
      sc[tid] = v;
    }
  }
  if (__syncthreads_or(nan) && tid == 0 && status != nullptr) raise_status(status, kStatusNonFinite);
  // rank of each expert inside its group
  int rg = 0;
  const int g = tid / gs;
  if ((gs & (gs - 1)) == 0) {
    const int lane_g = tid % gs;
    // unconditional shuffles with a compile-time trip count (a shuffle under a branch makes
    // the warp reconverge around it); only the count is predicated
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const float o = __shfl_sync(0xffffffffu, v, j, gs);
      rg += (int)((j < gs) & ((o > v) | ((o == v) & (j < lane_g))));
    }
  } else if (tid < E) {
    const int j0 = g * gs;
    for (int j = 0; j < gs; ++j) {
      const float o = sc[j0 + j];
      rg += (o > v) || (o == v && j0 + j < tid);
    }
  }
  if (tid < E) {
    if (rg == 0) s_top1[g] = v;
    if (rg == 1) s_top2[g] = v;
  }
  __syncthreads();
  if (tid < 32) s_gsc[tid] = tid >= G ? -4.0f : gs >= 2 ? __fadd_rn(s_top1[tid], s_top2[tid]) : s_top1[tid];
  __syncthreads();
  if (tid < 32) {
    const float mine = s_gsc[tid];
    int rank = 0;
#pragma unroll
    for (int h = 0; h < 32; ++h) {
      const float o = s_gsc[h];   // entries past G are never counted
      rank += (int)((h < G) & ((o > mine) | ((o == mine) & (h < tid))));
    }
    s_keep[tid] = tid < G && rank < topk_groups;
  }
  __syncthreads();
  // candidates: the best kc = min(gs, topk) of each kept group (exactly topk_groups are kept)
  const int kc = gs < topk ? gs : topk;
  const int n_cand = topk_groups * kc;
  if (tid < E && rg < kc && s_keep[g]) {
    int before = 0;
#pragma unroll
    for (int h = 0; h < 32; ++h) before += (h < g) ? s_keep[h] : 0;
    s_cv[before * kc + rg] = v;
    s_ce[before * kc + rg] = tid;
  }
  __syncthreads();
  if (n_cand <= 32) {
    if (tid < 32) {
      const float c = tid < n_cand ? s_cv[tid] : -4.0f;
      const int ce = tid < n_cand ? s_ce[tid] : 0x7FFFFFFF;
      int r = 0;
#pragma unroll
      for (int q = 0; q < 32; ++q) {   // lanes past n_cand hold -4: they never outrank
        const float o = __shfl_sync(0xffffffffu, c, q);
        const int oe = __shfl_sync(0xffffffffu, ce, q);
        r += (int)((o > c) | ((o == c) & (oe < ce)));
      }
      if (tid < n_cand && r < topk) {
        s_sel_s[r] = c;
        s_sel_e[r] = ce;
      }
    }
  } else if (tid < n_cand) {
    const float c = s_cv[tid];
    const int ce = s_ce[tid];
    int r = 0;
    for (int q = 0; q < n_cand; ++q) {
      const float o = s_cv[q];
      r += (o > c) || (o == c && s_ce[q] < ce);
    }
    if (r < topk) {
      s_sel_s[r] = c;
      s_sel_e[r] = ce;
    }
  }
  __syncthreads();
  if (tid < topk) {
    float sum = 0.f;
    for (int j = 0; j < topk; ++j) sum = __fadd_rn(sum, s_sel_s[j]);
    idx_out[tid] = s_sel_e[tid];
    w_out[tid] = __fdiv_rn(__fmul_rn(routed_scale, s_sel_s[tid]), sum);
  }
  __syncthreads();
}

}  // namespace nvfp4moe
