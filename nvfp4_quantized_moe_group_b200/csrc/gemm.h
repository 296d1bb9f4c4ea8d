// Interface of the grouped NVFP4 expert GEMMs (gemm.cu): tile sizes, arguments, launchers.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace nvfp4moe {

constexpr int kBlockM = 128;             // token rows per GEMM tile / expert segment padding
constexpr int kWeightTileRows = 128;     // rows of one pre-tiled weight tile (gate/up: 64 gate + 64 up)
constexpr int kBlockK = 256;             // K values per pipeline stage (128 bytes of E2M1)

struct GemmArgs {
  const uint8_t* b_tiles;      // weights, tiled: [E][n_total/128][ceil(K/256)][128 rows][128 B], swizzled
  const uint8_t* sfa;          // swizzled scales of A (padded rows)
  const uint8_t* sfb;          // swizzled scales of B, experts back to back
  const int32_t* mtile_prefix; // [E+1] (may point into a longer table: entries are global tile numbers)
  const int32_t* counts;       // [E]
  int E;                       // experts of this launch (weights, scales, per-expert scalars indexed 0..E-1)
  int K;                       // reduction length
  int n_total;                 // B rows per expert (2I for gate/up, H for down)
  uint32_t* status;            // the call's status word; a timeout already raised in it (by an
                               // earlier kernel of the call) makes the GEMM do no work
  uint64_t wait_ns;            // limit of each bounded wait (0: kWaitLimitNs)
  int* work_counter;           // zero at launch: items handed out beyond the first gridDim.x
  // gate/up epilogue
  uint8_t* hq_codes;           // [rows_cap][I/2]
  uint8_t* hq_sf;              // swizzled [rows_cap][I/16]
  const float* g_x;            // device scalar
  const float* g_gate;         // [E]
  const float* g_up;           // [E]
  const float* g_h;            // [E]
  int I;
  float* zero_acc;             // optional [zero_acc_elems] FP32 zeroed by the launch's epilogue
  int64_t zero_acc_elems;      // warps (a slice per work item; gate/up launch only)
  // down epilogue
  float* acc;                  // [T][H]
  float* const* acc_peers;     // optional: token t's row is acc_peers[t / rows_per_peer] +
  int64_t rows_per_peer;       //   (t % rows_per_peer) * H instead of acc + t * H
  const int32_t* row_pair;     // [rows_cap]
  const float* wts;            // [T*topk]
  const float* alpha_down;     // [E] = g_h * g_down
  int topk;
  int H;
  // FP8 variant (per-row activation scales, per-output-channel weight scales)
  const float* a_scale;        // gate/up: [rows_cap] scale of each segment row of A
  const float* w_scale;        // [E][n_total] weight channel scales (gate/up in packed column order)
  float* h32;                  // gate/up: [rows_cap][I] FP32 SwiGLU product
  const float* h_scale;        // down: [rows_cap] scale of each segment row of A (= h)
  // debug (NVFP4 gate/up): the FP32 SwiGLU product h of every pair before its requantisation,
  // [pairs][I] in grouping order (pair position = dbg_offsets[e] + row in the expert's
  // segment); nullptr on the hot path
  float* h_dbg;
  const int32_t* dbg_offsets;  // [E + 1], with h_dbg
};

// gemm.cu
// tma_a / tma_a32: the A rows with a 128-row / 32-row box (both 128 bytes wide).  Work items
// are 256 output columns wide: n_total (2I, H) must be a multiple of 256.
// decode: the configuration for segments that average fewer than 32 rows.
cudaError_t launch_gemm_gateup(const CUtensorMap& tma_a, const CUtensorMap& tma_a32, const GemmArgs& a,
                               int grid, bool decode, cudaStream_t stream);
cudaError_t launch_gemm_down(const CUtensorMap& tma_a, const CUtensorMap& tma_a32, const GemmArgs& a,
                             int grid, bool decode, cudaStream_t stream);
// Both GEMMs in one persistent launch (NVFP4, the configuration for segments that average
// fewer than 32 rows): gate_up and down as for the two launches above (the same grouping
// tables, status and work counter: gate_up's), tma_h / tma_h32 the maps of the down GEMM's A
// rows (h).  dep: one zeroed counter per 128-row tile of the launch; a down item starts once its
// tile's counter reaches 8 per gate/up column tile.  lag: gate/up items claimed, beyond the
// largest expert's, between an expert's last gate/up item and its first down item.
cudaError_t launch_gemm_fused(const CUtensorMap& tma_a, const CUtensorMap& tma_a32, const CUtensorMap& tma_h,
                              const CUtensorMap& tma_h32, const GemmArgs& gate_up, const GemmArgs& down, int* dep,
                              int lag, int grid, cudaStream_t stream);
// The FP8 W8A8 variants: A and B are E4M3 rows of K bytes (tensor maps over K-byte rows), the
// scales come from a_scale / w_scale / h_scale, and gate/up writes FP32 h to h32.
cudaError_t launch_gemm_gateup_fp8(const CUtensorMap& tma_a, const CUtensorMap& tma_a32, const GemmArgs& a,
                                   int grid, bool decode, cudaStream_t stream);
cudaError_t launch_gemm_down_fp8(const CUtensorMap& tma_a, const CUtensorMap& tma_a32, const GemmArgs& a,
                                 int grid, bool decode, cudaStream_t stream);
// Weight codes [rows][row_bytes] -> tiled operand layout: source row r is packed row
// (r / group) * group * mul + add * group + r % group; packed rows form 128-row tiles, each
// split into 128-byte K blocks stored as contiguous 16 KB images of the 128-byte-swizzled
// shared-memory tile.  The destination must be zero where row_bytes is not a multiple of 128.
cudaError_t launch_tile_weights(const uint8_t* src, int rows, int row_bytes, uint8_t* dst, int group, int mul,
                                int add, cudaStream_t stream);
// Encodes a 2D byte tensor map [rows][row_bytes] with a 128-byte x box_rows box, 128B swizzle.
int make_tma_2d(CUtensorMap* map, const void* base, uint64_t row_bytes, uint64_t rows, uint32_t box_rows);

}  // namespace nvfp4moe
