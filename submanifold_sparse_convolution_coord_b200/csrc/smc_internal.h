// Internal declarations of libsmc (not part of the C ABI).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/smc.h"

namespace smc {

constexpr int kTaps = 27;       // 3 x 3 x 3 offsets
constexpr int kCentreTap = 13;  // d = (0, 0, 0)
constexpr int kTileRows = 128;  // rows per tensor-core tile (UMMA M)

// Coordinate packing limits: 15 bits of batch, 16 bits per axis.
constexpr int32_t kMaxBatch = 1 << 15;
constexpr int32_t kMaxAxis = 1 << 16;

// Device status word values (written by kernels, read by the host).
constexpr int32_t kDevOk = 0;
constexpr int32_t kDevDuplicate = 1;
constexpr int32_t kDevRange = 2;
constexpr int32_t kDevTableFull = 4;
constexpr int32_t kDevTimeout = 8;

struct Plan {
  int64_t n = 0;
  int64_t n_tiles = 0;
  int64_t total_slots = 0;     // sum over tiles of active taps
  int32_t* nbr = nullptr;      // [n][27]
  uint32_t* mask = nullptr;    // [n] bit k = tap k has an active neighbour
  int32_t* perm = nullptr;     // [n] plan row -> voxel
  uint32_t* tile_mask = nullptr;  // [n_tiles]
  int32_t* tile_off = nullptr;    // [n_tiles + 1] first slot of each tile
  uint8_t* tile_taps = nullptr;   // [n_tiles][32] active taps, ascending
  int32_t* gidx = nullptr;        // [total_slots][128] voxel gathered per row, -1 = none
  int32_t* out_row = nullptr;     // [n_tiles * 128] voxel written per plan row, -1 = none
  int32_t* status = nullptr;      // device status word
  uint32_t* work_counter = nullptr;  // tensor-core kernel's item counter (+ finished CTAs)
  // group_order[G - 1][q]: the q-th work item's group of G consecutive tiles,
  // most taps first (G = 1, 2), so the largest items are handed out first
  int32_t* group_order[2] = {nullptr, nullptr};
  int64_t useful_pairs = 0;
  int64_t issued_rows_taps = 0;
};

// Index build (smc_index.cu).  Returns an smc_status.
int build_plan(const int32_t* coords, int64_t n, int32_t stride, int64_t table_capacity,
               int32_t order, cudaStream_t stream, Plan* plan);
void free_plan(Plan* plan);

// Tensor-core convolution (smc_conv_tc.cu).  feats/W/out in f16 or bf16.
// dense = true runs the K = 1 form (rows in order, one tap, no plan arrays).
int launch_conv_tc(const Plan& plan, bool dense, const void* feats, const void* W, void* out,
                   int cin, int cout, int dtype, cudaStream_t stream);
bool conv_tc_supported(int cin, int cout, int dtype);

// CUDA-core convolution (smc_conv_simt.cu): any cin, cout, dtype.
int launch_conv_simt(const Plan& plan, bool dense, const void* feats, const void* W, void* out,
                     int cin, int cout, int dtype, cudaStream_t stream);

}  // namespace smc
