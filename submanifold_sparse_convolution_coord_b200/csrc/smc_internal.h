// Internal declarations of libsmc (not part of the C ABI).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/smc.h"

namespace smc {

constexpr int kTaps = 27;       // 3 x 3 x 3 offsets
constexpr int kCentreTap = 13;  // d = (0, 0, 0)
constexpr int kTileRows = 128;  // rows per tensor-core tile (UMMA M)
constexpr int kBwdChunk = 32;   // tiles per CTA of the weight-gradient kernel

// Coordinate packing limits: 15 bits of batch, 16 bits per axis.
constexpr int32_t kMaxBatch = 1 << 15;
constexpr int32_t kMaxAxis = 1 << 16;

// Device status word values (written by kernels, read by the host).
constexpr int32_t kDevOk = 0;
constexpr int32_t kDevDuplicate = 1;
constexpr int32_t kDevRange = 2;
constexpr int32_t kDevTableFull = 4;
constexpr int32_t kDevTimeout = 8;
constexpr int32_t kDevLayout = 16;  // a kernel found its shared memory misaligned

struct Plan {
  void* arena = nullptr;       // one device allocation holding every array below
  int64_t n = 0;
  int64_t n_tiles = 0;
  int64_t total_slots = 0;     // sum over tiles of active taps
  int32_t* nbr = nullptr;      // [n][27]
  uint32_t* mask = nullptr;    // [n] bit k = tap k has an active neighbour
  int32_t* perm = nullptr;     // [n] plan row -> voxel
  uint32_t* tile_mask = nullptr;  // [n_tiles]
  int32_t* tile_off = nullptr;    // [n_tiles + 1] first slot of each tile
  int32_t* gidx = nullptr;        // [total_slots][128] voxel gathered per row, -1 = none
                                  // (room for 27 slots per tile)
  int32_t* out_row = nullptr;     // [n_tiles * 128] voxel written per plan row, -1 = none
  int32_t* status = nullptr;      // device status word
  // items[G - 1][q]: the q-th work item of G consecutive tiles (G = 1, 2),
  // most taps first, so the largest items are handed out first:
  // {first tile, its tap mask, the next tile's mask (0 if none or G = 1),
  //  first gather-index slot of the first tile}
  int4* items[2] = {nullptr, nullptr};
  // tap-major tile lists (weight gradient): entries tap_start[k] ..
  // tap_start[k + 1] - 1 of tap_tiles are {tile, gather-index slot} of the
  // tiles whose mask has tap k, in tile order; tap_chunk[k] is the first
  // weight-gradient chunk (kBwdChunk tiles) of tap k, tap_chunk[27] the count
  int2* tap_tiles = nullptr;     // [total_slots]
  int32_t* tap_start = nullptr;  // [28]
  int32_t* tap_chunk = nullptr;  // [28]
  int64_t useful_pairs = 0;
  int64_t issued_rows_taps = 0;
};

// Stream-ordered device memory from libsmc's own pool on the current device
// (smc_pool.cu): freed memory stays reserved for the next allocation.
cudaError_t dev_alloc(void** ptr, size_t bytes, cudaStream_t s);
cudaError_t dev_free(void* ptr, cudaStream_t s);

// Fused epilogue of a convolution: out = act(conv + bias) + residual, each
// part optional (null pointers, act = SMC_ACT_NONE).  bias [cout] and
// residual [n][cout] are in the convolution's dtype.
struct Epilogue {
  const void* bias = nullptr;
  const void* residual = nullptr;
  int act = 0;
};

// Index build (smc_index.cu).  Returns an smc_status.
int build_plan(const int32_t* coords, int64_t n, int32_t stride, int64_t table_capacity,
               int32_t order, int32_t lookup, cudaStream_t stream, Plan* plan);
void free_plan(Plan* plan);
// Rebuild the row order, tile plan and work items of a built plan in another
// order, from its neighbour map and masks (smc_index.cu).  Waits for the
// device first: no forward may be reading the plan.
int replan(Plan* plan, int32_t order, cudaStream_t stream);

// Tensor-core convolution (smc_conv_tc.cu).  feats/W/out in f16 or bf16.
// dense = true runs the K = 1 form (rows in order, one tap, no plan arrays).
// cfg selects a launch configuration (ConvConfig), -1 the default rule.
int launch_conv_tc(const Plan& plan, bool dense, const void* feats, const void* W, void* out,
                   int cin, int cout, int dtype, const Epilogue& ep, cudaStream_t stream,
                   int cfg = -1);
bool conv_tc_supported(int cin, int cout, int dtype);
// Launch configurations of the tensor-core kernel: output-column block (BN),
// tiles per work item (G), 128-channel units (k128) or tap pairs (pair).
enum ConvConfig : int {
  kCfg256G2 = 0,  // BN 256, two tiles per item sharing each W slice, one accumulator set
  kCfg256G1,      // BN 256, one tile per item
  kCfg256G1K2,    // BN 256, one tile per item, 128-channel units
  kCfg128G2K2,    // BN 128, two tiles per item, 128-channel units
  kCfg128G1K2,    // BN 128, one tile per item, 128-channel units
  kCfg128G1Pair,  // BN 128, one tile per item, two taps per unit (Cin = 64, K = 3)
  kCfg128G2,      // BN 128, two tiles per item, 64-channel units
  kCfg128G1,      // BN 128, one tile per item, 64-channel units
  kCfg64G1Pair,   // BN 64, one tile per item, two taps per unit (Cin = 64, K = 3)
  kCfg64G2,       // BN 64, two tiles per item, 64-channel units
  kCfg64G1,       // BN 64, one tile per item, 64-channel units
  kConvConfigs
};
bool conv_config_valid(int cfg, bool dense, int cin, int cout);
int conv_default_config(const Plan& plan, bool dense, int cin, int cout);
const char* conv_config_name(int cfg);

// Stable LSD radix sort of (key, value) pairs by the low `bits` bits of the
// key, 8 bits per pass (smc_sort.cu).  Reads buffer `cur`, ping-pongs between
// the two, and reports in *out_cur the buffer holding the result.  hist needs
// sort_hist_words(n) words.
size_t sort_hist_words(int64_t n);
// In-place exclusive scan of m uint32 counts (one block; for m up to a few
// million).
int scan_exclusive(uint32_t* data, int64_t m, cudaStream_t s);
template <class K>
int radix_sort(K* const keys[2], int32_t* const vals[2], int cur, int64_t n, int bits,
               uint32_t* hist, cudaStream_t s, int* out_cur);

// Wait limit of the kernels' bounded waits (smc_conv_tc.cu): 2 s, or
// SMC_DEBUG_WAIT_LIMIT_NS, read once per process.
uint64_t wait_limit_ns();

// Backward passes (smc_backward.cu).
// Wt[k][co][ci] = W[taps - 1 - k][ci][co] (dtype's element size).
int launch_weight_transpose(const void* W, void* Wt, int taps, int cin, int cout, int dtype,
                            cudaStream_t stream);
bool bwd_weight_tc_supported(int cin, int cout, int dtype);
int64_t bwd_weight_chunks(const Plan& plan, bool dense);
// Bytes of the weight-gradient workspace (partial sums); 0 = none needed.
size_t bwd_weight_workspace_bytes(const Plan& plan, bool dense, int cin, int cout, int dtype);
int launch_bwd_weight(const Plan& plan, bool dense, const void* feats, const void* grad, float* dW,
                      int cin, int cout, int dtype, void* workspace, uint64_t wait_ns,
                      cudaStream_t stream);

// x2 coordinate operations (smc_coords.cu).
int downsample2(const int32_t* coords, int64_t n, const void* feats, int c, int dtype,
                int32_t* out_coords, void* out_feats, int64_t* out_n, cudaStream_t s);
int subdivide2(const int32_t* coords, int64_t n, const void* feats, int c, int dtype,
               int32_t* out_coords, void* out_feats, cudaStream_t s);

// CUDA-core convolution (smc_conv_simt.cu): any cin, cout, dtype.
int launch_conv_simt(const Plan& plan, bool dense, const void* feats, const void* W, void* out,
                     int cin, int cout, int dtype, const Epilogue& ep, cudaStream_t stream);

}  // namespace smc
