/*
 * smc.h -- C ABI of libsmc, a submanifold sparse 3-D convolution (SubMConv3d)
 * for NVIDIA B200 (sm_100a).
 *
 * The operation (trellis_sparse_mlx README, "What's in it" and "Correctness"):
 * a sparse tensor is a set of N active voxels with coordinates (b, x, y, z)
 * and one feature row per voxel.  The submanifold convolution with a K x K x K
 * kernel (K = 3, or K = 1) produces one output row per INPUT voxel (the output
 * sites are exactly the input sites):
 *
 *     out[c] = sum over offsets d in {-1,0,1}^3 with c + stride*d active
 *              of feats[c + stride*d] @ W[k(d)]
 *
 * the cross-correlation convention (the row at c + d is gathered, not c - d).
 * Offsets are numbered k(d) = 9 (dx+1) + 3 (dy+1) + (dz+1), so k = 13 is the
 * centre.  Voxels of different batch index b are never neighbours.  The
 * README's "Performance" section is about caching the prepared device gather
 * index across calls; here that cache is the smc_handle_t.
 *
 * Conventions for every call:
 *   - "device pointer" = memory of the current CUDA device, contiguous,
 *     row-major, at least 16-byte aligned.  The caller owns every pointer it
 *     passes; the library never frees or retains them past the call.
 *   - Every function returns an smc_status (0 = SMC_OK) unless noted.  Errors
 *     found in the arguments are reported before anything is launched and
 *     leave every output buffer untouched.  Errors only the device can see
 *     (duplicate coordinates, out-of-range coordinates, a full hash table)
 *     are reported after the kernels that found them have run: the index
 *     build then frees what it allocated and writes no caller buffer, and
 *     smc_build_neighbor_map_static leaves map_dev undefined.
 *   - No call falls back to the CPU.  There is no alternative backend.
 */
#ifndef SMC_H_
#define SMC_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; 0 is the legacy default stream. */
typedef struct CUstream_st* smc_stream_t;

/* Opaque handle: the neighbour map and the tile plan of one coordinate set. */
typedef struct smc_index* smc_handle_t;

enum smc_status {
  SMC_OK = 0,
  SMC_ERR_INVALID = -1,     /* null pointer, negative size, misaligned pointer, bad K */
  SMC_ERR_DUPLICATE = -2,   /* the same (b,x,y,z) appears twice */
  SMC_ERR_RANGE = -3,       /* b outside [0, 32768) or x, y, z outside [0, 65536) */
  SMC_ERR_OOM = -4,         /* device allocation failed */
  SMC_ERR_CUDA = -5,        /* a CUDA runtime call or a launch failed */
  SMC_ERR_UNSUPPORTED = -6, /* a shape/dtype combination this build does not run */
  SMC_ERR_TABLE_FULL = -7,  /* the coordinate hash table ran out of slots */
  SMC_ERR_TIMEOUT = -8      /* a device-side wait gave up (see smc_device_status) */
};

enum smc_dtype { SMC_F32 = 0, SMC_F16 = 1, SMC_BF16 = 2 };

/* Row order used for the tile plan (smc_index_options.order). */
enum smc_order {
  SMC_ORDER_MASK = 0,  /* rows sorted by (number of active taps, Gray-code rank of the
                          tap mask): default */
  SMC_ORDER_INPUT = 1, /* rows in input order (ablation) */
  SMC_ORDER_GREEDY = 2 /* the mask order, then greedy packing inside segments of
                          1,024 rows: each tile grows by the masks that add the
                          fewest taps to its union (fewer taps multiplied; a
                          slower build) */
};

/* How neighbours are looked up (smc_index_options.lookup); both give the same
 * map, bit for bit. */
enum smc_lookup {
  SMC_LOOKUP_HASH = 0, /* open-addressing hash of packed coordinates: default */
  SMC_LOOKUP_SORT = 1  /* packed 64-bit keys radix-sorted, binary search per tap
                          ("Running TRELLIS.2 on a Mac (3/3)", "E. Vectorizing mesh
                          extraction": pack into int64, sort, searchsorted) */
};

typedef struct smc_index_options {
  int64_t table_capacity; /* hash slots; 0 = smallest power of two >= 2N.  A
                             value < N makes the build fail with
                             SMC_ERR_TABLE_FULL (used to test that path). */
  int32_t order;          /* enum smc_order */
  int32_t lookup;         /* enum smc_lookup */
} smc_index_options;

/*
 * Build the neighbour map and the tile plan of a coordinate set: the
 * "prepared device gather index" of the trellis_sparse_mlx README
 * ("Performance": caching it, not only the raw indice map, is what made the
 * layer compute-bound; "What's in it": a SparseTensor is coords [N,4] +
 * feats [N,C] with an indice-map cache).  Build once per coordinate set, then
 * run any number of smc_forward calls on the handle.
 *
 * coords_dev : device pointer, int32 [n][4] = (b, x, y, z), any row order.
 * n          : number of voxels, >= 0 (n == 0 gives an empty handle).
 * stride     : neighbour spacing, >= 1 (neighbours are at c + stride*d).
 * out_handle : receives the handle; caller releases it with smc_destroy.
 *
 * Runs on the legacy default stream and synchronises it before returning (it
 * reads the device status word: duplicates, range errors, table overflow).
 * coords_dev may be freed as soon as the call returns.
 * Errors: SMC_ERR_INVALID, _DUPLICATE, _RANGE, _OOM, _CUDA, _TABLE_FULL; on
 * error *out_handle is set to NULL.
 */
int smc_build_index(const int32_t* coords_dev, int64_t n, int32_t stride,
                    smc_handle_t* out_handle);

/* As smc_build_index, with options (NULL = defaults) and an explicit stream,
 * which the call synchronises before returning. */
int smc_build_index_ex(const int32_t* coords_dev, int64_t n, int32_t stride,
                       const smc_index_options* opts, smc_stream_t stream,
                       smc_handle_t* out_handle);

/* Largest n that smc_build_neighbor_map_static accepts. */
#define SMC_STATIC_MAX_VOXELS 524288

/*
 * Neighbour map with no device allocation by the library.  The pages this
 * library follows have no counterpart to this call; it exists for callers
 * that may not allocate device memory themselves: code running inside a
 * framework or server that reserves the GPU's memory up front and hands it out
 * from its own pool (a cudaMalloc beside that pool fails under its cap or
 * breaks its accounting), and latency-sensitive loops, where cudaMalloc and
 * cudaFree may synchronise the device and stall other streams.
 *
 * coords_dev : device pointer, int32 [n][4] = (b, x, y, z), 16-byte aligned.
 * n          : 0 <= n <= SMC_STATIC_MAX_VOXELS; a larger n returns
 *              SMC_ERR_UNSUPPORTED and launches nothing.
 * stride     : neighbour spacing, >= 1.
 * map_dev    : device pointer, int32 [n][27], written like
 *              smc_get_neighbor_map's output (-1 = no active neighbour).
 * stream     : the work is queued on this stream, which the call then
 *              synchronises to read the status word.  After
 *              SMC_ERR_DUPLICATE or SMC_ERR_RANGE the kernels have run and
 *              map_dev holds undefined values.
 *
 * Scratch: the coordinate hash table lives in one fixed array of static
 * device memory (about 18 MiB), reserved on every GPU that loads libsmc and
 * held until the process exits.  The first call on a device looks up that
 * array's device address (looked up again only if the device's CUDA context
 * changes, e.g. after cudaDeviceReset); make that first call before any
 * stream capture.
 * Every call, from any stream or host thread, uses the same array and clears
 * the part it needs first, so calls that overlap on the GPU race with each
 * other and must be serialised by the caller.
 * Errors: SMC_ERR_INVALID, _UNSUPPORTED, _DUPLICATE, _RANGE, _CUDA.
 */
int smc_build_neighbor_map_static(const int32_t* coords_dev, int64_t n, int32_t stride,
                                  int32_t* map_dev, smc_stream_t stream);

/*
 * SubMConv3d forward over the handle's voxels (trellis_sparse_mlx README,
 * "What's in it": the submanifold 3x3x3 and 1x1x1 sparse convolution;
 * "Correctness": feats[c+d] is gathered, cross-correlation).  Implements the
 * sum written at the top of this file.
 *
 * feats : device pointer, [n][cin] of dtype.
 * W     : device pointer, [K^3][cin][cout] of dtype, W[k][ci][co] (tap k as
 *         numbered above; for K = 1 the single tap is the centre).
 * out   : device pointer, [n][cout] of dtype; row i belongs to voxel i of the
 *         coordinates the handle was built from.  Written once per row, no
 *         atomics; every element is overwritten.
 * K     : 3 (uses the neighbour map) or 1 (per-row linear map, ignores it).
 * dtype : SMC_F16 / SMC_BF16 -- tensor cores, fp32 accumulation, output
 *         rounded to nearest; SMC_F32 -- CUDA cores, fp64 accumulation,
 *         output rounded once to fp32.
 * stream: the call is asynchronous on this stream and never synchronises.
 *         A forward only reads the handle (apart from setting its status
 *         word on a device error), so forwards on one handle may run on
 *         different streams at once.
 *
 * Tensor-core path when cin % 64 == 0 and cout % 64 == 0 (f16/bf16); any
 * other cin, cout >= 1 runs on the CUDA-core kernel.  feats and out must not
 * overlap.  The current device must be the one the handle was built on.
 * Errors: SMC_ERR_INVALID (null / misaligned pointers, K not 1 or 3, bad
 * dtype, cin or cout < 1, another current device), SMC_ERR_CUDA (launch
 * failure).  A device-side
 * wait that gives up is reported later by smc_device_status.
 */
int smc_forward(smc_handle_t h, const void* feats, const void* W, void* out, int K,
                int cin, int cout, int dtype, smc_stream_t stream);

/*
 * Launch-configuration search for smc_forward ("Metal-native replacement for
 * flex_gemm bottleneck?", "Open": autotuning of the tile shape and schedule).
 * Runs every tensor-core launch configuration valid for this layer shape
 * (output-column block, tiles per work item, 128-channel units or tap pairs)
 * on the given buffers, once to warm up and three times timed with CUDA
 * events on `stream`, and keeps the fastest in the handle for this
 * (K, cin, cout, dtype): later smc_forward / smc_forward_ex calls of that
 * shape use it.  Without a search they use a fixed rule.
 * Arguments as smc_forward; out is overwritten (it holds the forward result
 * afterwards).  chosen (host pointer, may be null) receives the configuration
 * id (name: smc_conv_config_name), or -1 when the shape runs on the CUDA
 * cores (nothing to choose).  Synchronises the stream.
 * Errors: as smc_forward; SMC_ERR_TIMEOUT when a candidate's device-side wait
 * gave up (the handle then keeps its previous choice).
 */
int smc_autotune(smc_handle_t h, const void* feats, const void* W, void* out, int K, int cin,
                 int cout, int dtype, smc_stream_t stream, int* chosen);

/* Static name of a launch configuration id ("cuda-cores" for -1). */
const char* smc_conv_config_name(int config);

/*
 * smc_autotune with the row order of the tile plan searched too
 * (search_orders != 0, K = 3): for SMC_ORDER_MASK and SMC_ORDER_GREEDY the
 * handle's plan is rebuilt in that order (smc_replan) and every launch
 * configuration timed; the handle keeps the fastest (order, configuration).
 * The order belongs to the whole handle, so it applies to every layer that
 * uses it.  chosen_order (host pointer, may be null) receives the order.
 * Synchronises the device; no other call may use the handle meanwhile.
 * Errors: as smc_autotune, plus those of smc_replan.
 */
int smc_autotune_ex(smc_handle_t h, const void* feats, const void* W, void* out, int K, int cin,
                    int cout, int dtype, int search_orders, smc_stream_t stream,
                    int* chosen_config, int* chosen_order);

/*
 * Rebuild the handle's tile plan (row order, tiles, gather index, work items,
 * tap lists) in another row order (enum smc_order) from the neighbour map
 * and tap masks it already holds; the neighbour map is unchanged and the
 * coordinates are not needed.  Waits for all work on the handle's device
 * first (a forward in flight reads the plan), then runs on `stream` and
 * synchronises it.  Configurations chosen by smc_autotune are dropped.
 * Errors: SMC_ERR_INVALID (null handle, bad order, another current device),
 * SMC_ERR_OOM (scratch), SMC_ERR_CUDA.
 */
int smc_replan(smc_handle_t h, int order, smc_stream_t stream);

/*
 * Input gradient of smc_forward ("Metal-native replacement for flex_gemm
 * bottleneck?", "Fixed" / "Open": the bwd-input pass next to fwd):
 *
 *     grad_in[j] = sum over (i, k) with voxel j at coords[i] + stride*d(k)
 *                  of grad_out[i] @ W[k]^T
 *
 * the adjoint of the forward sum in feats.  Because j is i's tap-k neighbour
 * exactly when i is j's tap-(26 - k) neighbour, this is the forward
 * convolution of grad_out with the weights W'[k] = W[26 - k]^T, and it runs on
 * the same kernels and tile plan.
 *
 * grad_out : device pointer, [n][cout] of dtype.
 * W        : device pointer, [K^3][cin][cout] of dtype (the forward weights).
 * grad_in  : device pointer, [n][cin] of dtype; every element is overwritten.
 * K, cin, cout, dtype, stream: as for smc_forward (cin and cout are the
 *         forward layer's).  Asynchronous; calls on one handle must be
 *         stream-ordered.  The transposed weights live in a workspace the
 *         handle owns, allocated stream-ordered from the library's memory pool
 *         the first time a call needs more than it holds.
 * Errors: as smc_forward, plus SMC_ERR_OOM.
 */
int smc_backward_input(smc_handle_t h, const void* grad_out, const void* W, void* grad_in, int K,
                       int cin, int cout, int dtype, smc_stream_t stream);

/*
 * Weight gradient of smc_forward (the bwd-weight pass of the same passage):
 *
 *     dW[k] = sum over voxels i with an active tap-k neighbour j
 *             of outer(feats[j], grad_out[i])          ([cin][cout] per tap)
 *
 * feats    : device pointer, [n][cin] of dtype (the forward input).
 * grad_out : device pointer, [n][cout] of dtype.
 * dW       : device pointer, float32 [K^3][cin][cout]; every element is
 *            overwritten (taps with no pair get zeros).  fp32 whatever dtype
 *            is: weight gradients are accumulated in fp32 (f16/bf16 inputs,
 *            tensor cores) or fp64 (f32 inputs, CUDA cores) and rounded once.
 * The sum over pairs is split over CTAs; the partial sums go to a workspace
 * the handle owns (allocated stream-ordered when it must grow) and are added
 * in a fixed order, so the result is deterministic.  Asynchronous; calls on
 * one handle must be stream-ordered.
 * Errors: as smc_forward, plus SMC_ERR_OOM.
 */
int smc_backward_weight(smc_handle_t h, const void* feats, const void* grad_out, float* dW, int K,
                        int cin, int cout, int dtype, smc_stream_t stream);

/*
 * x2 downsample of a sparse tensor by maximum (trellis_sparse_mlx README,
 * "What's in it": the downsample half of the subdivide / downsample row, "x2
 * max-pool", reduce="amax").  The parent of (b, x, y, z) is
 * (b, x >> 1, y >> 1, z >> 1); every parent appears once, in lexicographic
 * (b, x, y, z) order, and its row is the element-wise maximum of its
 * children's rows (an exact copy of one input value per element).
 *
 * coords_dev     : device pointer, int32 [n][4], any order, no duplicates
 *                  needed (duplicates simply share a parent).
 * feats_dev      : device pointer, [n][c] of dtype.
 * out_coords_dev : device pointer, int32 [n][4] (room for n parents).
 * out_feats_dev  : device pointer, [n][c] of dtype.
 * out_n          : host pointer, receives the number of parents m; rows
 *                  [0, m) of both outputs are written.
 * Queued on stream, which the call synchronises to read m back; its scratch
 * is allocated and freed stream-ordered from the library's memory pool.
 * Errors: SMC_ERR_INVALID, _RANGE (coordinates outside the packing limits;
 * outputs undefined), _OOM, _CUDA, _UNSUPPORTED (n >= 2^31).
 */
int smc_downsample2(const int32_t* coords_dev, int64_t n, const void* feats_dev, int c, int dtype,
                    int32_t* out_coords_dev, void* out_feats_dev, int64_t* out_n,
                    smc_stream_t stream);

/*
 * x2 subdivision (the subdivide half of the same row, "x2 coord expansion"):
 * voxel i's 8 children (b, 2x + dx, 2y + dy, 2z + dz) are rows 8 i + c,
 * c = 4 dx + 2 dy + dz, and each carries a copy of voxel i's row.
 *
 * coords_dev     : device pointer, int32 [n][4]; x, y, z must be below 32768
 *                  so the children stay inside the packing limits.
 * feats_dev      : device pointer, [n][c] of dtype.
 * out_coords_dev : device pointer, int32 [8 n][4].
 * out_feats_dev  : device pointer, [8 n][c] of dtype.
 * Synchronises stream to read the range check.  Errors: SMC_ERR_INVALID,
 * _RANGE (outputs undefined), _OOM, _CUDA, _UNSUPPORTED (n >= 2^28).
 */
int smc_subdivide2(const int32_t* coords_dev, int64_t n, const void* feats_dev, int c, int dtype,
                   int32_t* out_coords_dev, void* out_feats_dev, smc_stream_t stream);

/* Activation of the fused epilogue (smc_epilogue.activation). */
enum smc_activation {
  SMC_ACT_NONE = 0,
  SMC_ACT_RELU = 1, /* max(v, 0) */
  SMC_ACT_SILU = 2, /* v / (1 + exp(-v)) */
  SMC_ACT_GELU = 3  /* v / 2 * (1 + erf(v / sqrt 2)), the exact form */
};

/* Element-wise work fused into the convolution's epilogue. */
typedef struct smc_epilogue {
  const void* bias;     /* device pointer, [cout] of dtype, or NULL */
  const void* residual; /* device pointer, [n][cout] of dtype, or NULL; may not
                           overlap out */
  int32_t activation;   /* enum smc_activation */
  int32_t reserved;     /* must be 0 */
} smc_epilogue;

/*
 * smc_forward with a fused epilogue: out = act(conv + bias) + residual,
 * computed on the fp32 (fp64 for SMC_F32) accumulator before the one rounding
 * to dtype.  This is the layer shape of the sparse ResBlock (trellis_sparse_mlx
 * README, "What's in it": SparseLinear, SparseSiLU/GELU, SparseResBlock): a
 * convolution with bias, followed by an activation or closed by the skip
 * connection's sum, in one pass over the output.  ep == NULL is smc_forward.
 * Errors: as smc_forward; SMC_ERR_INVALID also for a bad activation, a
 * non-zero reserved field or misaligned bias / residual pointers.
 */
int smc_forward_ex(smc_handle_t h, const void* feats, const void* W, void* out, int K, int cin,
                   int cout, int dtype, const smc_epilogue* ep, smc_stream_t stream);

/* Copy the int32 [n][27] neighbour map (-1 = no active neighbour) into
 * map_dev, asynchronously on stream.  Entry [i][k] is the row j whose
 * coordinates are coords[i] + stride * d(k) in the same batch: the indice map
 * of the trellis_sparse_mlx README ("What's in it", SparseTensor's indice-map
 * cache), with -1 in place of its unnamed sentinel ("Performance"). */
int smc_get_neighbor_map(smc_handle_t h, int32_t* map_dev, smc_stream_t stream);

/* Work counts of the tile plan (the masked implicit GEMM skips every tap no
 * row of a 128-row tile uses, as mtlgemm's sorted_idx / valid_kernel masking
 * does in "Metal-native replacement for flex_gemm bottleneck?", "Fixed").
 * Host-side counts fixed at build time: useful_pairs = number of
 * (voxel, active neighbour) pairs, i.e. non-sentinel map entries;
 * issued_rows_taps = rows x taps the tensor-core kernel multiplies for K = 3
 * (128 rows per tile times the taps active anywhere in the tile).  Either
 * pointer may be NULL. */
int smc_get_plan_stats(smc_handle_t h, int64_t* useful_pairs, int64_t* issued_rows_taps);

/* Number of voxels and of 128-row tiles. Either pointer may be NULL. */
int smc_get_sizes(smc_handle_t h, int64_t* n, int64_t* n_tiles);

/* Copy the tile plan into device buffers, asynchronously on stream:
 * perm_dev int32 [n] (the voxel behind plan row p; tile t holds plan rows
 * [128 t, 128 t + 128)), tile_mask_dev uint32 [n_tiles] (bit k set when tap k
 * is multiplied for that tile).  Either pointer may be NULL. */
int smc_get_tile_plan(smc_handle_t h, int32_t* perm_dev, uint32_t* tile_mask_dev,
                      smc_stream_t stream);

/* Read and clear the handle's device status word (synchronises the stream):
 * SMC_OK, or SMC_ERR_TIMEOUT when a kernel gave up waiting. */
int smc_device_status(smc_handle_t h, smc_stream_t stream);

/* Release the handle's device memory.  Synchronous: it first waits for all
 * work queued on the handle's device, on every stream, so a forward still in
 * flight never reads freed memory.  NULL is ignored. */
void smc_destroy(smc_handle_t h);

/* Static string for a status code. */
const char* smc_status_string(int status);

/* Library version, major * 10000 + minor * 100 + patch. */
int smc_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SMC_H_ */
