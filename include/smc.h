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
 *   - Every function returns an smc_status (0 = SMC_OK) unless noted; on an
 *     error nothing has been launched and output buffers are untouched.
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
  SMC_ORDER_INPUT = 1  /* rows in input order (ablation) */
};

typedef struct smc_index_options {
  int64_t table_capacity; /* hash slots; 0 = smallest power of two >= 2N.  A
                             value < N makes the build fail with
                             SMC_ERR_TABLE_FULL (used to test that path). */
  int32_t order;          /* enum smc_order */
  int32_t reserved;       /* must be 0 */
} smc_index_options;

/*
 * Build the neighbour map and the tile plan of a coordinate set.
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
 *              synchronises to read the status word.
 *
 * Scratch: the coordinate hash table lives in one fixed array of static
 * device memory (about 14 MiB), reserved on every GPU that loads libsmc and
 * held until the process exits.  The first call on a device looks up that
 * array's device address; make that first call before any stream capture.
 * Every call, from any stream or host thread, uses the same array and clears
 * the part it needs first, so calls that overlap on the GPU race with each
 * other and must be serialised by the caller.
 * Errors: SMC_ERR_INVALID, _UNSUPPORTED, _DUPLICATE, _RANGE, _CUDA.
 */
int smc_build_neighbor_map_static(const int32_t* coords_dev, int64_t n, int32_t stride,
                                  int32_t* map_dev, smc_stream_t stream);

/*
 * SubMConv3d forward over the handle's voxels.
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
 *         Forward calls that use the same handle must be ordered (one stream,
 *         or events): the tensor-core kernel keeps its work counter in the
 *         handle.
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

/* Copy the int32 [n][27] neighbour map (-1 = no active neighbour) into
 * map_dev, asynchronously on stream. */
int smc_get_neighbor_map(smc_handle_t h, int32_t* map_dev, smc_stream_t stream);

/* Host-side counts fixed at build time: useful_pairs = number of
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

/* Release the handle's device memory (synchronous).  NULL is ignored. */
void smc_destroy(smc_handle_t h);

/* Static string for a status code. */
const char* smc_status_string(int status);

/* Library version, major * 10000 + minor * 100 + patch. */
int smc_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SMC_H_ */
