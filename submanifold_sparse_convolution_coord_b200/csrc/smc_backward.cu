// Backward passes of SubMConv3d ("Metal-native replacement for flex_gemm
// bottleneck?", "Fixed" / "Open": fwd / bwd-input / bwd-weight).
//
// The forward is linear in feats and in W; every term feats[j] @ W[k] it adds
// to out[i] (j = the tap-k neighbour of i) has two adjoints:
//
//   input gradient   grad_in[j] += grad_out[i] @ W[k]^T
//   weight gradient  dW[k]      += outer(feats[j], grad_out[i])
//
// Input gradient.  j is i's tap-k neighbour exactly when i is j's
// tap-(26 - k) neighbour (the offsets are mirror images), so grad_in is the
// forward convolution of grad_out with W'[k] = W[26 - k]^T: one small
// transpose kernel (k_weight_transpose) and then the forward kernels on the
// handle's own tile plan.
//
// Weight gradient.  For tap k, dW[k] = A_k^T G over the pairs of tap k: the
// tile plan already lists them, tile by tile (row r of tile t gathers voxel
// gidx[t, k][r] and belongs to voxel out_row[t][r]).  The tensor-core kernel
// (k_bwd_weight_tc) gives each CTA a chunk of up to kBwdChunk tiles of one tap
// and one (128-input-channel, BN-output-channel) block of dW[k]; it gathers
// the A rows (neighbour features) and G rows (the tile's output gradients)
// 64 rows at a time and accumulates D[ci][co] += A^T G on tcgen05 with both
// operands MN-major (the gathered rows are K), fp32 in tensor memory.  Each
// CTA writes its partial block; k_bwd_weight_reduce adds a tap's chunks in
// chunk order (deterministic, no atomics) into the fp32 dW.  fp32 inputs, and
// channel counts off the 64-grid, run on k_bwd_weight_simt (one thread per
// dW element, fp64 accumulation for fp32).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <algorithm>
#include <cstdlib>

#include "smc_internal.h"
#include "smc_ptx.cuh"

namespace smc {
namespace {

using namespace ptx;

template <class T>
__device__ __forceinline__ float to_f(T v);
template <>
__device__ __forceinline__ float to_f<__half>(__half v) {
  return __half2float(v);
}
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 v) {
  return __bfloat162float(v);
}
template <>
__device__ __forceinline__ float to_f<float>(float v) {
  return v;
}

// Wt[k][co][ci] = W[taps - 1 - k][ci][co], 32 x 32 tiles through shared memory.
template <class T>
__global__ void k_weight_transpose(const T* __restrict__ W, T* __restrict__ Wt, int taps, int cin,
                                   int cout) {
  __shared__ T tile[32][33];
  const int k = blockIdx.z;
  const int ci0 = blockIdx.y * 32, co0 = blockIdx.x * 32;
  const T* src = W + size_t(taps - 1 - k) * cin * cout;
  T* dst = Wt + size_t(k) * cin * cout;
  for (int y = threadIdx.y; y < 32; y += blockDim.y) {
    const int ci = ci0 + y, co = co0 + threadIdx.x;
    if (ci < cin && co < cout) tile[y][threadIdx.x] = src[size_t(ci) * cout + co];
  }
  __syncthreads();
  for (int y = threadIdx.y; y < 32; y += blockDim.y) {
    const int co = co0 + y, ci = ci0 + threadIdx.x;
    if (ci < cin && co < cout) dst[size_t(co) * cin + ci] = tile[threadIdx.x][y];
  }
}

// One thread per dW element (k, ci, co): the sum over tap k's pairs in tile
// order, accumulated in Acc (double for fp32 inputs).
template <class T, class Acc>
__global__ void k_bwd_weight_simt(const T* __restrict__ feats, const T* __restrict__ grad,
                                  const int2* __restrict__ tap_tiles,
                                  const int32_t* __restrict__ tap_start,
                                  const int32_t* __restrict__ gidx,
                                  const int32_t* __restrict__ out_row, int64_t n, int taps, int cin,
                                  int cout, int dense, float* __restrict__ dW) {
  const int64_t id = blockIdx.x * int64_t(blockDim.x) + threadIdx.x;
  if (id >= int64_t(taps) * cin * cout) return;
  const int co = int(id % cout);
  const int ci = int((id / cout) % cin);
  const int k = int(id / (int64_t(cin) * cout));
  Acc acc = 0;
  if (dense) {
    for (int64_t i = 0; i < n; ++i)
      acc += Acc(to_f(feats[i * cin + ci])) * Acc(to_f(grad[i * cout + co]));
  } else {
    for (int e = tap_start[k]; e < tap_start[k + 1]; ++e) {
      const int2 ts = tap_tiles[e];
      const int32_t* gi = gidx + int64_t(ts.y) * kTileRows;
      const int32_t* orow = out_row + int64_t(ts.x) * kTileRows;
      for (int r = 0; r < kTileRows; ++r) {
        const int32_t j = gi[r];
        if (j < 0) continue;
        const int32_t i = orow[r];
        acc += Acc(to_f(feats[int64_t(j) * cin + ci])) * Acc(to_f(grad[int64_t(i) * cout + co]));
      }
    }
  }
  dW[id] = float(acc);
}

// ----------------------------------------------------------------------------
// tensor-core weight gradient
// ----------------------------------------------------------------------------
constexpr int kBwdStages = 5;
constexpr int kBwdRows = 64;                   // gathered rows per stage (two per tile)
constexpr int kBwdAtom = kBwdRows * 128;       // one 64-channel column of a stage: 8 KB
constexpr int kBwdEpiWarps = 4;                // warps 0-3
constexpr int kBwdProdWarps = 8;               // warps 4-11
constexpr int kBwdMmaWarp = kBwdEpiWarps + kBwdProdWarps;  // warp 12
constexpr int kBwdThreads = 32 * (kBwdMmaWarp + 1);
constexpr int kBwdIdxBytes = 2 * kBwdChunk * kTileRows * 4;  // A and G row indices of a chunk

struct BwdArgs {
  const uint16_t* feats;
  const uint16_t* grad;
  const int32_t* gidx;
  const int32_t* out_row;
  const int2* tap_tiles;
  const int32_t* tap_start;
  const int32_t* tap_chunk;
  float* partial;  // [chunk][block][128][BN]
  int32_t* status;
  int64_t n;
  int n_tiles;
  int cin;
  int cout;
  int n_cob;     // cout / BN
  int n_blk;     // ceil(cin / 128) * n_cob
  int n_chunks;  // dense: ceil(n_tiles / kBwdChunk)
  int dense;
  uint64_t wait_ns;
};

template <int BN, bool BF16>
__global__ void __launch_bounds__(kBwdThreads, 1) k_bwd_weight_tc(const BwdArgs a) {
  constexpr int kGBytes = (BN / 64) * kBwdAtom;
  constexpr int kStageBytes = 2 * kBwdAtom + kGBytes;  // A: up to 128 channels, G: BN channels
  constexpr uint32_t kIdesc = make_idesc(BN, BF16) | (1u << 15);  // A MN-major too
  constexpr uint32_t kTmemCols = BN < 32 ? 32 : BN;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  int32_t* idx = reinterpret_cast<int32_t*>(smem + kBwdStages * kStageBytes);  // [2][chunk][128]
  uint64_t* bars = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(idx) + kBwdIdxBytes);
  // full[S], empty[S], idx, tfull, drain
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * kBwdStages + 3);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const uint32_t full0 = smem_addr(bars), empty0 = full0 + 8 * kBwdStages;
  const uint32_t idx_bar = empty0 + 8 * kBwdStages, tfull = idx_bar + 8, drain = tfull + 8;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // this CTA's chunk of tiles, tap and (input, output) channel block
  const int c = blockIdx.x / a.n_blk, blk = blockIdx.x % a.n_blk;
  const int cib = blk / a.n_cob, cob = blk % a.n_cob;
  const int cib_w = min(128, a.cin - cib * 128);  // 64 or 128 input channels
  int tap = 0, first = 0, count = 0;
  if (a.dense) {
    first = c * kBwdChunk;
    count = min(kBwdChunk, a.n_tiles - first);
  } else {
    while (tap < kTaps && a.tap_chunk[tap + 1] <= c) ++tap;
    if (tap < kTaps) {
      first = a.tap_start[tap] + (c - a.tap_chunk[tap]) * kBwdChunk;
      count = min(kBwdChunk, a.tap_start[tap + 1] - first);
    }
  }
  if (count <= 0) return;  // past the last chunk (the grid is an upper bound)
  const int n_stages = 2 * count;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kBwdStages; ++s) {
      mbar_init(full0 + 8 * s, kBwdProdWarps * 32);
      mbar_init(empty0 + 8 * s, 1);
    }
    mbar_init(idx_bar, 1);
    mbar_init(tfull, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == kBwdMmaWarp) tmem_alloc(smem_addr(tmem_slot), kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const Waits wt{abort_flag, a.status, a.wait_ns};
  int32_t* idx_a = idx;                        // [count][128] gathered voxel, -1 = zero row
  int32_t* idx_g = idx + kBwdChunk * kTileRows;  // [count][128] output voxel, -1 = zero row

  if (warp == kBwdEpiWarps && lane == 0) {
    // the chunk's row indices into shared memory
    if (a.dense) {
      mbar_arrive(idx_bar);
    } else {
      mbar_arrive_expect_tx(idx_bar, uint32_t(2 * count * kTileRows * 4));
      for (int e = 0; e < count; ++e) {
        const int2 ts = a.tap_tiles[first + e];
        bulk_load(smem_addr(idx_a + e * kTileRows), a.gidx + int64_t(ts.y) * kTileRows,
                  kTileRows * 4, idx_bar);
        bulk_load(smem_addr(idx_g + e * kTileRows), a.out_row + int64_t(ts.x) * kTileRows,
                  kTileRows * 4, idx_bar);
      }
    }
  }

  if (warp >= kBwdEpiWarps && warp < kBwdMmaWarp) {
    // ---------------- producers: gather A and G rows ----------------
    const int pt = threadIdx.x - 32 * kBwdEpiWarps;  // 0 .. 255
    const int a_chunks = (cib_w / 64) * 8;           // 16-byte chunks per A row
    constexpr int g_chunks = (BN / 64) * 8;
    bool ok = wt.wait(idx_bar, 0);
    // A stage is published (copies landed, proxy fence, arrival) once the next
    // stage's copies are issued, so two stages' copies stay in flight; the
    // last one after the loop.
    int pend = -1;
    for (int s = 0; s < n_stages && ok; ++s) {
      const int slot = s % kBwdStages;
      if (!wt.wait(empty0 + 8 * slot, ((s / kBwdStages) & 1) ^ 1)) {
        ok = false;
        break;
      }
      const int e = s >> 1, r0 = (s & 1) * kBwdRows;
      const int tile = a.dense ? first + e : 0;
      const uint32_t base = smem_addr(smem + slot * kStageBytes);
      for (int q = pt; q < kBwdRows * a_chunks; q += kBwdProdWarps * 32) {
        const int row = q / a_chunks, qq = q % a_chunks, atom = qq >> 3, ch = qq & 7;
        int64_t j;
        if (a.dense) {
          j = int64_t(tile) * kTileRows + r0 + row;
          if (j >= a.n) j = -1;
        } else {
          j = idx_a[e * kTileRows + r0 + row];
        }
        const uint16_t* src = j >= 0 ? a.feats + j * a.cin + cib * 128 + atom * 64 + ch * 8 : a.feats;
        cp_async_16(base + atom * kBwdAtom + row * 128 + ((ch ^ (row & 7)) << 4), src,
                    j >= 0 ? 16u : 0u);
      }
      for (int q = pt; q < kBwdRows * g_chunks; q += kBwdProdWarps * 32) {
        const int row = q / g_chunks, qq = q % g_chunks, atom = qq >> 3, ch = qq & 7;
        int64_t i;
        if (a.dense) {
          i = int64_t(tile) * kTileRows + r0 + row;
          if (i >= a.n) i = -1;
        } else {
          i = idx_g[e * kTileRows + r0 + row];
        }
        const uint16_t* src = i >= 0 ? a.grad + i * a.cout + cob * BN + atom * 64 + ch * 8 : a.grad;
        cp_async_16(base + 2 * kBwdAtom + atom * kBwdAtom + row * 128 + ((ch ^ (row & 7)) << 4),
                    src, i >= 0 ? 16u : 0u);
      }
      cp_async_commit();
      if (pend >= 0) {
        cp_async_wait_group<1>();
        fence_proxy_async_smem();
        mbar_arrive(full0 + 8 * pend);
      }
      pend = slot;
    }
    if (ok && pend >= 0) {
      cp_async_wait_group<0>();
      fence_proxy_async_smem();
      mbar_arrive(full0 + 8 * pend);
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
  } else if (warp == kBwdMmaWarp) {
    // ---------------- MMA: D[ci][co] += A^T G, K = gathered rows ----------------
    const uint32_t lbo_a = cib_w == 128 ? kBwdAtom : 0;  // 64 channels: both halves read the same
    bool ok = true;
    for (int s = 0; s < n_stages; ++s) {
      const int slot = s % kBwdStages;
      const bool ready = wt.wait(full0 + 8 * slot, (s / kBwdStages) & 1);
      if (!__all_sync(0xffffffffu, ready)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t base = smem_addr(smem + slot * kStageBytes);
      const uint64_t ad = desc_b_mnmajor(base, lbo_a);
      const uint64_t bd = desc_b_mnmajor(base + 2 * kBwdAtom, kBwdAtom);
#pragma unroll
      for (int kk = 0; kk < kBwdRows / 16; ++kk)
        umma_f16(tmem, ad + (2048 >> 4) * kk, bd + (2048 >> 4) * kk, kIdesc,
                 (s > 0 || kk > 0) ? 1u : 0u);
      umma_commit(empty0 + 8 * slot);
    }
    if (ok) umma_commit(tfull);
    umma_commit(drain);
    mbar_drain(drain, 0);
  } else if (warp < kBwdEpiWarps) {
    // ---------------- epilogue: the partial block to global memory ----------------
    const int row = warp * 32 + lane;  // input channel within the block
    bool have = wt.wait(tfull, 0);
    if (__all_sync(0xffffffffu, have)) {
      tc_fence_after();
      float* dst = a.partial + (int64_t(blockIdx.x) * 128 + row) * BN;
#pragma unroll 1
      for (int cc = 0; cc < BN / 32; ++cc) {
        uint32_t v[32];
        tmem_ld_x32(tmem + (uint32_t(warp * 32) << 16) + uint32_t(cc * 32), v);
        if (row < cib_w) {
          float4* d4 = reinterpret_cast<float4*>(dst + cc * 32);
#pragma unroll
          for (int q = 0; q < 8; ++q)
            d4[q] = make_float4(__uint_as_float(v[4 * q]), __uint_as_float(v[4 * q + 1]),
                                __uint_as_float(v[4 * q + 2]), __uint_as_float(v[4 * q + 3]));
        }
      }
    }
  }
  if (warp == kBwdEpiWarps && lane == 0 && !a.dense) mbar_drain(idx_bar, 0);
  tc_fence_before();
  __syncthreads();
  if (warp == kBwdMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// dW[k][ci][co] = sum of tap k's chunk partials, in chunk order.
__global__ void k_bwd_weight_reduce(const float* __restrict__ partial,
                                    const int32_t* __restrict__ tap_chunk, int taps, int cin,
                                    int cout, int bn, int n_cob, int n_blk, int dense_chunks,
                                    float* __restrict__ dW) {
  const int64_t id = blockIdx.x * int64_t(blockDim.x) + threadIdx.x;
  if (id >= int64_t(taps) * cin * cout) return;
  const int co = int(id % cout);
  const int ci = int((id / cout) % cin);
  const int k = int(id / (int64_t(cin) * cout));
  const int c0 = dense_chunks > 0 ? 0 : tap_chunk[k];
  const int c1 = dense_chunks > 0 ? dense_chunks : tap_chunk[k + 1];
  const int blk = (ci / 128) * n_cob + co / bn;
  const int64_t off = int64_t(ci % 128) * bn + co % bn;
  float acc = 0.f;
  for (int c = c0; c < c1; ++c) acc += partial[(int64_t(c) * n_blk + blk) * 128 * bn + off];
  dW[id] = acc;
}

inline unsigned grid_for(int64_t n, int threads) { return unsigned((n + threads - 1) / threads); }

template <int BN, bool BF16>
int launch_bwd_weight_tc(const Plan& plan, bool dense, const void* feats, const void* grad,
                         float* dW, int cin, int cout, float* partial, int64_t n_chunks,
                         uint64_t wait_ns, cudaStream_t stream) {
  constexpr int kStageBytes = 2 * kBwdAtom + (BN / 64) * kBwdAtom;
  constexpr int kSmem = 1024 + kBwdStages * kStageBytes + kBwdIdxBytes + 256;
  static_assert(kSmem <= 227 * 1024, "shared memory");
  auto kern = k_bwd_weight_tc<BN, BF16>;
  constexpr int kMaxDev = 64;
  static bool attr_set[kMaxDev] = {};
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return SMC_ERR_CUDA;
  if (!(dev >= 0 && dev < kMaxDev && attr_set[dev])) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem) !=
        cudaSuccess)
      return SMC_ERR_CUDA;
    if (dev >= 0 && dev < kMaxDev) attr_set[dev] = true;
  }
  BwdArgs a;
  a.feats = static_cast<const uint16_t*>(feats);
  a.grad = static_cast<const uint16_t*>(grad);
  a.gidx = plan.gidx;
  a.out_row = plan.out_row;
  a.tap_tiles = plan.tap_tiles;
  a.tap_start = plan.tap_start;
  a.tap_chunk = plan.tap_chunk;
  a.partial = partial;
  a.status = plan.status;
  a.n = plan.n;
  a.n_tiles = int(plan.n_tiles);
  a.cin = cin;
  a.cout = cout;
  a.n_cob = cout / BN;
  a.n_blk = (cin + 127) / 128 * a.n_cob;
  a.n_chunks = int(n_chunks);
  a.dense = dense ? 1 : 0;
  a.wait_ns = wait_ns;
  const int64_t grid = n_chunks * a.n_blk;
  if (grid > 0) {
    kern<<<unsigned(grid), kBwdThreads, kSmem, stream>>>(a);
    if (cudaGetLastError() != cudaSuccess) return SMC_ERR_CUDA;
  }
  const int taps = dense ? 1 : kTaps;
  k_bwd_weight_reduce<<<grid_for(int64_t(taps) * cin * cout, 256), 256, 0, stream>>>(
      partial, plan.tap_chunk, taps, cin, cout, BN, a.n_cob, a.n_blk, dense ? int(n_chunks) : 0,
      dW);
  return cudaGetLastError() == cudaSuccess ? SMC_OK : SMC_ERR_CUDA;
}

}  // namespace

int launch_weight_transpose(const void* W, void* Wt, int taps, int cin, int cout, int dtype,
                            cudaStream_t stream) {
  const dim3 grid((cout + 31) / 32, (cin + 31) / 32, taps), block(32, 8);
  if (dtype == SMC_F32)
    k_weight_transpose<float><<<grid, block, 0, stream>>>(static_cast<const float*>(W),
                                                         static_cast<float*>(Wt), taps, cin, cout);
  else
    k_weight_transpose<uint16_t><<<grid, block, 0, stream>>>(
        static_cast<const uint16_t*>(W), static_cast<uint16_t*>(Wt), taps, cin, cout);
  return cudaGetLastError() == cudaSuccess ? SMC_OK : SMC_ERR_CUDA;
}

bool bwd_weight_tc_supported(int cin, int cout, int dtype) {
  return (dtype == SMC_F16 || dtype == SMC_BF16) && cin > 0 && cout > 0 && cin % 64 == 0 &&
         cout % 64 == 0;
}

size_t bwd_weight_workspace_bytes(const Plan& plan, bool dense, int cin, int cout, int dtype) {
  if (!bwd_weight_tc_supported(cin, cout, dtype) || plan.n == 0) return 0;
  const int bn = cout % 128 == 0 ? 128 : 64;
  const int64_t n_blk = (cin + 127) / 128 * (cout / bn);
  return size_t(bwd_weight_chunks(plan, dense)) * n_blk * 128 * bn * sizeof(float);
}

int64_t bwd_weight_chunks(const Plan& plan, bool dense) {
  if (dense) return (plan.n_tiles + kBwdChunk - 1) / kBwdChunk;
  return (plan.total_slots + kBwdChunk - 1) / kBwdChunk + kTaps;  // upper bound
}

int launch_bwd_weight(const Plan& plan, bool dense, const void* feats, const void* grad, float* dW,
                      int cin, int cout, int dtype, void* workspace, uint64_t wait_ns,
                      cudaStream_t stream) {
  const int taps = dense ? 1 : kTaps;
  if (plan.n == 0) {
    return cudaMemsetAsync(dW, 0, size_t(taps) * cin * cout * sizeof(float), stream) ==
                   cudaSuccess
               ? SMC_OK
               : SMC_ERR_CUDA;
  }
  if (bwd_weight_tc_supported(cin, cout, dtype)) {
    float* partial = static_cast<float*>(workspace);
    const int64_t chunks = bwd_weight_chunks(plan, dense);
    const bool bf16 = dtype == SMC_BF16;
    if (cout % 128 == 0)
      return bf16 ? launch_bwd_weight_tc<128, true>(plan, dense, feats, grad, dW, cin, cout,
                                                    partial, chunks, wait_ns, stream)
                  : launch_bwd_weight_tc<128, false>(plan, dense, feats, grad, dW, cin, cout,
                                                     partial, chunks, wait_ns, stream);
    return bf16 ? launch_bwd_weight_tc<64, true>(plan, dense, feats, grad, dW, cin, cout, partial,
                                                 chunks, wait_ns, stream)
                : launch_bwd_weight_tc<64, false>(plan, dense, feats, grad, dW, cin, cout, partial,
                                                  chunks, wait_ns, stream);
  }
  const int64_t total = int64_t(taps) * cin * cout;
  const unsigned g = grid_for(total, 128);
  const int d = dense ? 1 : 0;
  switch (dtype) {
    case SMC_F32:
      k_bwd_weight_simt<float, double><<<g, 128, 0, stream>>>(
          static_cast<const float*>(feats), static_cast<const float*>(grad), plan.tap_tiles,
          plan.tap_start, plan.gidx, plan.out_row, plan.n, taps, cin, cout, d, dW);
      break;
    case SMC_F16:
      k_bwd_weight_simt<__half, float><<<g, 128, 0, stream>>>(
          static_cast<const __half*>(feats), static_cast<const __half*>(grad), plan.tap_tiles,
          plan.tap_start, plan.gidx, plan.out_row, plan.n, taps, cin, cout, d, dW);
      break;
    default:
      k_bwd_weight_simt<__nv_bfloat16, float><<<g, 128, 0, stream>>>(
          static_cast<const __nv_bfloat16*>(feats), static_cast<const __nv_bfloat16*>(grad),
          plan.tap_tiles, plan.tap_start, plan.gidx, plan.out_row, plan.n, taps, cin, cout, d,
          dW);
  }
  return cudaGetLastError() == cudaSuccess ? SMC_OK : SMC_ERR_CUDA;
}

}  // namespace smc
