// Output-stationary implicit-GEMM SubMConv3d on the sm_100a tensor cores.
//
// One CTA computes a 128-row x BN-column output tile.  For every tap the
// tile's plan marks active (the others are skipped), the CTA gathers the 128
// neighbour feature rows of that tap (zero rows for absent neighbours) and
// multiplies them by W[tap] with tcgen05.mma, accumulating in fp32 in tensor
// memory; each output row is then written exactly once, without atomics.
// This is the sum over offsets of the trellis_sparse_mlx README ("What's in
// it": out[c] = sum_d feats[c+d] @ W[d] over active neighbours) reorganised
// so that the dense work the README's fused [N, 27 Cin] x [27 Cin, Cout]
// matmul spends on absent neighbours is skipped a tile-tap at a time.
//
// Warp roles (192 threads):
//   warps 0-3  gather A: 16-byte cp.async copies of the neighbour rows into a
//              128-byte-swizzled K-major tile (zero-filled for -1), then the
//              epilogue (TMEM -> registers -> fp16/bf16 -> global);
//   warp 4     lane 0 loads the W[tap] slice with TMA (MN-major, 128B swizzle);
//   warp 5     allocates tensor memory; lane 0 issues the MMAs.
// Stages are handed over with mbarriers; every wait is bounded in time and a
// wait that runs out marks the CTA aborted and sets the status word.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <mutex>

#include "smc_internal.h"

namespace smc {
namespace {

constexpr int kThreads = 192;
constexpr int kBK = 64;                        // input channels per stage (128 bytes)
constexpr int kABytes = kTileRows * kBK * 2;   // 16 KB
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s

// ----------------------------------------------------------------------------
// PTX wrappers
// ----------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Wait for the phase of `bar` with parity `parity`, at most kWaitLimitNs.
// Returns false (and marks the CTA aborted) when the limit runs out or another
// thread of the CTA has already aborted.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          int32_t* status) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (*abort_flag) return false;
    if (global_ns() - t0 > kWaitLimitNs) {
      *abort_flag = 1;
      atomicOr(status, kDevTimeout);
      return false;
    }
  }
  return true;
}
// Bounded wait that ignores the abort flag: used on the abort path to let
// tensor-core work already issued finish before its memory is released.
__device__ __forceinline__ void mbar_drain(uint32_t bar, uint32_t parity) {
  const uint64_t t0 = global_ns();
  while (!mbar_try_wait(bar, parity) && global_ns() - t0 < kWaitLimitNs) {
  }
}

__device__ __forceinline__ void cp_async_16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void fence_async_proxy() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int c0, int c1,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void tma_prefetch_map(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void umma_f16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                         uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar)
               : "memory");
}
__device__ __forceinline__ void tmem_ld_x32(uint32_t taddr, uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
        "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]),
        "=r"(v[14]), "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]),
        "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]), "=r"(v[25]),
        "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptors (sm_100 UMMA format: start >> 4 in bits
// 0-13, leading byte offset >> 4 in 16-29, stride byte offset >> 4 in 32-45,
// version 1 in bit 46, layout type in 61-63 with 2 = 128-byte swizzle).
// A: K-major, rows of 128 bytes, 8-row swizzle atoms 1024 bytes apart.
__device__ __forceinline__ uint64_t desc_a_kmajor(uint32_t addr) {
  return uint64_t((addr >> 4) & 0x3FFFu) | (uint64_t(1) << 16) | (uint64_t(1024 >> 4) << 32) |
         (uint64_t(1) << 46) | (uint64_t(2) << 61);
}
// B: MN-major (W[tap] is [Cin][Cout] with Cout contiguous); 64-column blocks
// `lbo` bytes apart, 8-row (K) groups 1024 bytes apart.
__device__ __forceinline__ uint64_t desc_b_mnmajor(uint32_t addr, uint32_t lbo) {
  return uint64_t((addr >> 4) & 0x3FFFu) | (uint64_t((lbo >> 4) & 0x3FFFu) << 16) |
         (uint64_t(1024 >> 4) << 32) | (uint64_t(1) << 46) | (uint64_t(2) << 61);
}
// Instruction descriptor, kind::f16: fp32 accumulator, A K-major, B MN-major.
__host__ __device__ constexpr uint32_t make_idesc(int bn, bool bf16) {
  return (1u << 4) | ((bf16 ? 1u : 0u) << 7) | ((bf16 ? 1u : 0u) << 10) | (1u << 16) |
         (uint32_t(bn >> 3) << 17) | (uint32_t(kTileRows >> 4) << 24);
}

template <bool BF16>
__device__ __forceinline__ uint32_t pack2(uint32_t a, uint32_t b) {
  const float fa = __uint_as_float(a), fb = __uint_as_float(b);
  if constexpr (BF16) {
    __nv_bfloat162 h = __floats2bfloat162_rn(fa, fb);
    return *reinterpret_cast<uint32_t*>(&h);
  } else {
    __half2 h = __floats2half2_rn(fa, fb);
    return *reinterpret_cast<uint32_t*>(&h);
  }
}

struct ConvArgs {
  const uint16_t* feats;
  uint16_t* out;
  const int32_t* gidx;
  const int32_t* tile_off;
  const uint8_t* tile_taps;
  const int32_t* out_row;
  int32_t* status;
  int64_t n;
  int cin;
  int cout;
  int n_tiles;
  int dense;
};

template <int BN, int STAGES, int LAG, bool BF16>
__global__ void __launch_bounds__(kThreads, 1)
k_conv_tc(const __grid_constant__ CUtensorMap wmap, const ConvArgs args) {
  static_assert(BN % 64 == 0 && BN <= 256, "BN");
  static_assert(LAG >= 1 && LAG < STAGES, "LAG");
  constexpr int kBBytes = BN * kBK * 2;
  constexpr int kStageBytes = kABytes + kBBytes;
  constexpr uint32_t kTmemCols = BN < 32 ? 32 : BN;
  constexpr uint32_t kIdesc = make_idesc(BN, BF16);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * kStageBytes);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int tile = args.n_tiles - 1 - int(blockIdx.x);  // largest tap sets first
  const int n0 = int(blockIdx.y) * BN;
  const int kb_per_tap = args.cin / kBK;
  int slot0 = 0, ntaps = 1;
  if (!args.dense) {
    slot0 = args.tile_off[tile];
    ntaps = args.tile_off[tile + 1] - slot0;
  }
  const int iters = ntaps * kb_per_tap;
  const uint32_t full0 = smem_addr(bars);
  const uint32_t empty0 = smem_addr(bars + STAGES);
  const uint32_t accum_bar = smem_addr(bars + 2 * STAGES);

  if (tid == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full0 + 8 * s, 4 * 32 + 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    mbar_init(accum_bar, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 5) tmem_alloc(smem_addr(tmem_slot), kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp < 4) {
    // ---------------- gather producer ----------------
    const int chunk = tid & 7;  // 16-byte chunk of a row's 128-byte slice
    const int rsub = tid >> 3;  // rows rsub + 16 j, j = 0..7
    int g[8];
    int issued = 0;
    for (int it = 0; it < iters; ++it) {
      const int s = it / kb_per_tap;
      const int kb = it - s * kb_per_tap;
      if (kb == 0) {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int row = rsub + 16 * j;
          if (args.dense) {
            const int64_t r = int64_t(tile) * kTileRows + row;
            g[j] = r < args.n ? int(r) : -1;
          } else {
            g[j] = args.gidx[int64_t(slot0 + s) * kTileRows + row];
          }
        }
      }
      const int stage = it % STAGES;
      if (!mbar_wait(empty0 + 8 * stage, ((it / STAGES) & 1) ^ 1, abort_flag, args.status)) break;
      const uint32_t a_base = smem_addr(smem + stage * kStageBytes);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int row = rsub + 16 * j;
        const bool ok = g[j] >= 0;
        const uint16_t* src =
            ok ? args.feats + int64_t(g[j]) * args.cin + kb * kBK + chunk * 8 : args.feats;
        cp_async_16(a_base + row * 128 + ((chunk ^ (row & 7)) << 4), src, ok ? 16u : 0u);
      }
      cp_async_commit();
      ++issued;
      if (it >= LAG) {
        cp_async_wait<LAG>();
        fence_async_proxy();
        mbar_arrive(full0 + 8 * ((it - LAG) % STAGES));
      }
    }
    cp_async_wait<0>();
    fence_async_proxy();
    for (int it = issued > LAG ? issued - LAG : 0; it < issued; ++it)
      mbar_arrive(full0 + 8 * (it % STAGES));

    // ---------------- epilogue ----------------
    bool have = iters > 0 && mbar_wait(accum_bar, 0, abort_flag, args.status);
    have = __all_sync(0xffffffffu, have);  // tcgen05.ld below is warp-collective
    tc_fence_after();
    const int row = warp * 32 + lane;
    int32_t orow;
    if (args.dense) {
      const int64_t r = int64_t(tile) * kTileRows + row;
      orow = r < args.n ? int32_t(r) : -1;
    } else {
      orow = args.out_row[int64_t(tile) * kTileRows + row];
    }
    uint16_t* dst = args.out + int64_t(orow < 0 ? 0 : orow) * args.cout + n0;
#pragma unroll 1
    for (int cc = 0; cc < BN / 32; ++cc) {
      uint32_t v[32];
      if (have) {
        tmem_ld_x32(tmem + (uint32_t(warp * 32) << 16) + uint32_t(cc * 32), v);
      } else {
#pragma unroll
        for (int q = 0; q < 32; ++q) v[q] = 0u;
      }
      if (orow >= 0 && !*abort_flag) {
        uint4* d4 = reinterpret_cast<uint4*>(dst + cc * 32);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint4 w;
          w.x = pack2<BF16>(v[8 * q + 0], v[8 * q + 1]);
          w.y = pack2<BF16>(v[8 * q + 2], v[8 * q + 3]);
          w.z = pack2<BF16>(v[8 * q + 4], v[8 * q + 5]);
          w.w = pack2<BF16>(v[8 * q + 6], v[8 * q + 7]);
          d4[q] = w;
        }
      }
    }
  } else if (warp == 4) {
    // ---------------- W producer (TMA) ----------------
    if (lane == 0) {
      tma_prefetch_map(&wmap);
      for (int it = 0; it < iters; ++it) {
        const int s = it / kb_per_tap;
        const int kb = it - s * kb_per_tap;
        const int tap = args.dense ? 0 : int(args.tile_taps[int64_t(tile) * 32 + s]);
        const int stage = it % STAGES;
        if (!mbar_wait(empty0 + 8 * stage, ((it / STAGES) & 1) ^ 1, abort_flag, args.status))
          break;
        const uint32_t full = full0 + 8 * stage;
        mbar_arrive_expect_tx(full, kBBytes);
        const uint32_t b_base = smem_addr(smem + stage * kStageBytes + kABytes);
#pragma unroll
        for (int j = 0; j < BN / 64; ++j)
          tma_load_2d(b_base + j * (kBK * 128), &wmap, n0 + 64 * j, tap * args.cin + kb * kBK,
                      full);
      }
    }
    __syncwarp();
  } else {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      int done = 0;
      for (int it = 0; it < iters; ++it) {
        const int stage = it % STAGES;
        if (!mbar_wait(full0 + 8 * stage, (it / STAGES) & 1, abort_flag, args.status)) break;
        tc_fence_after();
        const uint32_t a_base = smem_addr(smem + stage * kStageBytes);
        const uint32_t b_base = a_base + kABytes;
#pragma unroll
        for (int k = 0; k < kBK / 16; ++k) {
          umma_f16(tmem, desc_a_kmajor(a_base + 32 * k), desc_b_mnmajor(b_base + 2048 * k, kBK * 128),
                   kIdesc, (it | k) != 0 ? 1u : 0u);
        }
        umma_commit(empty0 + 8 * stage);
        ++done;
      }
      umma_commit(accum_bar);
      if (done < iters) {
        // aborted: let the MMAs already issued finish before the memory goes away
        mbar_drain(accum_bar, 0);
      }
    }
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ----------------------------------------------------------------------------
// host side
// ----------------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    cudaGetLastError();
  });
  return fn;
}

template <int BN, int STAGES, int LAG, bool BF16>
int launch_cfg(const Plan& plan, bool dense, const void* feats, const void* W, void* out, int cin,
               int cout, cudaStream_t stream) {
  constexpr int kStageBytes = kABytes + BN * kBK * 2;
  constexpr int kSmem = STAGES * kStageBytes + 1024 + 256;
  auto kern = k_conv_tc<BN, STAGES, LAG, BF16>;
  static bool attr_set = false;
  if (!attr_set) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem) !=
        cudaSuccess)
      return SMC_ERR_CUDA;
    attr_set = true;
  }
  auto encode = get_encode_fn();
  if (!encode) return SMC_ERR_CUDA;
  const int taps = dense ? 1 : kTaps;
  CUtensorMap map;
  cuuint64_t dims[2] = {cuuint64_t(cout), cuuint64_t(taps) * cuuint64_t(cin)};
  cuuint64_t strides[1] = {cuuint64_t(cout) * 2};
  cuuint32_t box[2] = {64, kBK};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = encode(&map, BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                      2, const_cast<void*>(W), dims, strides, box, estr,
                      CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                      CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return SMC_ERR_CUDA;
  ConvArgs a;
  a.feats = static_cast<const uint16_t*>(feats);
  a.out = static_cast<uint16_t*>(out);
  a.gidx = plan.gidx;
  a.tile_off = plan.tile_off;
  a.tile_taps = plan.tile_taps;
  a.out_row = plan.out_row;
  a.status = plan.status;
  a.n = plan.n;
  a.cin = cin;
  a.cout = cout;
  a.n_tiles = int(plan.n_tiles);
  a.dense = dense ? 1 : 0;
  dim3 grid(unsigned(plan.n_tiles), unsigned(cout / BN));
  kern<<<grid, kThreads, kSmem, stream>>>(map, a);
  return cudaGetLastError() == cudaSuccess ? SMC_OK : SMC_ERR_CUDA;
}

template <bool BF16>
int launch_dtype(const Plan& plan, bool dense, const void* feats, const void* W, void* out,
                 int cin, int cout, cudaStream_t stream) {
  if (cout % 256 == 0) return launch_cfg<256, 4, 2, BF16>(plan, dense, feats, W, out, cin, cout, stream);
  if (cout % 128 == 0) return launch_cfg<128, 3, 1, BF16>(plan, dense, feats, W, out, cin, cout, stream);
  return launch_cfg<64, 4, 2, BF16>(plan, dense, feats, W, out, cin, cout, stream);
}

}  // namespace

bool conv_tc_supported(int cin, int cout, int dtype) {
  return (dtype == SMC_F16 || dtype == SMC_BF16) && cin > 0 && cout > 0 && cin % kBK == 0 &&
         cout % 64 == 0;
}

int launch_conv_tc(const Plan& plan, bool dense, const void* feats, const void* W, void* out,
                   int cin, int cout, int dtype, cudaStream_t stream) {
  if (plan.n == 0) return SMC_OK;
  if (!conv_tc_supported(cin, cout, dtype)) return SMC_ERR_UNSUPPORTED;
  if (dtype == SMC_BF16) return launch_dtype<true>(plan, dense, feats, W, out, cin, cout, stream);
  return launch_dtype<false>(plan, dense, feats, W, out, cin, cout, stream);
}

}  // namespace smc
