// Output-stationary implicit-GEMM SubMConv3d on the sm_100a tensor cores.
//
// A work item is a 128-row x BN-column output tile.  For every tap the tile's
// plan marks active (the others are skipped), the tile's 128 neighbour feature
// rows of that tap are gathered into shared memory (zero rows for absent
// neighbours) and multiplied by W[tap] with tcgen05.mma, accumulating in fp32
// in tensor memory; each output row is then written exactly once, without
// atomics.  This is the sum over offsets of the trellis_sparse_mlx README
// ("What's in it": out[c] = sum_d feats[c+d] @ W[d] over active neighbours)
// organised so that the dense work of the README's fused
// [N, 27 Cin] x [27 Cin, Cout] matmul is skipped one tile-tap at a time.
//
// Persistent kernel, one CTA per SM, 8 + WPS * STAGES warps:
//   warp 0      lane 0 loads the W[tap] slice of each stage with TMA
//               (MN-major, 128-byte swizzle), and for K = 1 also the stage's
//               contiguous feature rows (128 x 64 box, 128-byte swizzle);
//   warp 1      allocates tensor memory; with the last warp, issues the MMAs
//               (M = 128, N = BN, K = 16): warp 1 those of the even tiles of
//               a work item, the last warp those of the odd tiles.  A
//               tcgen05.mma keeps its issuing thread until the tensor core
//               accepts it (about one MMA time), so a single issuer's own
//               loop and waits between stages would idle the tensor core;
//               two issuers cover each other's gaps;
//   warps 2-5   epilogue: tensor memory -> registers -> fp16/bf16 -> global;
//               with two accumulator sets (NBUF = 2) it overlaps the MMAs of
//               the next work item;
//   warp 6      scheduler: takes work items (most taps first) from a global
//               counter and decodes each one's tile masks and slot offsets
//               into a small shared-memory queue read by every other role;
//   warps 7..   gather, WPS (4 or 2) warps per pipeline stage slot: warp q of
//               slot i copies rows 128/WPS q .. of every tile the stage feeds
//               (BK = 64 or 32 channels, 128 or 64 bytes per row) with 16-byte cp.async
//               (zero-filled for absent neighbours) into a 128-byte-swizzled
//               K-major tile; each lane's mbarrier arrival fires when its
//               copies land, so no thread waits on its copies.  Many warps
//               with few copies each keep enough copies in flight; fixed
//               owners per slot keep every parity wait on a slot's barrier at
//               most one phase ahead.
// Stages and accumulators are handed over with mbarriers; every wait is
// bounded in time and a wait that runs out marks the CTA aborted and sets the
// status word, so a fault in the pipeline ends the kernel instead of hanging.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <algorithm>
#include <cstdlib>
#include <mutex>

#include "smc_internal.h"

namespace smc {
namespace {

constexpr int kPrefetchWarp = 6;
constexpr int kFirstGatherWarp = 7;
// Warps: 0 W loader, 1 MMA (even tiles of a group), 2-5 epilogue, 6 scheduler,
// then WPS gather warps per stage slot (each copies 128 / WPS of a tile's
// rows), then the second MMA warp (odd tiles).
__host__ __device__ constexpr int threads_for(int stages, int wps) {
  return 32 * (kFirstGatherWarp + wps * stages + 1);
}
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

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int c0, int c1,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(bar)
      : "memory");
}
// 16-byte copy global -> shared; src_bytes = 0 writes 16 zero bytes.
__device__ __forceinline__ void cp_async_16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(src_bytes)
               : "memory");
}
// Arrive on `bar` once every cp.async this thread issued so far has landed
// (the arrival is counted in the barrier's expected count).
__device__ __forceinline__ void cp_async_arrive_noinc(uint32_t bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
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
// MMA issue and commit, called by all 32 lanes of a converged warp: elect.sync
// picks one lane (the same one every time, lane 0, as all lanes are active),
// which issues.  Keeping the warp converged lets the operands stay warp-uniform;
// the same lane issues every MMA and commit, as a commit tracks the MMAs of its
// own thread.
__device__ __forceinline__ void umma_f16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                         uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile(
      "{\n\t.reg .pred e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(
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
// A: K-major, rows of 2*BK bytes (128 or 64) with the matching swizzle
// (128-byte: layout 2, 64-byte: layout 4), 8-row atoms 16*BK bytes apart.
template <int BK>
__device__ __forceinline__ uint64_t desc_a_kmajor(uint32_t addr) {
  static_assert(BK == 64 || BK == 32, "BK");
  constexpr uint64_t kLayout = BK == 64 ? 2 : 4;
  constexpr uint64_t kSbo = 8 * BK * 2;
  return uint64_t((addr >> 4) & 0x3FFFu) | (uint64_t(1) << 16) | ((kSbo >> 4) << 32) |
         (uint64_t(1) << 46) | (kLayout << 61);
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
  const int32_t* gidx;        // [slots][128], -1 = absent
  const int32_t* tile_off;    // [n_tiles + 1] first slot of each tile
  const uint32_t* tile_mask;  // [n_tiles] active taps of each tile
  const int32_t* out_row;     // [n_tiles * 128], -1 = padding row
  const int32_t* group_order; // [n_groups] group of the q-th item, most taps first
  uint32_t* work_counter;     // [0] next item, [1] CTAs finished; both 0 between launches
  int32_t* status;
  int64_t n;
  int cin;
  int cout;
  int n_tiles;
  int n_groups;  // ceil(n_tiles / G)
  int n_blocks;  // cout / BN
  int dense;     // 1: K = 1, rows in order, one tap
};

// A work item is a group of G consecutive tiles (in plan order) and one
// BN-wide block of output channels.  The group's taps are the union of its
// tiles' taps; a W chunk is loaded once per stage and multiplied into every
// tile of the group that has that tap.  Items are numbered by the tap count of
// their group, most first (longest-processing-time order), and handed out
// dynamically, so every SM stays busy until the end.
template <int G>
struct Group {
  int w;         // item number, -1 = no more work
  int tile0;
  int n0;
  uint32_t all;  // union of the masks
  int rot;       // taps are visited starting at this tap (spreads W reads over L2)
  uint32_t mask[G];
  int slot0[G];  // first gather-index slot of each tile
};

template <int BN, int G>
__device__ __forceinline__ Group<G> group_of(const ConvArgs& a, int w) {
  Group<G> gr;
  gr.w = w;
  const int q = w / a.n_blocks;
  // groups with the largest tap sets first; K = 1 items are all alike
  gr.tile0 = (a.dense ? a.n_groups - 1 - q : a.group_order[q]) * G;
  gr.n0 = (w - q * a.n_blocks) * BN;
  gr.all = 0;
#pragma unroll
  for (int k = 0; k < G; ++k) {
    const int t = gr.tile0 + k;
    const bool live = t < a.n_tiles;
    gr.mask[k] = live ? (a.dense ? 1u : a.tile_mask[t]) : 0u;
    gr.slot0[k] = live && !a.dense ? a.tile_off[t] : 0;
    gr.all |= gr.mask[k];
  }
  gr.rot = a.dense ? 0 : int((unsigned(w) * 7u) % unsigned(kTaps));
  return gr;
}

// Taps of `all` in the order r, r+1, ..., 26, 0, ..., r-1 (set bits only).
__device__ __forceinline__ uint32_t rotate_taps(uint32_t all, int r) {
  constexpr uint32_t kAll = (1u << kTaps) - 1u;
  return r == 0 ? all : (((all >> r) | (all << (kTaps - r))) & kAll);
}
__device__ __forceinline__ int next_tap(uint32_t& rotated, int r) {
  const int b = __ffs(rotated) - 1;
  rotated &= rotated - 1u;
  const int t = b + r;
  return t >= kTaps ? t - kTaps : t;
}

// One gather warp's share of a stage: which tiles it copies and from where.
template <int G, int IDX>
struct GatherJob {
  int stage;
  uint32_t g;
  int kb;
  uint32_t tiles;    // bit k: tile k of the group has this tap
  int vidx[G][IDX];  // lane l: source row of local row 32 i + l of tile k (-1 = zero row)
};

// NBUF: accumulator sets in tensor memory (2: the epilogue of one item overlaps
// the MMAs of the next; 1: room for two 256-column tiles per item).
template <int BN, int BK, int STAGES, int G, int WPS, bool BF16, int NBUF>
__global__ void __launch_bounds__(threads_for(STAGES, WPS), 1)
k_conv_tc(const __grid_constant__ CUtensorMap wmap, const __grid_constant__ CUtensorMap fmap,
          const ConvArgs args) {
  static_assert(BN % 64 == 0 && BN <= 256, "BN");
  static_assert(BK == 64 || BK == 32, "BK");
  constexpr int kBK = BK;
  constexpr int kABytes = kTileRows * BK * 2;      // one tile's rows for one stage
  constexpr int kRowBytes = BK * 2;                 // 128 or 64
  constexpr int kChunks = kRowBytes / 16;           // 16-byte copies per row
  constexpr int kRowsPerInstr = 32 / kChunks;       // rows one warp copy instruction covers
  constexpr int kRowsPerWarp = kTileRows / WPS;     // rows of a tile one gather warp copies
  constexpr int kInstr = kRowsPerWarp / kRowsPerInstr;
  constexpr int kIdx = kRowsPerWarp / 32;           // gather indices held per lane
  static_assert(kRowsPerWarp % 32 == 0 && kInstr >= 1, "gather split");
  constexpr int kBBytes = BN * kBK * 2;
  constexpr int kStageBytes = G * kABytes + kBBytes;
  static_assert(NBUF == 1 || NBUF == 2, "accumulator sets");
  constexpr uint32_t kTmemCols = NBUF * G * BN;  // NBUF sets of G accumulators
  constexpr uint32_t kIdesc = make_idesc(BN, BF16);
  // Two MMA warps: a tcgen05.mma holds its issuing thread until the tensor core
  // takes it, so one issuer's own loop and barrier waits would leave the tensor
  // core idle between stages.  Warp 1 issues the even tiles of a group, the
  // last warp the odd ones (separate accumulators, so no ordering between
  // them is needed); both commit every stage.
  constexpr int kMmaWarp2 = kFirstGatherWarp + WPS * STAGES;
  // Work items published ahead of the producers.  An item taken from the
  // global counter cannot move to an idle SM any more, so a deeper queue
  // leaves a longer tail: one entry for the 64/128-column tiles (many short
  // items); two for 256-column tiles, whose long items would otherwise wait
  // for the scheduler's decode at every item boundary.
  constexpr int kQueue = BN == 256 ? 2 : 1;
  constexpr uint32_t kMmaWarps = 2;
  // readers of a queue entry: gather warps, W loader, both MMA warps (the
  // epilogue learns each item from MMA warp 1, one accumulator at a time)
  constexpr uint32_t kQueueReaders = WPS * STAGES + 1 + kMmaWarps;
  static_assert(kTmemCols >= 32 && kTmemCols <= 512 && (kTmemCols & (kTmemCols - 1)) == 0,
                "tensor memory columns");

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * kStageBytes);
  // barriers: full[S], empty[S], tfull[2], tempty[2], qfull[Q], qempty[Q], info[2]
  Group<G>* queue = reinterpret_cast<Group<G>*>(bars + 2 * STAGES + 6 + 2 * kQueue);
  Group<G>* acc_info = queue + kQueue;  // item held by each accumulator
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_info + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kb_per_tap = args.cin / kBK;
  const int total_work = args.n_groups * args.n_blocks;
  const uint32_t full0 = smem_addr(bars);
  const uint32_t empty0 = smem_addr(bars + STAGES);
  const uint32_t tfull0 = smem_addr(bars + 2 * STAGES);
  const uint32_t tempty0 = smem_addr(bars + 2 * STAGES + 2);
  const uint32_t qfull0 = smem_addr(bars + 2 * STAGES + 4);
  const uint32_t qempty0 = smem_addr(bars + 2 * STAGES + 4 + kQueue);
  const uint32_t info0 = smem_addr(bars + 2 * STAGES + 4 + 2 * kQueue);  // 2 barriers

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      // sparse: the gather lanes and the W loader; dense (K = 1): the loader
      // brings the contiguous A rows with TMA too
      mbar_init(full0 + 8 * s, args.dense ? 1 : WPS * 32 + 1);
      mbar_init(empty0 + 8 * s, kMmaWarps);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull0 + 8 * a, kMmaWarps);
      mbar_init(tempty0 + 8 * a, 4 * 32);
      mbar_init(info0 + 8 * a, 1);
    }
    for (int q = 0; q < kQueue; ++q) {
      mbar_init(qfull0 + 8 * q, 1);
      mbar_init(qempty0 + 8 * q, kQueueReaders);
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) tmem_alloc(smem_addr(tmem_slot), kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // Next work item from the queue; every unit (a warp, or one thread) reads
  // each entry once and releases it with one arrival.  warp_wide: all 32
  // lanes read and lane 0 releases after the warp has read.  Returns w = -1
  // at the end or when the CTA aborts.
  auto next_item = [&](uint32_t& j, bool warp_wide) -> Group<G> {
    Group<G> gr;
    const uint32_t q = j % kQueue;
    bool ok = mbar_wait(qfull0 + 8 * q, (j / kQueue) & 1, abort_flag, args.status);
    if (warp_wide) ok = __all_sync(0xffffffffu, ok);
    if (!ok) {
      gr.w = -1;
      return gr;
    }
    gr = queue[q];
    if (warp_wide) __syncwarp();
    if (!warp_wide || lane == 0) mbar_arrive(qempty0 + 8 * q);
    ++j;
    return gr;
  };

  if (warp == kPrefetchWarp) {
    // ---------------- scheduler: hands out items ----------------
    for (uint32_t j = 0;; ++j) {
      const uint32_t q = j % kQueue;
      int w = -1;
      if (lane == 0) {
        if (mbar_wait(qempty0 + 8 * q, ((j / kQueue) & 1) ^ 1, abort_flag, args.status)) {
          const uint32_t t = atomicAdd(args.work_counter, 1u);
          w = t < uint32_t(total_work) ? int(t) : -1;
        }
      }
      w = __shfl_sync(0xffffffffu, w, 0);
      Group<G> gr;
      if (w >= 0) {
        gr = group_of<BN, G>(args, w);
      } else {
        gr.w = -1;
      }
      if (lane == 0) {
        queue[q] = gr;
        mbar_arrive(qfull0 + 8 * q);  // release: publishes the entry
      }
      if (w < 0) break;
    }
  } else if (warp >= kFirstGatherWarp && warp < kMmaWarp2) {
    // ------------- gather warps: warps WPS i .. WPS i + WPS - 1 own stage slot i ----
    const int gw = (warp - kFirstGatherWarp) / WPS;  // slot
    const int rq = (warp - kFirstGatherWarp) % WPS;  // rows kRowsPerWarp * rq ...
    const int chunk = lane % kChunks;  // 16-byte chunk within a row slice
    const int rsub = lane / kChunks;   // instruction j copies local rows kRowsPerInstr j + rsub
    // Within an item, the index loads of an owned stage are issued one owned
    // stage ahead of its copies, so they overlap the wait for the slot.
    GatherJob<G, kIdx> pend;
    bool have_pend = false;
    bool ok = true;
    auto run = [&](const GatherJob<G, kIdx>& job) -> bool {
      // the source row of every copy, exchanged before the wait for the slot
      int vv[G][kInstr];
#pragma unroll
      for (int k = 0; k < G; ++k)
#pragma unroll
        for (int jj = 0; jj < kInstr; ++jj) {
          const int local = kRowsPerInstr * jj + rsub;
          vv[k][jj] = __shfl_sync(0xffffffffu, job.vidx[k][local / 32], local % 32);
        }
      if (!mbar_wait(empty0 + 8 * job.stage, ((job.g / STAGES) & 1) ^ 1, abort_flag,
                     args.status))
        return false;
      const uint32_t stage_base = smem_addr(smem + job.stage * kStageBytes);
      const uint16_t* src_col = args.feats + job.kb * kBK + chunk * 8;
#pragma unroll
      for (int k = 0; k < G; ++k) {
        if (!((job.tiles >> k) & 1u)) continue;
        const uint32_t a_base = stage_base + k * kABytes;
#pragma unroll
        for (int jj = 0; jj < kInstr; ++jj) {
          const int local = kRowsPerInstr * jj + rsub;
          const int v = vv[k][jj];
          const int row = kRowsPerWarp * rq + local;
          const uint16_t* src = v >= 0 ? src_col + int64_t(v) * args.cin : args.feats;
          // swizzled chunk: XOR with address bits 7.. (128-byte: row & 7; 64-byte: (row >> 1) & 3)
          const int pchunk = BK == 64 ? (chunk ^ (row & 7)) : (chunk ^ ((row >> 1) & 3));
          cp_async_16(a_base + row * kRowBytes + (pchunk << 4), src, v >= 0 ? 16u : 0u);
        }
      }
      cp_async_arrive_noinc(full0 + 8 * job.stage);
      return true;
    };
    uint32_t g = 0, j = 0;
    while (ok) {
      const Group<G> cur = next_item(j, true);
      if (cur.w < 0) break;
      if (args.dense) continue;  // the loader brings contiguous rows by TMA
      uint32_t rem = rotate_taps(cur.all, cur.rot);
      while (rem && ok) {
        const int tap = next_tap(rem, cur.rot);
        for (int kb = 0; kb < kb_per_tap && ok; ++kb, ++g) {
          const int stage = int(g % STAGES);
          if (stage != gw) continue;
          GatherJob<G, kIdx> job;
          job.stage = stage;
          job.g = g;
          job.kb = kb;
          job.tiles = 0;
#pragma unroll
          for (int k = 0; k < G; ++k) {
#pragma unroll
            for (int i = 0; i < kIdx; ++i) job.vidx[k][i] = -1;
            if (!((cur.mask[k] >> tap) & 1u)) continue;
            job.tiles |= 1u << k;
            const int slot = cur.slot0[k] + __popc(cur.mask[k] & ((1u << tap) - 1u));
#pragma unroll
            for (int i = 0; i < kIdx; ++i)
              job.vidx[k][i] =
                  args.gidx[int64_t(slot) * kTileRows + kRowsPerWarp * rq + 32 * i + lane];
          }
          if (have_pend) ok = run(pend);
          pend = job;
          have_pend = true;
        }
      }
      // Never carry a stage into the next item: the next owned stage may lie
      // several items ahead, which the queue only publishes once the MMA
      // warps have moved on -- and the MMA warps wait for this stage.
      if (have_pend && ok) ok = run(pend);
      have_pend = false;
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
  } else if (warp == 0) {
    // ---------------- W loader ----------------
    if (lane == 0) {
      tma_prefetch_map(&wmap);
      if (args.dense) tma_prefetch_map(&fmap);
      uint32_t g = 0, j = 0;
      bool ok = true;
      while (ok) {
        const Group<G> cur = next_item(j, false);
        if (cur.w < 0) break;
        uint32_t rem = rotate_taps(cur.all, cur.rot);
        while (rem && ok) {
          const int tap = next_tap(rem, cur.rot);
          for (int kb = 0; kb < kb_per_tap; ++kb, ++g) {
            const int stage = int(g % STAGES);
            if (!mbar_wait(empty0 + 8 * stage, ((g / STAGES) & 1) ^ 1, abort_flag, args.status)) {
              ok = false;
              break;
            }
            const uint32_t full = full0 + 8 * stage;
            const uint32_t stage_base = smem_addr(smem + stage * kStageBytes);
            if (args.dense) {
              uint32_t live = 0;
#pragma unroll
              for (int k = 0; k < G; ++k) live += cur.mask[k] != 0u ? 1u : 0u;
              mbar_arrive_expect_tx(full, kBBytes + live * kABytes);
#pragma unroll
              for (int k = 0; k < G; ++k)
                if (cur.mask[k] != 0u)
                  tma_load_2d(stage_base + k * kABytes, &fmap, kb * kBK,
                              (cur.tile0 + k) * kTileRows, full);
            } else {
              mbar_arrive_expect_tx(full, kBBytes);
            }
            const uint32_t b_base = stage_base + G * kABytes;
#pragma unroll
            for (int jj = 0; jj < BN / 64; ++jj)
              tma_load_2d(b_base + jj * (kBK * 128), &wmap, cur.n0 + 64 * jj,
                          tap * args.cin + kb * kBK, full);
          }
        }
      }
    }
    __syncwarp();
  } else if (warp == 1 || warp == kMmaWarp2) {
    // ---------------- MMA warps ----------------
    // The whole warp runs the loop (waits, item bookkeeping, descriptors) and
    // stays converged; one elected lane issues.
    const int mine = warp == 1 ? 0 : 1;  // this warp's tiles: k % 2 == mine
    uint32_t g = 0, j = 0, acc_iter = 0;
    bool ok = true;
    const uint64_t adesc0 = desc_a_kmajor<BK>(smem_addr(smem));
    const uint64_t bdesc0 = desc_b_mnmajor(smem_addr(smem) + G * kABytes, kBK * 128);
    while (ok) {
      const Group<G> cur = next_item(j, true);
      const uint32_t a = acc_iter % NBUF;
      const uint32_t use = acc_iter / NBUF;  // how many times set a was used before
      const bool free = mbar_wait(tempty0 + 8 * a, (use & 1) ^ 1, abort_flag, args.status);
      if (!__all_sync(0xffffffffu, free)) break;
      // tell the epilogue which item this accumulator will hold (or that there
      // are no more); the buffer's epilogue has finished with it
      if (mine == 0 && lane == 0) {
        acc_info[a] = cur;
        mbar_arrive(info0 + 8 * a);
      }
      __syncwarp();
      if (cur.w < 0) break;
      tc_fence_after();
      uint32_t started = 0;  // bit k: tile k's accumulator holds a partial sum
      uint32_t rem = rotate_taps(cur.all, cur.rot);
      while (rem && ok) {
        const int tap = next_tap(rem, cur.rot);
        uint32_t live = 0;  // tiles of the group that have this tap
#pragma unroll
        for (int k = 0; k < G; ++k) live |= ((cur.mask[k] >> tap) & 1u) << k;
        for (int kb = 0; kb < kb_per_tap; ++kb, ++g) {
          const int stage = int(g % STAGES);
          const bool ready = mbar_wait(full0 + 8 * stage, (g / STAGES) & 1, abort_flag, args.status);
          if (!__all_sync(0xffffffffu, ready)) {
            ok = false;
            break;
          }
          tc_fence_after();
          {
            // descriptors of this stage: the start-address field (bits 0-13,
            // 16-byte units) never carries, so offsets add to the 64-bit value
            const uint64_t soff = uint64_t(stage) * (kStageBytes >> 4);
#pragma unroll
            for (int k = 0; k < G; ++k) {
              if (!((live >> k) & 1u) || (k & 1) != mine) continue;
              const uint32_t d_tmem = tmem + (a * G + k) * BN;
              const uint64_t ad = adesc0 + soff + uint64_t(k * (kABytes >> 4));
              const uint64_t bd = bdesc0 + soff;
              const uint32_t acc = (started >> k) & 1u;
#pragma unroll
              for (int kk = 0; kk < kBK / 16; ++kk)
                umma_f16(d_tmem, ad + 2 * kk, bd + (2048 >> 4) * kk, kIdesc, kk != 0 ? 1u : acc);
            }
            umma_commit(empty0 + 8 * stage);
          }
          started |= live;
        }
      }
      umma_commit(tfull0 + 8 * a);
      if (!ok) mbar_drain(tfull0 + 8 * a, use & 1);
      ++acc_iter;
    }
  } else {
    // ---------------- epilogue (warps 2-5) ----------------
    const int quarter = warp & 3;  // tensor-memory lanes 32*quarter .. +31
    const int row = quarter * 32 + lane;
    uint32_t acc_iter = 0;
    while (true) {
      const uint32_t a = acc_iter % NBUF;
      const uint32_t use = acc_iter / NBUF;
      bool have = mbar_wait(info0 + 8 * a, use & 1, abort_flag, args.status);
      have = __all_sync(0xffffffffu, have);
      if (!have) break;
      const Group<G> gr = acc_info[a];
      if (gr.w < 0) break;
      int32_t orow[G];
#pragma unroll
      for (int k = 0; k < G; ++k) {
        const int64_t r = int64_t(gr.tile0 + k) * kTileRows + row;
        if (gr.mask[k] == 0)
          orow[k] = -1;
        else if (args.dense)
          orow[k] = r < args.n ? int32_t(r) : -1;
        else
          orow[k] = args.out_row[r];
      }
      have = mbar_wait(tfull0 + 8 * a, use & 1, abort_flag, args.status);
      have = __all_sync(0xffffffffu, have);  // tcgen05.ld below is warp-collective
      if (!have) break;
      tc_fence_after();
#pragma unroll
      for (int k = 0; k < G; ++k) {
        if (gr.mask[k] == 0) continue;  // past the last tile
        uint16_t* dst = args.out + int64_t(orow[k] < 0 ? 0 : orow[k]) * args.cout + gr.n0;
#pragma unroll 1
        for (int cc = 0; cc < BN / 32; ++cc) {
          uint32_t v[32];
          tmem_ld_x32(tmem + (uint32_t(quarter * 32) << 16) + (a * G + k) * BN + uint32_t(cc * 32),
                      v);
          if (orow[k] >= 0) {
            uint4* d4 = reinterpret_cast<uint4*>(dst + cc * 32);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              uint4 o;
              o.x = pack2<BF16>(v[8 * q + 0], v[8 * q + 1]);
              o.y = pack2<BF16>(v[8 * q + 2], v[8 * q + 3]);
              o.z = pack2<BF16>(v[8 * q + 4], v[8 * q + 5]);
              o.w = pack2<BF16>(v[8 * q + 6], v[8 * q + 7]);
              d4[q] = o;
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(tempty0 + 8 * a);
      ++acc_iter;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  // The last CTA to finish resets the item counter for the next launch (every
  // CTA's last atomicAdd on it happened before it got here).
  if (threadIdx.x == 0) {
    __threadfence();
    if (atomicAdd(args.work_counter + 1, 1u) == gridDim.x - 1) {
      atomicExch(args.work_counter, 0u);
      atomicExch(args.work_counter + 1, 0u);
    }
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

// SM count of the current device, cached per device.
int sm_count() {
  constexpr int kMaxDev = 64;
  static int cache[kMaxDev] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < kMaxDev && cache[dev] > 0) return cache[dev];
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 1) {
    cudaGetLastError();
    sms = 148;
  }
  if (dev >= 0 && dev < kMaxDev) cache[dev] = sms;
  return sms;
}

// 2-D row-major [rows][cols] tensor map with a (box_cols x box_rows) box;
// box_cols * 2 bytes is the swizzle width (128 or 64 bytes).
bool encode_2d(CUtensorMap* map, bool bf16, const void* base, uint64_t cols, uint64_t rows,
               uint32_t box_cols, uint32_t box_rows) {
  auto encode = get_encode_fn();
  if (!encode) return false;
  cuuint64_t dims[2] = {cuuint64_t(cols), cuuint64_t(rows)};
  cuuint64_t strides[1] = {cuuint64_t(cols) * 2};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  const CUtensorMapSwizzle swz =
      box_cols == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  return encode(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2,
                const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int BN, int BK, int STAGES, int G, int WPS, bool BF16, int NBUF = 2>
int launch_cfg(const Plan& plan, bool dense, const void* feats, const void* W, void* out, int cin,
               int cout, cudaStream_t stream) {
  constexpr int kStageBytes = G * kTileRows * BK * 2 + BN * BK * 2;
  constexpr int kSmem = STAGES * kStageBytes + 1024 + 512;
  static_assert(kSmem <= 227 * 1024, "shared memory");
  static_assert(threads_for(STAGES, WPS) <= 1024, "threads");
  auto kern = k_conv_tc<BN, BK, STAGES, G, WPS, BF16, NBUF>;
  // the shared-memory limit is a per-device function attribute: set it once
  // on each device this configuration runs on
  constexpr int kMaxDev = 64;
  static bool attr_set[kMaxDev] = {};
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return SMC_ERR_CUDA;
  const bool cached = dev >= 0 && dev < kMaxDev && attr_set[dev];
  if (!cached) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem) !=
        cudaSuccess)
      return SMC_ERR_CUDA;
    if (dev >= 0 && dev < kMaxDev) attr_set[dev] = true;
  }
  CUtensorMap wmap, fmap;
  const int taps = dense ? 1 : kTaps;
  if (!encode_2d(&wmap, BF16, W, uint64_t(cout), uint64_t(taps) * uint64_t(cin), 64, BK) ||
      !encode_2d(&fmap, BF16, feats, uint64_t(cin), uint64_t(plan.n), BK, kTileRows))
    return SMC_ERR_CUDA;
  ConvArgs a;
  a.feats = static_cast<const uint16_t*>(feats);
  a.out = static_cast<uint16_t*>(out);
  a.gidx = plan.gidx;
  a.tile_off = plan.tile_off;
  a.tile_mask = plan.tile_mask;
  a.out_row = plan.out_row;
  static_assert(G == 1 || G == 2, "work-item orders exist for one and two tiles per item");
  a.group_order = plan.group_order[G - 1];
  a.status = plan.status;
  a.n = plan.n;
  a.cin = cin;
  a.cout = cout;
  a.n_tiles = int(plan.n_tiles);
  a.n_blocks = cout / BN;
  a.n_groups = int((plan.n_tiles + G - 1) / G);
  a.dense = dense ? 1 : 0;
  a.work_counter = plan.work_counter;  // zero since the build; reset by each launch
  const int64_t work = int64_t(a.n_groups) * a.n_blocks;
  const int grid = int(std::min<int64_t>(work, sm_count()));
  kern<<<grid, threads_for(STAGES, WPS), kSmem, stream>>>(wmap, fmap, a);
  return cudaGetLastError() == cudaSuccess ? SMC_OK : SMC_ERR_CUDA;
}

// Tuning overrides, read once per process: SMC_TC_GROUP=1 or 2 (tiles per work
// item, default: 1 below 6 tiles per SM, else 2) and SMC_TC_BK=32 (32-channel
// stages, twice as many, 64-byte swizzle).
int env_int(const char* name) {
  const char* e = std::getenv(name);
  return e ? std::atoi(e) : 0;
}
int group_override() {
  static int v = env_int("SMC_TC_GROUP");
  return v;
}
int bk_override() {
  static int v = env_int("SMC_TC_BK");
  return v;
}

template <bool BF16>
int launch_dtype(const Plan& plan, bool dense, const void* feats, const void* W, void* out,
                 int cin, int cout, cudaStream_t stream) {
  // Few tiles per SM: one tile per work item, so every SM gets work and no SM
  // runs two heavy tiles back to back.
  const bool small = plan.n_tiles < int64_t(6) * sm_count();
  //            BN  BK  stages G WPS
  if (bk_override() == 32) {
    if (cout % 256 == 0)
      return launch_cfg<256, 32, 8, 1, 2, BF16>(plan, dense, feats, W, out, cin, cout, stream);
    if (cout % 128 == 0)
      return launch_cfg<128, 32, 8, 2, 2, BF16>(plan, dense, feats, W, out, cin, cout, stream);
    return launch_cfg<64, 32, 10, 2, 2, BF16>(plan, dense, feats, W, out, cin, cout, stream);
  }
  if ((group_override() == 1 || (small && group_override() != 2)) && cout % 256 != 0) {
    if (cout % 128 == 0)
      return launch_cfg<128, 64, 5, 1, 4, BF16>(plan, dense, feats, W, out, cin, cout, stream);
    return launch_cfg<64, 64, 6, 1, 4, BF16>(plan, dense, feats, W, out, cin, cout, stream);
  }
  if (cout % 256 == 0) {
    // sparse: two 256-column tiles per item share each W slice (single
    // accumulator set), as long as that leaves at least two items per SM;
    // dense (K = 1) items are short, so they keep the overlapped epilogue
    const int64_t items2 = (plan.n_tiles + 1) / 2 * (cout / 256);
    if (group_override() == 2 ||
        (group_override() == 0 && !dense && items2 >= 2 * int64_t(sm_count())))
      return launch_cfg<256, 64, 3, 2, 4, BF16, 1>(plan, dense, feats, W, out, cin, cout, stream);
    return launch_cfg<256, 64, 4, 1, 4, BF16>(plan, dense, feats, W, out, cin, cout, stream);
  }
  if (cout % 128 == 0)
    return launch_cfg<128, 64, 4, 2, 4, BF16>(plan, dense, feats, W, out, cin, cout, stream);
  return launch_cfg<64, 64, 5, 2, 4, BF16>(plan, dense, feats, W, out, cin, cout, stream);
}

}  // namespace

bool conv_tc_supported(int cin, int cout, int dtype) {
  return (dtype == SMC_F16 || dtype == SMC_BF16) && cin > 0 && cout > 0 && cin % 64 == 0 &&
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
