// Output-stationary implicit-GEMM SubMConv3d on the sm_100a tensor cores.
//
// A work item is a group of G consecutive 128-row tiles (in plan order) and
// one BN-wide block of output channels.  For every tap some tile of the group
// uses (the others are skipped), each such tile's 128 neighbour feature rows
// of that tap are gathered into shared memory (zero rows for absent
// neighbours) and multiplied by W[tap] with tcgen05.mma, accumulating in fp32
// in tensor memory; each output row is then written exactly once, without
// atomics.  This is the sum over offsets of the trellis_sparse_mlx README
// ("What's in it": out[c] = sum_d feats[c+d] @ W[d] over active neighbours)
// organised as the masked implicit GEMM of "Metal-native replacement for
// flex_gemm bottleneck?" ("Fixed": sorted rows, per-block valid taps, empty
// taps skipped), rather than the README's dense [N, 27 Cin] x [27 Cin, Cout]
// matmul.
//
// Pipeline units.  The taps of an item are walked in a rotated order; each
// tap is split into Cin / (64 KS) channel chunks ("stages"), KS = 2 (128
// channels) where Cin allows it for 128-column tiles, else 1.  A stage needs
// one W slice W[tap][64 KS ci][BN] (shared by the group's tiles) and, for
// every tile of the group that has the tap, one A unit: 128 gathered rows x
// 64 KS channels (16 KS KB).  W slices and A units live in two separate
// shared-memory rings, so an A unit is refilled as soon as its own MMAs are
// done, and a tile whose rows have landed is multiplied without waiting for
// the other tile.
//
// Work items are dealt to the CTAs statically, in snake order over the
// longest-first item list, and every role walks its CTA's items itself, so
// nothing is claimed or handed out at run time.
//
// Persistent kernel, one CTA per SM, 7 + NQ * WPS + 1 warps:
//   warp 0      W loader: lane 0 TMA-loads each stage's W slice (MN-major,
//               128-byte swizzle) into the W ring;
//   warp 1      allocates tensor memory; issues the MMAs (M = 128, N = BN,
//               K = 16) of the even tiles of each item.  The last warp
//               issues those of the odd tiles.  A tcgen05.mma keeps its
//               issuing thread until the tensor core accepts it, so two
//               issuers cover each other's loop and wait overheads;
//   warps 2-5   epilogue: tensor memory -> registers -> fp16/bf16 -> global,
//               overlapping the next item's MMAs when there are two
//               accumulator sets (NBUF = 2).  Where shared memory has room,
//               each warp passes its 32 rows through a staging block so that
//               every store writes 64-byte row pieces (8 rows per
//               instruction) rather than 16-byte pieces of 32 rows.  The
//               CTA's last item is stored together with the first four
//               gather warps, which are idle by then;
//   warp 6      index prefetcher: lane 0 bulk-copies the 128 gather indices
//               of each A unit into a ring of index blocks, running up to a
//               full ring of units ahead of the gathers;
//   warps 7..   NQ gather groups of WPS warps.  Units are dealt round-robin to
//               the groups; a group reads its unit's indices from shared
//               memory and copies the 128 rows with 16-byte cp.async into
//               128-byte-swizzled K-major tiles (zero-filled for absent
//               neighbours); each lane's arrival on the unit's barrier is
//               made by the hardware when its copies land, and the MMA warp
//               puts a proxy fence between that barrier and its reads.  For
//               K = 1 ("dense" mode) the rows are contiguous and one lane of
//               the group loads them with TMA.
// Every hand-over is an mbarrier.  Every wait is bounded in time; a wait that
// runs out marks the CTA aborted and sets the status word, and each role then
// waits (again bounded) for the asynchronous copies and MMAs it issued before
// the CTA frees tensor memory and exits.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <algorithm>
#include <cstdlib>
#include <mutex>

#include "smc_internal.h"
#include "smc_ptx.cuh"

namespace smc {
namespace {

using namespace ptx;

constexpr int kLoaderWarp = 0;
constexpr int kMmaWarp = 1;
constexpr int kIndexWarp = 6;
constexpr int kFirstGatherWarp = 7;
constexpr int kBK = 64;                          // channels per sub-chunk (128-byte rows)
constexpr int kSubBytes = kTileRows * kBK * 2;    // one A sub-tile: 128 rows x 64 channels
constexpr int kIdxBytes = kTileRows * 4;          // one unit's gather indices

__host__ __device__ constexpr int threads_for(int nq, int wps) {
  return 32 * (kFirstGatherWarp + nq * wps + 1);
}

struct ConvArgs {
  const uint16_t* feats;
  uint16_t* out;
  const int32_t* gidx;     // [slots][128], -1 = absent
  const int32_t* out_row;  // [n_tiles * 128], -1 = padding row
  const int4* items;       // [n_groups] {first tile, mask0, mask1, first slot}, most taps first
  int32_t* status;
  int64_t n;
  int cin;
  int cout;
  int n_tiles;
  int n_groups;  // ceil(n_tiles / G)
  int n_blocks;  // cout / BN
  int dense;     // 1: K = 1, rows in order, one tap, no plan arrays
  uint64_t wait_ns;
  const uint16_t* bias;      // [cout] or null: epilogue act(acc + bias) + residual
  const uint16_t* residual;  // [n][cout] or null
  int act;                   // enum smc_activation
};

template <bool BF16>
__device__ __forceinline__ float half_to_float(uint16_t h) {
  if constexpr (BF16)
    return __uint_as_float(uint32_t(h) << 16);
  else
    return __half2float(__ushort_as_half(h));
}

// Adds 32 fp16/bf16 values (four 16-byte words, element order) to v.
template <bool BF16>
__device__ __forceinline__ void add_halves(uint32_t (&v)[32], const uint4 (&h)[4]) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint32_t w[4] = {h[q].x, h[q].y, h[q].z, h[q].w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      v[8 * q + 2 * e] = __float_as_uint(__uint_as_float(v[8 * q + 2 * e]) +
                                         half_to_float<BF16>(uint16_t(w[e] & 0xFFFFu)));
      v[8 * q + 2 * e + 1] = __float_as_uint(__uint_as_float(v[8 * q + 2 * e + 1]) +
                                             half_to_float<BF16>(uint16_t(w[e] >> 16)));
    }
  }
}

// act(acc + bias) on 32 consecutive columns of one output row, in fp32.  The
// activation is chosen once per call, and SiLU uses the fast exponential and
// division (their error, a few fp32 ulps, is far below the output's one
// rounding; for very negative x the divisor is infinite and the result the
// limit 0).
template <bool BF16>
__device__ __forceinline__ void bias_activation(uint32_t (&v)[32], const ConvArgs& a, int col) {
  if (a.bias) {
    const uint4* b4 = reinterpret_cast<const uint4*>(a.bias + col);
    uint4 b[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) b[q] = __ldg(b4 + q);
    add_halves<BF16>(v, b);
  }
  switch (a.act) {
    case SMC_ACT_RELU:
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] = __float_as_uint(fmaxf(__uint_as_float(v[i]), 0.f));
      break;
    case SMC_ACT_SILU:
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const float x = __uint_as_float(v[i]);
        v[i] = __float_as_uint(__fdividef(x, 1.f + __expf(-x)));
      }
      break;
    case SMC_ACT_GELU:
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const float x = __uint_as_float(v[i]);
        v[i] = __float_as_uint(0.5f * x * (1.f + erff(x * 0.7071067811865476f)));
      }
      break;
    default:
      break;
  }
}

// The residual's 32 columns of one output row (zeros when there is none or
// the row is padding), loaded one chunk ahead of their use.
template <bool BF16>
__device__ __forceinline__ void load_residual(uint4 (&r)[4], const ConvArgs& a, int32_t row,
                                              int col) {
  if (a.residual && row >= 0) {
    const uint4* r4 = reinterpret_cast<const uint4*>(a.residual + int64_t(row) * a.cout + col);
#pragma unroll
    for (int q = 0; q < 4; ++q) r[q] = __ldg(r4 + q);
  } else {
#pragma unroll
    for (int q = 0; q < 4; ++q) r[q] = make_uint4(0u, 0u, 0u, 0u);
  }
}

// A work item as every role of a CTA decodes it.
template <int G>
struct Item {
  int w;         // item number, -1 = no more work
  int tile0;
  int n0;        // first output channel
  uint32_t all;  // union of the tiles' tap masks
  int rot;       // taps are visited starting at this one (spreads W reads over L2)
  uint32_t mask[G];
  int slot0[G];  // first gather-index slot of each tile
};

// The j-th item of this CTA: items are dealt over the CTAs in snake order
// (CTA c takes c, 2 P - 1 - c, 2 P + c, ... of the longest-first list, P CTAs),
// so every CTA gets a similar mix of long and short items and no item has to
// be claimed at run time.  -1 past the end.
__device__ __forceinline__ int item_of(uint32_t j, int total) {
  const int64_t p = gridDim.x, c = blockIdx.x;
  const int64_t w = int64_t(j) * p + ((j & 1u) ? p - 1 - c : c);
  return w < total ? int(w) : -1;
}
// The 16-byte record of item w (sparse mode), loaded one item ahead of use.
template <bool DENSE>
__device__ __forceinline__ int4 item_record(const ConvArgs& a, int w) {
  if (w < 0 || DENSE) return make_int4(0, 0, 0, 0);
  return __ldg(a.items + w / a.n_blocks);
}

template <int BN, int G, bool DENSE>
__device__ __forceinline__ Item<G> decode_item(const ConvArgs& a, int w, int4 r) {
  Item<G> it;
  it.w = w;
  const int q = w / a.n_blocks;
  it.n0 = (w - q * a.n_blocks) * BN;
  if constexpr (DENSE) {
    it.tile0 = q * G;
#pragma unroll
    for (int k = 0; k < G; ++k) {
      it.mask[k] = it.tile0 + k < a.n_tiles ? 1u : 0u;
      it.slot0[k] = 0;
    }
    it.rot = 0;
  } else {
    it.tile0 = r.x;
    it.mask[0] = uint32_t(r.y);
    it.slot0[0] = r.w;
    if constexpr (G == 2) {
      it.mask[1] = uint32_t(r.z);
      it.slot0[1] = r.w + __popc(uint32_t(r.y));
    }
    it.rot = int((unsigned(w) * 7u) % unsigned(kTaps));
  }
  it.all = 0;
#pragma unroll
  for (int k = 0; k < G; ++k) it.all |= it.mask[k];
  return it;
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
// The taps of one stage: ta, and with tap pairing (64-channel inputs, two
// taps per 128-channel unit) the next tap of the item's list, or -1.
struct StageTaps {
  int ta, tb;
};
template <bool PAIR>
__device__ __forceinline__ StageTaps next_stage_taps(uint32_t& rem, int rot) {
  StageTaps t;
  t.ta = next_tap(rem, rot);
  t.tb = (PAIR && rem) ? next_tap(rem, rot) : -1;
  return t;
}
// Sub-chunks of a stage that tile k multiplies (bit s = sub-chunk s): with
// pairing, sub-chunk s is tap s of the pair; otherwise the KS sub-chunks are
// consecutive 64-channel chunks of one tap.
template <int G, int KS, bool PAIR>
__device__ __forceinline__ uint32_t sub_live(const Item<G>& it, int k, StageTaps t) {
  const uint32_t m = it.mask[k];
  if constexpr (PAIR)
    return ((m >> t.ta) & 1u) | (t.tb >= 0 ? ((m >> t.tb) & 1u) << 1 : 0u);
  else
    return ((m >> t.ta) & 1u) ? ((1u << KS) - 1u) : 0u;
}
// Tiles of the group with any sub-chunk in the stage (bit k = tile k).
template <int G, int KS, bool PAIR>
__device__ __forceinline__ uint32_t stage_live(const Item<G>& it, StageTaps t) {
  uint32_t live = 0;
#pragma unroll
  for (int k = 0; k < G; ++k) live |= (sub_live<G, KS, PAIR>(it, k, t) != 0u ? 1u : 0u) << k;
  return live;
}
// Gather-index slot of tile k's tap t (the tile has the tap).
template <int G>
__device__ __forceinline__ int index_slot(const Item<G>& it, int k, int t) {
  return it.slot0[k] + __popc(it.mask[k] & ((1u << t) - 1u));
}

// Shared-memory layout: A ring, W ring, index ring (the rings), then the
// barriers and the small per-CTA state (the tail), then, when the rings leave
// room for it, the epilogue's output staging: per epilogue warp 32 rows of 32
// output columns, each row's 64 bytes padded to 80 so that both the row-wise
// writes and the column-wise reads are free of bank conflicts.
constexpr int kStageRowBytes = 80;
constexpr int kStageBytes = 4 * 32 * kStageRowBytes;
template <int BN, int NA, int NW, int KS, bool PAIR>
__host__ __device__ constexpr int smem_rings() {
  return NA * (KS * kSubBytes + (PAIR ? 2 : 1) * kIdxBytes) + NW * KS * BN * kBK * 2;
}
template <int NA, int NW, int G>
__host__ __device__ constexpr int smem_tail() {
  return ((4 * NA + 2 * NW + 9) * 8 + 2 * int(sizeof(Item<G>)) + 16 + 15) & ~15;
}
template <int BN, int NA, int NW, int G, int KS, bool PAIR>
__host__ __device__ constexpr bool staged_output() {
  return smem_rings<BN, NA, NW, KS, PAIR>() + smem_tail<NA, NW, G>() + kStageBytes <= 227 * 1024;
}
template <int BN, int NA, int NW, int G, int KS, bool PAIR>
__host__ __device__ constexpr int smem_bytes() {
  return smem_rings<BN, NA, NW, KS, PAIR>() + smem_tail<NA, NW, G>() +
         (staged_output<BN, NA, NW, G, KS, PAIR>() ? kStageBytes : 0);
}

// NA: A units in flight (16 KS KB each), NW: W slices in flight, NQ gather
// groups of WPS warps, NBUF accumulator sets in tensor memory (2: the epilogue
// of one item overlaps the MMAs of the next; 1: room for two 256-column
// tiles), KS: 64-channel sub-chunks per unit, PAIR: the two sub-chunks are
// two taps of 64-channel rows (else KS chunks of one tap), EPI: the fused
// epilogue (bias, activation, residual) is applied, DENSE: K = 1 (contiguous
// rows loaded by TMA, one tap, no plan arrays); each is its own instantiation
// so that a kernel carries only the code it runs.
template <int BN, int NA, int NW, int G, int WPS, int NQ, bool BF16, int NBUF, int KS, bool PAIR,
          bool EPI, bool DENSE>
__global__ void __launch_bounds__(threads_for(NQ, WPS), 1)
k_conv_tc(const __grid_constant__ CUtensorMap wmap, const __grid_constant__ CUtensorMap fmap,
          const ConvArgs args) {
  static_assert(BN % 64 == 0 && BN <= 256, "BN");
  // Each A slot belongs to one gather group (slot = unit % NA, group = unit %
  // NQ): a group fills its slots in phase order, so no wait on a slot barrier
  // can be two phases behind, and the abort path can tell which of its loads
  // may still be in flight.
  static_assert(NA % NQ == 0, "every A slot is owned by one gather group");
  // a stage has at most G units, so each gather group has at most one of them
  static_assert(NQ >= G, "one unit per gather group and stage");
  // the first four gather warps (consecutive warps: one per tensor-memory lane
  // quarter) store half of the CTA's last item
  static_assert(NQ * WPS >= 4, "four gather warps help store the last item");
  // The two MMA warps take the even and odd tiles of an item and meet only at
  // the W ring, so one can run up to NW stages (NW * G units) ahead of the
  // other.  Its wait on an A slot must never be two phases ahead of the
  // barrier: a slot is reused every NA units, hence NW * G <= NA.
  static_assert(NW * G <= NA, "MMA warps drift by at most one A slot phase");
  static_assert(NBUF == 1 || NBUF == 2, "accumulator sets");
  static_assert(KS == 1 || KS == 2, "64-channel sub-chunks per unit");
  static_assert(!PAIR || KS == 2, "tap pairing puts two taps in one 128-channel unit");
  constexpr int kIdxSlot = (PAIR ? 2 : 1) * kIdxBytes;  // index blocks of one unit
  constexpr int kAUnitBytes = KS * kSubBytes;    // one A unit: 128 rows x 64 KS channels
  constexpr int kWBytes = BN * kBK * 2;          // one W sub-slice: 64 input channels x BN
  constexpr int kWStage = KS * kWBytes;          // the W of one unit
  constexpr int kRowsPerWarp = kTileRows / WPS;  // rows of a unit one gather warp copies
  constexpr int kInstr = kRowsPerWarp / 4;       // a warp copy instruction covers 4 rows
  static_assert(kRowsPerWarp % 4 == 0 && kInstr >= 1, "gather split");
  constexpr uint32_t kTmemCols = NBUF * G * BN;  // NBUF sets of G accumulators
  static_assert(kTmemCols >= 32 && kTmemCols <= 512 && (kTmemCols & (kTmemCols - 1)) == 0,
                "tensor memory columns");
  constexpr uint32_t kIdesc = make_idesc(BN, BF16);
  constexpr int kMmaWarp2 = kFirstGatherWarp + NQ * WPS;
  constexpr uint32_t kMmaWarps = 2;

  // The rings start at the beginning of dynamic shared memory (the kernel
  // has no static shared variables), which the 128-byte swizzle needs
  // 1024-byte aligned; a launch where it is not reports that and does nothing.
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if ((smem_addr(smem_raw) & 1023u) != 0) {
    if (threadIdx.x == 0) atomicOr(args.status, kDevLayout);
    return;
  }
  uint8_t* a_ring = smem_raw;                               // NA x kAUnitBytes
  uint8_t* w_ring = a_ring + NA * kAUnitBytes;              // NW x kWStage
  int32_t* idx_ring = reinterpret_cast<int32_t*>(w_ring + NW * kWStage);  // NA x kIdxSlot
  uint64_t* bars = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(idx_ring) + NA * kIdxSlot);
  // barriers: afull[NA] aempty[NA] ifull[NA] iempty[NA] wfull[NW] wempty[NW]
  //           tfull[2] tempty[2] info[2] drain[2] lastdone
  constexpr int kBars = 4 * NA + 2 * NW + 6 + 2 + 1;
  constexpr bool kStaged = staged_output<BN, NA, NW, G, KS, PAIR>();
  Item<G>* acc_info = reinterpret_cast<Item<G>*>(bars + kBars);  // item of each accumulator set
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_info + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  uint8_t* out_stage = smem_raw + smem_rings<BN, NA, NW, KS, PAIR>() + smem_tail<NA, NW, G>();

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kb_per_tap = PAIR ? 1 : args.cin / (kBK * KS);  // stages per tap (pair)
  const int total_work = args.n_groups * args.n_blocks;
  const uint32_t afull0 = smem_addr(bars);
  const uint32_t aempty0 = afull0 + 8 * NA;
  const uint32_t ifull0 = aempty0 + 8 * NA;
  const uint32_t iempty0 = ifull0 + 8 * NA;
  const uint32_t wfull0 = iempty0 + 8 * NA;
  const uint32_t wempty0 = wfull0 + 8 * NW;
  const uint32_t tfull0 = wempty0 + 8 * NW;
  const uint32_t tempty0 = tfull0 + 16;
  const uint32_t info0 = tempty0 + 16;
  const uint32_t drain0 = info0 + 16;
  const uint32_t lastdone = drain0 + 16;  // the CTA's last item's MMAs are done
  const uint32_t a_base = smem_addr(a_ring);
  const uint32_t w_base = smem_addr(w_ring);
  const uint32_t i_base = smem_addr(idx_ring);

  if (threadIdx.x == 0) {
    for (int s = 0; s < NA; ++s) {
      // sparse: every lane of the unit's gather group; dense: the lane that
      // TMA-loads the contiguous rows
      mbar_init(afull0 + 8 * s, DENSE ? 1 : WPS * 32);
      mbar_init(aempty0 + 8 * s, 1);
      mbar_init(ifull0 + 8 * s, 1);
      mbar_init(iempty0 + 8 * s, WPS);
    }
    for (int s = 0; s < NW; ++s) {
      mbar_init(wfull0 + 8 * s, 1);
      mbar_init(wempty0 + 8 * s, kMmaWarps);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull0 + 8 * a, kMmaWarps);
      mbar_init(tempty0 + 8 * a, 4 * 32);
      mbar_init(info0 + 8 * a, 1);
      mbar_init(drain0 + 8 * a, 1);
    }
    mbar_init(lastdone, kMmaWarps);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == kMmaWarp) tmem_alloc(smem_addr(tmem_slot), kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const Waits wt{abort_flag, args.status, args.wait_ns};

  // Every role walks the CTA's items itself, in the same order: next_item
  // decodes the j-th item from the record loaded by the previous call and
  // starts the load of the following record.  w = -1 after the last item.
  auto next_item = [&](uint32_t& j, int4& rec) -> Item<G> {
    Item<G> it;
    const int w = item_of(j, total_work);
    if (w < 0) {
      it.w = -1;
      return it;
    }
    it = decode_item<BN, G, DENSE>(args, w, rec);
    ++j;
    rec = item_record<DENSE>(args, item_of(j, total_work));
    return it;
  };
  auto first_record = [&]() { return item_record<DENSE>(args, item_of(0, total_work)); };

  // Epilogue pieces, used by the epilogue warps and, for the CTA's last item,
  // by the first four gather warps.  A warp handles the tensor-memory lanes
  // (rows) 32 * (warp % 4) ... + 31 of every tile of the item.
  constexpr int kChunks = BN / 32;  // 32-column chunks of a tile
  auto output_rows = [&](const Item<G>& it, int32_t (&orow)[G]) {
    const int row = (warp & 3) * 32 + lane;
#pragma unroll
    for (int k = 0; k < G; ++k) {
      const int64_t r = int64_t(it.tile0 + k) * kTileRows + row;
      if (it.mask[k] == 0)
        orow[k] = -1;
      else if (DENSE)
        orow[k] = r < args.n ? int32_t(r) : -1;
      else
        orow[k] = args.out_row[r];
    }
  };
  // Chunks cc0 .. cc1 - 1 of every tile of the item in accumulator set a.
  auto store_columns = [&](const Item<G>& it, uint32_t a, const int32_t (&orow)[G], int cc0,
                           int cc1, uint8_t* st_rows) {
    const int quarter = warp & 3;
#pragma unroll
    for (int k = 0; k < G; ++k) {
      if (it.mask[k] == 0) continue;  // past the last tile
      uint16_t* dst = args.out + int64_t(orow[k] < 0 ? 0 : orow[k]) * args.cout + it.n0;
      uint4 res[4];  // the fused epilogue's residual, one chunk ahead
      if constexpr (EPI) load_residual<BF16>(res, args, orow[k], it.n0 + cc0 * 32);
#pragma unroll 1
      for (int cc = cc0; cc < cc1; ++cc) {
        uint32_t v[32];
        tmem_ld_x32(tmem + (uint32_t(quarter * 32) << 16) + (a * G + k) * BN + uint32_t(cc * 32),
                    v);
        if constexpr (EPI) {
          // act(acc + bias) + residual, before the one rounding
          uint4 cur[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) cur[q] = res[q];
          if (cc + 1 < cc1) load_residual<BF16>(res, args, orow[k], it.n0 + (cc + 1) * 32);
          if (orow[k] >= 0) {
            bias_activation<BF16>(v, args, it.n0 + cc * 32);
            add_halves<BF16>(v, cur);
          }
        }
        if constexpr (kStaged) {
          // this lane's row piece into the warp's staging rows, then each
          // store writes 64-byte pieces of 8 rows (4 lanes per row)
          uint4* mine_row = reinterpret_cast<uint4*>(st_rows + lane * kStageRowBytes);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint4 o;
            o.x = pack2<BF16>(v[8 * q + 0], v[8 * q + 1]);
            o.y = pack2<BF16>(v[8 * q + 2], v[8 * q + 3]);
            o.z = pack2<BF16>(v[8 * q + 4], v[8 * q + 5]);
            o.w = pack2<BF16>(v[8 * q + 6], v[8 * q + 7]);
            mine_row[q] = o;
          }
          __syncwarp();
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int r = 8 * i + (lane >> 2), c = lane & 3;
            const int32_t orr = __shfl_sync(0xffffffffu, orow[k], r);
            const uint4 val = *reinterpret_cast<const uint4*>(st_rows + r * kStageRowBytes + c * 16);
            if (orr >= 0)
              *reinterpret_cast<uint4*>(args.out + int64_t(orr) * args.cout + it.n0 + cc * 32 +
                                        c * 8) = val;
          }
          __syncwarp();  // the rows are read before the next chunk overwrites them
          continue;
        }
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
  };

  if (warp == kLoaderWarp) {
    // ---------------- W loader ----------------
    if (lane == 0) {
      tma_prefetch_map(&wmap);
      uint32_t s = 0, j = 0;
      int4 rec = first_record();
      bool ok = true;
      while (ok) {
        const Item<G> it = next_item(j, rec);
        if (it.w < 0) break;
        uint32_t rem = rotate_taps(it.all, it.rot);
        while (rem && ok) {
          const StageTaps st = next_stage_taps<PAIR>(rem, it.rot);
          const int nsub = (PAIR && st.tb < 0) ? 1 : KS;  // an unpaired last tap
          for (int kb = 0; kb < kb_per_tap; ++kb, ++s) {
            const uint32_t ws = s % NW;
            if (!wt.wait(wempty0 + 8 * ws, ((s / NW) & 1) ^ 1)) {
              ok = false;
              break;
            }
            const uint32_t full = wfull0 + 8 * ws;
            mbar_arrive_expect_tx(full, nsub * kWBytes);
            const uint32_t dst = w_base + ws * kWStage;
#pragma unroll
            for (int sub = 0; sub < KS; ++sub) {
              if (sub >= nsub) break;
              const int row = PAIR ? (sub ? st.tb : st.ta) * args.cin
                                   : st.ta * args.cin + (kb * KS + sub) * kBK;
#pragma unroll
              for (int jj = 0; jj < BN / 64; ++jj)
                tma_load_2d(dst + sub * kWBytes + jj * (kBK * 128), &wmap, it.n0 + 64 * jj, row,
                            full);
            }
          }
        }
      }
      // the slices still in flight land before the CTA's shared memory goes
      for (uint32_t d = 0; d < NW && d < s; ++d) {
        const uint32_t t = s - 1 - d;
        mbar_drain(wfull0 + 8 * (t % NW), (t / NW) & 1);
      }
    }
    __syncwarp();
  } else if (warp == kIndexWarp) {
    // ---------------- index prefetcher ----------------
    if (lane == 0) {
      uint32_t u = 0, j = 0;
      int4 rec = first_record();
      bool ok = true;
      while (ok) {
        const Item<G> it = next_item(j, rec);
        if (it.w < 0) break;
        if (DENSE) continue;  // K = 1 has no gather index
        uint32_t rem = rotate_taps(it.all, it.rot);
        while (rem && ok) {
          const StageTaps st = next_stage_taps<PAIR>(rem, it.rot);
          for (int kb = 0; kb < kb_per_tap && ok; ++kb) {
#pragma unroll
            for (int k = 0; k < G; ++k) {
              const uint32_t sl = sub_live<G, KS, PAIR>(it, k, st);
              if (sl == 0u) continue;
              const uint32_t is = u % NA;
              if (!wt.wait(iempty0 + 8 * is, ((u / NA) & 1) ^ 1)) {
                ok = false;
                break;
              }
              // the gathers' reads of this block (generic proxy) come before the
              // bulk copy that overwrites it (async proxy)
              fence_proxy_async_smem();
              const uint32_t full = ifull0 + 8 * is;
              if constexpr (PAIR) {
                mbar_arrive_expect_tx(full, uint32_t(__popc(sl)) * kIdxBytes);
#pragma unroll
                for (int sub = 0; sub < 2; ++sub)
                  if ((sl >> sub) & 1u)
                    bulk_load(i_base + is * kIdxSlot + sub * kIdxBytes,
                              args.gidx + int64_t(index_slot(it, k, sub ? st.tb : st.ta)) * kTileRows,
                              kIdxBytes, full);
              } else {
                mbar_arrive_expect_tx(full, kIdxBytes);
                bulk_load(i_base + is * kIdxSlot,
                          args.gidx + int64_t(index_slot(it, k, st.ta)) * kTileRows, kIdxBytes,
                          full);
              }
              ++u;
            }
          }
        }
      }
      for (uint32_t d = 0; d < NA && d < u; ++d) {
        const uint32_t t = u - 1 - d;
        mbar_drain(ifull0 + 8 * (t % NA), (t / NA) & 1);
      }
    }
    __syncwarp();
  } else if (warp >= kFirstGatherWarp && warp < kMmaWarp2) {
    // ---------------- gather groups ----------------
    const int grp = (warp - kFirstGatherWarp) / WPS;  // units u with u % NQ == grp
    const int wq = (warp - kFirstGatherWarp) % WPS;   // rows kRowsPerWarp * wq ...
    const int chunk = lane & 7;   // 16-byte chunk of a 128-byte row
    const int rsub = lane >> 3;   // instruction i copies rows 4 i + rsub of the warp's share
    const int row0 = kRowsPerWarp * wq;
    if (DENSE && wq == 0 && lane == 0) tma_prefetch_map(&fmap);
    uint32_t u = 0, j = 0;
    int4 rec = first_record();
    int last_dense = -1;  // last unit this group TMA-loaded (dense mode)
    bool ok = true;
    Item<G> last_it;
    uint32_t n_items = 0;
    while (ok) {
      const Item<G> it = next_item(j, rec);
      if (it.w < 0) break;
      last_it = it;
      ++n_items;
      uint32_t rem = rotate_taps(it.all, it.rot);
      while (rem && ok) {
        const StageTaps st = next_stage_taps<PAIR>(rem, it.rot);
        for (int kb = 0; kb < kb_per_tap && ok; ++kb) {
          // the group's unit of this stage, if any (at most one: NQ >= G);
          // one copy of the code below serves every tile of the group
          int k = -1;
          uint32_t my = 0, sl = 0;
#pragma unroll
          for (int t = 0; t < G; ++t) {
            const uint32_t l = sub_live<G, KS, PAIR>(it, t, st);
            if (l == 0u) continue;
            const uint32_t un = u++;
            if (int(un % NQ) == grp) {
              k = t;
              my = un;
              sl = l;
            }
          }
          if (k < 0) continue;
          {
            const uint32_t slot = my % NA, ph = (my / NA) & 1;
            const uint32_t dst = a_base + slot * kAUnitBytes;
            if constexpr (DENSE) {
              if (wq == 0 && lane == 0) {
                if (!wt.wait(aempty0 + 8 * slot, ph ^ 1)) {
                  ok = false;
                } else {
                  mbar_arrive_expect_tx(afull0 + 8 * slot, kAUnitBytes);
#pragma unroll
                  for (int sub = 0; sub < KS; ++sub)
                    tma_load_2d(dst + sub * kSubBytes, &fmap, (kb * KS + sub) * kBK,
                                (it.tile0 + k) * kTileRows, afull0 + 8 * slot);
                  last_dense = int(my);
                }
              }
              ok = __shfl_sync(0xffffffffu, ok, 0);
              if (!ok) break;
              continue;
            }
            // the unit's source rows, read from the index ring
            bool got = wt.wait(ifull0 + 8 * slot, ph);
            if (!__all_sync(0xffffffffu, got)) {
              ok = false;
              break;
            }
            constexpr int kSets = PAIR ? 2 : 1;  // index blocks of the unit
            int v[kSets][kInstr];
            const int32_t* idx = idx_ring + slot * (kIdxSlot / 4) + row0 + rsub;
#pragma unroll
            for (int q = 0; q < kSets; ++q)
#pragma unroll
              for (int i = 0; i < kInstr; ++i) v[q][i] = idx[q * kTileRows + 4 * i];
            // the block is refilled by a bulk copy (async proxy) once released:
            // order these generic-proxy reads before that write
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(iempty0 + 8 * slot);
            got = wt.wait(aempty0 + 8 * slot, ph ^ 1);
            if (!__all_sync(0xffffffffu, got)) {
              ok = false;
              break;
            }
            const uint16_t* src_col = args.feats + (PAIR ? 0 : kb * (KS * kBK)) + chunk * 8;
#pragma unroll
            for (int i = 0; i < kInstr; ++i) {
              const int row = row0 + 4 * i + rsub;
              // 128-byte swizzle: chunk c of row r sits at chunk c ^ (r & 7)
              const uint32_t d = dst + row * 128 + ((chunk ^ (row & 7)) << 4);
#pragma unroll
              for (int sub = 0; sub < KS; ++sub) {
                if (PAIR && !((sl >> sub) & 1u)) continue;  // that tap is not the tile's
                const int r = v[PAIR ? sub : 0][i];
                const uint16_t* src =
                    r >= 0 ? src_col + int64_t(r) * args.cin + (PAIR ? 0 : sub * kBK) : args.feats;
                cp_async_16(d + sub * kSubBytes, src, r >= 0 ? 16u : 0u);
              }
            }
            // one arrival per lane on the slot's barrier, made by the hardware
            // once this lane's copies have landed; the MMA warp orders them
            // before its tensor-core reads with a proxy fence
            cp_async_arrive_noinc(afull0 + 8 * slot);
          }
        }
      }
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
    if (ok && n_items > 0 && warp - kFirstGatherWarp < 4) {
      // help store the CTA's last item (the second half of its columns) once
      // its MMAs are done; the A ring is free by then and holds the staging rows
      const uint32_t a = (n_items - 1) % NBUF;
      int32_t orow[G];
      output_rows(last_it, orow);
      // one phase only, so the wait cannot mistake an earlier item for it
      const bool have = wt.wait(lastdone, 0);
      if (__all_sync(0xffffffffu, have)) {
        tc_fence_after();
        // the A ring was last written by copies and read by the tensor core
        // (async proxy); order that before these staging writes
        fence_proxy_async_smem();
        store_columns(last_it, a, orow, kChunks / 2, kChunks,
                      a_ring + (warp & 3) * (32 * kStageRowBytes));
      }
    }
    if (last_dense >= 0) {
      // TMA loads this lane issued that may not have landed: the latest unit
      // of each of the group's NA / NQ slots (earlier ones were consumed)
      for (int d = 0; d < NA / NQ && last_dense - d * NQ >= 0; ++d) {
        const uint32_t t = uint32_t(last_dense - d * NQ);
        mbar_drain(afull0 + 8 * (t % NA), (t / NA) & 1);
      }
    }
    __syncwarp();
  } else if (warp == kMmaWarp || warp == kMmaWarp2) {
    // ---------------- MMA warps ----------------
    // The whole warp runs the loop (waits, bookkeeping, descriptors) and stays
    // converged; one elected lane issues.
    const uint32_t mine = warp == kMmaWarp ? 0u : 1u;  // this warp's tiles: k % 2 == mine
    uint32_t u = 0, s = 0, j = 0, acc_iter = 0;
    int4 rec = first_record();
    bool ok = true;
    const uint64_t adesc0 = desc_a_kmajor(a_base);
    const uint64_t bdesc0 = desc_b_mnmajor(w_base, kBK * 128);
    while (ok) {
      const Item<G> it = next_item(j, rec);
      const uint32_t a = acc_iter % NBUF;
      const uint32_t use = acc_iter / NBUF;  // earlier uses of accumulator set a
      const bool free = wt.wait(tempty0 + 8 * a, (use & 1) ^ 1);
      if (!__all_sync(0xffffffffu, free)) break;
      // tell the epilogue which item this accumulator set will hold (or that
      // there are no more); its previous contents have been stored
      if (mine == 0 && lane == 0) {
        acc_info[a] = it;
        mbar_arrive(info0 + 8 * a);
      }
      __syncwarp();
      if (it.w < 0) break;
      tc_fence_after();
      uint32_t started = 0;  // bit k: tile k's accumulator holds a partial sum
      uint32_t rem = rotate_taps(it.all, it.rot);
      while (rem && ok) {
        const StageTaps st = next_stage_taps<PAIR>(rem, it.rot);
        const uint32_t live = stage_live<G, KS, PAIR>(it, st);
        for (int kb = 0; kb < kb_per_tap; ++kb, ++s) {
          const uint32_t ws = s % NW;
          // Both warps wait for every W slice, even one they do not multiply:
          // a warp commits each stage's release (count 2), and without this
          // wait a warp with no tiles for a run of stages could commit into
          // the next use of a slot before the other warp released this one.
          const bool ready = wt.wait(wfull0 + 8 * ws, (s / NW) & 1);
          if (!__all_sync(0xffffffffu, ready)) {
            ok = false;
            break;
          }
          const uint64_t bd = bdesc0 + uint64_t(ws) * (kWStage >> 4);
          // this warp's unit of the stage (its tile, if the tile has the tap);
          // one copy of the code below serves both tiles
          int k = -1;
          uint32_t my = 0, sl = 0;
#pragma unroll
          for (int t = 0; t < G; ++t) {
            const uint32_t l = sub_live<G, KS, PAIR>(it, t, st);
            if (l == 0u) continue;
            const uint32_t un = u++;
            if ((uint32_t(t) & 1u) == mine) {
              k = t;
              my = un;
              sl = l;
            }
          }
          if (k >= 0) {
            const uint32_t slot = my % NA;
            const bool landed = wt.wait(afull0 + 8 * slot, (my / NA) & 1);
            if (!__all_sync(0xffffffffu, landed)) {
              ok = false;
              break;
            }
            // the rows were written by cp.async (generic proxy) or TMA: order
            // them before the tensor core's (async-proxy) reads
            if (!DENSE) fence_proxy_async_smem();
            tc_fence_after();
            // descriptors: the start-address field (bits 0-13, 16-byte units)
            // never carries, so byte offsets add to the 64-bit value
            const uint64_t ad = adesc0 + uint64_t(slot) * (kAUnitBytes >> 4);
            const uint32_t d_tmem = tmem + (a * G + k) * BN;
            uint32_t acc = (started >> k) & 1u;  // 0 for the tile's first MMA of the item
#pragma unroll
            for (int sub = 0; sub < KS; ++sub) {
              if (PAIR && !((sl >> sub) & 1u)) continue;  // that tap is not the tile's
#pragma unroll
              for (int k16 = 0; k16 < kBK / 16; ++k16) {
                umma_f16(d_tmem, ad + uint64_t(sub) * (kSubBytes >> 4) + 2 * k16,
                         bd + uint64_t(sub) * (kWBytes >> 4) + (2048 >> 4) * k16, kIdesc, acc);
                acc = 1u;
              }
            }
            umma_commit(aempty0 + 8 * slot);
          }
          if (!ok) break;
          umma_commit(wempty0 + 8 * ws);
          started |= live;
        }
      }
      if (!ok) break;
      umma_commit(tfull0 + 8 * a);
      if (item_of(j, total_work) < 0) umma_commit(lastdone);
      ++acc_iter;
    }
    // every MMA this warp issued completes before tensor memory and the
    // operand rings are released (a no-op wait on the normal path)
    umma_commit(drain0 + 8 * mine);
    mbar_drain(drain0 + 8 * mine, 0);
  } else {
    // ---------------- epilogue (warps 2-5) ----------------
    uint32_t acc_iter = 0;
    while (true) {
      const uint32_t a = acc_iter % NBUF;
      const uint32_t use = acc_iter / NBUF;
      bool have = wt.wait(info0 + 8 * a, use & 1);
      if (!__all_sync(0xffffffffu, have)) break;
      const Item<G> it = acc_info[a];
      if (it.w < 0) break;
      int32_t orow[G];
      output_rows(it, orow);
      have = wt.wait(tfull0 + 8 * a, use & 1);
      if (!__all_sync(0xffffffffu, have)) break;  // tcgen05.ld below is warp-collective
      tc_fence_after();
      // the CTA's last item: the second half of the columns is stored by the
      // first four gather warps, which have nothing left to do
      const bool last = item_of(acc_iter + 1, total_work) < 0;
      store_columns(it, a, orow, 0, last ? kChunks / 2 : kChunks,
                    out_stage + (warp & 3) * (32 * kStageRowBytes));
      tc_fence_before();
      mbar_arrive(tempty0 + 8 * a);
      ++acc_iter;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
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

// 2-D row-major [rows][cols] tensor map with a (64 x box_rows) box and the
// 128-byte swizzle (64 half-precision columns are one 128-byte row).
bool encode_2d(CUtensorMap* map, bool bf16, const void* base, uint64_t cols, uint64_t rows,
               uint32_t box_rows) {
  auto encode = get_encode_fn();
  if (!encode) return false;
  cuuint64_t dims[2] = {cuuint64_t(cols), cuuint64_t(rows)};
  cuuint64_t strides[1] = {cuuint64_t(cols) * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return encode(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2,
                const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int BN, int NA, int NW, int G, int WPS, int NQ, bool BF16, int NBUF, int KS,
          bool PAIR, bool EPI, bool DENSE>
int launch_cfg(const Plan& plan, bool dense, const void* feats, const void* W, void* out, int cin,
               int cout, const Epilogue& ep, cudaStream_t stream) {
  constexpr int kSmem = smem_bytes<BN, NA, NW, G, KS, PAIR>();
  static_assert(kSmem <= 227 * 1024, "shared memory");
  static_assert(threads_for(NQ, WPS) <= 1024, "threads");
  static_assert(!(PAIR && DENSE), "tap pairs exist for K = 3 only");
  auto kern = k_conv_tc<BN, NA, NW, G, WPS, NQ, BF16, NBUF, KS, PAIR, EPI, DENSE>;
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
  if (!encode_2d(&wmap, BF16, W, uint64_t(cout), uint64_t(taps) * uint64_t(cin), kBK) ||
      !encode_2d(&fmap, BF16, feats, uint64_t(cin), uint64_t(plan.n), kTileRows))
    return SMC_ERR_CUDA;
  ConvArgs a;
  a.feats = static_cast<const uint16_t*>(feats);
  a.out = static_cast<uint16_t*>(out);
  a.gidx = plan.gidx;
  a.out_row = plan.out_row;
  static_assert(G == 1 || G == 2, "work-item records exist for one and two tiles per item");
  a.items = plan.items[G - 1];
  a.status = plan.status;
  a.n = plan.n;
  a.cin = cin;
  a.cout = cout;
  a.n_tiles = int(plan.n_tiles);
  a.n_blocks = cout / BN;
  a.n_groups = int((plan.n_tiles + G - 1) / G);
  a.dense = dense ? 1 : 0;
  a.wait_ns = wait_limit_ns();
  a.bias = static_cast<const uint16_t*>(ep.bias);
  a.residual = static_cast<const uint16_t*>(ep.residual);
  a.act = ep.act;
  const int64_t work = int64_t(a.n_groups) * a.n_blocks;
  const int grid = int(std::min<int64_t>(work, sm_count()));
  kern<<<grid, threads_for(NQ, WPS), kSmem, stream>>>(wmap, fmap, a);
  return cudaGetLastError() == cudaSuccess ? SMC_OK : SMC_ERR_CUDA;
}

// Tuning override, read once per process: SMC_TC_GROUP=1 or 2 (tiles per work
// item; default: 1 below 6 tiles per SM, else 2).
int group_override() {
  static const int v = [] {
    const char* e = std::getenv("SMC_TC_GROUP");
    return e ? std::atoi(e) : 0;
  }();
  return v;
}

// The launch configurations, by id (see the ConvConfig enumeration in
// smc_internal.h for what each one is).
template <bool BF16>
int launch_config(int cfg, const Plan& plan, bool dense, const void* feats, const void* W,
                  void* out, int cin, int cout, const Epilogue& ep, cudaStream_t stream) {
  // the fused epilogue (bias, activation, residual) is its own instantiation,
  // so the plain convolution carries none of its code
  const bool epi = ep.bias || ep.residual || ep.act != SMC_ACT_NONE;
#define SMC_CFG(...)                                                                     \
  if (dense) return epi ? launch_cfg<__VA_ARGS__, true, true>(plan, dense, feats, W, out, cin, \
                                                              cout, ep, stream)             \
                        : launch_cfg<__VA_ARGS__, false, true>(plan, dense, feats, W, out, cin, \
                                                               cout, ep, stream);           \
  return epi ? launch_cfg<__VA_ARGS__, true, false>(plan, dense, feats, W, out, cin, cout, ep,    \
                                                    stream)                                 \
             : launch_cfg<__VA_ARGS__, false, false>(plan, dense, feats, W, out, cin, cout, ep,   \
                                                     stream)
  // tap pairs (K = 3 only): no K = 1 instantiation
#define SMC_CFG_SPARSE(...)                                                              \
  if (dense) return SMC_ERR_INVALID;                                                     \
  return epi ? launch_cfg<__VA_ARGS__, true, false>(plan, dense, feats, W, out, cin, cout, ep,    \
                                                    stream)                                 \
             : launch_cfg<__VA_ARGS__, false, false>(plan, dense, feats, W, out, cin, cout, ep,   \
                                                     stream)
  switch (cfg) {  //            BN  NA NW G WPS NQ        NBUF KS PAIR
    case kCfg256G2: SMC_CFG(256, 9, 2, 2, 4, 3, BF16, 1, 1, false);
    case kCfg256G1: SMC_CFG(256, 9, 2, 1, 4, 3, BF16, 2, 1, false);
    case kCfg256G1K2: SMC_CFG(256, 2, 2, 1, 4, 2, BF16, 2, 2, false);
    case kCfg128G2K2: SMC_CFG(128, 4, 2, 2, 4, 2, BF16, 2, 2, false);
    case kCfg128G1K2: SMC_CFG(128, 4, 2, 1, 4, 2, BF16, 2, 2, false);
    case kCfg128G1Pair: SMC_CFG_SPARSE(128, 4, 2, 1, 4, 2, BF16, 2, 2, true);
    case kCfg128G2: SMC_CFG(128, 10, 3, 2, 2, 5, BF16, 2, 1, false);
    case kCfg128G1: SMC_CFG(128, 10, 3, 1, 2, 5, BF16, 2, 1, false);
    case kCfg64G1Pair: SMC_CFG_SPARSE(64, 5, 2, 1, 2, 5, BF16, 2, 2, true);
    case kCfg64G2: SMC_CFG(64, 12, 2, 2, 2, 6, BF16, 2, 1, false);
    case kCfg64G1: SMC_CFG(64, 12, 2, 1, 2, 6, BF16, 2, 1, false);
    default: return SMC_ERR_INVALID;
  }
#undef SMC_CFG
#undef SMC_CFG_SPARSE
}

}  // namespace

bool conv_config_valid(int cfg, bool dense, int cin, int cout) {
  if (cin % 64 != 0 || cout % 64 != 0) return false;
  switch (cfg) {
    case kCfg256G2:
    case kCfg256G1:
      return cout % 256 == 0;
    case kCfg256G1K2:
      return cout % 256 == 0 && cin % 128 == 0;
    case kCfg128G2K2:
    case kCfg128G1K2:
      return cout % 128 == 0 && cin % 128 == 0;
    case kCfg128G1Pair:
      return cout % 128 == 0 && cin == 64 && !dense;
    case kCfg128G2:
    case kCfg128G1:
      return cout % 128 == 0;
    case kCfg64G1Pair:
      return cin == 64 && !dense;
    case kCfg64G2:
    case kCfg64G1:
      return true;
    default:
      return false;
  }
}

const char* conv_config_name(int cfg) {
  static const char* const kNames[kConvConfigs] = {
      "bn256-g2",     "bn256-g1",  "bn256-g1-k128", "bn128-g2-k128", "bn128-g1-k128",
      "bn128-g1-pair", "bn128-g2",  "bn128-g1",      "bn64-g1-pair",  "bn64-g2",
      "bn64-g1"};
  return cfg >= 0 && cfg < kConvConfigs ? kNames[cfg] : "cuda-cores";
}

int conv_default_config(const Plan& plan, bool dense, int cin, int cout) {
  // Test and tuning override, read at every call: SMC_TC_CONFIG=<id> forces
  // a configuration wherever it is valid.
  if (const char* e = std::getenv("SMC_TC_CONFIG")) {
    const int c = std::atoi(e);
    if (conv_config_valid(c, dense, cin, cout)) return c;
  }
  // Few tiles per SM: one tile per work item, so every SM gets work and no SM
  // runs two heavy tiles back to back.
  const bool small = plan.n_tiles < int64_t(6) * sm_count();
  const bool g1 = group_override() == 1 || (small && group_override() != 2);
  if (cout % 256 == 0) {
    // sparse: two 256-column tiles per item share each W slice (one
    // accumulator set), as long as that leaves at least two items per SM;
    // dense (K = 1) items are short, so they keep the overlapped epilogue
    const int64_t items2 = (plan.n_tiles + 1) / 2 * (cout / 256);
    if (group_override() == 2 ||
        (group_override() == 0 && !dense && items2 >= 2 * int64_t(sm_count())))
      return kCfg256G2;
    // K = 1: 128-channel units (half the hand-offs per multiply)
    if (dense && cin % 128 == 0) return kCfg256G1K2;
    return kCfg256G1;
  }
  if (cout % 128 == 0) {
    // 128 input channels per unit where Cin allows: half the hand-offs per
    // multiply of the 64-channel unit
    if (cin % 128 == 0) return g1 ? kCfg128G1K2 : kCfg128G2K2;
    // 64 input channels and few tiles per SM (a short chain of units per
    // SM, bound by hand-off latency): two taps per 128-channel unit.  With
    // many tiles the 64-channel units keep more rows in flight and win.
    if (cin == 64 && !dense && g1) return kCfg128G1Pair;
    return g1 ? kCfg128G1 : kCfg128G2;
  }
  if (cin == 64 && !dense && g1) return kCfg64G1Pair;
  return g1 ? kCfg64G1 : kCfg64G2;
}

// A test sets SMC_DEBUG_WAIT_LIMIT_NS tiny to exercise the abort path.
uint64_t wait_limit_ns() {
  static const uint64_t v = [] {
    const char* e = std::getenv("SMC_DEBUG_WAIT_LIMIT_NS");
    const long long x = e ? std::atoll(e) : 0;
    return x > 0 ? uint64_t(x) : uint64_t(2000000000ull);
  }();
  return v;
}

bool conv_tc_supported(int cin, int cout, int dtype) {
  return (dtype == SMC_F16 || dtype == SMC_BF16) && cin > 0 && cout > 0 && cin % 64 == 0 &&
         cout % 64 == 0;
}

int launch_conv_tc(const Plan& plan, bool dense, const void* feats, const void* W, void* out,
                   int cin, int cout, int dtype, const Epilogue& ep, cudaStream_t stream,
                   int cfg) {
  if (plan.n == 0) return SMC_OK;
  if (!conv_tc_supported(cin, cout, dtype)) return SMC_ERR_UNSUPPORTED;
  if (cfg < 0) cfg = conv_default_config(plan, dense, cin, cout);
  if (!conv_config_valid(cfg, dense, cin, cout)) return SMC_ERR_INVALID;
  if (dtype == SMC_BF16)
    return launch_config<true>(cfg, plan, dense, feats, W, out, cin, cout, ep, stream);
  return launch_config<false>(cfg, plan, dense, feats, W, out, cin, cout, ep, stream);
}

}  // namespace smc
