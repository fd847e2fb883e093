// Index build: coordinate hash, neighbour map, row ordering and tile plan.
//
// This is the "prepared device gather index" of the trellis_sparse_mlx README
// ("Performance": caching the prepared index, not only the raw indice map,
// is what made the layer compute-bound), built once per coordinate set:
//
//   1. insert   every voxel's packed key (b:15 | x:16 | y:16 | z:16 bits) into
//               an open-addressing table (linear probing, Fibonacci hashing);
//   2. query    the 27 neighbours c + stride*d of every voxel (one warp per
//               voxel, one lane per tap) -> int32 map [n][27] (-1 = absent)
//               and a 27-bit tap mask per voxel;
//   3. order    rows by (popcount(mask), Gray-code rank of mask) with a stable
//               LSD radix sort, so a 128-row tile holds voxels whose active
//               taps coincide;
//   4. plan     per tile, the OR of its rows' masks (the taps the tensor-core
//               kernel multiplies; the others are skipped) and a compact
//               gather index [tile][active tap][128 rows];
//   5. items    for work items of one and of two consecutive tiles, the
//               groups in decreasing order of their union's tap count (one
//               block-wide stable counting sort, or a radix pass for more
//               than 49,152 tiles), so the convolution deals its largest
//               items first, each written as a 16-byte record (first tile,
//               tap masks, first gather-index slot) that each role of the
//               convolution reads with one load.
#include <algorithm>
#include <cstdio>
#include <cstring>

#include "smc_internal.h"

namespace smc {
namespace {

constexpr uint64_t kEmptyKey = ~0ull;

// One open-addressing slot: the packed key and the row it maps to, 16 bytes,
// so a probe is a single load.  An empty slot holds kEmptyKey.
struct __align__(16) Slot {
  unsigned long long key;
  int32_t val;
  int32_t pad;
};

// Fibonacci (multiplicative) hashing, Knuth, The Art of Computer Programming
// vol. 3, section 6.4: a table of 2^b slots takes the top b bits of
// key * 2^64 / phi.  The hash is linear in the key, and a neighbour's packed
// key is the voxel's key plus a per-offset constant (when every coordinate
// stays in range), so the query computes one product per voxel and adds a
// per-offset product for each of the 27 taps.
constexpr uint64_t kFib = 0x9E3779B97F4A7C15ull;
__device__ __forceinline__ uint64_t hash_slot(uint64_t prod, int shift) {
  return shift >= 64 ? 0ull : prod >> shift;  // shift = 64 - b (a one-slot table has b = 0)
}

__device__ __forceinline__ uint64_t pack_key(int64_t b, int64_t x, int64_t y, int64_t z) {
  return (uint64_t(b) << 48) | (uint64_t(x) << 32) | (uint64_t(y) << 16) | uint64_t(z);
}

__device__ __forceinline__ bool axis_ok(int64_t v) { return v >= 0 && v < kMaxAxis; }

__global__ void k_insert(const int4* __restrict__ coords, int64_t n, Slot* table,
                         uint64_t cap_mask, int shift, int32_t* status) {
  const int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x;
  if (i >= n) return;
  const int4 c = coords[i];
  if (c.x < 0 || c.x >= kMaxBatch || !axis_ok(c.y) || !axis_ok(c.z) || !axis_ok(c.w)) {
    atomicOr(status, kDevRange);
    return;
  }
  const uint64_t key = pack_key(c.x, c.y, c.z, c.w);
  uint64_t slot = hash_slot(key * kFib, shift);
  for (uint64_t probe = 0; probe <= cap_mask; ++probe) {
    const unsigned long long prev =
        atomicCAS(&table[slot].key, (unsigned long long)kEmptyKey, (unsigned long long)key);
    if (prev == kEmptyKey) {
      table[slot].val = int32_t(i);
      return;
    }
    if (prev == key) {
      atomicOr(status, kDevDuplicate);
      return;
    }
    slot = (slot + 1) & cap_mask;
  }
  atomicOr(status, kDevTableFull);
}

// One warp per voxel, lane k < 27 looks up tap k: the map row is written by
// consecutive lanes and the tap mask is the warp's ballot.
constexpr int kNbrWarps = 8;

__global__ void __launch_bounds__(kNbrWarps * 32)
k_neighbors(const int4* __restrict__ coords, int64_t n, int32_t stride,
            const Slot* __restrict__ table, uint64_t cap_mask, int shift,
            int32_t* __restrict__ nbr, uint32_t* __restrict__ mask) {
  const int lane = threadIdx.x & 31;
  const int64_t i = blockIdx.x * int64_t(kNbrWarps) + (threadIdx.x >> 5);
  if (i >= n) return;  // warp-uniform
  const int k = lane < kTaps ? lane : 0;
  const int64_t sx = int64_t(stride) * (k / 9 - 1);
  const int64_t sy = int64_t(stride) * ((k / 3) % 3 - 1);
  const int64_t sz = int64_t(stride) * (k % 3 - 1);
  // the tap's key offset (sx, sy, sz in the x, y, z fields), two's complement
  const uint64_t dprod = uint64_t(sx * 4294967296ll + sy * 65536ll + sz) * kFib;
  const int4 c = coords[i];
  int32_t found = -1;
  if (lane < kTaps) {
    const int64_t x = int64_t(c.y) + sx, y = int64_t(c.z) + sy, z = int64_t(c.w) + sz;
    if (axis_ok(x) && axis_ok(y) && axis_ok(z)) {
      const uint64_t key = pack_key(c.x, x, y, z);
      uint64_t slot = hash_slot(pack_key(c.x, c.y, c.z, c.w) * kFib + dprod, shift);
      for (uint64_t probe = 0; probe <= cap_mask; ++probe) {
        const Slot e = table[slot];
        if (e.key == key) {
          found = e.val;
          break;
        }
        if (e.key == kEmptyKey) break;
        slot = (slot + 1) & cap_mask;
      }
    }
    nbr[i * kTaps + lane] = found;
  }
  const uint32_t m = __ballot_sync(0xffffffffu, found >= 0) & ((1u << kTaps) - 1u);
  if (lane == 0) mask[i] = m;
}

// ---------------------------------------------------------------------------
// Sort-based lookup (the alternative to the hash): coordinates packed
// injectively into one 64-bit key, the (key, row) pairs radix-sorted, and
// every neighbour found by binary search over the sorted keys -- the
// pack-into-int64 + sort + searchsorted vectorisation of "Running TRELLIS.2 on
// a Mac (3/3)", section "E. Vectorizing mesh extraction".
// ---------------------------------------------------------------------------
__global__ void k_pack_keys(const int4* __restrict__ coords, int64_t n,
                            unsigned long long* __restrict__ keys, int32_t* __restrict__ vals,
                            int32_t* status) {
  const int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x;
  if (i >= n) return;
  const int4 c = coords[i];
  if (c.x < 0 || c.x >= kMaxBatch || !axis_ok(c.y) || !axis_ok(c.z) || !axis_ok(c.w)) {
    atomicOr(status, kDevRange);
    keys[i] = ~0ull - uint64_t(i);  // unique, above every valid key: matches nothing
  } else {
    keys[i] = pack_key(c.x, c.y, c.z, c.w);
  }
  vals[i] = int32_t(i);
}

__global__ void k_sorted_dups(const unsigned long long* __restrict__ keys, int64_t n,
                              int32_t* status) {
  const int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x;
  if (i >= 1 && i < n && keys[i] == keys[i - 1]) atomicOr(status, kDevDuplicate);
}

__global__ void __launch_bounds__(kNbrWarps * 32)
k_neighbors_sorted(const int4* __restrict__ coords, int64_t n, int32_t stride,
                   const unsigned long long* __restrict__ skeys, const int32_t* __restrict__ svals,
                   int32_t* __restrict__ nbr, uint32_t* __restrict__ mask) {
  const int lane = threadIdx.x & 31;
  const int64_t i = blockIdx.x * int64_t(kNbrWarps) + (threadIdx.x >> 5);
  if (i >= n) return;  // warp-uniform
  const int k = lane < kTaps ? lane : 0;
  const int4 c = coords[i];
  int32_t found = -1;
  if (lane < kTaps) {
    const int64_t x = int64_t(c.y) + int64_t(stride) * (k / 9 - 1);
    const int64_t y = int64_t(c.z) + int64_t(stride) * ((k / 3) % 3 - 1);
    const int64_t z = int64_t(c.w) + int64_t(stride) * (k % 3 - 1);
    if (axis_ok(x) && axis_ok(y) && axis_ok(z)) {
      const unsigned long long key = pack_key(c.x, x, y, z);
      int64_t lo = 0, hi = n;  // first position with skeys[pos] >= key
      while (lo < hi) {
        const int64_t mid = (lo + hi) >> 1;
        if (skeys[mid] < key)
          lo = mid + 1;
        else
          hi = mid;
      }
      if (lo < n && skeys[lo] == key) found = svals[lo];
    }
    nbr[i * kTaps + lane] = found;
  }
  const uint32_t m = __ballot_sync(0xffffffffu, found >= 0) & ((1u << kTaps) - 1u);
  if (lane == 0) mask[i] = m;
}

// ---------------------------------------------------------------------------
// Greedy tile packing (SMC_ORDER_GREEDY).  The mask-sorted rows are cut into
// segments of kGreedySeg rows, one CTA each.  Inside a segment, equal masks
// are contiguous; each tile starts from the first mask with rows left, then
// alternates (a) taking, in order, every mask whose taps are already in the
// tile's union, and (b) taking the one mask that adds the fewest new taps
// (most rows on ties), until 128 rows.  The tensor-core kernel multiplies
// 128 rows per tap of a tile's union, so fewer union taps is less work.
// Output: a plan-row permutation with the same tile layout as the sort.
// ---------------------------------------------------------------------------
constexpr int kGreedySeg = 1024;    // rows per segment (a multiple of 128)
constexpr int kGreedyThreads = 256;
constexpr int kGreedyPer = kGreedySeg / kGreedyThreads;  // distinct masks per thread, at most

// Block-wide exclusive scan of one value per thread (kGreedyThreads threads);
// returns the prefix, *total gets the sum.
__device__ __forceinline__ int block_scan(int v, int* total, int* wsum) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = lane < kGreedyThreads / 32 ? wsum[lane] : 0;
    int wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += t;
    }
    if (lane < kGreedyThreads / 32) wsum[lane] = wi - w;  // exclusive warp offsets
    if (lane == kGreedyThreads / 32 - 1) wsum[32] = wi;
  }
  __syncthreads();
  const int r = wsum[warp] + incl - v;
  *total = wsum[32];
  __syncthreads();
  return r;
}

// Block-wide minimum of a 64-bit key (kGreedyThreads threads).
__device__ __forceinline__ unsigned long long block_min(unsigned long long v,
                                                       unsigned long long* wmin) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = min(v, __shfl_xor_sync(0xffffffffu, v, o));
  if (lane == 0) wmin[warp] = v;
  __syncthreads();
  if (warp == 0) {
    unsigned long long w = lane < kGreedyThreads / 32 ? wmin[lane] : ~0ull;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) w = min(w, __shfl_xor_sync(0xffffffffu, w, o));
    if (lane == 0) wmin[32] = w;
  }
  __syncthreads();
  const unsigned long long r = wmin[32];
  __syncthreads();
  return r;
}

__global__ void __launch_bounds__(kGreedyThreads)
k_greedy_tiles(const int32_t* __restrict__ sorted_rows, const uint32_t* __restrict__ mask,
               int64_t n, int32_t* __restrict__ perm) {
  extern __shared__ uint32_t gsm[];
  uint32_t* u = gsm;                                          // distinct masks, in order
  int32_t* rows = reinterpret_cast<int32_t*>(u + kGreedySeg);    // the segment's sorted rows
  uint16_t* live = reinterpret_cast<uint16_t*>(rows + kGreedySeg);  // rows left per mask
  uint16_t* next = live + kGreedySeg;                         // next row to take (segment offset)
  __shared__ int wsum[33];
  __shared__ unsigned long long wmin[33];
  const int64_t base = int64_t(blockIdx.x) * kGreedySeg;
  const int len = int(n - base < int64_t(kGreedySeg) ? n - base : int64_t(kGreedySeg));
  const int t0 = threadIdx.x * kGreedyPer;  // this thread's rows, then its distinct masks

  for (int i = threadIdx.x; i < len; i += kGreedyThreads) rows[i] = sorted_rows[base + i];
  __syncthreads();
  // run-length encode the segment's masks: distinct index of each head row
  int heads = 0;
  uint32_t prev = t0 > 0 && t0 < len ? mask[rows[t0 - 1]] : 0u;
  for (int i = t0; i < t0 + kGreedyPer && i < len; ++i) {
    const uint32_t m = mask[rows[i]];
    heads += (i == 0 || m != prev) ? 1 : 0;
    prev = m;
  }
  int d = 0;
  int q = block_scan(heads, &d, wsum);
  prev = t0 > 0 && t0 < len ? mask[rows[t0 - 1]] : 0u;
  for (int i = t0; i < t0 + kGreedyPer && i < len; ++i) {
    const uint32_t m = mask[rows[i]];
    if (i == 0 || m != prev) {
      u[q] = m;
      next[q] = uint16_t(i);
      ++q;
    }
    prev = m;
  }
  __syncthreads();
  for (int k = t0; k < t0 + kGreedyPer; ++k)
    if (k < d) live[k] = uint16_t((k + 1 < d ? int(next[k + 1]) : len) - int(next[k]));
  __syncthreads();

  // take `t` rows of distinct mask k into plan rows out, out + 1, ...
  auto take = [&](int k, int t, int64_t out) {
    const int r0 = next[k];
    for (int j = 0; j < t; ++j) perm[out + j] = rows[r0 + j];
  };

  int64_t out = base;
  const int64_t end = base + len;
  while (out < end) {
    // a new tile from the first mask with rows left
    unsigned long long key = ~0ull;
    for (int k = t0; k < t0 + kGreedyPer && k < d; ++k)
      if (live[k] > 0) {
        key = k;
        break;
      }
    key = block_min(key, wmin);
    uint32_t U = u[key];
    int fill = 0;
    bool pick_next = false;  // the first mask is taken by the subset pass below
    while (fill < kTileRows) {
      if (pick_next) {
        // the mask adding the fewest taps to U, most rows on ties, first index
        unsigned long long best = ~0ull;
        for (int k = t0; k < t0 + kGreedyPer && k < d; ++k) {
          if (live[k] == 0) continue;
          const unsigned add = __popc(u[k] & ~U);
          const unsigned rows = min(int(live[k]), kTileRows - fill);
          const unsigned long long kk =
              (uint64_t(add) << 40) | (uint64_t(kTileRows - rows) << 24) | uint64_t(k);
          best = min(best, kk);
        }
        best = block_min(best, wmin);
        if (best == ~0ull) break;  // the segment is used up
        const int k = int(best & 0xFFFFFF);
        U |= u[k];
      }
      pick_next = true;
      // every mask inside U, in order, until the tile is full
      int mine = 0;
      for (int k = t0; k < t0 + kGreedyPer && k < d; ++k)
        if (live[k] > 0 && (u[k] & ~U) == 0u) mine += live[k];
      int total = 0;
      int pre = block_scan(mine, &total, wsum);
      for (int k = t0; k < t0 + kGreedyPer && k < d; ++k) {
        if (live[k] == 0 || (u[k] & ~U) != 0u) continue;
        const int t = max(0, min(int(live[k]), kTileRows - fill - pre));
        if (t > 0) {
          take(k, t, out + fill + pre);
          next[k] = uint16_t(next[k] + t);
          live[k] = uint16_t(live[k] - t);
        }
        pre += live[k] + t;  // this mask's rows before the take, for the next mask
      }
      fill = min(kTileRows, fill + total);
      __syncthreads();
      if (fill >= kTileRows || out + fill >= end) break;
    }
    out += fill;
  }
}

// Sort key: popcount in the top 5 bits (so tiles come out lightest to
// heaviest), then the rank of the 27-bit mask in reflected Gray-code order
// (the prefix XOR of the mask): consecutive masks in that order differ in one
// tap, so a 128-row run covers fewer distinct taps than in plain binary order.
__global__ void k_sort_keys(const uint32_t* __restrict__ mask, int64_t n, uint32_t* keys,
                            int32_t* vals) {
  const int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x;
  if (i >= n) return;
  const uint32_t m = mask[i];
  uint32_t r = m;
  r ^= r >> 1;
  r ^= r >> 2;
  r ^= r >> 4;
  r ^= r >> 8;
  r ^= r >> 16;
  keys[i] = (uint32_t(__popc(m)) << 27) | r;
  vals[i] = int32_t(i);
}

__global__ void k_iota(int32_t* out, int64_t n) {
  const int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x;
  if (i < n) out[i] = int32_t(i);
}

// One block of 128 threads per tile: OR of the rows' masks, its tap count,
// and the two plan counters (useful pairs, issued rows x taps).
__global__ void __launch_bounds__(kTileRows)
k_tile_mask(const int32_t* __restrict__ perm, const uint32_t* __restrict__ mask, int64_t n,
            uint32_t* __restrict__ tile_mask, uint32_t* __restrict__ tile_ntaps,
            unsigned long long* stats) {
  __shared__ uint32_t s_or[kTileRows / 32], s_pop[kTileRows / 32];
  const int64_t p = blockIdx.x * int64_t(kTileRows) + threadIdx.x;
  const uint32_t m = p < n ? mask[perm[p]] : 0u;
  const uint32_t wor = __reduce_or_sync(0xffffffffu, m);
  const uint32_t wpop = __reduce_add_sync(0xffffffffu, uint32_t(__popc(m)));
  if ((threadIdx.x & 31) == 0) {
    s_or[threadIdx.x >> 5] = wor;
    s_pop[threadIdx.x >> 5] = wpop;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t o = 0, pop = 0;
    for (int w = 0; w < kTileRows / 32; ++w) {
      o |= s_or[w];
      pop += s_pop[w];
    }
    tile_mask[blockIdx.x] = o;
    tile_ntaps[blockIdx.x] = __popc(o);
    atomicAdd(&stats[0], (unsigned long long)pop);
    atomicAdd(&stats[1], (unsigned long long)__popc(o) * kTileRows);
  }
}

// One block of 128 threads per tile: for each active tap of the tile, the
// voxel each plan row gathers (or -1), and the voxel each row writes.
__global__ void __launch_bounds__(kTileRows)
k_tile_gather(const int32_t* __restrict__ perm, const int32_t* __restrict__ nbr, int64_t n,
              const uint32_t* __restrict__ tile_mask, const int32_t* __restrict__ tile_off,
              int32_t* __restrict__ gidx, int32_t* __restrict__ out_row) {
  const int64_t tile = blockIdx.x;
  const int64_t p = tile * kTileRows + threadIdx.x;
  const int32_t v = p < n ? perm[p] : -1;
  out_row[p] = v;
  uint32_t m = tile_mask[tile];
  const int64_t off = tile_off[tile];
  int s = 0;
  while (m) {
    const int t = __ffs(m) - 1;
    m &= m - 1;
    gidx[(off + s) * kTileRows + threadIdx.x] = v >= 0 ? nbr[int64_t(v) * kTaps + t] : -1;
    ++s;
  }
}

// Sort keys of the work-item groups: group g covers tiles g*G .. g*G+G-1; its
// key is 27 minus the tap count of their union, listed from the last group to
// the first, so a stable ascending sort yields most taps first and, among
// equal tap counts, the later (heavier-masked) groups first.
__global__ void k_group_keys(const uint32_t* __restrict__ tile_mask, int64_t n_tiles, int G,
                             int64_t n_groups, uint32_t* __restrict__ keys,
                             int32_t* __restrict__ vals) {
  const int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x;
  if (i >= n_groups) return;
  const int64_t g = n_groups - 1 - i;
  uint32_t u = 0;
  for (int k = 0; k < G; ++k) {
    const int64_t t = g * G + k;
    if (t < n_tiles) u |= tile_mask[t];
  }
  keys[i] = uint32_t(kTaps - __popc(u));
  vals[i] = int32_t(g);
}

// Work items of G = blockIdx.x + 1 tiles in one block: the same order as
// k_group_keys + a stable sort + k_item_records (most union taps first; among
// equal counts the later group first), as a stable counting sort over the 28
// possible keys, each key a block-wide scan of per-thread counts.  The keys
// are cached in shared memory (one byte per group, up to kItemSortMax tiles).
constexpr int kItemSortMax = 49152;  // within the default 48 KB of dynamic shared memory

__global__ void __launch_bounds__(1024)
k_item_order(const uint32_t* __restrict__ tile_mask, const int32_t* __restrict__ tile_off,
             int64_t n_tiles, int4* __restrict__ items1, int4* __restrict__ items2) {
  extern __shared__ uint8_t key_of[];  // [ng]: 27 - tap count, in listing order i
  __shared__ int wsum[33];
  const int G = blockIdx.x + 1;
  int4* items = G == 1 ? items1 : items2;
  const int ng = int((n_tiles + G - 1) / G);
  const int per = (ng + 1023) / 1024;
  const int i0 = threadIdx.x * per, i1 = min(ng, i0 + per);
  for (int i = i0; i < i1; ++i) {
    const int64_t g = ng - 1 - i;  // listed from the last group to the first
    uint32_t u = tile_mask[g * G];
    if (G == 2 && g * G + 1 < n_tiles) u |= tile_mask[g * G + 1];
    key_of[i] = uint8_t(kTaps - __popc(u));
  }
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int base = 0;
  for (int v = 0; v <= kTaps; ++v) {
    int c = 0;
    for (int i = i0; i < i1; ++i) c += key_of[i] == v ? 1 : 0;
    // block-wide exclusive scan of c
    int incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      const int w = wsum[lane];
      int wi = w;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, wi, o);
        if (lane >= o) wi += t;
      }
      wsum[lane] = wi - w;
      if (lane == 31) wsum[32] = wi;
    }
    __syncthreads();
    int pos = base + wsum[warp] + incl - c;
    const int total = wsum[32];
    for (int i = i0; i < i1; ++i) {
      if (key_of[i] != v) continue;
      const int64_t t = int64_t(ng - 1 - i) * G;
      int4 r;
      r.x = int(t);
      r.y = int(tile_mask[t]);
      r.z = (G == 2 && t + 1 < n_tiles) ? int(tile_mask[t + 1]) : 0;
      r.w = tile_off[t];
      items[pos++] = r;
    }
    base += total;
    __syncthreads();
  }
}

// Tap-major tile lists (see Plan::tap_tiles), one block per tap.
__global__ void __launch_bounds__(1024)
k_tap_count(const uint32_t* __restrict__ tile_mask, int64_t n_tiles, int32_t* __restrict__ count) {
  __shared__ int32_t part[32];
  const int k = blockIdx.x;
  int32_t c = 0;
  for (int64_t t = threadIdx.x; t < n_tiles; t += blockDim.x) c += (tile_mask[t] >> k) & 1u;
  c = __reduce_add_sync(0xffffffffu, c);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = c;
  __syncthreads();
  if (threadIdx.x < 32) {
    int32_t v = threadIdx.x < blockDim.x / 32 ? part[threadIdx.x] : 0;
    v = __reduce_add_sync(0xffffffffu, v);
    if (threadIdx.x == 0) count[k] = v;
  }
}

__global__ void k_tap_scan(const int32_t* __restrict__ count, int32_t* __restrict__ tap_start,
                           int32_t* __restrict__ tap_chunk, int chunk) {
  if (threadIdx.x != 0) return;
  int32_t s = 0, c = 0;
  for (int k = 0; k < kTaps; ++k) {
    tap_start[k] = s;
    tap_chunk[k] = c;
    s += count[k];
    c += (count[k] + chunk - 1) / chunk;
  }
  tap_start[kTaps] = s;
  tap_chunk[kTaps] = c;
}

__global__ void __launch_bounds__(1024)
k_tap_fill(const uint32_t* __restrict__ tile_mask, const int32_t* __restrict__ tile_off,
           int64_t n_tiles, const int32_t* __restrict__ tap_start, int2* __restrict__ tap_tiles) {
  __shared__ int32_t wsum[32];
  __shared__ int32_t base;
  const int k = blockIdx.x;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) base = tap_start[k];
  __syncthreads();
  for (int64_t t0 = 0; t0 < n_tiles; t0 += blockDim.x) {
    const int64_t t = t0 + threadIdx.x;
    const uint32_t m = t < n_tiles ? tile_mask[t] : 0u;
    const int has = (m >> k) & 1u;
    const uint32_t ballot = __ballot_sync(0xffffffffu, has);
    if (lane == 0) wsum[warp] = __popc(ballot);
    __syncthreads();
    int32_t before = 0, total = 0;
    for (int w = 0; w < int(blockDim.x / 32); ++w) {
      before += w < warp ? wsum[w] : 0;
      total += wsum[w];
    }
    if (has) {
      const int32_t pos = base + before + __popc(ballot & ((1u << lane) - 1u));
      tap_tiles[pos] = make_int2(int(t), tile_off[t] + __popc(m & ((1u << k) - 1u)));
    }
    __syncthreads();
    if (threadIdx.x == 0) base += total;
    __syncthreads();
  }
}

// Work-item records in the sorted group order (see Plan::items).
__global__ void k_item_records(const int32_t* __restrict__ order, int64_t n_groups, int G,
                               const uint32_t* __restrict__ tile_mask,
                               const int32_t* __restrict__ tile_off, int64_t n_tiles,
                               int4* __restrict__ items) {
  const int64_t q = blockIdx.x * int64_t(blockDim.x) + threadIdx.x;
  if (q >= n_groups) return;
  const int64_t t = int64_t(order[q]) * G;
  int4 r;
  r.x = int(t);
  r.y = int(tile_mask[t]);
  r.z = (G == 2 && t + 1 < n_tiles) ? int(tile_mask[t + 1]) : 0;
  r.w = tile_off[t];
  items[q] = r;
}

inline int log2_pow2(uint64_t v) {  // v a power of two
  int b = 0;
  while ((uint64_t(1) << b) < v) ++b;
  return b;
}

inline unsigned grid_for(int64_t n, int threads) {
  return unsigned((n + threads - 1) / threads);
}

int status_from_device(int32_t dev) {
  if (dev & kDevDuplicate) return SMC_ERR_DUPLICATE;
  if (dev & kDevRange) return SMC_ERR_RANGE;
  if (dev & kDevTableFull) return SMC_ERR_TABLE_FULL;
  if (dev & kDevTimeout) return SMC_ERR_TIMEOUT;
  return SMC_OK;
}

// Carves one allocation into 256-byte-aligned arrays.  A first pass with a
// null base only measures.
struct Carve {
  uint8_t* base = nullptr;
  size_t off = 0;
  template <class T>
  T* take(size_t count) {
    off = (off + 255) & ~size_t(255);
    T* p = reinterpret_cast<T*>(base + off);
    off += (count ? count : 1) * sizeof(T);
    return p;
  }
};

// Device counters written by the build and read back once at its end.
struct BuildCounters {
  int32_t status;
  int32_t total_slots;          // copy of tile_off[n_tiles], for the one read-back
  unsigned long long stats[2];  // useful pairs, issued rows x taps
};

// The plan's arrays in one arena (sizes are upper bounds where they depend on
// the tile masks, so nothing has to be read back before the end).
void carve_plan(Carve& c, Plan* p, BuildCounters** ctr) {
  const int64_t n = p->n, nt = p->n_tiles;
  *ctr = c.take<BuildCounters>(1);
  p->nbr = c.take<int32_t>(size_t(n) * kTaps);
  p->mask = c.take<uint32_t>(size_t(n));
  p->perm = c.take<int32_t>(size_t(n));
  p->tile_mask = c.take<uint32_t>(size_t(nt));
  p->tile_off = c.take<int32_t>(size_t(nt) + 1);
  p->gidx = c.take<int32_t>(size_t(nt) * kTaps * kTileRows);
  p->out_row = c.take<int32_t>(size_t(nt) * kTileRows);
  p->items[0] = c.take<int4>(size_t(nt));
  p->items[1] = c.take<int4>(size_t((nt + 1) / 2));
  p->tap_tiles = c.take<int2>(size_t(nt) * kTaps);
  p->tap_start = c.take<int32_t>(kTaps + 1);
  p->tap_chunk = c.take<int32_t>(kTaps + 1);
}

struct Scratch {
  Slot* table = nullptr;
  unsigned long long* ckeys[2] = {nullptr, nullptr};  // packed coordinates (sort lookup)
  uint32_t* skeys[2] = {nullptr, nullptr};
  int32_t* svals[2] = {nullptr, nullptr};
  uint32_t* hist = nullptr;
  int32_t* tap_count = nullptr;
  uint32_t* gkeys[2] = {nullptr, nullptr};
  int32_t* gvals = nullptr;
  int32_t* gorder = nullptr;
};

void carve_scratch(Carve& c, Scratch* sc, int64_t n, int64_t nt, uint64_t cap, bool sorted) {
  sc->table = c.take<Slot>(sorted ? 0 : size_t(cap));
  for (int i = 0; i < 2; ++i) sc->ckeys[i] = c.take<unsigned long long>(sorted ? size_t(n) : 0);
  for (int i = 0; i < 2; ++i) {
    sc->skeys[i] = c.take<uint32_t>(size_t(n));
    sc->svals[i] = c.take<int32_t>(size_t(n));
    sc->gkeys[i] = c.take<uint32_t>(size_t(nt));
  }
  sc->hist = c.take<uint32_t>(sort_hist_words(n));
  sc->tap_count = c.take<int32_t>(kTaps);
  sc->gvals = c.take<int32_t>(size_t(nt));
  sc->gorder = c.take<int32_t>(size_t(nt));
}

#define SMC_TRY(expr)             \
  do {                            \
    int rc_ = (expr);             \
    if (rc_ != SMC_OK) return rc_; \
  } while (0)

#define SMC_LAUNCHED()                                     \
  do {                                                     \
    if (cudaGetLastError() != cudaSuccess) return SMC_ERR_CUDA; \
  } while (0)

uint64_t table_slots(int64_t n, int64_t table_capacity) {
  uint64_t cap = 64;
  if (table_capacity > 0) {
    cap = 1;
    while (cap < uint64_t(table_capacity)) cap <<= 1;
    if (cap > uint64_t(table_capacity)) cap >>= 1;  // largest power of two <= request
    if (cap == 0) cap = 1;
  } else {
    while (cap < uint64_t(2 * n)) cap <<= 1;
  }
  return cap;
}

// Steps 3-5 of the build (row order, tile plan, work items) and the one
// read-back, from the neighbour map and masks already in the plan's arena;
// the build's counters must be zero.
int order_and_tile(Plan* plan, BuildCounters* ctr, const Scratch& sc, int32_t order,
                   cudaStream_t s) {
  const int64_t n = plan->n, nt = plan->n_tiles;
  // 3. row order
  if (order == SMC_ORDER_MASK) {
    // four 8-bit passes end where they started: sort straight into perm
    int32_t* vals[2] = {plan->perm, sc.svals[1]};
    k_sort_keys<<<grid_for(n, 256), 256, 0, s>>>(plan->mask, n, sc.skeys[0], vals[0]);
    SMC_LAUNCHED();
    int cur = 0;
    SMC_TRY(radix_sort(sc.skeys, vals, 0, n, 32, sc.hist, s, &cur));
    if (cur != 0 && cudaMemcpyAsync(plan->perm, vals[cur], size_t(n) * sizeof(int32_t),
                                    cudaMemcpyDeviceToDevice, s) != cudaSuccess)
      return SMC_ERR_CUDA;
  } else if (order == SMC_ORDER_GREEDY) {
    k_sort_keys<<<grid_for(n, 256), 256, 0, s>>>(plan->mask, n, sc.skeys[0], sc.svals[0]);
    SMC_LAUNCHED();
    int cur = 0;
    SMC_TRY(radix_sort(sc.skeys, sc.svals, 0, n, 32, sc.hist, s, &cur));
    constexpr int kSmem = kGreedySeg * (4 + 4 + 2 + 2);
    // the shared-memory limit is a per-device function attribute
    constexpr int kMaxDev = 64;
    static bool attr_set[kMaxDev] = {};
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return SMC_ERR_CUDA;
    if (!(dev >= 0 && dev < kMaxDev && attr_set[dev])) {
      if (cudaFuncSetAttribute(k_greedy_tiles, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               kSmem) != cudaSuccess)
        return SMC_ERR_CUDA;
      if (dev >= 0 && dev < kMaxDev) attr_set[dev] = true;
    }
    k_greedy_tiles<<<grid_for(n, kGreedySeg), kGreedyThreads, kSmem, s>>>(sc.svals[cur],
                                                                          plan->mask, n, plan->perm);
    SMC_LAUNCHED();
  } else {
    k_iota<<<grid_for(n, 256), 256, 0, s>>>(plan->perm, n);
    SMC_LAUNCHED();
  }

  // 4. tile plan: masks and tap counts, slot offsets, gather index
  k_tile_mask<<<unsigned(nt), kTileRows, 0, s>>>(plan->perm, plan->mask, n, plan->tile_mask,
                                                  reinterpret_cast<uint32_t*>(plan->tile_off),
                                                  ctr->stats);
  if (cudaMemsetAsync(plan->tile_off + nt, 0, sizeof(int32_t), s) != cudaSuccess)
    return SMC_ERR_CUDA;
  SMC_TRY(scan_exclusive(reinterpret_cast<uint32_t*>(plan->tile_off), nt + 1, s));
  k_tile_gather<<<unsigned(nt), kTileRows, 0, s>>>(plan->perm, plan->nbr, n, plan->tile_mask,
                                                    plan->tile_off, plan->gidx, plan->out_row);
  SMC_LAUNCHED();

  // tap-major tile lists for the weight gradient
  k_tap_count<<<kTaps, 1024, 0, s>>>(plan->tile_mask, nt, sc.tap_count);
  k_tap_scan<<<1, 32, 0, s>>>(sc.tap_count, plan->tap_start, plan->tap_chunk, kBwdChunk);
  k_tap_fill<<<kTaps, 1024, 0, s>>>(plan->tile_mask, plan->tile_off, nt, plan->tap_start,
                                    plan->tap_tiles);
  SMC_LAUNCHED();

  // 5. work items of one and two tiles, most taps first
  if (nt <= kItemSortMax) {
    k_item_order<<<2, 1024, size_t(nt), s>>>(plan->tile_mask, plan->tile_off, nt, plan->items[0],
                                             plan->items[1]);
    SMC_LAUNCHED();
  } else {
    // one stable radix pass over the (27 - tap count) keys, below 256
    for (int G = 1; G <= 2; ++G) {
      const int64_t ng = (nt + G - 1) / G;
      k_group_keys<<<grid_for(ng, 256), 256, 0, s>>>(plan->tile_mask, nt, G, ng, sc.gkeys[0],
                                                      sc.gvals);
      int32_t* gv[2] = {sc.gvals, sc.gorder};
      int gcur = 0;
      SMC_TRY(radix_sort(sc.gkeys, gv, 0, ng, 8, sc.hist, s, &gcur));
      k_item_records<<<grid_for(ng, 256), 256, 0, s>>>(gv[gcur], ng, G, plan->tile_mask,
                                                        plan->tile_off, nt, plan->items[G - 1]);
      SMC_LAUNCHED();
    }
  }

  // the one read-back: status word, plan counters, slot count
  if (cudaMemcpyAsync(&ctr->total_slots, plan->tile_off + nt, sizeof(int32_t),
                      cudaMemcpyDeviceToDevice, s) != cudaSuccess)
    return SMC_ERR_CUDA;
  BuildCounters h;
  if (cudaMemcpyAsync(&h, ctr, sizeof(h), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return SMC_ERR_CUDA;
  SMC_TRY(status_from_device(h.status));
  plan->total_slots = h.total_slots;
  plan->useful_pairs = int64_t(h.stats[0]);
  plan->issued_rows_taps = int64_t(h.stats[1]);
  return SMC_OK;
}

int build_plan_impl(const int32_t* coords, int64_t n, int32_t stride, int64_t table_capacity,
                    int32_t order, int32_t lookup, cudaStream_t s, Plan* plan,
                    void** scratch_mem) {
  const bool sorted = lookup == SMC_LOOKUP_SORT;
  const int4* c4 = reinterpret_cast<const int4*>(coords);
  plan->n = n;
  plan->n_tiles = (n + kTileRows - 1) / kTileRows;
  const int64_t nt = plan->n_tiles;
  const uint64_t cap = n > 0 ? table_slots(n, table_capacity) : 1;

  // two allocations: the plan's arena (kept) and the build's scratch (freed)
  Carve pc;
  BuildCounters* ctr = nullptr;
  carve_plan(pc, plan, &ctr);
  if (dev_alloc(&plan->arena, pc.off, s) != cudaSuccess) {
    cudaGetLastError();
    plan->arena = nullptr;
    return SMC_ERR_OOM;
  }
  pc = Carve{static_cast<uint8_t*>(plan->arena), 0};
  carve_plan(pc, plan, &ctr);
  plan->status = &ctr->status;
  if (cudaMemsetAsync(ctr, 0, sizeof(BuildCounters), s) != cudaSuccess) return SMC_ERR_CUDA;
  if (n == 0) return SMC_OK;

  Carve scc;
  Scratch sc;
  carve_scratch(scc, &sc, n, nt, cap, sorted);
  if (dev_alloc(scratch_mem, scc.off, s) != cudaSuccess) {
    cudaGetLastError();
    *scratch_mem = nullptr;
    return SMC_ERR_OOM;
  }
  scc = Carve{static_cast<uint8_t*>(*scratch_mem), 0};
  carve_scratch(scc, &sc, n, nt, cap, sorted);

  // 1. lookup structure; 2. neighbour map and masks
  if (sorted) {
    k_pack_keys<<<grid_for(n, 256), 256, 0, s>>>(c4, n, sc.ckeys[0], sc.svals[0], plan->status);
    SMC_LAUNCHED();
    int cur = 0;
    SMC_TRY(radix_sort(sc.ckeys, sc.svals, 0, n, 64, sc.hist, s, &cur));
    k_sorted_dups<<<grid_for(n, 256), 256, 0, s>>>(sc.ckeys[cur], n, plan->status);
    k_neighbors_sorted<<<grid_for(n, kNbrWarps), kNbrWarps * 32, 0, s>>>(
        c4, n, stride, sc.ckeys[cur], sc.svals[cur], plan->nbr, plan->mask);
  } else {
    if (cudaMemsetAsync(sc.table, 0xFF, cap * sizeof(Slot), s) != cudaSuccess)
      return SMC_ERR_CUDA;
    const int shift = 64 - log2_pow2(cap);
    k_insert<<<grid_for(n, 256), 256, 0, s>>>(c4, n, sc.table, cap - 1, shift, plan->status);
    k_neighbors<<<grid_for(n, kNbrWarps), kNbrWarps * 32, 0, s>>>(c4, n, stride, sc.table, cap - 1,
                                                                  shift, plan->nbr, plan->mask);
  }
  SMC_LAUNCHED();

  return order_and_tile(plan, ctr, sc, order, s);
}

}  // namespace

void free_plan(Plan* plan) {
  // A forward queued on any stream (including non-blocking ones, which the
  // legacy stream does not order) may still read the plan: wait for all work
  // on the device before handing the buffers back.
  cudaDeviceSynchronize();
  cudaGetLastError();
  if (plan->arena) {
    dev_free(plan->arena, nullptr);
    cudaStreamSynchronize(nullptr);
  }
  *plan = Plan{};
}

int replan(Plan* plan, int32_t order, cudaStream_t s) {
  if (plan->n == 0) return SMC_OK;
  // a forward queued on any stream may still read the plan being rewritten
  if (cudaDeviceSynchronize() != cudaSuccess) return SMC_ERR_CUDA;
  // the counters sit at the start of the arena (carve_plan)
  BuildCounters* ctr = static_cast<BuildCounters*>(plan->arena);
  if (cudaMemsetAsync(&ctr->total_slots, 0, sizeof(BuildCounters) - sizeof(int32_t), s) !=
      cudaSuccess)
    return SMC_ERR_CUDA;
  Carve scc;
  Scratch sc;
  carve_scratch(scc, &sc, plan->n, plan->n_tiles, 1, false);
  void* mem = nullptr;
  if (dev_alloc(&mem, scc.off, s) != cudaSuccess) {
    cudaGetLastError();
    return SMC_ERR_OOM;
  }
  scc = Carve{static_cast<uint8_t*>(mem), 0};
  carve_scratch(scc, &sc, plan->n, plan->n_tiles, 1, false);
  const int rc = order_and_tile(plan, ctr, sc, order, s);
  dev_free(mem, s);
  if (rc != SMC_OK) {
    cudaGetLastError();
    cudaStreamSynchronize(s);
  }
  return rc;
}

int build_plan(const int32_t* coords, int64_t n, int32_t stride, int64_t table_capacity,
               int32_t order, int32_t lookup, cudaStream_t stream, Plan* plan) {
  void* scratch = nullptr;
  int rc = build_plan_impl(coords, n, stride, table_capacity, order, lookup, stream, plan,
                           &scratch);
  if (scratch) dev_free(scratch, stream);  // stream-ordered after the build's kernels
  if (rc != SMC_OK) {
    cudaGetLastError();
    cudaStreamSynchronize(stream);
    free_plan(plan);
  }
  return rc;
}

}  // namespace smc

// ---------------------------------------------------------------------------
// Allocation-free neighbour map: smc_build_neighbor_map_static.
//
// For callers that may not allocate device memory themselves (see the header):
// the same insert and query kernels as the index build above, with the hash
// table in a fixed-size array of static device memory that every device
// loading this library reserves once, for the life of the process.
// ---------------------------------------------------------------------------
#include <cuda.h>

#include <mutex>

namespace smc {
namespace {

constexpr int64_t kStaticMaxVoxels = SMC_STATIC_MAX_VOXELS;
constexpr int64_t kStaticSlots = 2 * kStaticMaxVoxels;  // load factor <= 1/2

struct StaticScratch {
  Slot table[kStaticSlots];
  uint32_t mask[kStaticMaxVoxels];
  int32_t status;
};

// Host code may not use this name as a device address: the pointer passed to
// the kernels comes from cudaGetSymbolAddress, once per device.
static __device__ __align__(256) StaticScratch g_static_scratch;

constexpr int kMaxDevices = 128;
std::mutex g_static_mutex;
StaticScratch* g_static_ptr[kMaxDevices] = {};
unsigned long long g_static_ctx[kMaxDevices] = {};  // context the address belongs to

// Unique id of the calling thread's current CUDA context (0 when the driver
// cannot tell).  A device address is only valid in the context it came from;
// after cudaDeviceReset the device gets a new context with a new id.
unsigned long long current_context_id() {
  using GetCurrent = CUresult (*)(CUcontext*);
  using GetId = CUresult (*)(CUcontext, unsigned long long*);
  static GetCurrent get_current = nullptr;
  static GetId get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<GetCurrent>(p);
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<GetId>(p);
    cudaGetLastError();
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx ||
      get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

// Device address of the static scratch array on the current device.  The
// lookup runs once per device and context (with that device current); when
// the context id is unknown it runs on every call.
int static_scratch(StaticScratch** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return SMC_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) return SMC_ERR_UNSUPPORTED;
  // 0 before the thread's first CUDA call that binds a context: then the
  // lookup below (which binds it) runs and records the id it ran under
  const unsigned long long ctx = current_context_id();
  std::lock_guard<std::mutex> lock(g_static_mutex);
  if (!g_static_ptr[dev] || ctx == 0 || g_static_ctx[dev] != ctx) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || !p) {
      cudaGetLastError();
      g_static_ptr[dev] = nullptr;
      return SMC_ERR_CUDA;
    }
    g_static_ptr[dev] = static_cast<StaticScratch*>(p);
    g_static_ctx[dev] = current_context_id();
  }
  *out = g_static_ptr[dev];
  return SMC_OK;
}

}  // namespace
}  // namespace smc

extern "C" int smc_build_neighbor_map_static(const int32_t* coords_dev, int64_t n, int32_t stride,
                                             int32_t* map_dev, smc_stream_t stream) {
  using namespace smc;
  if (n < 0 || stride < 1) return SMC_ERR_INVALID;
  if (n > kStaticMaxVoxels) return SMC_ERR_UNSUPPORTED;
  if (n == 0) return SMC_OK;
  if (!coords_dev || !map_dev) return SMC_ERR_INVALID;
  if ((reinterpret_cast<uintptr_t>(coords_dev) & 15u) != 0) return SMC_ERR_INVALID;
  StaticScratch* sc = nullptr;
  int rc = static_scratch(&sc);
  if (rc != SMC_OK) return rc;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint64_t cap = 64;
  while (cap < uint64_t(2 * n)) cap <<= 1;
  // The array keeps the previous call's contents: reset the slots this call
  // probes and the status word before use.
  if (cudaMemsetAsync(sc->table, 0xFF, cap * sizeof(Slot), s) != cudaSuccess ||
      cudaMemsetAsync(&sc->status, 0, sizeof(int32_t), s) != cudaSuccess)
    return SMC_ERR_CUDA;
  const int4* c4 = reinterpret_cast<const int4*>(coords_dev);
  const int shift = 64 - log2_pow2(cap);
  k_insert<<<grid_for(n, 256), 256, 0, s>>>(c4, n, sc->table, cap - 1, shift, &sc->status);
  k_neighbors<<<grid_for(n, kNbrWarps), kNbrWarps * 32, 0, s>>>(c4, n, stride, sc->table, cap - 1,
                                                                shift, map_dev, sc->mask);
  if (cudaGetLastError() != cudaSuccess) return SMC_ERR_CUDA;
  int32_t dev_status = 0;
  if (cudaMemcpyAsync(&dev_status, &sc->status, sizeof(int32_t), cudaMemcpyDeviceToHost, s) !=
          cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return SMC_ERR_CUDA;
  return status_from_device(dev_status);
}
