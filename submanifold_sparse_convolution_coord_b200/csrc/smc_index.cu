// Index build: coordinate hash, neighbour map, row ordering and tile plan.
//
// This is the "prepared device gather index" of the trellis_sparse_mlx README
// ("Performance": caching the prepared index, not only the raw indice map,
// is what made the layer compute-bound), built once per coordinate set:
//
//   1. insert   every voxel's packed key (b:15 | x:16 | y:16 | z:16 bits) into
//               an open-addressing table (linear probing, SplitMix64 mixer);
//   2. query    the 27 neighbours c + stride*d of every voxel -> int32 map
//               [n][27] (-1 = absent) and a 27-bit tap mask per voxel;
//   3. order    rows by (popcount(mask), Gray-code rank of mask) with a stable
//               LSD radix sort, so a 128-row tile holds voxels whose active
//               taps coincide;
//   4. plan     per tile, the OR of its rows' masks (the taps the tensor-core
//               kernel multiplies; the others are skipped) and a compact
//               gather index [tile][active tap][128 rows];
//   5. items    for work items of one and of two consecutive tiles, the
//               groups in decreasing order of their union's tap count (one
//               stable radix pass), so the convolution hands out its largest
//               items first.
#include <algorithm>
#include <cstdio>
#include <cstring>

#include "smc_internal.h"

namespace smc {
namespace {

constexpr uint64_t kEmptyKey = ~0ull;

// SplitMix64 output mixer (Steele, Lea and Flood, "Fast splittable
// pseudorandom number generators", OOPSLA 2014).
__device__ __forceinline__ uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xbf58476d1ce4e5b9ull;
  z = (z ^ (z >> 27)) * 0x94d049bb133111ebull;
  return z ^ (z >> 31);
}

__device__ __forceinline__ uint64_t pack_key(int64_t b, int64_t x, int64_t y, int64_t z) {
  return (uint64_t(b) << 48) | (uint64_t(x) << 32) | (uint64_t(y) << 16) | uint64_t(z);
}

__device__ __forceinline__ bool axis_ok(int64_t v) { return v >= 0 && v < kMaxAxis; }

__global__ void k_insert(const int4* __restrict__ coords, int64_t n, uint64_t* keys,
                         int32_t* vals, uint64_t cap_mask, int32_t* status) {
  const int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x;
  if (i >= n) return;
  const int4 c = coords[i];
  if (c.x < 0 || c.x >= kMaxBatch || !axis_ok(c.y) || !axis_ok(c.z) || !axis_ok(c.w)) {
    atomicOr(status, kDevRange);
    return;
  }
  const uint64_t key = pack_key(c.x, c.y, c.z, c.w);
  uint64_t slot = mix64(key) & cap_mask;
  for (uint64_t probe = 0; probe <= cap_mask; ++probe) {
    const unsigned long long prev = atomicCAS(reinterpret_cast<unsigned long long*>(keys + slot),
                                              (unsigned long long)kEmptyKey,
                                              (unsigned long long)key);
    if (prev == kEmptyKey) {
      vals[slot] = int32_t(i);
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

// 32 voxels per block, one thread per (voxel, tap): the map is written with
// consecutive threads on consecutive words.
constexpr int kNbrVoxels = 32;
constexpr int kNbrThreads = kNbrVoxels * kTaps;  // 864

__global__ void __launch_bounds__(kNbrThreads)
k_neighbors(const int4* __restrict__ coords, int64_t n, int32_t stride,
            const uint64_t* __restrict__ keys, const int32_t* __restrict__ vals,
            uint64_t cap_mask, int32_t* __restrict__ nbr, uint32_t* __restrict__ mask) {
  __shared__ uint32_t smask[kNbrVoxels];
  if (threadIdx.x < kNbrVoxels) smask[threadIdx.x] = 0;
  __syncthreads();
  const int local = threadIdx.x / kTaps;
  const int k = threadIdx.x - local * kTaps;
  const int64_t i = blockIdx.x * int64_t(kNbrVoxels) + local;
  if (i < n) {
    const int4 c = coords[i];
    const int64_t x = int64_t(c.y) + int64_t(stride) * (k / 9 - 1);
    const int64_t y = int64_t(c.z) + int64_t(stride) * ((k / 3) % 3 - 1);
    const int64_t z = int64_t(c.w) + int64_t(stride) * (k % 3 - 1);
    int32_t found = -1;
    if (axis_ok(x) && axis_ok(y) && axis_ok(z)) {
      const uint64_t key = pack_key(c.x, x, y, z);
      uint64_t slot = mix64(key) & cap_mask;
      for (uint64_t probe = 0; probe <= cap_mask; ++probe) {
        const uint64_t kk = keys[slot];
        if (kk == key) {
          found = vals[slot];
          break;
        }
        if (kk == kEmptyKey) break;
        slot = (slot + 1) & cap_mask;
      }
    }
    nbr[i * kTaps + k] = found;
    if (found >= 0) atomicOr(&smask[local], 1u << k);
  }
  __syncthreads();
  if (threadIdx.x < kNbrVoxels) {
    const int64_t ii = blockIdx.x * int64_t(kNbrVoxels) + threadIdx.x;
    if (ii < n) mask[ii] = smask[threadIdx.x];
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

// ---------------------------------------------------------------------------
// Stable LSD radix sort, 8 bits per pass: per-block digit histograms, one
// exclusive scan in (digit, block) order, then a stable scatter that ranks
// equal digits inside a block in index order.
// ---------------------------------------------------------------------------
constexpr int kSortThreads = 256;
constexpr int kSortRounds = 16;
constexpr int kSortTile = kSortThreads * kSortRounds;  // 4096 items per block

__global__ void __launch_bounds__(kSortThreads)
k_radix_hist(const uint32_t* __restrict__ keys, int64_t n, int shift, uint32_t* hist,
             int nblocks) {
  __shared__ uint32_t h[256];
  h[threadIdx.x] = 0;
  __syncthreads();
  const int64_t base = blockIdx.x * int64_t(kSortTile);
  for (int j = 0; j < kSortRounds; ++j) {
    const int64_t idx = base + j * kSortThreads + threadIdx.x;
    if (idx < n) atomicAdd(&h[(keys[idx] >> shift) & 255u], 1u);
  }
  __syncthreads();
  hist[int64_t(threadIdx.x) * nblocks + blockIdx.x] = h[threadIdx.x];
}

// In-place exclusive scan of m 32-bit counts by one block of 1024 threads.
__global__ void __launch_bounds__(1024) k_scan_exclusive(uint32_t* data, int64_t m) {
  __shared__ uint32_t part[1024];
  const int64_t per = (m + 1023) / 1024;
  const int64_t lo = std::min<int64_t>(threadIdx.x * per, m);
  const int64_t hi = std::min<int64_t>(lo + per, m);
  uint32_t s = 0;
  for (int64_t i = lo; i < hi; ++i) s += data[i];
  part[threadIdx.x] = s;
  __syncthreads();
  for (int off = 1; off < 1024; off <<= 1) {
    const uint32_t v = threadIdx.x >= unsigned(off) ? part[threadIdx.x - off] : 0u;
    __syncthreads();
    part[threadIdx.x] += v;
    __syncthreads();
  }
  uint32_t run = threadIdx.x ? part[threadIdx.x - 1] : 0u;
  for (int64_t i = lo; i < hi; ++i) {
    const uint32_t v = data[i];
    data[i] = run;
    run += v;
  }
}

__global__ void __launch_bounds__(kSortThreads)
k_radix_scatter(const uint32_t* __restrict__ keys_in, const int32_t* __restrict__ vals_in,
                uint32_t* __restrict__ keys_out, int32_t* __restrict__ vals_out, int64_t n,
                int shift, const uint32_t* __restrict__ offsets, int nblocks) {
  constexpr int kWarps = kSortThreads / 32;
  __shared__ uint32_t run[256];
  __shared__ uint32_t wcnt[kWarps][256];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  run[tid] = offsets[int64_t(tid) * nblocks + blockIdx.x];
  for (int w = 0; w < kWarps; ++w) wcnt[w][tid] = 0;
  __syncthreads();
  const int64_t base = blockIdx.x * int64_t(kSortTile);
  for (int j = 0; j < kSortRounds; ++j) {
    const int64_t idx = base + j * kSortThreads + tid;
    const bool valid = idx < n;
    const uint32_t key = valid ? keys_in[idx] : 0u;
    const int32_t val = valid ? vals_in[idx] : 0;
    const uint32_t d = valid ? ((key >> shift) & 255u) : (256u + lane);  // invalid lanes never match
    const uint32_t peers = __match_any_sync(0xffffffffu, d);
    const uint32_t rank = __popc(peers & ((1u << lane) - 1u));
    if (valid && rank == 0) wcnt[warp][d] = __popc(peers);
    __syncthreads();
    if (valid) {
      uint32_t pos = run[d] + rank;
      for (int w = 0; w < warp; ++w) pos += wcnt[w][d];
      keys_out[pos] = key;
      vals_out[pos] = val;
    }
    __syncthreads();
    uint32_t tot = 0;
    for (int w = 0; w < kWarps; ++w) {
      tot += wcnt[w][tid];
      wcnt[w][tid] = 0;
    }
    run[tid] += tot;
    __syncthreads();
  }
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

// One block of 128 threads per tile: the tile's tap list and, for each active
// tap, the voxel each plan row gathers (or -1).
__global__ void __launch_bounds__(kTileRows)
k_tile_gather(const int32_t* __restrict__ perm, const int32_t* __restrict__ nbr, int64_t n,
              const uint32_t* __restrict__ tile_mask, const int32_t* __restrict__ tile_off,
              uint8_t* __restrict__ tile_taps, int32_t* __restrict__ gidx,
              int32_t* __restrict__ out_row) {
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
    if (threadIdx.x == 0) tile_taps[tile * 32 + s] = uint8_t(t);
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

template <class T>
int dev_alloc(T** p, size_t count, cudaStream_t s) {
  *p = nullptr;
  if (count == 0) count = 1;
  if (cudaMallocAsync(reinterpret_cast<void**>(p), count * sizeof(T), s) != cudaSuccess) {
    cudaGetLastError();
    return SMC_ERR_OOM;
  }
  return SMC_OK;
}

template <class T>
void dev_free(T*& p, cudaStream_t s) {
  if (p) cudaFreeAsync(p, s);
  p = nullptr;
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

struct Scratch {
  uint64_t* keys = nullptr;
  int32_t* vals = nullptr;
  uint32_t* skeys[2] = {nullptr, nullptr};
  int32_t* svals[2] = {nullptr, nullptr};
  uint32_t* hist = nullptr;
  uint32_t* tile_ntaps = nullptr;
  unsigned long long* stats = nullptr;
  uint32_t* gkeys[2] = {nullptr, nullptr};
  int32_t* gvals = nullptr;
  uint32_t* ghist = nullptr;
  void release(cudaStream_t s) {
    dev_free(gkeys[0], s);
    dev_free(gkeys[1], s);
    dev_free(gvals, s);
    dev_free(ghist, s);
    dev_free(keys, s);
    dev_free(vals, s);
    for (int i = 0; i < 2; ++i) {
      dev_free(skeys[i], s);
      dev_free(svals[i], s);
    }
    dev_free(hist, s);
    dev_free(tile_ntaps, s);
    dev_free(stats, s);
  }
};

#define SMC_TRY(expr)             \
  do {                            \
    int rc_ = (expr);             \
    if (rc_ != SMC_OK) return rc_; \
  } while (0)

#define SMC_LAUNCHED()                                     \
  do {                                                     \
    if (cudaGetLastError() != cudaSuccess) return SMC_ERR_CUDA; \
  } while (0)

int build_plan_impl(const int32_t* coords, int64_t n, int32_t stride, int64_t table_capacity,
                    int32_t order, cudaStream_t s, Plan* plan, Scratch& sc) {
  const int4* c4 = reinterpret_cast<const int4*>(coords);
  SMC_TRY(dev_alloc(&plan->status, 1, s));
  SMC_TRY(dev_alloc(&plan->work_counter, 64, s));
  if (cudaMemsetAsync(plan->work_counter, 0, 64 * sizeof(uint32_t), s) != cudaSuccess)
    return SMC_ERR_CUDA;
  if (cudaMemsetAsync(plan->status, 0, sizeof(int32_t), s) != cudaSuccess) return SMC_ERR_CUDA;
  plan->n = n;
  plan->n_tiles = (n + kTileRows - 1) / kTileRows;
  if (n == 0) return SMC_OK;

  // 1. hash insert
  uint64_t cap = 64;
  if (table_capacity > 0) {
    cap = 1;
    while (cap < uint64_t(table_capacity)) cap <<= 1;
    if (cap > uint64_t(table_capacity)) cap >>= 1;  // largest power of two <= request
    if (cap == 0) cap = 1;
  } else {
    while (cap < uint64_t(2 * n)) cap <<= 1;
  }
  SMC_TRY(dev_alloc(&sc.keys, cap, s));
  SMC_TRY(dev_alloc(&sc.vals, cap, s));
  if (cudaMemsetAsync(sc.keys, 0xFF, cap * sizeof(uint64_t), s) != cudaSuccess) return SMC_ERR_CUDA;
  k_insert<<<grid_for(n, 256), 256, 0, s>>>(c4, n, sc.keys, sc.vals, cap - 1, plan->status);
  SMC_LAUNCHED();

  // 2. neighbour map and masks
  SMC_TRY(dev_alloc(&plan->nbr, size_t(n) * kTaps, s));
  SMC_TRY(dev_alloc(&plan->mask, size_t(n), s));
  k_neighbors<<<grid_for(n, kNbrVoxels), kNbrThreads, 0, s>>>(c4, n, stride, sc.keys, sc.vals,
                                                               cap - 1, plan->nbr, plan->mask);
  SMC_LAUNCHED();
  dev_free(sc.keys, s);
  dev_free(sc.vals, s);

  // 3. row order
  SMC_TRY(dev_alloc(&plan->perm, size_t(n), s));
  if (order == SMC_ORDER_MASK) {
    const int nblocks = int((n + kSortTile - 1) / kSortTile);
    for (int i = 0; i < 2; ++i) {
      SMC_TRY(dev_alloc(&sc.skeys[i], size_t(n), s));
      SMC_TRY(dev_alloc(&sc.svals[i], size_t(n), s));
    }
    SMC_TRY(dev_alloc(&sc.hist, size_t(256) * nblocks, s));
    k_sort_keys<<<grid_for(n, 256), 256, 0, s>>>(plan->mask, n, sc.skeys[0], sc.svals[0]);
    SMC_LAUNCHED();
    int cur = 0;
    for (int shift = 0; shift < 32; shift += 8) {
      k_radix_hist<<<nblocks, kSortThreads, 0, s>>>(sc.skeys[cur], n, shift, sc.hist, nblocks);
      k_scan_exclusive<<<1, 1024, 0, s>>>(sc.hist, int64_t(256) * nblocks);
      k_radix_scatter<<<nblocks, kSortThreads, 0, s>>>(sc.skeys[cur], sc.svals[cur],
                                                       sc.skeys[cur ^ 1], sc.svals[cur ^ 1], n,
                                                       shift, sc.hist, nblocks);
      SMC_LAUNCHED();
      cur ^= 1;
    }
    if (cudaMemcpyAsync(plan->perm, sc.svals[cur], size_t(n) * sizeof(int32_t),
                        cudaMemcpyDeviceToDevice, s) != cudaSuccess)
      return SMC_ERR_CUDA;
  } else {
    k_iota<<<grid_for(n, 256), 256, 0, s>>>(plan->perm, n);
    SMC_LAUNCHED();
  }

  // 4. tile plan
  const int64_t nt = plan->n_tiles;
  SMC_TRY(dev_alloc(&plan->tile_mask, size_t(nt), s));
  SMC_TRY(dev_alloc(&sc.tile_ntaps, size_t(nt) + 1, s));
  SMC_TRY(dev_alloc(&sc.stats, 2, s));
  if (cudaMemsetAsync(sc.tile_ntaps, 0, (size_t(nt) + 1) * sizeof(uint32_t), s) != cudaSuccess ||
      cudaMemsetAsync(sc.stats, 0, 2 * sizeof(unsigned long long), s) != cudaSuccess)
    return SMC_ERR_CUDA;
  k_tile_mask<<<unsigned(nt), kTileRows, 0, s>>>(plan->perm, plan->mask, n, plan->tile_mask,
                                                  sc.tile_ntaps, sc.stats);
  k_scan_exclusive<<<1, 1024, 0, s>>>(sc.tile_ntaps, nt + 1);
  SMC_LAUNCHED();

  struct {
    uint32_t total;
    int32_t status;
    unsigned long long stats[2];
  } h{};
  if (cudaMemcpyAsync(&h.total, sc.tile_ntaps + nt, sizeof(uint32_t), cudaMemcpyDeviceToHost, s) !=
          cudaSuccess ||
      cudaMemcpyAsync(&h.status, plan->status, sizeof(int32_t), cudaMemcpyDeviceToHost, s) !=
          cudaSuccess ||
      cudaMemcpyAsync(h.stats, sc.stats, sizeof(h.stats), cudaMemcpyDeviceToHost, s) !=
          cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return SMC_ERR_CUDA;
  SMC_TRY(status_from_device(h.status));
  plan->total_slots = h.total;
  plan->useful_pairs = int64_t(h.stats[0]);
  plan->issued_rows_taps = int64_t(h.stats[1]);
  plan->tile_off = reinterpret_cast<int32_t*>(sc.tile_ntaps);  // ownership moves to the plan
  sc.tile_ntaps = nullptr;

  SMC_TRY(dev_alloc(&plan->tile_taps, size_t(nt) * 32, s));
  SMC_TRY(dev_alloc(&plan->gidx, size_t(plan->total_slots) * kTileRows, s));
  SMC_TRY(dev_alloc(&plan->out_row, size_t(nt) * kTileRows, s));
  k_tile_gather<<<unsigned(nt), kTileRows, 0, s>>>(plan->perm, plan->nbr, n, plan->tile_mask,
                                                    plan->tile_off, plan->tile_taps, plan->gidx,
                                                    plan->out_row);
  SMC_LAUNCHED();

  // 5. work-item order for one and two tiles per item: one stable radix pass
  // over the (27 - tap count) keys, which are below 256
  {
    const int gblocks = int((nt + kSortTile - 1) / kSortTile);
    SMC_TRY(dev_alloc(&sc.gkeys[0], size_t(nt), s));
    SMC_TRY(dev_alloc(&sc.gkeys[1], size_t(nt), s));
    SMC_TRY(dev_alloc(&sc.gvals, size_t(nt), s));
    SMC_TRY(dev_alloc(&sc.ghist, size_t(256) * gblocks, s));
    for (int G = 1; G <= 2; ++G) {
      const int64_t ng = (nt + G - 1) / G;
      const int nb = int((ng + kSortTile - 1) / kSortTile);
      SMC_TRY(dev_alloc(&plan->group_order[G - 1], size_t(ng), s));
      k_group_keys<<<grid_for(ng, 256), 256, 0, s>>>(plan->tile_mask, nt, G, ng, sc.gkeys[0],
                                                      sc.gvals);
      k_radix_hist<<<nb, kSortThreads, 0, s>>>(sc.gkeys[0], ng, 0, sc.ghist, nb);
      k_scan_exclusive<<<1, 1024, 0, s>>>(sc.ghist, int64_t(256) * nb);
      k_radix_scatter<<<nb, kSortThreads, 0, s>>>(sc.gkeys[0], sc.gvals, sc.gkeys[1],
                                                  plan->group_order[G - 1], ng, 0, sc.ghist, nb);
      SMC_LAUNCHED();
    }
  }
  if (cudaStreamSynchronize(s) != cudaSuccess) return SMC_ERR_CUDA;
  return SMC_OK;
}

}  // namespace

void free_plan(Plan* plan) {
  cudaStream_t s = nullptr;
  dev_free(plan->nbr, s);
  dev_free(plan->mask, s);
  dev_free(plan->perm, s);
  dev_free(plan->tile_mask, s);
  dev_free(plan->tile_off, s);
  dev_free(plan->tile_taps, s);
  dev_free(plan->gidx, s);
  dev_free(plan->out_row, s);
  dev_free(plan->status, s);
  dev_free(plan->work_counter, s);
  dev_free(plan->group_order[0], s);
  dev_free(plan->group_order[1], s);
  cudaStreamSynchronize(s);
}

int build_plan(const int32_t* coords, int64_t n, int32_t stride, int64_t table_capacity,
               int32_t order, cudaStream_t stream, Plan* plan) {
  Scratch sc;
  int rc = build_plan_impl(coords, n, stride, table_capacity, order, stream, plan, sc);
  sc.release(stream);
  if (rc != SMC_OK) {
    cudaGetLastError();
    free_plan(plan);
    *plan = Plan{};
  }
  cudaStreamSynchronize(stream);
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
#include <mutex>

namespace smc {
namespace {

constexpr int64_t kStaticMaxVoxels = SMC_STATIC_MAX_VOXELS;
constexpr int64_t kStaticSlots = 2 * kStaticMaxVoxels;  // load factor <= 1/2

struct StaticScratch {
  uint64_t keys[kStaticSlots];
  int32_t vals[kStaticSlots];
  uint32_t mask[kStaticMaxVoxels];
  int32_t status;
};

// Host code may not use this name as a device address: the pointer passed to
// the kernels comes from cudaGetSymbolAddress, once per device.
static __device__ __align__(256) StaticScratch g_static_scratch;

constexpr int kMaxDevices = 128;
std::mutex g_static_mutex;
StaticScratch* g_static_ptr[kMaxDevices] = {};

int static_scratch(StaticScratch** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return SMC_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) return SMC_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_static_mutex);
  if (!g_static_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || !p) {
      cudaGetLastError();
      return SMC_ERR_CUDA;
    }
    g_static_ptr[dev] = static_cast<StaticScratch*>(p);
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
  if (cudaMemsetAsync(sc->keys, 0xFF, cap * sizeof(uint64_t), s) != cudaSuccess ||
      cudaMemsetAsync(&sc->status, 0, sizeof(int32_t), s) != cudaSuccess)
    return SMC_ERR_CUDA;
  const int4* c4 = reinterpret_cast<const int4*>(coords_dev);
  k_insert<<<grid_for(n, 256), 256, 0, s>>>(c4, n, sc->keys, sc->vals, cap - 1, &sc->status);
  k_neighbors<<<grid_for(n, kNbrVoxels), kNbrThreads, 0, s>>>(c4, n, stride, sc->keys, sc->vals,
                                                               cap - 1, map_dev, sc->mask);
  if (cudaGetLastError() != cudaSuccess) return SMC_ERR_CUDA;
  int32_t dev_status = 0;
  if (cudaMemcpyAsync(&dev_status, &sc->status, sizeof(int32_t), cudaMemcpyDeviceToHost, s) !=
          cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return SMC_ERR_CUDA;
  return status_from_device(dev_status);
}
