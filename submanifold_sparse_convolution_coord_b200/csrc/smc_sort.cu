// Stable LSD radix sort of (key, value) pairs on the GPU, 8 bits per pass,
// used by the tile plan (32-bit mask keys, 8-bit work-item keys) and by the
// packed-coordinate operations (64-bit keys: the sort-based neighbour lookup
// and the x2 downsample).
//
// One pass: per-block digit histograms ([block][digit]); a column pass turns
// them into each block's exclusive offset within its digit and appends the
// digit totals; the scatter adds the digit's start (an exclusive scan of the
// totals, redone by every block) and ranks equal digits inside a block in
// index order (warp match, then earlier warps), so equal keys keep their
// order.
#include <algorithm>
#include <cstdint>

#include "smc_internal.h"

namespace smc {
namespace {

constexpr int kSortThreads = 256;
constexpr int kSortRounds = 16;
constexpr int kSortTile = kSortThreads * kSortRounds;  // 4096 items per block

template <class K>
__global__ void __launch_bounds__(kSortThreads)
k_radix_hist(const K* __restrict__ keys, int64_t n, int shift, uint32_t* hist) {
  __shared__ uint32_t h[256];
  h[threadIdx.x] = 0;
  __syncthreads();
  const int64_t base = blockIdx.x * int64_t(kSortTile);
  for (int j = 0; j < kSortRounds; ++j) {
    const int64_t idx = base + j * kSortThreads + threadIdx.x;
    if (idx < n) atomicAdd(&h[uint32_t(keys[idx] >> shift) & 255u], 1u);
  }
  __syncthreads();
  hist[int64_t(blockIdx.x) * 256 + threadIdx.x] = h[threadIdx.x];
}

// One thread per digit: hist[b][d] <- sum of hist[b'][d] for b' < b, and the
// digit's total into hist[nblocks][d].
__global__ void __launch_bounds__(256) k_radix_colscan(uint32_t* hist, int nblocks) {
  const int d = threadIdx.x;
  uint32_t run = 0;
  int b = 0;
  for (; b + 4 <= nblocks; b += 4) {
    const uint32_t v0 = hist[int64_t(b) * 256 + d], v1 = hist[int64_t(b + 1) * 256 + d];
    const uint32_t v2 = hist[int64_t(b + 2) * 256 + d], v3 = hist[int64_t(b + 3) * 256 + d];
    hist[int64_t(b) * 256 + d] = run;
    hist[int64_t(b + 1) * 256 + d] = run + v0;
    hist[int64_t(b + 2) * 256 + d] = run + v0 + v1;
    hist[int64_t(b + 3) * 256 + d] = run + v0 + v1 + v2;
    run += v0 + v1 + v2 + v3;
  }
  for (; b < nblocks; ++b) {
    const uint32_t v = hist[int64_t(b) * 256 + d];
    hist[int64_t(b) * 256 + d] = run;
    run += v;
  }
  hist[int64_t(nblocks) * 256 + d] = run;
}

template <class K>
__global__ void __launch_bounds__(kSortThreads)
k_radix_scatter(const K* __restrict__ keys_in, const int32_t* __restrict__ vals_in,
                K* __restrict__ keys_out, int32_t* __restrict__ vals_out, int64_t n, int shift,
                const uint32_t* __restrict__ hist, int nblocks) {
  constexpr int kWarps = kSortThreads / 32;
  __shared__ uint32_t run[256];
  __shared__ uint32_t wcnt[kWarps][256];
  __shared__ uint32_t wsum[kWarps];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // start of digit tid: exclusive scan of the digit totals
  const uint32_t tot = hist[int64_t(nblocks) * 256 + tid];
  uint32_t incl = tot;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) wsum[warp] = incl;
  for (int w = 0; w < kWarps; ++w) wcnt[w][tid] = 0;
  __syncthreads();
  uint32_t before = 0;
  for (int w = 0; w < warp; ++w) before += wsum[w];
  run[tid] = before + incl - tot + hist[int64_t(blockIdx.x) * 256 + tid];
  __syncthreads();
  const int64_t base = blockIdx.x * int64_t(kSortTile);
  for (int j = 0; j < kSortRounds; ++j) {
    const int64_t idx = base + j * kSortThreads + tid;
    const bool valid = idx < n;
    const K key = valid ? keys_in[idx] : K(0);
    const int32_t val = valid ? vals_in[idx] : 0;
    const uint32_t d = valid ? (uint32_t(key >> shift) & 255u) : (256u + lane);  // never matches
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
    uint32_t t = 0;
    for (int w = 0; w < kWarps; ++w) {
      t += wcnt[w][tid];
      wcnt[w][tid] = 0;
    }
    run[tid] += t;
    __syncthreads();
  }
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

}  // namespace

int scan_exclusive(uint32_t* data, int64_t m, cudaStream_t s) {
  if (m > 0) k_scan_exclusive<<<1, 1024, 0, s>>>(data, m);
  return cudaGetLastError() == cudaSuccess ? SMC_OK : SMC_ERR_CUDA;
}

size_t sort_hist_words(int64_t n) {
  const int64_t nb = (n + kSortTile - 1) / kSortTile;
  return size_t(256) * size_t(nb + 1);
}

template <class K>
int radix_sort(K* const keys[2], int32_t* const vals[2], int cur, int64_t n, int bits,
               uint32_t* hist, cudaStream_t s, int* out_cur) {
  const int nb = int((n + kSortTile - 1) / kSortTile);
  for (int shift = 0; shift < bits; shift += 8) {
    if (n > 0) {
      k_radix_hist<K><<<nb, kSortThreads, 0, s>>>(keys[cur], n, shift, hist);
      k_radix_colscan<<<1, 256, 0, s>>>(hist, nb);
      k_radix_scatter<K><<<nb, kSortThreads, 0, s>>>(keys[cur], vals[cur], keys[cur ^ 1],
                                                     vals[cur ^ 1], n, shift, hist, nb);
      if (cudaGetLastError() != cudaSuccess) return SMC_ERR_CUDA;
    }
    cur ^= 1;
  }
  *out_cur = cur;
  return SMC_OK;
}

template int radix_sort<uint32_t>(uint32_t* const[2], int32_t* const[2], int, int64_t, int,
                                  uint32_t*, cudaStream_t, int*);
template int radix_sort<unsigned long long>(unsigned long long* const[2], int32_t* const[2], int,
                                            int64_t, int, uint32_t*, cudaStream_t, int*);

}  // namespace smc
