// x2 coordinate operations of the sparse tensor (trellis_sparse_mlx README,
// "What's in it": subdivide / downsample -- x2 coordinate expansion; x2
// max-pool, upstream passing reduce="amax" although its docstring says
// "average").
//
// Downsample: every voxel's parent is (b, x >> 1, y >> 1, z >> 1).  The parent
// keys are packed into 64 bits and radix-sorted with their rows; equal keys
// form one segment per parent (heads flagged, then an exclusive scan numbers
// them), the parents come out in packed-key order, which is lexicographic
// (b, x, y, z), and each parent's row is the element-wise maximum over its
// segment.  Subdivide: each voxel's 8 children (b, 2x + dx, 2y + dy, 2z + dz),
// child c = 4 dx + 2 dy + dz, in parent order, copy the parent's row.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cstdint>

#include "smc_internal.h"

namespace smc {
namespace {

__device__ __forceinline__ unsigned long long pack4(int b, int x, int y, int z) {
  return (uint64_t(uint32_t(b)) << 48) | (uint64_t(uint32_t(x)) << 32) |
         (uint64_t(uint32_t(y)) << 16) | uint64_t(uint32_t(z));
}

__global__ void k_parent_keys(const int4* __restrict__ coords, int64_t n,
                              unsigned long long* __restrict__ keys, int32_t* __restrict__ vals,
                              int32_t* status) {
  const int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x;
  if (i >= n) return;
  const int4 c = coords[i];
  if (c.x < 0 || c.x >= kMaxBatch || c.y < 0 || c.y >= kMaxAxis || c.z < 0 || c.z >= kMaxAxis ||
      c.w < 0 || c.w >= kMaxAxis) {
    atomicOr(status, kDevRange);
    keys[i] = ~0ull - uint64_t(i);
  } else {
    keys[i] = pack4(c.x, c.y >> 1, c.z >> 1, c.w >> 1);
  }
  vals[i] = int32_t(i);
}

// heads[i] = 1 where a new key starts in sorted order; heads[n] = 0.
__global__ void k_segment_heads(const unsigned long long* __restrict__ keys, int64_t n,
                                uint32_t* __restrict__ heads) {
  const int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x;
  if (i < n) heads[i] = (i == 0 || keys[i] != keys[i - 1]) ? 1u : 0u;
  if (i == n) heads[n] = 0u;
}

// After the scan, seg[i] numbers the segment of sorted position i (at heads).
__global__ void k_segment_write(const unsigned long long* __restrict__ keys, int64_t n,
                                const uint32_t* __restrict__ seg, int32_t* __restrict__ start,
                                int4* __restrict__ out_coords) {
  const int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x;
  if (i >= n) return;
  const bool head = i == 0 || keys[i] != keys[i - 1];
  if (head) {
    const uint32_t p = seg[i];
    const unsigned long long k = keys[i];
    start[p] = int32_t(i);
    out_coords[p] = make_int4(int(k >> 48), int((k >> 32) & 0xFFFF), int((k >> 16) & 0xFFFF),
                              int(k & 0xFFFF));
  }
  if (i == n - 1) start[seg[n]] = int32_t(n);  // end of the last segment
}

template <class T>
__device__ __forceinline__ float as_float(T v);
template <>
__device__ __forceinline__ float as_float<float>(float v) {
  return v;
}
template <>
__device__ __forceinline__ float as_float<__half>(__half v) {
  return __half2float(v);
}
template <>
__device__ __forceinline__ float as_float<__nv_bfloat16>(__nv_bfloat16 v) {
  return __bfloat162float(v);
}

// One thread per (parent, channel): the maximum over the parent's segment.
// The result is one of the inputs, so it is stored exactly.
template <class T>
__global__ void k_segment_max(const T* __restrict__ feats, int c, const int32_t* __restrict__ rows,
                              const int32_t* __restrict__ start, const uint32_t* __restrict__ seg_end,
                              int64_t n, T* __restrict__ out) {
  const int64_t id = blockIdx.x * int64_t(blockDim.x) + threadIdx.x;
  const int64_t m = *seg_end;  // number of parents
  if (id >= m * c) return;
  const int64_t p = id / c;
  const int ch = int(id - p * c);
  T best = feats[int64_t(rows[start[p]]) * c + ch];
  for (int32_t r = start[p] + 1; r < start[p + 1]; ++r) {
    const T v = feats[int64_t(rows[r]) * c + ch];
    if (as_float(v) > as_float(best)) best = v;
  }
  out[p * c + ch] = best;
}

template <class T>
__global__ void k_subdivide(const int4* __restrict__ coords, int64_t n, const T* __restrict__ feats,
                            int c, int4* __restrict__ out_coords, T* __restrict__ out_feats,
                            int32_t* status) {
  const int64_t id = blockIdx.x * int64_t(blockDim.x) + threadIdx.x;
  if (id >= 8 * n) return;
  const int64_t i = id >> 3;
  const int child = int(id & 7);
  const int4 p = coords[i];
  const int dx = child >> 2, dy = (child >> 1) & 1, dz = child & 1;
  if (p.x < 0 || p.x >= kMaxBatch || p.y < 0 || 2 * p.y + 1 >= kMaxAxis || p.z < 0 ||
      2 * p.z + 1 >= kMaxAxis || p.w < 0 || 2 * p.w + 1 >= kMaxAxis) {
    if (child == 0) atomicOr(status, kDevRange);
    return;
  }
  out_coords[id] = make_int4(p.x, 2 * p.y + dx, 2 * p.z + dy, 2 * p.w + dz);
  const T* src = feats + i * c;
  T* dst = out_feats + id * c;
  for (int ch = 0; ch < c; ++ch) dst[ch] = src[ch];
}

inline unsigned grid_for(int64_t n, int threads) { return unsigned((n + threads - 1) / threads); }

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

struct DownScratch {
  int32_t* status;
  unsigned long long* keys[2];
  int32_t* vals[2];
  uint32_t* hist;
  uint32_t* seg;      // [n + 1]
  int32_t* start;     // [n + 1]
};

void carve_down(Carve& c, DownScratch* d, int64_t n) {
  d->status = c.take<int32_t>(1);
  for (int i = 0; i < 2; ++i) {
    d->keys[i] = c.take<unsigned long long>(size_t(n));
    d->vals[i] = c.take<int32_t>(size_t(n));
  }
  d->hist = c.take<uint32_t>(sort_hist_words(n));
  d->seg = c.take<uint32_t>(size_t(n) + 1);
  d->start = c.take<int32_t>(size_t(n) + 1);
}

int status_of(int32_t v) {
  if (v & kDevRange) return SMC_ERR_RANGE;
  return v == 0 ? SMC_OK : SMC_ERR_CUDA;
}

}  // namespace

int downsample2(const int32_t* coords, int64_t n, const void* feats, int c, int dtype,
                int32_t* out_coords, void* out_feats, int64_t* out_n, cudaStream_t s) {
  Carve cv;
  DownScratch d;
  carve_down(cv, &d, n);
  void* mem = nullptr;
  if (dev_alloc(&mem, cv.off, s) != cudaSuccess) {
    cudaGetLastError();
    return SMC_ERR_OOM;
  }
  cv = Carve{static_cast<uint8_t*>(mem), 0};
  carve_down(cv, &d, n);
  int rc = SMC_OK;
  int cur = 0;
  const int4* c4 = reinterpret_cast<const int4*>(coords);
  if (cudaMemsetAsync(d.status, 0, sizeof(int32_t), s) != cudaSuccess) rc = SMC_ERR_CUDA;
  if (rc == SMC_OK) {
    k_parent_keys<<<grid_for(n, 256), 256, 0, s>>>(c4, n, d.keys[0], d.vals[0], d.status);
    rc = cudaGetLastError() == cudaSuccess ? SMC_OK : SMC_ERR_CUDA;
  }
  if (rc == SMC_OK) rc = radix_sort(d.keys, d.vals, 0, n, 64, d.hist, s, &cur);
  if (rc == SMC_OK) {
    k_segment_heads<<<grid_for(n + 1, 256), 256, 0, s>>>(d.keys[cur], n, d.seg);
    rc = scan_exclusive(d.seg, n + 1, s);
  }
  if (rc == SMC_OK) {
    k_segment_write<<<grid_for(n, 256), 256, 0, s>>>(d.keys[cur], n, d.seg, d.start,
                                                      reinterpret_cast<int4*>(out_coords));
    const unsigned g = grid_for(n * int64_t(c), 256);
    switch (dtype) {
      case SMC_F32:
        k_segment_max<float><<<g, 256, 0, s>>>(static_cast<const float*>(feats), c, d.vals[cur],
                                               d.start, d.seg + n, n,
                                               static_cast<float*>(out_feats));
        break;
      case SMC_F16:
        k_segment_max<__half><<<g, 256, 0, s>>>(static_cast<const __half*>(feats), c, d.vals[cur],
                                                d.start, d.seg + n, n,
                                                static_cast<__half*>(out_feats));
        break;
      default:
        k_segment_max<__nv_bfloat16><<<g, 256, 0, s>>>(
            static_cast<const __nv_bfloat16*>(feats), c, d.vals[cur], d.start, d.seg + n, n,
            static_cast<__nv_bfloat16*>(out_feats));
    }
    rc = cudaGetLastError() == cudaSuccess ? SMC_OK : SMC_ERR_CUDA;
  }
  struct {
    int32_t status;
    uint32_t m;
  } h{};
  if (rc == SMC_OK &&
      (cudaMemcpyAsync(&h.status, d.status, sizeof(int32_t), cudaMemcpyDeviceToHost, s) !=
           cudaSuccess ||
       cudaMemcpyAsync(&h.m, d.seg + n, sizeof(uint32_t), cudaMemcpyDeviceToHost, s) !=
           cudaSuccess ||
       cudaStreamSynchronize(s) != cudaSuccess))
    rc = SMC_ERR_CUDA;
  dev_free(mem, s);
  if (rc == SMC_OK) rc = status_of(h.status);
  if (rc == SMC_OK) *out_n = int64_t(h.m);
  return rc;
}

int subdivide2(const int32_t* coords, int64_t n, const void* feats, int c, int dtype,
               int32_t* out_coords, void* out_feats, cudaStream_t s) {
  int32_t* status = nullptr;
  if (dev_alloc(reinterpret_cast<void**>(&status), sizeof(int32_t), s) != cudaSuccess) {
    cudaGetLastError();
    return SMC_ERR_OOM;
  }
  int rc = cudaMemsetAsync(status, 0, sizeof(int32_t), s) == cudaSuccess ? SMC_OK : SMC_ERR_CUDA;
  const int4* c4 = reinterpret_cast<const int4*>(coords);
  int4* o4 = reinterpret_cast<int4*>(out_coords);
  const unsigned g = grid_for(8 * n, 256);
  if (rc == SMC_OK) {
    switch (dtype) {
      case SMC_F32:
        k_subdivide<float><<<g, 256, 0, s>>>(c4, n, static_cast<const float*>(feats), c, o4,
                                             static_cast<float*>(out_feats), status);
        break;
      default:
        k_subdivide<uint16_t><<<g, 256, 0, s>>>(c4, n, static_cast<const uint16_t*>(feats), c, o4,
                                                static_cast<uint16_t*>(out_feats), status);
    }
    rc = cudaGetLastError() == cudaSuccess ? SMC_OK : SMC_ERR_CUDA;
  }
  int32_t h = 0;
  if (rc == SMC_OK &&
      (cudaMemcpyAsync(&h, status, sizeof(int32_t), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
       cudaStreamSynchronize(s) != cudaSuccess))
    rc = SMC_ERR_CUDA;
  dev_free(status, s);
  if (rc == SMC_OK) rc = status_of(h);
  return rc;
}

}  // namespace smc
