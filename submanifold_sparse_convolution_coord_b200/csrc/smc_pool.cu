// Device memory of libsmc: one stream-ordered memory pool per device, owned
// by the library.  Memory a build or a handle gives back stays reserved in
// the pool (release threshold: unlimited), so the next index build reuses it
// instead of mapping fresh device memory; the pool is trimmed only when an
// allocation would otherwise fail.
#include <mutex>

#include "smc_internal.h"

namespace smc {
namespace {

constexpr int kMaxDev = 64;
cudaMemPool_t g_pool[kMaxDev] = {};
std::mutex g_pool_mu;

// The pool of the current device, created on first use; null if the device
// has no memory-pool support (then the device's default pool is used).
cudaMemPool_t pool_of_current_device(int* dev_out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) {
    cudaGetLastError();
    *dev_out = -1;
    return nullptr;
  }
  *dev_out = dev;
  std::lock_guard<std::mutex> lock(g_pool_mu);
  if (g_pool[dev]) return g_pool[dev];
  cudaMemPoolProps props = {};
  props.allocType = cudaMemAllocationTypePinned;
  props.handleTypes = cudaMemHandleTypeNone;
  props.location.type = cudaMemLocationTypeDevice;
  props.location.id = dev;
  cudaMemPool_t p = nullptr;
  if (cudaMemPoolCreate(&p, &props) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  uint64_t keep = ~0ull;
  cudaMemPoolSetAttribute(p, cudaMemPoolAttrReleaseThreshold, &keep);
  cudaGetLastError();
  g_pool[dev] = p;
  return p;
}

}  // namespace

cudaError_t dev_alloc(void** ptr, size_t bytes, cudaStream_t s) {
  int dev = -1;
  cudaMemPool_t p = pool_of_current_device(&dev);
  if (!p) return cudaMallocAsync(ptr, bytes, s);
  cudaError_t e = cudaMallocFromPoolAsync(ptr, bytes, p, s);
  if (e == cudaErrorMemoryAllocation) {
    // memory held by the pool but not in use goes back before giving up
    cudaGetLastError();
    cudaStreamSynchronize(s);
    cudaMemPoolTrimTo(p, 0);
    e = cudaMallocFromPoolAsync(ptr, bytes, p, s);
  }
  return e;
}

cudaError_t dev_free(void* ptr, cudaStream_t s) { return cudaFreeAsync(ptr, s); }

}  // namespace smc
