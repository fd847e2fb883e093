// SubMConv3d on the CUDA cores, for fp32 features and for channel counts the
// tensor-core kernel does not tile (cin or cout not a multiple of 64).
//
// out[i][co] = sum over taps k with nbr[i][k] = j >= 0 of
//              sum_ci feats[j][ci] * W[k][ci][co]
// (trellis_sparse_mlx README, "What's in it" / "Correctness": the output at
// each input voxel sums feats[c+d] @ W[d] over its active neighbours.)
// Accumulation runs in tap order, then input-channel order: in fp64 for fp32
// features (so the fp32 result is the exact sum rounded once), in fp32 FMA for
// fp16/bf16 features.  The optional epilogue act(acc + bias) + residual runs
// in the accumulator's precision before the one rounding.  One thread
// per (row, output channel); a block is 32 output channels x 8 rows, so the
// weight reads of a warp are consecutive and the feature reads are broadcasts.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "smc_internal.h"

namespace smc {
namespace {

template <class T>
__device__ __forceinline__ float to_f(T v);
template <>
__device__ __forceinline__ float to_f<float>(float v) {
  return v;
}
template <>
__device__ __forceinline__ float to_f<__half>(__half v) {
  return __half2float(v);
}
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 v) {
  return __bfloat162float(v);
}
template <class T>
__device__ __forceinline__ T from_f(float v);
template <>
__device__ __forceinline__ float from_f<float>(float v) {
  return v;
}
template <>
__device__ __forceinline__ __half from_f<__half>(float v) {
  return __float2half_rn(v);
}
template <>
__device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}

template <class T>
struct Acc {
  using type = float;
};
template <>
struct Acc<float> {
  using type = double;
};

__device__ __forceinline__ float act_apply(float v, int act) {
  switch (act) {
    case SMC_ACT_RELU:
      return fmaxf(v, 0.f);
    case SMC_ACT_SILU:
      return v / (1.f + expf(-v));
    case SMC_ACT_GELU:
      return 0.5f * v * (1.f + erff(v * 0.7071067811865476f));
    default:
      return v;
  }
}
__device__ __forceinline__ double act_apply(double v, int act) {
  switch (act) {
    case SMC_ACT_RELU:
      return fmax(v, 0.0);
    case SMC_ACT_SILU:
      return v / (1.0 + exp(-v));
    case SMC_ACT_GELU:
      return 0.5 * v * (1.0 + erf(v * 0.7071067811865476));
    default:
      return v;
  }
}

template <class T>
__global__ void __launch_bounds__(256)
k_conv_simt(const T* __restrict__ feats, const T* __restrict__ W, T* __restrict__ out,
            const int32_t* __restrict__ nbr, int64_t n, int cin, int cout, int dense,
            const T* __restrict__ bias, const T* __restrict__ residual, int act) {
  const int64_t i = blockIdx.x * int64_t(blockDim.y) + threadIdx.y;
  const int co = blockIdx.y * blockDim.x + threadIdx.x;
  if (i >= n || co >= cout) return;
  using A = typename Acc<T>::type;
  A acc = A(0);
  const int taps = dense ? 1 : kTaps;
  for (int k = 0; k < taps; ++k) {
    const int64_t j = dense ? i : int64_t(nbr[i * kTaps + k]);
    if (j < 0) continue;
    const T* f = feats + j * cin;
    const T* w = W + int64_t(k) * cin * cout + co;
    for (int ci = 0; ci < cin; ++ci)
      acc = fma(A(to_f(f[ci])), A(to_f(w[int64_t(ci) * cout])), acc);
  }
  if (bias) acc += A(to_f(bias[co]));
  acc = act_apply(acc, act);
  if (residual) acc += A(to_f(residual[i * cout + co]));
  out[i * cout + co] = from_f<T>(float(acc));
}

template <class T>
int launch_t(const Plan& plan, bool dense, const void* feats, const void* W, void* out, int cin,
             int cout, const Epilogue& ep, cudaStream_t stream) {
  dim3 block(32, 8);
  dim3 grid(unsigned((plan.n + 7) / 8), unsigned((cout + 31) / 32));
  k_conv_simt<T><<<grid, block, 0, stream>>>(
      static_cast<const T*>(feats), static_cast<const T*>(W), static_cast<T*>(out), plan.nbr,
      plan.n, cin, cout, dense ? 1 : 0, static_cast<const T*>(ep.bias),
      static_cast<const T*>(ep.residual), ep.act);
  return cudaGetLastError() == cudaSuccess ? SMC_OK : SMC_ERR_CUDA;
}

}  // namespace

int launch_conv_simt(const Plan& plan, bool dense, const void* feats, const void* W, void* out,
                     int cin, int cout, int dtype, const Epilogue& ep, cudaStream_t stream) {
  if (plan.n == 0) return SMC_OK;
  switch (dtype) {
    case SMC_F32:
      return launch_t<float>(plan, dense, feats, W, out, cin, cout, ep, stream);
    case SMC_F16:
      return launch_t<__half>(plan, dense, feats, W, out, cin, cout, ep, stream);
    case SMC_BF16:
      return launch_t<__nv_bfloat16>(plan, dense, feats, W, out, cin, cout, ep, stream);
    default:
      return SMC_ERR_INVALID;
  }
}

}  // namespace smc
