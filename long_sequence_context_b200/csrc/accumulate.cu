// accumulate.cu -- acc[i] += x[i] with fp32 accumulators: the gradient sums of
// the multi-rank ring backward, where every (q chunk, kv chunk) block adds its
// dQ, dK, dV terms into running sums ("Megatron-LM source analysis: Context
// Parallel", section 2: the backward mirrors the forward's exchange, each
// block contributing to the gradients of its q and kv chunks).
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>

#include "cpattn.h"
#include "kernels.h"

namespace cpattn {
namespace {

// 4 elements per thread (n % 4 == 0 and 16-byte aligned pointers are checked by the caller)
template <typename T>
__global__ void __launch_bounds__(256) accumulate_kernel(float* __restrict__ acc, const T* __restrict__ x,
                                                        long n4) {
  for (long i = (long)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += (long)gridDim.x * blockDim.x) {
    float4 a = reinterpret_cast<float4*>(acc)[i];
    float v[4];
    if constexpr (sizeof(T) == 4) {
      const float4 b = reinterpret_cast<const float4*>(x)[i];
      v[0] = b.x; v[1] = b.y; v[2] = b.z; v[3] = b.w;
    } else {
      const uint2 b = reinterpret_cast<const uint2*>(x)[i];
      const __nv_bfloat162 lo = *reinterpret_cast<const __nv_bfloat162*>(&b.x);
      const __nv_bfloat162 hi = *reinterpret_cast<const __nv_bfloat162*>(&b.y);
      v[0] = __low2float(lo); v[1] = __high2float(lo); v[2] = __low2float(hi); v[3] = __high2float(hi);
    }
    a.x += v[0]; a.y += v[1]; a.z += v[2]; a.w += v[3];
    reinterpret_cast<float4*>(acc)[i] = a;
  }
}

}  // namespace
}  // namespace cpattn

using namespace cpattn;

extern "C" int cpattn_accumulate(float* acc, const void* x, long n, int dtype, void* stream) {
  NvtxRange nv("cpattn_accumulate");
  if (dtype != CPATTN_BF16 && dtype != CPATTN_FP32) return CPATTN_ERR_DTYPE;
  if (n < 0 || n % 4 != 0) return CPATTN_ERR_SHAPE;
  if (n == 0) return CPATTN_OK;
  if (!acc || !x) return CPATTN_ERR_ARG;
  if ((reinterpret_cast<uintptr_t>(acc) & 15u) || (reinterpret_cast<uintptr_t>(x) & 15u))
    return CPATTN_ERR_ALIGN;
  int dev = 0;
  cudaGetDevice(&dev);
  const long n4 = n / 4;
  const long blocks = std::min<long>((n4 + 255) / 256, (long)num_sms(dev) * 16);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  prof_begin(kKAccumulate, s);
  if (dtype == CPATTN_BF16)
    accumulate_kernel<__nv_bfloat16><<<(unsigned)blocks, 256, 0, s>>>(acc, static_cast<const __nv_bfloat16*>(x), n4);
  else
    accumulate_kernel<float><<<(unsigned)blocks, 256, 0, s>>>(acc, static_cast<const float*>(x), n4);
  prof_end(kKAccumulate, s);
  if (cudaGetLastError() != cudaSuccess) return CPATTN_ERR_CUDA;
  add_launches(1);
  return CPATTN_OK;
}
