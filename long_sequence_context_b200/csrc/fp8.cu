// fp8.cu -- e4m3 inputs for the FP8 ring-attention forward ("Megatron-LM source
// analysis: Context Parallel", section 4: FP8 attention under context
// parallelism, to save memory): the per-tensor maximum |x|, the quantiser and
// the C entry points of the FP8 path.
//
// Quantisation (per tensor): s = 448 / max|x| in fp32 (1 for an all-zero
// tensor), code = e4m3(fp32(x * s)), rounded to nearest even and saturated to
// +-448 by the hardware conversion.  The value a code stands for is code / s.
// V is written transposed per head ([B][H][D][S]) so that the P.V product of
// the tensor-core kernel takes both operands K-major.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>

#include "cpattn.h"
#include "kernels.h"

namespace cpattn {
namespace {

template <typename T>
__device__ __forceinline__ float ld(const T* p, long i);
template <>
__device__ __forceinline__ float ld<float>(const float* p, long i) { return p[i]; }
template <>
__device__ __forceinline__ float ld<__nv_bfloat16>(const __nv_bfloat16* p, long i) {
  return __bfloat162float(p[i]);
}

// max|x| over n elements into *amax (which the launcher zeroes first): per
// thread, then warp, then block, then one atomicMax on the bit pattern
// (non-negative floats order like their bits).
template <typename T>
__global__ void __launch_bounds__(256) amax_kernel(const T* __restrict__ x, long n,
                                                   unsigned* __restrict__ amax) {
  float m = 0.f;
  for (long i = (long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long)gridDim.x * blockDim.x)
    m = fmaxf(m, fabsf(ld(x, i)));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  __shared__ float wm[8];
  if ((threadIdx.x & 31) == 0) wm[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    float b = wm[0];
    for (int w = 1; w < 8; ++w) b = fmaxf(b, wm[w]);
    atomicMax(amax, __float_as_uint(b));
  }
}

__device__ __forceinline__ float scale_from(const float* amax) {
  const float a = *amax;
  return a > 0.f ? __fdiv_rn(448.f, a) : 1.f;
}

__device__ __forceinline__ uint16_t e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// codes in the input's layout: 8 elements (8 bytes out) per thread
template <typename T>
__global__ void __launch_bounds__(256) quant_kernel(const T* __restrict__ x, long n8,
                                                    const float* __restrict__ amax,
                                                    uint2* __restrict__ out) {
  const float s = scale_from(amax);
  for (long i = (long)blockIdx.x * blockDim.x + threadIdx.x; i < n8; i += (long)gridDim.x * blockDim.x) {
    float f[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) f[e] = __fmul_rn(ld(x, 8 * i + e), s);
    uint2 o;
    o.x = (uint32_t)e4m3x2(f[0], f[1]) | ((uint32_t)e4m3x2(f[2], f[3]) << 16);
    o.y = (uint32_t)e4m3x2(f[4], f[5]) | ((uint32_t)e4m3x2(f[6], f[7]) << 16);
    out[i] = o;
  }
}

// codes transposed per head: x [BH][S][D] -> out [BH][D][S].  A block takes 64
// rows of one head: reads them row-wise (coalesced), writes 64-byte runs of
// every d column (coalesced) through a shared-memory tile.
template <typename T, int D>
__global__ void __launch_bounds__(256) quant_t_kernel(const T* __restrict__ x, int S,
                                                      const float* __restrict__ amax,
                                                      uint8_t* __restrict__ out) {
  __shared__ uint8_t tile[D][64 + 4];
  const float s = scale_from(amax);
  const long bh = blockIdx.y;
  const int s0 = blockIdx.x * 64;
  const T* src = x + (bh * S + s0) * (long)D;
  for (int idx = threadIdx.x; idx < 64 * D / 2; idx += blockDim.x) {
    const int r = (2 * idx) / D, d = (2 * idx) % D;
    const uint16_t c = e4m3x2(__fmul_rn(ld(src, (long)r * D + d), s),
                              __fmul_rn(ld(src, (long)r * D + d + 1), s));
    tile[d][r] = (uint8_t)(c & 0xFF);
    tile[d + 1][r] = (uint8_t)(c >> 8);
  }
  __syncthreads();
  uint8_t* dst = out + (bh * D) * (long)S + s0;
  for (int idx = threadIdx.x; idx < D * 16; idx += blockDim.x) {
    const int d = idx / 16, w = idx % 16;  // 16 words of 4 bytes per d row
    const uint32_t v = (uint32_t)tile[d][4 * w] | ((uint32_t)tile[d][4 * w + 1] << 8) |
                       ((uint32_t)tile[d][4 * w + 2] << 16) | ((uint32_t)tile[d][4 * w + 3] << 24);
    *reinterpret_cast<uint32_t*>(dst + (long)d * S + 4 * w) = v;
  }
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace cpattn

using namespace cpattn;

extern "C" {

int cpattn_amax(const void* x, long n, int dtype, float* amax, void* stream) {
  NvtxRange nv("cpattn_amax");
  if (dtype != CPATTN_BF16 && dtype != CPATTN_FP32) return CPATTN_ERR_DTYPE;
  if (n < 0) return CPATTN_ERR_SHAPE;
  if (!amax || (n > 0 && !x)) return CPATTN_ERR_ARG;
  if ((reinterpret_cast<uintptr_t>(amax) & 3u) != 0) return CPATTN_ERR_ALIGN;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(amax, 0, sizeof(float), s) != cudaSuccess) return CPATTN_ERR_CUDA;
  if (n == 0) return CPATTN_OK;
  int dev = 0;
  cudaGetDevice(&dev);
  const long blocks = std::min<long>((n + 255) / 256, (long)num_sms(dev) * 8);
  unsigned* a = reinterpret_cast<unsigned*>(amax);
  prof_begin(kKQuant, s);
  if (dtype == CPATTN_BF16)
    amax_kernel<__nv_bfloat16><<<(unsigned)blocks, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(x), n, a);
  else
    amax_kernel<float><<<(unsigned)blocks, 256, 0, s>>>(static_cast<const float*>(x), n, a);
  prof_end(kKQuant, s);
  if (cudaGetLastError() != cudaSuccess) return CPATTN_ERR_CUDA;
  add_launches(1);
  return CPATTN_OK;
}

int cpattn_quantize_e4m3(const void* x, int dtype, int BH, int S, int D, int transpose,
                         const float* amax, uint8_t* out, void* stream) {
  NvtxRange nv("cpattn_quantize_e4m3");
  if (dtype != CPATTN_BF16 && dtype != CPATTN_FP32) return CPATTN_ERR_DTYPE;
  if (BH < 1 || S < 1 || (D != 64 && D != 128)) return CPATTN_ERR_SHAPE;
  if (BH > 65535) return CPATTN_ERR_SHAPE;
  if (transpose && S % 64 != 0) return CPATTN_ERR_SHAPE;
  if (!x || !amax || !out) return CPATTN_ERR_ARG;
  if (!aligned16(x) || !aligned16(out) || (reinterpret_cast<uintptr_t>(amax) & 3u))
    return CPATTN_ERR_ALIGN;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const long n = (long)BH * S * D;
  int dev = 0;
  cudaGetDevice(&dev);
  prof_begin(kKQuant, s);
  if (!transpose) {
    const long n8 = n / 8;
    const long blocks = std::min<long>((n8 + 255) / 256, (long)num_sms(dev) * 16);
    if (dtype == CPATTN_BF16)
      quant_kernel<__nv_bfloat16><<<(unsigned)blocks, 256, 0, s>>>(
          static_cast<const __nv_bfloat16*>(x), n8, amax, reinterpret_cast<uint2*>(out));
    else
      quant_kernel<float><<<(unsigned)blocks, 256, 0, s>>>(static_cast<const float*>(x), n8, amax,
                                                           reinterpret_cast<uint2*>(out));
  } else {
    const dim3 grid(S / 64, BH);
    if (dtype == CPATTN_BF16) {
      const auto* xb = static_cast<const __nv_bfloat16*>(x);
      if (D == 64) quant_t_kernel<__nv_bfloat16, 64><<<grid, 256, 0, s>>>(xb, S, amax, out);
      else quant_t_kernel<__nv_bfloat16, 128><<<grid, 256, 0, s>>>(xb, S, amax, out);
    } else {
      const auto* xf = static_cast<const float*>(x);
      if (D == 64) quant_t_kernel<float, 64><<<grid, 256, 0, s>>>(xf, S, amax, out);
      else quant_t_kernel<float, 128><<<grid, 256, 0, s>>>(xf, S, amax, out);
    }
  }
  prof_end(kKQuant, s);
  if (cudaGetLastError() != cudaSuccess) return CPATTN_ERR_CUDA;
  add_launches(1);
  return CPATTN_OK;
}

int cpattn_fwd_fp8(const uint8_t* q8, const uint8_t* k8, const uint8_t* vt8, const float* amax,
                   void* o, float* lse, int B, int H, int S, int D, int cp_size, int causal,
                   float scale, void* stream) {
  NvtxRange nv("cpattn_fwd_fp8");
  int st = check_attention_shape(B, H, S, D, cp_size, causal, scale, CPATTN_BF16);
  if (st != CPATTN_OK) return st;
  if (D != 128) return CPATTN_ERR_SHAPE;
  const int n_chunks = causal ? 2 * cp_size : cp_size;
  if ((S / n_chunks) % 128 != 0) return CPATTN_ERR_SHAPE;
  if ((long long)B * H * S >= (1LL << 31)) return CPATTN_ERR_SHAPE;
  if (!q8 || !k8 || !vt8 || !amax || !o || !lse) return CPATTN_ERR_ARG;
  if (!aligned16(q8) || !aligned16(k8) || !aligned16(vt8) || !aligned16(o) || !aligned16(lse) ||
      (reinterpret_cast<uintptr_t>(amax) & 3u))
    return CPATTN_ERR_ALIGN;
  unsigned* err = device_error_word();
  if (!err) return CPATTN_ERR_CUDA;
  AttnShape sh;
  sh.B = B;
  sh.H = H;
  sh.S = S;
  sh.D = D;
  sh.g = make_geom(S, cp_size, causal);
  sh.scale = scale;
  sh.bf16 = 1;
  const int n = launch_tc_fwd_fp8(sh, q8, k8, vt8, amax, o, lse, err, static_cast<cudaStream_t>(stream));
  if (n < 0) return CPATTN_ERR_CUDA;
  add_launches(n);
  return CPATTN_OK;
}

}  // extern "C"
