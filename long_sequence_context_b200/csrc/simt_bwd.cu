// simt_bwd.cu -- CUDA-core recompute backward (fp32 problems and bf16 shapes
// outside the tcgen05 kernels).  Three launches, no atomics:
//   1. delta_i = sum_d dO_id O_id                      (one warp per row)
//   2. dK, dV: a block owns 16 keys and walks, in ring order, every q row that
//      sees them (the mirror of the forward ring: at step t the keys' K/V sit
//      on rank owner + t), recomputing P = exp(s - LSE), dP = dO.v,
//      dS = P (dP - delta), dV += P dO, dK += scale dS q
//   3. dQ: a block owns 16 q rows and walks their K/V blocks in forward ring
//      order, dQ += scale dS k.
// Ring rule and block kinds: ring.cuh ("Configuring RingAttention+
// FlashAttention for CP", section 3 code and note 2, section 5 item 1).
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "kernels.h"

namespace cpattn {

namespace {

constexpr float kLog2e = 1.4426950408889634f;

template <typename T>
__device__ __forceinline__ float ld_f(const T* p, long i);
template <>
__device__ __forceinline__ float ld_f<float>(const float* p, long i) { return p[i]; }
template <>
__device__ __forceinline__ float ld_f<__nv_bfloat16>(const __nv_bfloat16* p, long i) {
  return __bfloat162float(p[i]);
}
template <typename T>
__device__ __forceinline__ void st_f(T* p, long i, float x);
template <>
__device__ __forceinline__ void st_f<float>(float* p, long i, float x) { p[i] = x; }
template <>
__device__ __forceinline__ void st_f<__nv_bfloat16>(__nv_bfloat16* p, long i, float x) {
  p[i] = __float2bfloat16_rn(x);
}

// sum over the 8 lanes of an aligned group
__device__ __forceinline__ float group8_sum(float x) {
  x += __shfl_xor_sync(0xffffffffu, x, 1);
  x += __shfl_xor_sync(0xffffffffu, x, 2);
  x += __shfl_xor_sync(0xffffffffu, x, 4);
  return x;
}

template <typename T, int D>
__global__ void delta_kernel(const T* __restrict__ o, const T* __restrict__ dout,
                             float* __restrict__ delta, long rows) {
  const long row = (long)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  float acc = 0.f;
  for (int d = lane; d < D; d += 32) acc += ld_f(o, row * D + d) * ld_f(dout, row * D + d);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (lane == 0) delta[row] = acc;
}

// Output of one gradient element: written in the tensor's dtype, or, in
// accumulate mode (acc != nullptr), added to the fp32 accumulator.  Each
// element belongs to one thread of the launch.
template <typename T>
__device__ __forceinline__ void out_f(T* p, float* acc, long i, float x) {
  if (acc)
    acc[i] += x;
  else
    st_f(p, i, x);
}

constexpr int kTile = 16;   // keys (dK/dV kernel) or rows (dQ kernel) per block
constexpr int kBatch = 8;   // rows / keys staged in shared memory at a time

// grid (n_chunks * ceil(c/16), B*H), block 128: thread = (key t/8, d-slice t%8).
// Block x owns keys [j0, j0 + 16) of kv chunk x / ceil(c/16); keys at or past
// the chunk's end read no input and write nothing.
template <typename T, int D>
__global__ void __launch_bounds__(128) dkdv_kernel(const T* __restrict__ q, const T* __restrict__ k,
                                                   const T* __restrict__ v,
                                                   const float* __restrict__ lse,
                                                   const T* __restrict__ dout,
                                                   const float* __restrict__ delta,
                                                   T* __restrict__ dk, T* __restrict__ dv,
                                                   float* __restrict__ dk_acc_out,
                                                   float* __restrict__ dv_acc_out,
                                                   RingGeom g, float scale) {
  constexpr int SL = D / 8;
  __shared__ float Qs[kBatch][D], dOs[kBatch][D], Ls[kBatch], Ds[kBatch];
  const long bh = blockIdx.y;
  const long base = bh * (long)g.S * D;
  const int bpc = (g.c + kTile - 1) / kTile;
  const int b = blockIdx.x / bpc;         // kv chunk of these keys
  const int j0 = b * g.c + (blockIdx.x % bpc) * kTile;
  const int kj = threadIdx.x / 8, sl = threadIdx.x % 8;
  const int key = j0 + kj;
  const bool key_in = key < (b + 1) * g.c;
  float kr[SL], vr[SL], dk_acc[SL], dv_acc[SL];
#pragma unroll
  for (int i = 0; i < SL; ++i) {
    kr[i] = key_in ? ld_f(k, base + (long)key * D + sl * SL + i) : 0.f;
    vr[i] = key_in ? ld_f(v, base + (long)key * D + sl * SL + i) : 0.f;
    dk_acc[i] = 0.f;
    dv_acc[i] = 0.f;
  }
  const float scale_log2 = scale * kLog2e;
  const int owner = chunk_owner(g, b);    // rank whose K/V these are
  for (int t = 0; t < g.N; ++t) {
    const int r = (owner + t) % g.N;      // rank holding this K/V at step t
    for (int s = 0; s < slots(g); ++s) {
      const int a = rank_chunk(g, r, s);
      const int kind = block_kind(g, a, b);
      if (kind == kSkip) continue;
      int i0 = a * g.c;
      if (kind == kDiag && i0 < j0) i0 = j0;  // rows before the first key see none of them
      const int i1 = (a + 1) * g.c;
      for (int ib = i0; ib < i1; ib += kBatch) {
        __syncthreads();
        for (int idx = threadIdx.x; idx < kBatch * D; idx += blockDim.x) {
          const int rr = idx / D, d = idx % D;
          const bool in = ib + rr < i1;
          Qs[rr][d] = in ? ld_f(q, base + (long)(ib + rr) * D + d) : 0.f;
          dOs[rr][d] = in ? ld_f(dout, base + (long)(ib + rr) * D + d) : 0.f;
        }
        if (threadIdx.x < kBatch) {
          const bool in = ib + threadIdx.x < i1;
          Ls[threadIdx.x] = in ? lse[bh * g.S + ib + threadIdx.x] : INFINITY;
          Ds[threadIdx.x] = in ? delta[bh * g.S + ib + threadIdx.x] : 0.f;
        }
        __syncthreads();
        for (int rr = 0; rr < kBatch; ++rr) {
          const int row = ib + rr;
          float sdot = 0.f, pdot = 0.f;
#pragma unroll
          for (int i = 0; i < SL; ++i) {
            sdot = fmaf(Qs[rr][sl * SL + i], kr[i], sdot);
            pdot = fmaf(dOs[rr][sl * SL + i], vr[i], pdot);
          }
          sdot = group8_sum(sdot);
          pdot = group8_sum(pdot);
          const bool valid = row < i1 && (kind != kDiag || key <= row);
          const float p = valid ? exp2f(sdot * scale_log2 - Ls[rr] * kLog2e) : 0.f;
          const float ds = p * (pdot - Ds[rr]);
#pragma unroll
          for (int i = 0; i < SL; ++i) {
            dv_acc[i] = fmaf(p, dOs[rr][sl * SL + i], dv_acc[i]);
            dk_acc[i] = fmaf(ds, Qs[rr][sl * SL + i], dk_acc[i]);
          }
        }
      }
    }
  }
  if (!key_in) return;
#pragma unroll
  for (int i = 0; i < SL; ++i) {
    out_f(dk, dk_acc_out, base + (long)key * D + sl * SL + i, dk_acc[i] * scale);
    out_f(dv, dv_acc_out, base + (long)key * D + sl * SL + i, dv_acc[i]);
  }
}

// grid (n_chunks * ceil(c/16), B*H), block 128: thread = (row t/8, d-slice t%8).
// Block x owns rows [i0, i0 + 16) of q chunk x / ceil(c/16); rows at or past
// the chunk's end read no input and write nothing.
template <typename T, int D>
__global__ void __launch_bounds__(128) dq_kernel(const T* __restrict__ q, const T* __restrict__ k,
                                                 const T* __restrict__ v,
                                                 const float* __restrict__ lse,
                                                 const T* __restrict__ dout,
                                                 const float* __restrict__ delta,
                                                 T* __restrict__ dq, float* __restrict__ dq_acc_out,
                                                 RingGeom g, float scale) {
  constexpr int SL = D / 8;
  __shared__ float Ks[kBatch][D], Vs[kBatch][D];
  const long bh = blockIdx.y;
  const long base = bh * (long)g.S * D;
  const int bpc = (g.c + kTile - 1) / kTile;
  const int a = blockIdx.x / bpc;  // q chunk of these rows
  const int i0 = a * g.c + (blockIdx.x % bpc) * kTile;
  const int ri = threadIdx.x / 8, sl = threadIdx.x % 8;
  const int row = i0 + ri;
  const bool row_in = row < (a + 1) * g.c;
  float qr[SL], dor[SL], acc[SL];
#pragma unroll
  for (int i = 0; i < SL; ++i) {
    qr[i] = row_in ? ld_f(q, base + (long)row * D + sl * SL + i) : 0.f;
    dor[i] = row_in ? ld_f(dout, base + (long)row * D + sl * SL + i) : 0.f;
    acc[i] = 0.f;
  }
  const float lse2 = row_in ? lse[bh * g.S + row] * kLog2e : INFINITY;
  const float dlt = row_in ? delta[bh * g.S + row] : 0.f;
  const float scale_log2 = scale * kLog2e;
  const int rank = chunk_owner(g, a);
  for (int t = 0; t < g.N; ++t) {
    const int src = step_src(g, rank, t);
    for (int s = 0; s < slots(g); ++s) {
      const int b = rank_chunk(g, src, s);
      const int kind = block_kind(g, a, b);
      if (kind == kSkip) continue;
      const int jb = b * g.c;
      int je = jb + g.c;
      if (kind == kDiag && je > i0 + kTile) je = i0 + kTile;
      for (int kb = jb; kb < je; kb += kBatch) {
        __syncthreads();
        for (int idx = threadIdx.x; idx < kBatch * D; idx += blockDim.x) {
          const int jj = idx / D, d = idx % D;
          const bool in = kb + jj < je;
          Ks[jj][d] = in ? ld_f(k, base + (long)(kb + jj) * D + d) : 0.f;
          Vs[jj][d] = in ? ld_f(v, base + (long)(kb + jj) * D + d) : 0.f;
        }
        __syncthreads();
        for (int jj = 0; jj < kBatch; ++jj) {
          const int key = kb + jj;
          float sdot = 0.f, pdot = 0.f;
#pragma unroll
          for (int i = 0; i < SL; ++i) {
            sdot = fmaf(qr[i], Ks[jj][sl * SL + i], sdot);
            pdot = fmaf(dor[i], Vs[jj][sl * SL + i], pdot);
          }
          sdot = group8_sum(sdot);
          pdot = group8_sum(pdot);
          const bool valid = key < je && (kind != kDiag || key <= row);
          const float p = valid ? exp2f(sdot * scale_log2 - lse2) : 0.f;
          const float ds = p * (pdot - dlt);
#pragma unroll
          for (int i = 0; i < SL; ++i) acc[i] = fmaf(ds, Ks[jj][sl * SL + i], acc[i]);
        }
      }
    }
  }
  if (!row_in) return;
#pragma unroll
  for (int i = 0; i < SL; ++i) out_f(dq, dq_acc_out, base + (long)row * D + sl * SL + i, acc[i] * scale);
}

template <typename T, int D>
int run_bwd(const AttnShape& sh, const void* q, const void* k, const void* v, const void* o,
            const float* lse, const void* dout, void* dq, void* dk, void* dv, float* ws_delta,
            int acc_f32, cudaStream_t stream) {
  const long rows = (long)sh.B * sh.H * sh.S;
  const T* Q = static_cast<const T*>(q);
  const T* K = static_cast<const T*>(k);
  const T* V = static_cast<const T*>(v);
  const T* O = static_cast<const T*>(o);
  const T* dO = static_cast<const T*>(dout);
  prof_begin(kKDelta, stream);
  delta_kernel<T, D><<<(unsigned)((rows + 7) / 8), 256, 0, stream>>>(O, dO, ws_delta, rows);
  prof_end(kKDelta, stream);
  if (cudaGetLastError() != cudaSuccess) return -1;
  dim3 grid(sh.g.n_chunks * ((sh.g.c + kTile - 1) / kTile), sh.B * sh.H);
  prof_begin(kKSimtDkdv, stream);
  float* acc_dk = acc_f32 ? static_cast<float*>(dk) : nullptr;
  float* acc_dv = acc_f32 ? static_cast<float*>(dv) : nullptr;
  float* acc_dq = acc_f32 ? static_cast<float*>(dq) : nullptr;
  dkdv_kernel<T, D><<<grid, 128, 0, stream>>>(Q, K, V, lse, dO, ws_delta,
                                              acc_f32 ? nullptr : static_cast<T*>(dk),
                                              acc_f32 ? nullptr : static_cast<T*>(dv), acc_dk,
                                              acc_dv, sh.g, sh.scale);
  prof_end(kKSimtDkdv, stream);
  if (cudaGetLastError() != cudaSuccess) return -1;
  prof_begin(kKSimtDq, stream);
  dq_kernel<T, D><<<grid, 128, 0, stream>>>(Q, K, V, lse, dO, ws_delta,
                                            acc_f32 ? nullptr : static_cast<T*>(dq), acc_dq, sh.g,
                                            sh.scale);
  prof_end(kKSimtDq, stream);
  if (cudaGetLastError() != cudaSuccess) return -1;
  return 3;
}

}  // namespace

int launch_simt_bwd(const AttnShape& sh, const void* q, const void* k, const void* v,
                    const void* o, const float* lse, const void* dout, void* dq, void* dk,
                    void* dv, float* ws_delta, int acc_f32, cudaStream_t stream) {
  if (sh.bf16) {
    if (sh.D == 64)
      return run_bwd<__nv_bfloat16, 64>(sh, q, k, v, o, lse, dout, dq, dk, dv, ws_delta, acc_f32,
                                        stream);
    return run_bwd<__nv_bfloat16, 128>(sh, q, k, v, o, lse, dout, dq, dk, dv, ws_delta, acc_f32,
                                       stream);
  }
  if (sh.D == 64)
    return run_bwd<float, 64>(sh, q, k, v, o, lse, dout, dq, dk, dv, ws_delta, acc_f32, stream);
  return run_bwd<float, 128>(sh, q, k, v, o, lse, dout, dq, dk, dv, ws_delta, acc_f32, stream);
}

}  // namespace cpattn
