// simt_fwd.cu -- CUDA-core (no tensor core) kernels for the ring forward, the
// standalone log-sum-exp merge and the fp32 -> dtype finalisation.
//
// These carry fp32 problems at full fp32 precision (tf32 tensor-core MMAs
// cannot hold a 1e-4 error bar) and any bf16 shape the tcgen05 kernels do not
// take.  Ring walk and block kinds come from ring.cuh ("Configuring
// RingAttention+FlashAttention for CP", section 3 code and note 2; section 5,
// item 1 for the zigzag).
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "kernels.h"

namespace cpattn {

namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

template <typename T>
__device__ __forceinline__ float to_f(T x);
template <>
__device__ __forceinline__ float to_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

constexpr int kRowsPerBlock = 16;  // 4 warps x 4 rows, all in one chunk (rows past its end idle)
constexpr int kRowsPerWarp = 4;
constexpr int kKeyTile = 32;       // one key per lane

// grid: (n_chunks * ceil(c / 16), B*H), block 128.  Block x covers rows
// [row0, row0 + 16) of chunk x / ceil(c / 16); rows at or past the chunk's end
// read no input and write nothing, so any chunk length c works.  Steps
// [t0, t1) of the ring; online softmax in the log2 domain across every
// non-SKIP block.
template <typename T, int D>
__global__ void __launch_bounds__(128) simt_fwd_kernel(const T* __restrict__ q,
                                                       const T* __restrict__ k,
                                                       const T* __restrict__ v, void* o_out,
                                                       float* __restrict__ lse_out, RingGeom g,
                                                       float scale_log2, int t0, int t1,
                                                       int final_out) {
  constexpr int DW = D / 32;  // output columns per lane
  __shared__ float Qs[kRowsPerBlock][D];
  __shared__ float Ks[kKeyTile][D + 1];
  __shared__ float Vs[kKeyTile][D];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long bh = blockIdx.y;
  const int bpc = (g.c + kRowsPerBlock - 1) / kRowsPerBlock;  // blocks per chunk
  const int a = blockIdx.x / bpc;       // q chunk of this block
  const int row0 = a * g.c + (blockIdx.x % bpc) * kRowsPerBlock;
  const int row_end = (a + 1) * g.c;    // rows at or past it belong to the next chunk
  const long base = bh * (long)g.S * D;

  for (int idx = threadIdx.x; idx < kRowsPerBlock * D; idx += blockDim.x)
    Qs[idx / D][idx % D] = (row0 + idx / D < row_end) ? to_f(q[base + (long)row0 * D + idx]) : 0.f;

  float m[kRowsPerWarp], l[kRowsPerWarp], acc[kRowsPerWarp][DW];
#pragma unroll
  for (int r = 0; r < kRowsPerWarp; ++r) {
    m[r] = -INFINITY;
    l[r] = 0.f;
#pragma unroll
    for (int i = 0; i < DW; ++i) acc[r][i] = 0.f;
  }

  const int rank = chunk_owner(g, a);   // virtual rank holding it
  for (int t = t0; t < t1; ++t) {
    const int src = step_src(g, rank, t);
    for (int s = 0; s < slots(g); ++s) {
      const int b = rank_chunk(g, src, s);
      const int kind = block_kind(g, a, b);
      if (kind == kSkip) continue;
      const int kb = b * g.c;
      int ke = kb + g.c;
      if (kind == kDiag && ke > row0 + kRowsPerBlock) ke = row0 + kRowsPerBlock;
      for (int kt = kb; kt < ke; kt += kKeyTile) {
        __syncthreads();
        for (int idx = threadIdx.x; idx < kKeyTile * D; idx += blockDim.x) {
          const int j = idx / D, d = idx % D;
          const bool in = kt + j < ke;
          Ks[j][d] = in ? to_f(k[base + (long)(kt + j) * D + d]) : 0.f;
          Vs[j][d] = in ? to_f(v[base + (long)(kt + j) * D + d]) : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int r = 0; r < kRowsPerWarp; ++r) {
          const int lr = warp * kRowsPerWarp + r;
          const int row = row0 + lr;
          const int key = kt + lane;
          const bool valid = key < ke && (kind != kDiag || key <= row);
          float dot = 0.f;
#pragma unroll 8
          for (int d = 0; d < D; ++d) dot = fmaf(Qs[lr][d], Ks[lane][d], dot);
          const float sc = valid ? dot * scale_log2 : -INFINITY;
          const float mx = warp_max(sc);
          const float m_new = fmaxf(m[r], mx);
          if (m_new == -INFINITY) continue;  // nothing visible yet (warp-uniform)
          const float alpha = exp2f(m[r] - m_new);
          const float p = valid ? exp2f(sc - m_new) : 0.f;
          l[r] = l[r] * alpha + warp_sum(p);
#pragma unroll
          for (int i = 0; i < DW; ++i) acc[r][i] *= alpha;
          for (int j = 0; j < kKeyTile; ++j) {
            const float pj = __shfl_sync(0xffffffffu, p, j);
#pragma unroll
            for (int i = 0; i < DW; ++i) acc[r][i] = fmaf(pj, Vs[j][lane + 32 * i], acc[r][i]);
          }
          m[r] = m_new;
        }
      }
    }
  }

#pragma unroll
  for (int r = 0; r < kRowsPerWarp; ++r) {
    const int row = row0 + warp * kRowsPerWarp + r;
    if (row >= row_end) continue;  // warp-uniform: the four rows of a warp are consecutive
    const long ro = base + (long)row * D;
    const bool empty = (l[r] == 0.f);
    const float inv = empty ? 0.f : 1.f / l[r];
#pragma unroll
    for (int i = 0; i < DW; ++i) {
      const float val = acc[r][i] * inv;
      if (final_out) {
        if (sizeof(T) == 2)
          reinterpret_cast<__nv_bfloat16*>(o_out)[ro + lane + 32 * i] = __float2bfloat16_rn(val);
        else
          reinterpret_cast<float*>(o_out)[ro + lane + 32 * i] = val;
      } else {
        reinterpret_cast<float*>(o_out)[ro + lane + 32 * i] = val;
      }
    }
    if (lane == 0) lse_out[bh * g.S + row] = empty ? -INFINITY : (m[r] + log2f(l[r])) * kLn2;
  }
}

// One thread group of D/4 lanes per row, float4 accesses.
template <int D>
__global__ void __launch_bounds__(256) merge_kernel(float* __restrict__ o_acc,
                                                    float* __restrict__ lse_acc,
                                                    const float* __restrict__ o_part,
                                                    const float* __restrict__ lse_part,
                                                    long rows) {
  constexpr int TPR = D / 4;  // threads per row
  const long row = (long)blockIdx.x * (256 / TPR) + threadIdx.x / TPR;
  const int c4 = threadIdx.x % TPR;
  const bool active = row < rows;
  const float la = active ? lse_acc[row] : -INFINITY;
  const float lb = active ? lse_part[row] : -INFINITY;
  __syncwarp();  // every lane of the row has read lse_acc before it is rewritten
  if (!active || lb == -INFINITY) return;  // empty partial: accumulator unchanged
  float4* oa = reinterpret_cast<float4*>(o_acc + row * D) + c4;
  const float4 pb = reinterpret_cast<const float4*>(o_part + row * D)[c4];
  float wa, wb, lnew;
  if (la == -INFINITY) {
    wa = 0.f;
    wb = 1.f;
    lnew = lb;
  } else {
    const float mx = fmaxf(la, lb);
    lnew = mx + logf(expf(la - mx) + expf(lb - mx));
    wa = expf(la - lnew);
    wb = expf(lb - lnew);
  }
  float4 a4 = (la == -INFINITY) ? make_float4(0.f, 0.f, 0.f, 0.f) : *oa;
  a4.x = wa * a4.x + wb * pb.x;
  a4.y = wa * a4.y + wb * pb.y;
  a4.z = wa * a4.z + wb * pb.z;
  a4.w = wa * a4.w + wb * pb.w;
  *oa = a4;
  if (c4 == 0) lse_acc[row] = lnew;
}

__global__ void finalize_bf16_kernel(const float4* __restrict__ src, uint2* __restrict__ dst,
                                     long n4) {
  for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < n4;
       i += (long)gridDim.x * blockDim.x) {
    const float4 x = src[i];
    __nv_bfloat162 lo = __floats2bfloat162_rn(x.x, x.y);
    __nv_bfloat162 hi = __floats2bfloat162_rn(x.z, x.w);
    uint2 u;
    u.x = *reinterpret_cast<uint32_t*>(&lo);
    u.y = *reinterpret_cast<uint32_t*>(&hi);
    dst[i] = u;
  }
}

__global__ void copy_f4_kernel(const float4* __restrict__ src, float4* __restrict__ dst, long n4) {
  for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < n4;
       i += (long)gridDim.x * blockDim.x)
    dst[i] = src[i];
}

int grid_for(long n, int threads) {
  long b = (n + threads - 1) / threads;
  if (b > 148L * 32) b = 148L * 32;
  if (b < 1) b = 1;
  return (int)b;
}

}  // namespace

int launch_simt_fwd(const AttnShape& sh, const void* q, const void* k, const void* v, void* o,
                    float* lse, int t0, int t1, int final_out, unsigned* err,
                    cudaStream_t stream) {
  (void)err;
  const int bpc = (sh.g.c + kRowsPerBlock - 1) / kRowsPerBlock;
  dim3 grid(sh.g.n_chunks * bpc, sh.B * sh.H);
  const float sl2 = sh.scale * kLog2e;
  prof_begin(kKSimtFwd, stream);
  if (sh.bf16) {
    auto* qq = static_cast<const __nv_bfloat16*>(q);
    auto* kk = static_cast<const __nv_bfloat16*>(k);
    auto* vv = static_cast<const __nv_bfloat16*>(v);
    if (sh.D == 64)
      simt_fwd_kernel<__nv_bfloat16, 64><<<grid, 128, 0, stream>>>(qq, kk, vv, o, lse, sh.g, sl2, t0, t1, final_out);
    else
      simt_fwd_kernel<__nv_bfloat16, 128><<<grid, 128, 0, stream>>>(qq, kk, vv, o, lse, sh.g, sl2, t0, t1, final_out);
  } else {
    auto* qq = static_cast<const float*>(q);
    auto* kk = static_cast<const float*>(k);
    auto* vv = static_cast<const float*>(v);
    if (sh.D == 64)
      simt_fwd_kernel<float, 64><<<grid, 128, 0, stream>>>(qq, kk, vv, o, lse, sh.g, sl2, t0, t1, final_out);
    else
      simt_fwd_kernel<float, 128><<<grid, 128, 0, stream>>>(qq, kk, vv, o, lse, sh.g, sl2, t0, t1, final_out);
  }
  prof_end(kKSimtFwd, stream);
  return cudaGetLastError() == cudaSuccess ? 1 : -1;
}

int launch_merge(float* o_acc, float* lse_acc, const float* o_part, const float* lse_part,
                 long rows, int D, cudaStream_t stream) {
  if (rows == 0) return 0;
  const int rpb = 256 / (D / 4);
  const long blocks = (rows + rpb - 1) / rpb;
  prof_begin(kKMerge, stream);
  if (D == 64)
    merge_kernel<64><<<(unsigned)blocks, 256, 0, stream>>>(o_acc, lse_acc, o_part, lse_part, rows);
  else
    merge_kernel<128><<<(unsigned)blocks, 256, 0, stream>>>(o_acc, lse_acc, o_part, lse_part, rows);
  prof_end(kKMerge, stream);
  return cudaGetLastError() == cudaSuccess ? 1 : -1;
}

int launch_finalize(const float* o_acc, void* o, long rows, int D, int bf16, cudaStream_t stream) {
  const long n4 = rows * D / 4;
  if (n4 == 0) return 0;
  prof_begin(kKFinalize, stream);
  if (bf16)
    finalize_bf16_kernel<<<grid_for(n4, 256), 256, 0, stream>>>(
        reinterpret_cast<const float4*>(o_acc), reinterpret_cast<uint2*>(o), n4);
  else
    copy_f4_kernel<<<grid_for(n4, 256), 256, 0, stream>>>(reinterpret_cast<const float4*>(o_acc),
                                                          reinterpret_cast<float4*>(o), n4);
  prof_end(kKFinalize, stream);
  return cudaGetLastError() == cudaSuccess ? 1 : -1;
}

}  // namespace cpattn
