// gemm.cu -- the attention layer's projection GEMMs on the tcgen05 tensor cores:
//   C[M][N] = op(A) op(B) (+ bias[N]),  bf16 operands and result, fp32 accumulation,
// row-major, with each operand either K-major (A stored [M][K], B stored [N][K]:
// the nn.Linear weight layout) or MN-major (A stored [K][M], B stored [K][N]).
// The layer's five products are of three kinds ("Configuring
// RingAttention+FlashAttention for CP", section 3 code: q/k/v_proj and
// out_proj, nn.Linear(E, E) with bias):
//   forward  x W^T + b          A K-major,  B K-major, bias epilogue
//   dX, dOm  dY W               A K-major,  B MN-major
//   dW       dY^T X             A MN-major, B MN-major
//
// Kernel: persistent, one CTA per SM, BM x 256 output tiles, k-blocks of 64.
//   warp 0    TMA producer: A and B k-blocks into a kStages-deep ring
//   warp 1    MMA issuer (one thread) and TMEM owner
//   warps 2.. epilogue: TMEM -> registers (+ bias) -> bf16 -> global memory
// BM = 128: 4 MMAs (M=128, N=256, K=16) per k-block into one of two 256-column
//   TMEM accumulators, so four epilogue warps overlap the next tile's main loop
//   (48 KB per stage, 4 stages).
// BM = 256: the two 128-row halves of the A tile share each B tile (8 MMAs per
//   k-block into two 256-column accumulators, 64 KB per stage, 3 stages): a
//   third less operand traffic per FLOP; eight epilogue warps drain both
//   halves before the next tile starts.
// Shared-memory tiles use the 128-byte swizzle.  K-major tiles are rows of 64
// k-elements (128 B); MN-major tiles are 64-element MN chunks of 64 k-rows,
// chunk after chunk (the descriptor's leading byte offset is the chunk stride).
// Ragged edges: TMA fills out-of-range elements with zeros (no contribution to
// the K sum); the epilogue stores only rows < M and 8-column groups < N.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "kernels.h"
#include "sm100.cuh"
#include "tmap.h"

namespace cpattn {
namespace {

using namespace sm100;

template <int BM>
struct GemmCfg {
  static constexpr int kBM = BM, kBN = 256, kBK = 64;
  static constexpr int kHalves = BM / 128;          // 128-row accumulators per tile
  static constexpr int kStages = BM == 128 ? 4 : 3;
  static constexpr int kABytes = kBM * kBK * 2;     // 16 / 32 KB
  static constexpr int kBBytes = kBN * kBK * 2;     // 32 KB
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kChunkBytes = 64 * kBK * 2;  // one MN-major 64 x 64 chunk: 8 KB
  static constexpr int kOffBar = kStages * kStageBytes;
  static constexpr int kSmemBytes = 1024 + kOffBar + 256;
  static constexpr int kEpiWarps = 4 * kHalves;
  static constexpr int kThreads = 64 + 32 * kEpiWarps;
  static constexpr int kAccBufs = BM == 128 ? 2 : 1;  // accumulator sets in TMEM
  static constexpr int kGroupM = BM == 128 ? 8 : 4;   // m-blocks per raster group (L2 reuse of B)
  static_assert(kAccBufs * kHalves * kBN == 512, "TMEM columns");
};

struct GemmParams {
  int M, N, K;
  int num_m, num_n, tiles, nk;
  __nv_bfloat16* C;
  const __nv_bfloat16* bias;  // [N] or null
  unsigned* err;
};

template <int GROUP_M>
__device__ __forceinline__ void tile_coords(const GemmParams& P, int t, int& m_blk, int& n_blk) {
  const int per_group = GROUP_M * P.num_n;
  const int g = t / per_group, r = t % per_group;
  const int first_m = g * GROUP_M;
  const int gm = min(P.num_m - first_m, GROUP_M);
  m_blk = first_m + r % gm;
  n_blk = r / gm;
}

template <int A_MN, int B_MN, int BM>
__global__ void __launch_bounds__(GemmCfg<BM>::kThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const GemmParams P) {
  using C = GemmCfg<BM>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* full = bars;                      // [kStages]
  uint64_t* empty = bars + C::kStages;        // [kStages]
  uint64_t* acc_full = bars + 2 * C::kStages;  // [2]
  uint64_t* acc_empty = acc_full + 2;          // [2]
  uint64_t* drain = acc_full + 4;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_full + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 32 * C::kEpiWarps);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tmA);
    prefetch_tensormap(&tmB);
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int grid = gridDim.x, cta = blockIdx.x;

  if (warp == 0) {
    // ------------------------------------------------------------- TMA --
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (int t = cta; t < P.tiles && ok; t += grid) {
        int mb, nb;
        tile_coords<C::kGroupM>(P, t, mb, nb);
        const int m0 = mb * C::kBM, n0 = nb * C::kBN;
        for (int kb = 0; kb < P.nk; ++kb, ++it) {
          const int s = it % C::kStages;
          if (it >= (uint32_t)C::kStages &&
              !mbar_wait(&empty[s], ((it / C::kStages) - 1) & 1, abort_flag, P.err)) {
            ok = false;
            break;
          }
          uint8_t* sA = smem + s * C::kStageBytes;
          uint8_t* sB = sA + C::kABytes;
          const int k0 = kb * C::kBK;
          mbar_expect_tx(&full[s], C::kStageBytes);
          if (A_MN) {
#pragma unroll
            for (int j = 0; j < C::kBM / 64; ++j)
              tma_load_2d(sA + j * C::kChunkBytes, &tmA, &full[s], m0 + 64 * j, k0);
          } else {
            tma_load_2d(sA, &tmA, &full[s], k0, m0);  // box: 64 k x BM rows
          }
          if (B_MN) {
#pragma unroll
            for (int j = 0; j < C::kBN / 64; ++j)
              tma_load_2d(sB + j * C::kChunkBytes, &tmB, &full[s], n0 + 64 * j, k0);
          } else {
            tma_load_2d(sB, &tmB, &full[s], k0, n0);
          }
        }
      }
      if (*abort_flag) {
        // let loads already in flight land before shared memory is released
        const uint32_t first = it > (uint32_t)C::kStages ? it - C::kStages : 0;
        const unsigned long long t0 = globaltimer();
        for (uint32_t i = first; i < it; ++i)
          while (!mbar_try_wait(&full[i % C::kStages], (i / C::kStages) & 1) &&
                 globaltimer() - t0 < kWaitLimitNs) {
          }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMA --
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, C::kBN, A_MN, B_MN);
      // the second 128-row half of A: 128 rows of 128 B further (K-major), or
      // two 64-row MN chunks further (MN-major) -- 16 KB either way
      constexpr uint32_t kHalfA = 16384;
      // K-major: 16 k-elements = 32 bytes along the swizzled row; MN-major: 16
      // k-rows = 2048 bytes (two 8-row groups of 128 B)
      constexpr uint32_t kStepA = A_MN ? 2048 : 32, kStepB = B_MN ? 2048 : 32;
      constexpr uint32_t lboA = A_MN ? C::kChunkBytes : 16, lboB = B_MN ? C::kChunkBytes : 16;
      uint32_t it = 0, lt = 0;
      bool ok = true;
      for (int t = cta; t < P.tiles && ok; t += grid, ++lt) {
        const uint32_t acc = C::kAccBufs == 2 ? (lt & 1) : 0;
        const uint32_t use = C::kAccBufs == 2 ? (lt >> 1) : lt;  // earlier uses of this set
        if (use >= 1 && !mbar_wait(&acc_empty[acc], (use - 1) & 1, abort_flag, P.err)) break;
        tc_fence_after();
        const uint32_t tacc = tmem_base + acc * C::kHalves * C::kBN;
        for (int kb = 0; kb < P.nk; ++kb, ++it) {
          const int s = it % C::kStages;
          if (!mbar_wait(&full[s], (it / C::kStages) & 1, abort_flag, P.err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t aA = smem_u32(smem + s * C::kStageBytes);
          const uint64_t dA = smem_desc_sw128(aA, lboA, 1024);
          const uint64_t dB = smem_desc_sw128(aA + C::kABytes, lboB, 1024);
#pragma unroll
          for (int kk = 0; kk < C::kBK / 16; ++kk)
#pragma unroll
            for (int h = 0; h < C::kHalves; ++h)
              mma_ss(tacc + h * C::kBN, desc_at(dA, h * kHalfA + kk * kStepA),
                     desc_at(dB, kk * kStepB), idesc, (kb > 0 || kk > 0) ? 1u : 0u);
          tc_commit(&empty[s]);
        }
        if (!ok) break;
        tc_commit(&acc_full[acc]);
      }
      tc_commit(drain);
      const unsigned long long t0 = globaltimer();
      while (!mbar_try_wait(drain, 0) && globaltimer() - t0 < kWaitLimitNs) {
      }
    }
    __syncwarp();
  } else {
    // -------------------------------------------------------- epilogue --
    // warps 2..5 -> TMEM lane quarters 2, 3, 0, 1 of the first 128-row half,
    // warps 6..9 (BM = 256) the same quarters of the second half
    const int quarter = warp & 3;
    const int half = (warp - 2) >> 2;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    uint32_t lt = 0;
    for (int t = cta; t < P.tiles; t += grid, ++lt) {
      const uint32_t acc = C::kAccBufs == 2 ? (lt & 1) : 0;
      const uint32_t use = C::kAccBufs == 2 ? (lt >> 1) : lt;
      if (!mbar_wait_warp(&acc_full[acc], use & 1, abort_flag, P.err)) break;
      tc_fence_after();
      int mb, nb;
      tile_coords<C::kGroupM>(P, t, mb, nb);
      const int row = mb * C::kBM + half * 128 + quarter * 32 + lane;
      const int n0 = nb * C::kBN;
      const uint32_t tacc = tmem_base + lane_off + (acc * C::kHalves + half) * C::kBN;
#pragma unroll 1
      for (int cb = 0; cb < C::kBN; cb += 32) {
        if (n0 + cb >= P.N) break;  // warp-uniform
        uint32_t v[32];
        tmem_ld32<0>(tacc + cb, v);
        tmem_wait_ld();
        if (row < P.M) {
          __nv_bfloat16* dst = P.C + (long)row * P.N + n0 + cb;
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            if (n0 + cb + 8 * g >= P.N) break;
            float f[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) f[e] = __uint_as_float(v[8 * g + e]);
            if (P.bias) {
              const uint4 braw = *reinterpret_cast<const uint4*>(P.bias + n0 + cb + 8 * g);
              const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&braw);
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                f[2 * e] += __low2float(b2[e]);
                f[2 * e + 1] += __high2float(b2[e]);
              }
            }
            uint4 o;
            o.x = pack_bf16x2(f[0], f[1]);
            o.y = pack_bf16x2(f[2], f[3]);
            o.z = pack_bf16x2(f[4], f[5]);
            o.w = pack_bf16x2(f[6], f[7]);
            *reinterpret_cast<uint4*>(dst + 8 * g) = o;
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&acc_empty[acc]);
    }
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

template <int A_MN, int B_MN, int BM>
int launch(const void* A, const void* B, const void* bias, void* Cm, int M, int N, int K,
           unsigned* err, cudaStream_t stream) {
  using C = GemmCfg<BM>;
  CUtensorMap ta, tb;
  // A: K-major [M][K] (box 64 k x 128 rows) or MN-major [K][M] (box 64 m x 64 k)
  const bool okA = A_MN ? make_tmap_bf16_2d(&ta, A, K, M, 64, 64)
                        : make_tmap_bf16_2d(&ta, A, M, K, 64, C::kBM);
  const bool okB = B_MN ? make_tmap_bf16_2d(&tb, B, K, N, 64, 64)
                        : make_tmap_bf16_2d(&tb, B, N, K, 64, C::kBN);
  if (!okA || !okB) return -1;
  GemmParams P;
  P.M = M;
  P.N = N;
  P.K = K;
  P.num_m = (M + C::kBM - 1) / C::kBM;
  P.num_n = (N + C::kBN - 1) / C::kBN;
  P.tiles = P.num_m * P.num_n;
  P.nk = (K + C::kBK - 1) / C::kBK;
  P.C = static_cast<__nv_bfloat16*>(Cm);
  P.bias = static_cast<const __nv_bfloat16*>(bias);
  P.err = err;
  static std::atomic<unsigned long long> attr_done{0};
  if (!smem_attr_once(gemm_kernel<A_MN, B_MN, BM>, C::kSmemBytes, attr_done)) return -1;
  int dev = 0;
  cudaGetDevice(&dev);
  int grid = num_sms(dev);
  if (grid > P.tiles) grid = P.tiles;
  prof_begin(kKGemm, stream);
  gemm_kernel<A_MN, B_MN, BM><<<grid, C::kThreads, C::kSmemBytes, stream>>>(ta, tb, P);
  prof_end(kKGemm, stream);
  return cudaGetLastError() == cudaSuccess ? 1 : -1;
}

}  // namespace

int gemm_check(int M, int N, int K) {
  if (M < 1 || N < 1 || K < 1) return 2;
  if (M % 8 || N % 8 || K % 8) return 2;  // 16-byte rows for TMA and the epilogue's stores
  if ((long long)M * N >= (1LL << 31) || (long long)M * K >= (1LL << 40) ||
      (long long)N * K >= (1LL << 40))
    return 2;
  return 0;
}

// 128-row tiles (kGemmBM = 128) or 256-row tiles (256)
constexpr int kGemmBM = 256;

int launch_gemm(const void* A, const void* B, const void* bias, void* C, int M, int N, int K,
                int a_mn, int b_mn, unsigned* err, cudaStream_t stream) {
  constexpr int BM = kGemmBM;
  if (a_mn && b_mn) return launch<1, 1, BM>(A, B, bias, C, M, N, K, err, stream);
  if (a_mn) return launch<1, 0, BM>(A, B, bias, C, M, N, K, err, stream);
  if (b_mn) return launch<0, 1, BM>(A, B, bias, C, M, N, K, err, stream);
  return launch<0, 0, BM>(A, B, bias, C, M, N, K, err, stream);
}

}  // namespace cpattn
