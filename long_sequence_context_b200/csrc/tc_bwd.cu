// tc_bwd.cu -- tcgen05 tensor-core recompute backward for bf16, D in {64,128}.
//
// Gradient of the ring forward (cpattn_fwd): for every non-SKIP (q chunk, kv
// chunk) block, recompute P = exp(scale q.k - LSE) from the saved LSE (DIAG
// blocks masked), then dV += P^T dO, dP = dO V^T, dS = P (dP - delta) with
// delta_i = dO_i . O_i, dK += scale dS^T Q, dQ += scale dS K.  The walk over
// q tiles for a given K/V tile mirrors the forward ring: at step t the K/V of
// rank `owner` sits on rank owner + t ("Megatron-LM source analysis: Context
// Parallel", section 2: the backward mirrors the forward's exchange; ring rule
// and zigzag from "Configuring RingAttention+FlashAttention for CP", section 3
// code and section 5 item 1).
//
// Launches: (1) preprocess: delta = rowsum(dO * O), zero the fp32 dQ
// accumulator; (2) the main kernel below; (3) dQ = scale * accumulator -> bf16.
//
// Main kernel: persistent, one 128-key K/V tile per work item (longest first).
// CTA roles (320 threads):
//   warps 0-3  "softmax": thread = key row (TMEM lane); turns S^T, dP^T into
//              P^T, dS^T (bf16, written back into TMEM for the dV / dK MMAs)
//              and dS (into shared memory, the A operand of the dQ MMA);
//              epilogue of dK, dV
//   warps 4-7  dQ: thread = query row; reads the dQ tile from TMEM and adds it
//              into the fp32 accumulator in global memory (vector reductions)
//   warp  8    TMA: K, V once per item; Q, dO per q tile (two stages)
//   warp  9    MMA issuer and TMEM owner
// TMEM (512 columns): S^T [0,128), dP^T [128,256), dV, dK accumulators; for
// D = 128 the dQ tile (two N = 64 halves) lands in the upper halves of the
// S^T and dP^T regions, free once P^T and dS^T occupy their lower halves.
// Per q tile the MMA thread issues S^T, dP^T | dQ | dV, dK, so the dQ read-out
// overlaps the dV / dK MMAs.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "kernels.h"
#include "sm100.cuh"
#include "tmap.h"

namespace cpattn {

namespace {

using namespace sm100;

constexpr float kLog2e = 1.4426950408889634f;

template <int D>
struct BwdCfg {
  static constexpr int kTileBytes = 128 * D * 2;  // bf16 128-row tile
  static constexpr int kSubBytes = 128 * 128;     // one 64-column swizzled block
  static constexpr int kQStages = 2;
  static constexpr int kThreads = 320;
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kTileBytes;
  static constexpr int kOffQ = 2 * kTileBytes;  // stage s: Q at +2s*tile, dO at +(2s+1)*tile
  static constexpr int kOffDS = kOffQ + kQStages * 2 * kTileBytes;
  static constexpr int kDSBytes = 128 * 128 * 2;
  static constexpr int kOffLD = kOffDS + kDSBytes;  // stage s: LSE[128], delta[128] (fp32)
  static constexpr int kLDBytes = 1024;
  static constexpr int kOffBar = kOffLD + kQStages * kLDBytes;
  // no alignment slack: the dynamic shared window starts 1024-byte aligned
  // (checked at kernel entry)
  static constexpr int kSmemBytes = kOffBar + 256;
  static constexpr bool kSplitDq = (D == 128);
  static constexpr uint32_t kColS = 0, kColDP = 128, kColDV = 256;
  static constexpr uint32_t kColDK = (D == 128) ? 384 : 320;
  static constexpr uint32_t kColDQ = 384;  // D = 64 only
  static constexpr int kDqN = kSplitDq ? D / 2 : D;
  static constexpr uint32_t kIdescST = idesc_bf16_f32(128, 128, 0, 0);
  static constexpr uint32_t kIdescAcc = idesc_bf16_f32(128, D, 0, 1);
  static constexpr uint32_t kIdescDQ = idesc_bf16_f32(128, kDqN, 1, 1);
};

struct BwdParams {
  RingGeom g;
  int BH;
  int T;        // 128-row tiles per chunk
  int tiles;    // 128-row tiles per head (S / 128)
  int n_items;  // BH * tiles
  int G;        // heads per scheduling group (divides BH)
  float sl2;    // scale * log2(e)
  float scale;
  const float* lse;
  const float* delta;
  float* dq_acc;
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  unsigned* err;
};

// Walks, for K/V tile jt, the q tiles that see it in mirror ring order.
struct QIter {
  int b, owner, jt, t, s, it, it_end, diag;
  __device__ __forceinline__ void init(const BwdParams& P, int kv_tile) {
    jt = kv_tile;
    b = jt / P.T;
    owner = chunk_owner(P.g, b);
    t = 0;
    s = -1;
    it = it_end = 0;
    diag = 0;
  }
  __device__ __forceinline__ bool next_segment(const BwdParams& P) {
    while (true) {
      ++s;
      if (s >= slots(P.g)) {
        s = 0;
        ++t;
      }
      if (t >= P.g.N) return false;
      const int r = (owner + t) % P.g.N;  // rank holding this K/V at step t
      const int a = rank_chunk(P.g, r, s);
      const int kind = block_kind(P.g, a, b);
      if (kind == kSkip) continue;
      diag = kind == kDiag;
      it = diag ? jt : a * P.T;  // in a DIAG block only q tiles at or after jt see it
      it_end = (a + 1) * P.T;
      if (it < it_end) return true;
    }
  }
  // next q tile; is_diag: the q tile shares the K/V tile's positions (mask inside)
  __device__ __forceinline__ bool next(const BwdParams& P, int& qt, int& is_diag) {
    while (it >= it_end)
      if (!next_segment(P)) return false;
    qt = it++;
    is_diag = diag && qt == jt;
    return true;
  }
};

// Work index -> (K/V tile, head).  Heads are taken G at a time, so the CTAs
// busy at any moment share a few heads' Q, dO and dQ accumulator in L2; inside
// a group K/V tiles go in ascending position (most q tiles first).
__device__ __forceinline__ void decode_item(const BwdParams& P, int w, int& jt, int& bh) {
  const int per_group = P.G * P.tiles;
  const int g = w / per_group, r = w % per_group;
  jt = r / P.G;
  bh = g * P.G + r % P.G;
}

__device__ __forceinline__ int snake_item(int round, int cta, int grid) {
  return round * grid + ((round & 1) ? (grid - 1 - cta) : cta);
}

template <int D>
__global__ void __launch_bounds__(320, 1)
    tc_bwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                  const __grid_constant__ CUtensorMap tmdQ, const BwdParams P) {
  using C = BwdCfg<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_raw;
  if (smem_u32(smem) & 1023u) {  // swizzled tiles need 1024-byte alignment
    if (threadIdx.x == 0) atomicOr(P.err, kErrLayout);
    return;
  }
  uint8_t* sK = smem + C::kOffK;
  uint8_t* sV = smem + C::kOffV;
  uint8_t* sDS = smem + C::kOffDS;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* kv_full = bars + 0;
  uint64_t* kv_empty = bars + 1;
  uint64_t* q_full = bars + 2;   // [2]
  uint64_t* q_empty = bars + 4;  // [2]
  uint64_t* s_ready = bars + 6;
  uint64_t* p_ready = bars + 7;
  uint64_t* dq_ready = bars + 8;
  uint64_t* dq_free = bars + 9;
  uint64_t* kv_done = bars + 10;
  uint64_t* acc_free = bars + 11;
  uint64_t* drain = bars + 12;
  uint64_t* stage_full = bars + 13;  // dQ rows written to the staging tile (128 arrivals)
  uint64_t* stage_free = bars + 14;  // staging tile read by the TMA reduction
  uint64_t* ds_free = bars + 15;     // dS buffer free again for the next q tile
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 16);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    mbar_init(kv_empty, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1);
    }
    mbar_init(s_ready, 1);
    mbar_init(p_ready, 128);
    mbar_init(dq_ready, 1);
    mbar_init(dq_free, 128);
    mbar_init(kv_done, 1);
    mbar_init(acc_free, 128);
    mbar_init(drain, 1);
    mbar_init(stage_full, 128);
    mbar_init(stage_free, 1);
    mbar_init(ds_free, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 9) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  if (warp == 8 && lane == 0) {
    prefetch_tensormap(&tmQ);
    prefetch_tensormap(&tmK);
    prefetch_tensormap(&tmV);
    prefetch_tensormap(&tmdO);
    prefetch_tensormap(&tmdQ);
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int grid = gridDim.x, cta = blockIdx.x;
  const int S = P.g.S;

  if (warp < 4) {
    // ------------------------------------------------- P^T, dS^T (softmax) --
    const int rloc = warp * 32 + lane;  // key row within the K/V tile
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    const uint32_t tS = tmem_base + lane_off + C::kColS;
    const uint32_t tDP = tmem_base + lane_off + C::kColDP;
    const uint32_t tDV = tmem_base + lane_off + C::kColDV;
    const uint32_t tDK = tmem_base + lane_off + C::kColDK;
    uint32_t s_cnt = 0, items = 0;
    bool ok = true;
    for (int round = 0; ok; ++round) {
      const int w = snake_item(round, cta, grid);
      if (w >= P.n_items) break;
      int jt, bh;
      decode_item(P, w, jt, bh);
      QIter qi;
      qi.init(P, jt);
      int qt, dg;
      while (qi.next(P, qt, dg)) {
        if (!mbar_wait_warp(s_ready, s_cnt & 1, abort_flag, P.err)) { ok = false; break; }
        // the dS buffer doubles as the dQ staging tile of the previous q tile
        if (s_cnt > 0 && !mbar_wait_warp(ds_free, (s_cnt - 1) & 1, abort_flag, P.err)) {
          ok = false;
          break;
        }
        // LSE and delta of this q tile arrived with its Q / dO stage
        if (!mbar_wait_warp(&q_full[s_cnt & 1], (s_cnt >> 1) & 1, abort_flag, P.err)) {
          ok = false;
          break;
        }
        const float4* lse4 = reinterpret_cast<const float4*>(smem + C::kOffLD + (s_cnt & 1) * C::kLDBytes);
        const float4* dl4 = lse4 + 32;
        ++s_cnt;
        tc_fence_after();
#pragma unroll
        for (int cb = 0; cb < 128; cb += 32) {
          uint32_t sv[32], dpv[32];
          tmem_ld32<0>(tS + cb, sv);
          tmem_ld32<0>(tDP + cb, dpv);
          tmem_wait_ld();
          uint32_t pk[16], dsk[16];
#pragma unroll
          for (int c4 = 0; c4 < 8; ++c4) {
            const float4 L = lse4[(cb >> 2) + c4];
            const float4 Dl = dl4[(cb >> 2) + c4];
            const float lv[4] = {L.x, L.y, L.z, L.w};
            const float dv_[4] = {Dl.x, Dl.y, Dl.z, Dl.w};
            float p[4], ds[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int c = cb + 4 * c4 + e;  // q column within the tile
              float pe = ex2(fmaf(__uint_as_float(sv[4 * c4 + e]), P.sl2, -lv[e] * kLog2e));
              if (dg && rloc > c) pe = 0.f;  // key after query: masked
              p[e] = pe;
              ds[e] = pe * (__uint_as_float(dpv[4 * c4 + e]) - dv_[e]);
            }
            pk[2 * c4] = pack_bf16x2(p[0], p[1]);
            pk[2 * c4 + 1] = pack_bf16x2(p[2], p[3]);
            dsk[2 * c4] = pack_bf16x2(ds[0], ds[1]);
            dsk[2 * c4 + 1] = pack_bf16x2(ds[2], ds[3]);
          }
          tmem_st16<0>(tS + cb / 2, pk);
          tmem_st16<0>(tDP + cb / 2, dsk);
          // dS into shared memory as the MN-major A operand of the dQ MMA:
          // row = key (K index), 64-query swizzled atoms along M
          uint8_t* rowp = sDS + (cb >> 6) * C::kSubBytes + rloc * 128;
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int chunk = ((cb & 63) >> 3) + u;
            *reinterpret_cast<uint4*>(rowp + ((chunk ^ (rloc & 7)) << 4)) =
                make_uint4(dsk[4 * u], dsk[4 * u + 1], dsk[4 * u + 2], dsk[4 * u + 3]);
          }
        }
        tmem_wait_st();
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(p_ready);
      }
      if (!ok) break;
      // epilogue: dV, dK of this K/V tile
      if (!mbar_wait_warp(kv_done, items & 1, abort_flag, P.err)) break;
      ++items;
      tc_fence_after();
      const long orow = ((long)bh * S + (long)jt * 128 + rloc) * D;
#pragma unroll
      for (int which = 0; which < 2; ++which) {
        const uint32_t src = which ? tDK : tDV;
        const float mul = which ? P.scale : 1.f;
        __nv_bfloat16* dst = which ? P.dk : P.dv;
#pragma unroll
        for (int cb = 0; cb < D; cb += 32) {
          uint32_t ov[32];
          tmem_ld32<0>(src + cb, ov);
          tmem_wait_ld();
          uint4* d4 = reinterpret_cast<uint4*>(dst + orow + cb);
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint4 u;
            u.x = pack_bf16x2(__uint_as_float(ov[8 * c + 0]) * mul, __uint_as_float(ov[8 * c + 1]) * mul);
            u.y = pack_bf16x2(__uint_as_float(ov[8 * c + 2]) * mul, __uint_as_float(ov[8 * c + 3]) * mul);
            u.z = pack_bf16x2(__uint_as_float(ov[8 * c + 4]) * mul, __uint_as_float(ov[8 * c + 5]) * mul);
            u.w = pack_bf16x2(__uint_as_float(ov[8 * c + 6]) * mul, __uint_as_float(ov[8 * c + 7]) * mul);
            d4[c] = u;
          }
        }
      }
      tc_fence_before();
      mbar_arrive(acc_free);
    }
  } else if (warp < 8) {
    // -------------------------------------------------- dQ read-out + add --
    const int quarter = warp - 4;
    const int rloc = quarter * 32 + lane;  // query row within the q tile
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const bool leader = (quarter == 0);  // warp 4 issues the TMA reductions
    uint32_t dq_cnt = 0, use_cnt = 0, free_cnt = 0;
    bool ok = true;
    for (int round = 0; ok; ++round) {
      const int w = snake_item(round, cta, grid);
      if (w >= P.n_items) break;
      int jt, bh;
      decode_item(P, w, jt, bh);
      QIter qi;
      qi.init(P, jt);
      int qt, dg;
      while (qi.next(P, qt, dg)) {
        if (!mbar_wait_warp(dq_ready, dq_cnt & 1, abort_flag, P.err)) { ok = false; break; }
        ++dq_cnt;
        tc_fence_after();
        uint32_t v[D];
        if constexpr (C::kSplitDq) {
          tmem_ld32<0>(tmem_base + lane_off + C::kColS + 64, v);
          tmem_ld32<32>(tmem_base + lane_off + C::kColS + 96, v);
          tmem_ld32<64>(tmem_base + lane_off + C::kColDP + 64, v);
          tmem_ld32<96>(tmem_base + lane_off + C::kColDP + 96, v);
        } else {
          tmem_ld32<0>(tmem_base + lane_off + C::kColDQ, v);
          tmem_ld32<32>(tmem_base + lane_off + C::kColDQ + 32, v);
        }
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(dq_free);
        // Add the tile into the fp32 accumulator with TMA reductions, 64
        // columns at a time, staged in the dS buffer (free: the dQ MMA that
        // read it is complete) as two 128-row x 32-column swizzled boxes.
#pragma unroll
        for (int h = 0; h < D / 64; ++h) {
          if (h > 0) {
            if (!mbar_wait_warp(stage_free, free_cnt & 1, abort_flag, P.err)) { ok = false; break; }
            ++free_cnt;
          }
#pragma unroll
          for (int b = 0; b < 2; ++b) {
            uint8_t* rowp = sDS + b * C::kSubBytes + rloc * 128;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              const int col = 64 * h + 32 * b + 4 * c;
              *reinterpret_cast<uint4*>(rowp + ((c ^ (rloc & 7)) << 4)) =
                  make_uint4(v[col], v[col + 1], v[col + 2], v[col + 3]);
            }
          }
          fence_proxy_async_smem();
          mbar_arrive(stage_full);
          if (leader) {
            if (!mbar_wait_warp(stage_full, use_cnt & 1, abort_flag, P.err)) { ok = false; break; }
            if (lane == 0) {
              const int y = bh * S + qt * 128;
              tma_reduce_add_2d(&tmdQ, sDS, 64 * h, y);
              tma_reduce_add_2d(&tmdQ, sDS + C::kSubBytes, 64 * h + 32, y);
              bulk_commit_group();
              bulk_wait_read_all();
              mbar_arrive(h + 1 < D / 64 ? stage_free : ds_free);
            }
            __syncwarp();
          }
          ++use_cnt;
        }
        if (!ok) break;
      }
    }
    if (leader && lane == 0) bulk_wait_all();
  } else if (warp == 8) {
    // ----------------------------------------------------------------- TMA --
    uint32_t items = 0, q_cnt = 0;
    bool ok = true;
    for (int round = 0; ok; ++round) {
      const int w = snake_item(round, cta, grid);
      if (w >= P.n_items) break;
      int jt, bh;
      decode_item(P, w, jt, bh);
      const int rowbase = bh * S;
      if (items > 0 && !mbar_wait_warp(kv_empty, (items - 1) & 1, abort_flag, P.err)) break;
      if (lane == 0) {
        mbar_expect_tx(kv_full, 2 * C::kTileBytes);
#pragma unroll
        for (int sb = 0; sb < D / 64; ++sb) {
          tma_load_2d(sK + sb * C::kSubBytes, &tmK, kv_full, sb * 64, rowbase + jt * 128);
          tma_load_2d(sV + sb * C::kSubBytes, &tmV, kv_full, sb * 64, rowbase + jt * 128);
        }
      }
      __syncwarp();
      ++items;
      QIter qi;
      qi.init(P, jt);
      int qt, dg;
      while (qi.next(P, qt, dg)) {
        const int st = q_cnt & 1;
        if (q_cnt >= 2 && !mbar_wait_warp(&q_empty[st], ((q_cnt >> 1) - 1) & 1, abort_flag, P.err)) {
          ok = false;
          break;
        }
        if (lane == 0) {
          uint8_t* sq = smem + C::kOffQ + (2 * st) * C::kTileBytes;
          uint8_t* sdo = sq + C::kTileBytes;
          uint8_t* sld = smem + C::kOffLD + st * C::kLDBytes;
          mbar_expect_tx(&q_full[st], 2 * C::kTileBytes + C::kLDBytes);
#pragma unroll
          for (int sb = 0; sb < D / 64; ++sb) {
            tma_load_2d(sq + sb * C::kSubBytes, &tmQ, &q_full[st], sb * 64, rowbase + qt * 128);
            tma_load_2d(sdo + sb * C::kSubBytes, &tmdO, &q_full[st], sb * 64, rowbase + qt * 128);
          }
          const long r0 = (long)rowbase + qt * 128;
          bulk_load(sld, P.lse + r0, 512, &q_full[st]);
          bulk_load(sld + 512, P.delta + r0, 512, &q_full[st]);
        }
        __syncwarp();
        ++q_cnt;
      }
    }
    if (*abort_flag) {
      // let loads already in flight land before shared memory is released
      const unsigned long long t0 = globaltimer();
      if (items > 0)
        while (!mbar_try_wait(kv_full, (items - 1) & 1) && globaltimer() - t0 < kWaitLimitNs) {
        }
      for (uint32_t i = q_cnt > 2 ? q_cnt - 2 : 0; i < q_cnt; ++i)
        while (!mbar_try_wait(&q_full[i & 1], (i >> 1) & 1) && globaltimer() - t0 < kWaitLimitNs) {
        }
    }
  } else {
    // ----------------------------------------------------------------- MMA --
    const uint32_t tS = tmem_base + C::kColS, tDP = tmem_base + C::kColDP;
    const uint32_t tDV = tmem_base + C::kColDV, tDK = tmem_base + C::kColDK;
    const uint32_t aK = smem_u32(sK), aV = smem_u32(sV), aDS = smem_u32(sDS);
    uint32_t items = 0, q_cnt = 0;
    bool ok = true;
    for (int round = 0; ok; ++round) {
      const int w = snake_item(round, cta, grid);
      if (w >= P.n_items) break;
      int jt, bh;
      decode_item(P, w, jt, bh);
      if (!mbar_wait_warp(kv_full, items & 1, abort_flag, P.err)) break;
      tc_fence_after();
      QIter qi;
      qi.init(P, jt);
      int qt, dg;
      bool first = true;
      while (qi.next(P, qt, dg)) {
        const int st = q_cnt & 1;
        const uint32_t aQ = smem_u32(smem + C::kOffQ + (2 * st) * C::kTileBytes);
        const uint32_t adO = aQ + C::kTileBytes;
        if (!mbar_wait_warp(&q_full[st], (q_cnt >> 1) & 1, abort_flag, P.err)) { ok = false; break; }
        if (C::kSplitDq && q_cnt > 0 &&
            !mbar_wait_warp(dq_free, (q_cnt - 1) & 1, abort_flag, P.err)) { ok = false; break; }
        tc_fence_after();
        if (lane == 0) {
          // S^T = K Q^T and dP^T = V dO^T (both operands K-major)
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * C::kSubBytes + (kk & 3) * 32;
            mma_ss(tS, smem_desc_sw128(aK + off, 16, 1024), smem_desc_sw128(aQ + off, 16, 1024),
                   C::kIdescST, kk > 0 ? 1u : 0u);
          }
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * C::kSubBytes + (kk & 3) * 32;
            mma_ss(tDP, smem_desc_sw128(aV + off, 16, 1024), smem_desc_sw128(adO + off, 16, 1024),
                   C::kIdescST, kk > 0 ? 1u : 0u);
          }
          tc_commit(s_ready);
        }
        __syncwarp();
        if (!mbar_wait_warp(p_ready, q_cnt & 1, abort_flag, P.err)) { ok = false; break; }
        if (!C::kSplitDq && q_cnt > 0 &&
            !mbar_wait_warp(dq_free, (q_cnt - 1) & 1, abort_flag, P.err)) { ok = false; break; }
        tc_fence_after();
        if (lane == 0) {
          // dQ = dS K: A = dS (MN-major, 2 atoms of 64 queries), B = K (MN-major over d)
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint64_t a = smem_desc_sw128(aDS + kk * 2048, C::kSubBytes, 1024);
            if constexpr (C::kSplitDq) {
              mma_ss(tS + 64, a, smem_desc_sw128(aK + kk * 2048, C::kSubBytes, 1024), C::kIdescDQ,
                     kk > 0 ? 1u : 0u);
              mma_ss(tDP + 64, a, smem_desc_sw128(aK + C::kSubBytes + kk * 2048, C::kSubBytes, 1024),
                     C::kIdescDQ, kk > 0 ? 1u : 0u);
            } else {
              mma_ss(tmem_base + C::kColDQ, a, smem_desc_sw128(aK + kk * 2048, C::kSubBytes, 1024),
                     C::kIdescDQ, kk > 0 ? 1u : 0u);
            }
          }
          tc_commit(dq_ready);
        }
        __syncwarp();
        if (first && items > 0 && !mbar_wait_warp(acc_free, (items - 1) & 1, abort_flag, P.err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (lane == 0) {
          // dV += P^T dO, dK += dS^T Q (A from TMEM, B MN-major over d)
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t acc = (first && kk == 0) ? 0u : 1u;
            mma_ts(tDV, tS + kk * 8, smem_desc_sw128(adO + kk * 2048, C::kSubBytes, 1024),
                   C::kIdescAcc, acc);
            mma_ts(tDK, tDP + kk * 8, smem_desc_sw128(aQ + kk * 2048, C::kSubBytes, 1024),
                   C::kIdescAcc, acc);
          }
          tc_commit(&q_empty[st]);
        }
        __syncwarp();
        first = false;
        ++q_cnt;
      }
      if (!ok) break;
      if (lane == 0) {
        tc_commit(kv_empty);
        tc_commit(kv_done);
      }
      __syncwarp();
      ++items;
    }
    if (lane == 0) tc_commit(drain);
    __syncwarp();
    const unsigned long long t0 = globaltimer();
    while (!mbar_try_wait(drain, 0) && globaltimer() - t0 < kWaitLimitNs) {
    }
  }

  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

// delta_i = sum_d dO_id O_id (fp32) and a zeroed dQ accumulator row; one warp per row
template <int D>
__global__ void __launch_bounds__(256) bwd_pre_kernel(const __nv_bfloat16* __restrict__ o,
                                                      const __nv_bfloat16* __restrict__ dout,
                                                      float* __restrict__ delta,
                                                      float* __restrict__ dq_acc, long rows) {
  const long row = (long)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  constexpr int E = D / 32;  // elements per lane
  float acc = 0.f;
  const __nv_bfloat16* op = o + row * D + lane * E;
  const __nv_bfloat16* dp = dout + row * D + lane * E;
#pragma unroll
  for (int e = 0; e < E; e += 2) {
    const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(op + e);
    const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(dp + e);
    acc = fmaf(__low2float(a), __low2float(b), acc);
    acc = fmaf(__high2float(a), __high2float(b), acc);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (lane == 0) delta[row] = acc;
  float* z = dq_acc + row * D + lane * E;
#pragma unroll
  for (int e = 0; e < E; e += 2) *reinterpret_cast<float2*>(z + e) = make_float2(0.f, 0.f);
}

// dq = bf16(scale * dq_acc), four elements per thread-iteration
__global__ void dq_convert_kernel(const float4* __restrict__ acc, uint2* __restrict__ dq, float scale,
                                  long n4) {
  for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < n4;
       i += (long)gridDim.x * blockDim.x) {
    const float4 x = acc[i];
    uint2 u;
    u.x = pack_bf16x2(x.x * scale, x.y * scale);
    u.y = pack_bf16x2(x.z * scale, x.w * scale);
    dq[i] = u;
  }
}

template <int D>
int launch_impl(const AttnShape& sh, const void* q, const void* k, const void* v, const void* o,
                const float* lse, const void* dout, void* dq, void* dk, void* dv, float* ws_dq,
                float* ws_delta, unsigned* err, cudaStream_t stream) {
  using C = BwdCfg<D>;
  const long rows = (long)sh.B * sh.H * sh.S;
  CUtensorMap mq, mk, mv, mdo, mdq;
  if (!make_tmap_bf16_2d(&mq, q, rows, D, 64, 128) || !make_tmap_bf16_2d(&mk, k, rows, D, 64, 128) ||
      !make_tmap_bf16_2d(&mv, v, rows, D, 64, 128) || !make_tmap_bf16_2d(&mdo, dout, rows, D, 64, 128) ||
      !make_tmap_f32_2d(&mdq, ws_dq, rows, D, 32, 128))
    return -1;
  int launched = 0;
  prof_begin(kKDelta, stream);
  bwd_pre_kernel<D><<<(unsigned)((rows + 7) / 8), 256, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(dout), ws_delta, ws_dq,
      rows);
  prof_end(kKDelta, stream);
  if (cudaGetLastError() != cudaSuccess) return -1;
  ++launched;

  BwdParams P;
  P.g = sh.g;
  P.BH = sh.B * sh.H;
  P.T = sh.g.c / 128;
  P.tiles = sh.S / 128;
  P.n_items = P.BH * P.tiles;
  P.G = (P.BH % 2 == 0) ? 2 : 1;
  P.sl2 = sh.scale * kLog2e;
  P.scale = sh.scale;
  P.lse = lse;
  P.delta = ws_delta;
  P.dq_acc = ws_dq;
  P.dk = static_cast<__nv_bfloat16*>(dk);
  P.dv = static_cast<__nv_bfloat16*>(dv);
  P.err = err;
  static bool attr_set[2] = {false, false};
  if (!attr_set[D == 128]) {
    if (cudaFuncSetAttribute(tc_bwd_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             C::kSmemBytes) != cudaSuccess)
      return -1;
    attr_set[D == 128] = true;
  }
  int dev = 0;
  cudaGetDevice(&dev);
  int grid = num_sms(dev);
  if (grid > P.n_items) grid = P.n_items;
  prof_begin(kKTcBwd, stream);
  tc_bwd_kernel<D><<<grid, C::kThreads, C::kSmemBytes, stream>>>(mq, mk, mv, mdo, mdq, P);
  prof_end(kKTcBwd, stream);
  if (cudaGetLastError() != cudaSuccess) return -1;
  ++launched;

  const long n4 = rows * D / 4;
  long blocks = (n4 + 255) / 256;
  if (blocks > 148L * 16) blocks = 148L * 16;
  prof_begin(kKDqConvert, stream);
  dq_convert_kernel<<<(unsigned)blocks, 256, 0, stream>>>(reinterpret_cast<const float4*>(ws_dq),
                                                          reinterpret_cast<uint2*>(dq), sh.scale, n4);
  prof_end(kKDqConvert, stream);
  if (cudaGetLastError() != cudaSuccess) return -1;
  ++launched;
  return launched;
}

}  // namespace

bool tc_bwd_supported(const AttnShape& sh) {
  if (!sh.bf16) return false;
  if (sh.D != 64 && sh.D != 128) return false;
  if (sh.g.c % 128 != 0) return false;
  if ((long long)sh.B * sh.H * sh.S >= (1LL << 31)) return false;
  return true;
}

int launch_tc_bwd(const AttnShape& sh, const void* q, const void* k, const void* v,
                  const void* o, const float* lse, const void* dout, void* dq, void* dk,
                  void* dv, float* ws_dq, float* ws_delta, unsigned* err, cudaStream_t stream) {
  if (sh.D == 64)
    return launch_impl<64>(sh, q, k, v, o, lse, dout, dq, dk, dv, ws_dq, ws_delta, err, stream);
  return launch_impl<128>(sh, q, k, v, o, lse, dout, dq, dk, dv, ws_dq, ws_delta, err, stream);
}

}  // namespace cpattn
