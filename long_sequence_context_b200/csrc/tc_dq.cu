// tc_dq.cu -- tcgen05 dQ kernel of the recompute backward (bf16, D in {64,128}).
//
// One 128-row Q tile per work item (longest first); its 128-key K/V tiles are
// walked in forward ring order.  Per K/V tile j:
//   S_j  = Q K_j^T,  dP_j = dO V_j^T                  (TMEM, fp32)
//   P_j  = exp2(S_j * scale * log2 e - LSE * log2 e)   (DIAG tiles masked)
//   dS_j = P_j (dP_j - delta)                          (bf16, back into TMEM)
//   dQ  += dS_j K_j                                    (A = dS_j from TMEM)
// dQ accumulates in TMEM and is written once, scaled, as bf16 (in accumulate
// mode: added once into the caller's fp32 dQ sum): no reductions.
//
// Overlap.  S is double-buffered; the elementwise work of a tile is split into
// an exponential phase that needs only S_j and a dS phase that needs dP_j.  The
// MMA thread issues, after the dS of tile j is in TMEM: dP_{j+1}, dQ_j,
// S_{j+2}.  So the exponentials of tile j+1 run while dP_{j+1} is computed, and
// the tensor core is busy while the elementwise warps work.
//
// TMEM (512 columns): S0 [0,128) S1 [128,256) dP [256,384) dQ [384,384+D).
// Roles (384 threads): warps 0-7 elementwise (warp w: TMEM lanes 32*(w%4)..,
// score columns 64*(w/4)..; 208 registers via setmaxnreg), warp 8 TMA (Q, dO
// per item; a ring of K / V tiles), warp 9 MMA issuer and TMEM owner, warps
// 10-11 only complete the third warpgroup (88 registers).  One CTA per Q tile,
// longest first.  dS of column half h is packed as
// bf16 into columns [64 h, 64 h + 32) of its S buffer.
// Sources: "Configuring RingAttention+FlashAttention for CP", section 3 code and
// note 2, section 5 item 1 (ring walk, mask, zigzag); the gradient is that of
// the forward ("Megatron-LM source analysis: Context Parallel", section 2).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "bwd_common.cuh"
#include "kernels.h"
#include "sm100.cuh"
#include "tmap.h"

namespace cpattn {
namespace bwd {

namespace {

using namespace sm100;

template <int D>
struct DqCfg {
  static constexpr int kTileBytes = 128 * D * 2;      // bf16 128-row tile
  static constexpr int kSubBytes = 128 * 128;         // one 64-column swizzled block
  static constexpr int kStages = D == 128 ? 5 : 10;   // K / V slots
  static constexpr int kOffQ = 0;
  static constexpr int kOffDO = kTileBytes;
  static constexpr int kOffKV = 2 * kTileBytes;
  static constexpr int kOffBar = kOffKV + kStages * kTileBytes;
  static constexpr int kSmemBytes = 1024 + kOffBar + 256;
  static constexpr uint32_t kColDP = 256, kColDQ = 384;
  __device__ static constexpr uint32_t col_s(int b) { return 128 * b; }
  static constexpr uint32_t kIdescS = idesc_bf16_f32(128, 128, 0, 0);
  static constexpr uint32_t kIdescDQ = idesc_bf16_f32(128, D, 0, 1);
};

// TMEM column of the packed bf16 pair for score columns (c, c+1): column half
// h = c / 64 packs into [64 h, 64 h + 32).
__device__ __forceinline__ uint32_t packed_col(int c) { return (c & 64) + ((c & 63) >> 1); }
// TMEM column of k-step kk (16 score columns) of the packed operand
__device__ __forceinline__ uint32_t packed_kstep(int kk) { return (kk >= 4 ? 64 : 0) + (kk & 3) * 8; }

template <int D>
__global__ void __launch_bounds__(384, 1)
    tc_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                 const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                 const BwdParams P) {
  using C = DqCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sQ = smem + C::kOffQ;
  uint8_t* sdO = smem + C::kOffDO;
  uint8_t* sKV = smem + C::kOffKV;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* kv_full = bars;                  // [kStages]
  uint64_t* kv_empty = bars + C::kStages;    // [kStages]
  uint64_t* q_full = bars + 2 * C::kStages;
  uint64_t* q_empty = q_full + 1;
  uint64_t* s_ready = q_full + 2;            // [2] one per S buffer
  uint64_t* dp_ready = q_full + 4;
  uint64_t* p_ready = q_full + 5;            // dS of the tile written to TMEM
  uint64_t* dq_done = q_full + 6;
  uint64_t* acc_free = q_full + 7;
  uint64_t* drain = q_full + 8;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(q_full + 9);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    mbar_init(&s_ready[0], 1);
    mbar_init(&s_ready[1], 1);
    mbar_init(dp_ready, 1);
    mbar_init(p_ready, 256);
    mbar_init(dq_done, 1);
    mbar_init(acc_free, 256);
    mbar_init(drain, 1);
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
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int grid = gridDim.x, cta = blockIdx.x;
  const int S = P.g.S;

  if (warp < 8) {
    // ---------------------------------------------------------- elementwise --
    regs_inc<208>();
    const int quarter = warp & 3, half = warp >> 2;
    const int rloc = quarter * 32 + lane;  // query row within the Q tile
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const uint32_t tDP = tmem_base + lane_off + C::kColDP + half * 64;
    uint32_t j_cnt = 0, items = 0;
    bool ok = true;
    for (int round = 0; ok; ++round) {
      const int w = snake_item(round, cta, grid);
      if (w >= P.n_items) break;
      int qt, bh;
      decode_item(P, w, true, qt, bh);
      const long row = (long)bh * S + (long)qt * 128 + rloc;
      const float lse2 = P.lse2[row];
      const float dlt = P.delta[row];
      KIter<128> ki;
      ki.init(P, qt);
      int kt, doff;
      while (ki.next(P, kt, doff)) {
        const int b = j_cnt & 1;
        const uint32_t tS = tmem_base + lane_off + C::col_s(b) + half * 64;
        // exponential phase: needs S_j only
        if (!mbar_wait_warp(&s_ready[b], (j_cnt >> 1) & 1, abort_flag, P.err)) { ok = false; break; }
        tc_fence_after();
        float p[64];
#pragma unroll
        for (int ch = 0; ch < 2; ++ch) {
          uint32_t sv[32];
          tmem_ld32<0>(tS + ch * 32, sv);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            float pe = ex2(fmaf(__uint_as_float(sv[c]), P.sl2, -lse2));
            if (doff >= 0 && half * 64 + ch * 32 + c > rloc) pe = 0.f;  // key after query
            p[ch * 32 + c] = pe;
          }
        }
        // dS phase: needs dP_j
        if (!mbar_wait_warp(dp_ready, j_cnt & 1, abort_flag, P.err)) { ok = false; break; }
        ++j_cnt;
        tc_fence_after();
#pragma unroll
        for (int ch = 0; ch < 2; ++ch) {
          uint32_t dpv[32], dsk[16];
          tmem_ld32<0>(tDP + ch * 32, dpv);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 32; c += 2)
            dsk[c >> 1] = pack_bf16x2(p[ch * 32 + c] * (__uint_as_float(dpv[c]) - dlt),
                                      p[ch * 32 + c + 1] * (__uint_as_float(dpv[c + 1]) - dlt));
          tmem_st16<0>(tmem_base + lane_off + C::col_s(b) + packed_col(half * 64 + ch * 32), dsk);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(p_ready);
      }
      if (!ok) break;
      if (!mbar_wait_warp(dq_done, items & 1, abort_flag, P.err)) break;
      ++items;
      tc_fence_after();
#pragma unroll
      for (int cb = 0; cb < D / 2; cb += 32) {
        const int col = half * (D / 2) + cb;
        uint32_t v[32];
        tmem_ld32<0>(tmem_base + lane_off + C::kColDQ + col, v);
        tmem_wait_ld();
        if (P.acc_f32)
          add_row32(P.dq_acc + row * D + col, v, P.scale);
        else
          store_row32(P.dq + row * D + col, v, P.scale);
      }
      tc_fence_before();
      mbar_arrive(acc_free);
    }
  } else {
    regs_dec<88>();
  }
  if (warp == 8) {
    // ----------------------------------------------------------------- TMA --
    uint32_t kv_idx = 0, items = 0;
    bool ok = true;
    for (int round = 0; ok; ++round) {
      const int w = snake_item(round, cta, grid);
      if (w >= P.n_items) break;
      int qt, bh;
      decode_item(P, w, true, qt, bh);
      const int rowbase = bh * S;
      if (items > 0 && !mbar_wait_warp(q_empty, (items - 1) & 1, abort_flag, P.err)) break;
      if (lane == 0) {
        mbar_expect_tx(q_full, 2 * C::kTileBytes);
#pragma unroll
        for (int sb = 0; sb < D / 64; ++sb) {
          tma_load_2d(sQ + sb * C::kSubBytes, &tmQ, q_full, sb * 64, rowbase + qt * 128);
          tma_load_2d(sdO + sb * C::kSubBytes, &tmdO, q_full, sb * 64, rowbase + qt * 128);
        }
      }
      __syncwarp();
      ++items;
      KIter<128> ki;
      ki.init(P, qt);
      int kt, doff;
      while (ki.next(P, kt, doff)) {
        for (int which = 0; which < 2; ++which) {
          const int s = kv_idx % C::kStages;
          if (kv_idx >= (uint32_t)C::kStages &&
              !mbar_wait_warp(&kv_empty[s], ((kv_idx / C::kStages) - 1) & 1, abort_flag, P.err)) {
            ok = false;
            break;
          }
          if (lane == 0) {
            mbar_expect_tx(&kv_full[s], C::kTileBytes);
            const CUtensorMap* map = which ? &tmV : &tmK;
#pragma unroll
            for (int sb = 0; sb < D / 64; ++sb)
              tma_load_2d(sKV + s * C::kTileBytes + sb * C::kSubBytes, map, &kv_full[s], sb * 64,
                          rowbase + kt * 128);
          }
          __syncwarp();
          ++kv_idx;
        }
        if (!ok) break;
      }
    }
    if (*abort_flag) {
      const unsigned long long t0 = globaltimer();
      if (items > 0)
        while (!mbar_try_wait(q_full, (items - 1) & 1) && globaltimer() - t0 < kWaitLimitNs) {
        }
      const uint32_t first = kv_idx > (uint32_t)C::kStages ? kv_idx - C::kStages : 0;
      for (uint32_t i = first; i < kv_idx; ++i)
        while (!mbar_try_wait(&kv_full[i % C::kStages], (i / C::kStages) & 1) &&
               globaltimer() - t0 < kWaitLimitNs) {
        }
    }
  } else if (warp == 9) {
    // ----------------------------------------------------------------- MMA --
    const uint32_t tDP = tmem_base + C::kColDP, tDQ = tmem_base + C::kColDQ;
    const uint32_t aQ = smem_u32(sQ), adO = smem_u32(sdO), aKV = smem_u32(sKV);
    uint32_t kv_idx = 0, j_cnt = 0, items = 0;
    bool ok = true;
    // slot of K / V tile t of the current item: kv_base + 2t (+1 for V)
    auto slot_of = [&](uint32_t idx) { return idx % C::kStages; };
    auto phase_of = [&](uint32_t idx) { return (idx / C::kStages) & 1; };
    // One descriptor per operand tile; k-steps are constant offsets from it.
    const uint64_t dQ0 = smem_desc_sw128(aQ, 16, 1024), ddO0 = smem_desc_sw128(adO, 16, 1024);
    auto issue_s = [&](int buf, uint32_t slotK) {
      const uint64_t dk = smem_desc_sw128(aKV + slotK * C::kTileBytes, 16, 1024);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = (kk >> 2) * C::kSubBytes + (kk & 3) * 32;
        mma_ss(tmem_base + C::col_s(buf), desc_at(dQ0, off), desc_at(dk, off), C::kIdescS,
               kk > 0 ? 1u : 0u);
      }
    };
    auto issue_dp = [&](uint32_t slotV) {
      const uint64_t dv = smem_desc_sw128(aKV + slotV * C::kTileBytes, 16, 1024);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = (kk >> 2) * C::kSubBytes + (kk & 3) * 32;
        mma_ss(tDP, desc_at(ddO0, off), desc_at(dv, off), C::kIdescS, kk > 0 ? 1u : 0u);
      }
    };
    for (int round = 0; ok; ++round) {
      const int w = snake_item(round, cta, grid);
      if (w >= P.n_items) break;
      int qt, bh;
      decode_item(P, w, true, qt, bh);
      // number of K/V tiles of this item
      KIter<128> ki;
      ki.init(P, qt);
      int n = 0, kt, doff;
      while (ki.next(P, kt, doff)) ++n;
      const uint32_t base = kv_idx;
      kv_idx += 2 * n;
      if (!mbar_wait_warp(q_full, items & 1, abort_flag, P.err)) break;
      tc_fence_after();
      // prologue: S_0, dP_0, S_1
      for (int t = 0; t < 2 && t < n; ++t) {
        if (!mbar_wait_warp(&kv_full[slot_of(base + 2 * t)], phase_of(base + 2 * t), abort_flag, P.err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (lane == 0) {
          issue_s((j_cnt + t) & 1, slot_of(base + 2 * t));
          tc_commit(&s_ready[(j_cnt + t) & 1]);
        }
        __syncwarp();
        if (t == 0) {
          if (!mbar_wait_warp(&kv_full[slot_of(base + 1)], phase_of(base + 1), abort_flag, P.err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (lane == 0) {
            issue_dp(slot_of(base + 1));
            tc_commit(dp_ready);
            tc_commit(&kv_empty[slot_of(base + 1)]);
          }
          __syncwarp();
        }
      }
      if (!ok) break;
      for (int t = 0; t < n; ++t) {
        // dS_t in TMEM: the elementwise warps are done with S_t and dP_t
        if (!mbar_wait_warp(p_ready, j_cnt & 1, abort_flag, P.err)) { ok = false; break; }
        if (t == 0 && items > 0 && !mbar_wait_warp(acc_free, (items - 1) & 1, abort_flag, P.err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (t + 1 < n) {  // dP_{t+1}
          const uint32_t iv = base + 2 * (t + 1) + 1;
          if (!mbar_wait_warp(&kv_full[slot_of(iv)], phase_of(iv), abort_flag, P.err)) { ok = false; break; }
          tc_fence_after();
          if (lane == 0) {
            issue_dp(slot_of(iv));
            tc_commit(dp_ready);
            tc_commit(&kv_empty[slot_of(iv)]);
          }
          __syncwarp();
        }
        if (lane == 0) {  // dQ += dS_t K_t
          const uint32_t tDS = tmem_base + C::col_s(j_cnt & 1);
          const uint64_t dk = smem_desc_sw128(aKV + slot_of(base + 2 * t) * C::kTileBytes,
                                              C::kSubBytes, 1024);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ts(tDQ, tDS + packed_kstep(kk), desc_at(dk, kk * 2048), C::kIdescDQ,
                   (t == 0 && kk == 0) ? 0u : 1u);
          tc_commit(&kv_empty[slot_of(base + 2 * t)]);
        }
        __syncwarp();
        if (t + 2 < n) {  // S_{t+2} into the buffer dS_t occupied
          const uint32_t ik = base + 2 * (t + 2);
          if (!mbar_wait_warp(&kv_full[slot_of(ik)], phase_of(ik), abort_flag, P.err)) { ok = false; break; }
          tc_fence_after();
          if (lane == 0) {
            issue_s(j_cnt & 1, slot_of(ik));
            tc_commit(&s_ready[j_cnt & 1]);
          }
          __syncwarp();
        }
        ++j_cnt;
      }
      if (!ok) break;
      if (lane == 0) {
        tc_commit(q_empty);
        tc_commit(dq_done);
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

}  // namespace

template <int D>
int launch_tc_dq(const BwdParams& P, const CUtensorMap& mq, const CUtensorMap& mk,
                 const CUtensorMap& mv, const CUtensorMap& mdo, int grid, cudaStream_t stream) {
  using C = DqCfg<D>;
  static std::atomic<unsigned long long> attr_done{0};
  if (!smem_attr_once(tc_dq_kernel<D>, C::kSmemBytes, attr_done)) return -1;
  prof_begin(kKTcDq, stream);
  tc_dq_kernel<D><<<grid, 384, C::kSmemBytes, stream>>>(mq, mk, mv, mdo, P);
  prof_end(kKTcDq, stream);
  return cudaGetLastError() == cudaSuccess ? 1 : -1;
}

template int launch_tc_dq<64>(const BwdParams&, const CUtensorMap&, const CUtensorMap&,
                              const CUtensorMap&, const CUtensorMap&, int, cudaStream_t);
template int launch_tc_dq<128>(const BwdParams&, const CUtensorMap&, const CUtensorMap&,
                               const CUtensorMap&, const CUtensorMap&, int, cudaStream_t);

}  // namespace bwd
}  // namespace cpattn
