// tc_bwd.cu -- tcgen05 tensor-core recompute backward for bf16, D in {64,128}:
// the preprocess, the dK / dV kernel and the launch sequence (the dQ kernel is
// in tc_dq.cu).
//
// Gradient of the ring forward (cpattn_fwd): for every non-SKIP (q chunk, kv
// chunk) block, recompute P = exp(scale q.k - LSE) from the saved LSE (DIAG
// blocks masked), then dV += P^T dO, dP = dO V^T, dS = P (dP - delta) with
// delta_i = dO_i . O_i, dK += scale dS^T Q, dQ += scale dS K.
// ("Megatron-LM source analysis: Context Parallel", section 2: the backward
// mirrors the forward's exchange; ring rule and zigzag from "Configuring
// RingAttention+FlashAttention for CP", section 3 code and section 5 item 1.)
//
// Launches:
//   1. preprocess: delta_i = rowsum(dO_i * O_i), LSE_i * log2(e)   (workspace)
//   2. dK / dV kernel: one 128-key K/V tile per work item; walks the q tiles
//      that see it in mirror ring order (at step t the K/V of rank `owner` sits
//      on rank owner + t): S^T = K Q^T, dP^T = V dO^T (TMEM), P^T (bf16, to
//      shared memory) and dS^T (bf16, back into TMEM), dV += P^T dO,
//      dK += dS^T Q (A from TMEM).
//   3. dQ kernel: one Q tile per work item, dQ accumulated in TMEM and written
//      once; no reductions.  At D = 128 with an even number of tiles per chunk
//      it runs on two SMs per pair of Q tiles (tc_dq2.cu, cta_group::2 MMAs),
//      otherwise on one SM per Q tile (tc_dq.cu).
// Computing dQ in its own kernel recomputes S and dP once more but removes the
// fp32 dQ reduction traffic, which on this GPU costs more than the extra
// tensor work.
//
// dK / dV kernel: one CTA per K/V tile, 384 threads.  Warps 0-7 do the
// elementwise work: warp w owns TMEM lanes 32*(w%4).. (one key row per thread)
// and the column half w/4 of each 128-column score tile.  Warp 8 issues TMA
// loads, warp 9 the MMAs (one thread) and owns TMEM; warps 10-11 only complete
// the third warpgroup (setmaxnreg: 200 registers for the elementwise warps,
// 104 for the rest; 384 x 168 at launch).
// TMEM (512 columns): S^T [0,128) dP^T [128,256) dV [256,256+D) dK [384,384+D)
// (D = 64: dK at 320).  The elementwise warps read S^T out of TMEM at once and
// release it, so the next q tile's S^T is computed during their exponential
// phase; P^T goes to shared memory (the A operand of dV += P^T dO, K-major,
// 128-byte swizzle) and dS^T back into dP^T's columns, packed: column half h
// into [128 + 64 h, 128 + 64 h + 32), so neither half overwrites values the
// other is still reading.  The MMA thread tests the barriers of its next MMA
// group between the MMAs of the current one.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "bwd_common.cuh"
#include "kernels.h"
#include "sm100.cuh"
#include "tmap.h"

namespace cpattn {
namespace bwd {

template <int D>
int launch_tc_dq(const BwdParams& P, const CUtensorMap& mq, const CUtensorMap& mk,
                 const CUtensorMap& mv, const CUtensorMap& mdo, int grid, cudaStream_t stream);
// two-SM dQ kernel (tc_dq2.cu): D = 128 and an even number of tiles per chunk
bool tc_dq2_supported(const BwdParams& P, int D);
int launch_tc_dq2(const BwdParams& P, const void* k, const void* v, long rows, cudaStream_t stream);

namespace {

using namespace sm100;

constexpr float kLog2e = 1.4426950408889634f;

// TMEM column of the packed bf16 pair for score columns (c, c+1) of a tile:
// column half h = c / 64 packs into [64 h, 64 h + 32).
__device__ __forceinline__ uint32_t packed_col(int c) { return (c & 64) + ((c & 63) >> 1); }
// TMEM column of k-step kk (16 score columns) of a packed bf16 operand
__device__ __forceinline__ uint32_t packed_kstep(int kk) { return (kk >= 4 ? 64 : 0) + (kk & 3) * 8; }

// ===================================================================== dK/dV ==
template <int D>
struct DkdvCfg {
  static constexpr int kTileBytes = 128 * D * 2;
  static constexpr int kSubBytes = 128 * 128;
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kTileBytes;
  static constexpr int kOffQ = 2 * kTileBytes;  // stage s: Q at +2s tiles, dO at +(2s+1)
  static constexpr int kStages = D == 128 ? 2 : 4;
  static constexpr int kOffLD = kOffQ + kStages * 2 * kTileBytes;  // stage s: LSE2[128], delta[128]
  static constexpr int kLDBytes = 1024;
  // P^T of the current q tile, bf16 [128 keys][128 q] as two 64-column swizzled
  // blocks: the A operand (K-major) of dV += P^T dO
  static constexpr int kOffP = kOffLD + kStages * kLDBytes;
  static constexpr int kDataBytes = kOffP + 128 * 128 * 2;
  static constexpr int kBarBytes = 256;
  // the barriers sit in the alignment slack in front of the 1024-aligned data
  // when it has room for them, else behind the data
  static constexpr int kSmemBytes = 1024 + kDataBytes;
  static constexpr uint32_t kColS = 0, kColDP = 128, kColDV = 256;
  static constexpr uint32_t kColDK = (D == 128) ? 384 : 320;
  static constexpr uint32_t kIdescST = idesc_bf16_f32(128, 128, 0, 0);
  static constexpr uint32_t kIdescAcc = idesc_bf16_f32(128, D, 0, 1);
  static_assert(kOffP % 1024 == 0, "swizzled P^T blocks need 1024-byte alignment");
  static_assert(kSmemBytes <= 232448, "shared memory per CTA");
};

template <int D>
__global__ void __launch_bounds__(384, 1)
    tc_dkdv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                   const BwdParams P) {
  using C = DkdvCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  // (chosen on the 32-bit shared-window address, so that the barrier
  // addresses stay constant offsets of one 32-bit base)
  const uint32_t raw_s = smem_u32(smem_raw), data_s = smem_u32(smem);
  const uint32_t bar_s = (data_s - raw_s >= (uint32_t)C::kBarBytes) ? raw_s : data_s + C::kDataBytes;
  uint8_t* bar_area = static_cast<uint8_t*>(__cvta_shared_to_generic(bar_s));
  uint8_t* sK = smem + C::kOffK;
  uint8_t* sV = smem + C::kOffV;
  uint8_t* sP = smem + C::kOffP;
  uint64_t* bars = reinterpret_cast<uint64_t*>(bar_area);
  uint64_t* kv_full = bars + 0;
  uint64_t* kv_empty = bars + 1;
  uint64_t* q_full = bars + 2;             // [kStages]
  uint64_t* q_empty = q_full + C::kStages;  // [kStages]
  uint64_t* s_ready = q_empty + C::kStages;  // S^T of the q tile in TMEM
  uint64_t* dp_ready = s_ready + 1;          // dP^T of the q tile in TMEM
  uint64_t* pa_ready = s_ready + 2;          // P^T in shared memory (256 arrivals)
  uint64_t* pb_ready = s_ready + 3;          // dS^T written back (256 arrivals)
  uint64_t* kv_done = s_ready + 4;
  uint64_t* acc_free = s_ready + 5;
  uint64_t* drain = s_ready + 6;
  uint64_t* s_free = s_ready + 7;            // S^T read out of TMEM (256 arrivals)
  uint64_t* p_free = s_ready + 8;            // dV MMA done reading P^T
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(s_ready + 9);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    mbar_init(kv_empty, 1);
    for (int i = 0; i < C::kStages; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1);
    }
    mbar_init(s_ready, 1);
    mbar_init(dp_ready, 1);
    mbar_init(pa_ready, 256);
    mbar_init(pb_ready, 256);
    mbar_init(kv_done, 1);
    mbar_init(acc_free, 256);
    mbar_init(drain, 1);
    mbar_init(s_free, 256);
    mbar_init(p_free, 1);
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
    // ---------------------------------------------------- P^T and dS^T --
    regs_inc<200>();
    const int quarter = warp & 3, half = warp >> 2;
    const int rloc = quarter * 32 + lane;  // key row within the K/V tile
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const uint32_t tS = tmem_base + lane_off + C::kColS;
    const uint32_t tDP = tmem_base + lane_off + C::kColDP;
    // this thread's 128-byte row of P^T: key rloc, q columns [64 half, 64 half + 64)
    uint8_t* prow = sP + half * C::kSubBytes + rloc * 128;
    uint32_t s_cnt = 0, items = 0;
    bool ok = true;
    for (int round = 0; ok; ++round) {
      const int w = snake_item(round, cta, grid);
      if (w >= P.n_items) break;
      int jt, bh;
      decode_item(P, w, false, jt, bh);
      QIter qi;
      qi.init(P, jt);
      int qt, dg;
      while (qi.next(P, qt, dg)) {
        const int st = s_cnt % C::kStages;
        // exponential phase: S^T is read out of TMEM at once (the next q tile's
        // S^T may then be computed into the same columns); P^T goes to shared
        // memory for dV
        if (!mbar_wait_warp(s_ready, s_cnt & 1, abort_flag, P.err) ||
            !mbar_wait_warp(&q_full[st], (s_cnt / C::kStages) & 1, abort_flag, P.err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t sv[64];
        tmem_ld32<0>(tS + half * 64, sv);
        tmem_ld32<32>(tS + half * 64 + 32, sv);
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(s_free);
        const float4* l4 = reinterpret_cast<const float4*>(smem + C::kOffLD + st * C::kLDBytes);
        const float4* d4 = l4 + 32;
        float p[64];
        const float2 sl = make_float2(P.sl2, P.sl2);
#pragma unroll
        for (int c4 = 0; c4 < 16; ++c4) {
          const float4 L = l4[half * 16 + c4];
          const float2 x01 = ffma2(make_float2(__uint_as_float(sv[4 * c4]), __uint_as_float(sv[4 * c4 + 1])), sl,
                                   make_float2(-L.x, -L.y));
          const float2 x23 = ffma2(make_float2(__uint_as_float(sv[4 * c4 + 2]), __uint_as_float(sv[4 * c4 + 3])), sl,
                                   make_float2(-L.z, -L.w));
          p[4 * c4 + 0] = ex2(x01.x);
          p[4 * c4 + 1] = ex2(x01.y);
          p[4 * c4 + 2] = ex2(x23.x);
          p[4 * c4 + 3] = ex2(x23.y);
        }
        if (dg) {
          // diagonal tile: keys after the query are masked
#pragma unroll
          for (int c = 0; c < 64; ++c)
            if (rloc > half * 64 + c) p[c] = 0.f;
        }
        // the previous q tile's dV MMA must be done reading P^T
        if (s_cnt > 0 && !mbar_wait_warp(p_free, (s_cnt - 1) & 1, abort_flag, P.err)) {
          ok = false;
          break;
        }
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
          const uint4 u = make_uint4(pack_bf16x2(p[8 * ch], p[8 * ch + 1]), pack_bf16x2(p[8 * ch + 2], p[8 * ch + 3]),
                                     pack_bf16x2(p[8 * ch + 4], p[8 * ch + 5]), pack_bf16x2(p[8 * ch + 6], p[8 * ch + 7]));
          *reinterpret_cast<uint4*>(prow + ((ch ^ (rloc & 7)) << 4)) = u;
        }
        fence_proxy_async_smem();
        mbar_arrive(pa_ready);
        // dS phase: needs dP^T; dS^T goes back to TMEM for dK
        if (!mbar_wait_warp(dp_ready, s_cnt & 1, abort_flag, P.err)) { ok = false; break; }
        ++s_cnt;
        tc_fence_after();
        uint32_t dpv[64];
        tmem_ld32<0>(tDP + half * 64, dpv);
        tmem_ld32<32>(tDP + half * 64 + 32, dpv);
        tmem_wait_ld();
#pragma unroll
        for (int ch = 0; ch < 2; ++ch) {
          const int cb = half * 64 + ch * 32;
          uint32_t dsk[16];
#pragma unroll
          for (int c4 = 0; c4 < 8; ++c4) {
            const float4 Dl = d4[(cb >> 2) + c4];
            const int e0 = ch * 32 + 4 * c4;
            const float2 ds01 = fmul2(make_float2(p[e0], p[e0 + 1]),
                                      fsub2(make_float2(__uint_as_float(dpv[e0]), __uint_as_float(dpv[e0 + 1])),
                                            make_float2(Dl.x, Dl.y)));
            const float2 ds23 = fmul2(make_float2(p[e0 + 2], p[e0 + 3]),
                                      fsub2(make_float2(__uint_as_float(dpv[e0 + 2]), __uint_as_float(dpv[e0 + 3])),
                                            make_float2(Dl.z, Dl.w)));
            dsk[2 * c4] = pack_bf16x2(ds01.x, ds01.y);
            dsk[2 * c4 + 1] = pack_bf16x2(ds23.x, ds23.y);
          }
          tmem_st16<0>(tDP + packed_col(cb), dsk);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(pb_ready);
      }
      if (!ok) break;
      // epilogue: this warp writes columns [half*D/2, half*D/2 + D/2) of dV, dK
      if (!mbar_wait_warp(kv_done, items & 1, abort_flag, P.err)) break;
      ++items;
      tc_fence_after();
      const long orow = ((long)bh * S + (long)jt * 128 + rloc) * D;
#pragma unroll
      for (int cb = 0; cb < D / 2; cb += 32) {
        const int col = half * (D / 2) + cb;
        uint32_t ov[32];
        tmem_ld32<0>(tmem_base + lane_off + C::kColDV + col, ov);
        tmem_wait_ld();
        if (P.acc_f32)
          add_row32(P.dv_acc + orow + col, ov, 1.f);
        else
          store_row32(P.dv + orow + col, ov, 1.f);
        tmem_ld32<0>(tmem_base + lane_off + C::kColDK + col, ov);
        tmem_wait_ld();
        if (P.acc_f32)
          add_row32(P.dk_acc + orow + col, ov, P.scale);
        else
          store_row32(P.dk + orow + col, ov, P.scale);
      }
      tc_fence_before();
      mbar_arrive(acc_free);
    }
  } else {
    regs_dec<104>();
  }
  if (warp == 8) {
    // ----------------------------------------------------------------- TMA --
    uint32_t items = 0, q_cnt = 0;
    bool ok = true;
    for (int round = 0; ok; ++round) {
      const int w = snake_item(round, cta, grid);
      if (w >= P.n_items) break;
      int jt, bh;
      decode_item(P, w, false, jt, bh);
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
        const int st = q_cnt % C::kStages;
        if (q_cnt >= (uint32_t)C::kStages &&
            !mbar_wait_warp(&q_empty[st], ((q_cnt / C::kStages) - 1) & 1, abort_flag, P.err)) {
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
          bulk_load(sld, P.lse2 + r0, 512, &q_full[st]);
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
      const uint32_t first = q_cnt > (uint32_t)C::kStages ? q_cnt - C::kStages : 0;
      for (uint32_t i = first; i < q_cnt; ++i)
        while (!mbar_try_wait(&q_full[i % C::kStages], (i / C::kStages) & 1) &&
               globaltimer() - t0 < kWaitLimitNs) {
        }
    }
  } else if (warp == 9) {
    // ----------------------------------------------------------------- MMA --
    // One thread issues every MMA (the other lanes wait at the end).
    if (lane == 0) {
      const uint32_t tS = tmem_base + C::kColS, tDP = tmem_base + C::kColDP;
      const uint32_t tDV = tmem_base + C::kColDV, tDK = tmem_base + C::kColDK;
      const uint32_t aK = smem_u32(sK), aV = smem_u32(sV);
      uint32_t items = 0, q_cnt = 0;
      bool ok = true;
      auto q_addr = [&](uint32_t cnt) {
        return smem_u32(smem + C::kOffQ + (2 * (cnt % C::kStages)) * C::kTileBytes);
      };
      // One descriptor per operand tile per MMA group; k-steps are constant
      // offsets from it.
      const uint32_t aP = smem_u32(sP);
      // The barriers of the next MMA group are tested between the MMAs of the
      // current one (Probe), so that their latency overlaps queued tensor work.
      Probe pa, pb;
      auto mid = [&](int kk) {
        if (kk == 1 || kk == 6) {
          pa.test();
          pb.test();
        }
      };
      // S^T = K Q^T and dP^T = V dO^T (both operands K-major)
      auto issue_st = [&](uint32_t aQ) {
        const uint64_t dK0 = smem_desc_sw128(aK, 16, 1024), dq = smem_desc_sw128(aQ, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * C::kSubBytes + (kk & 3) * 32;
          mma_ss(tS, desc_at(dK0, off), desc_at(dq, off), C::kIdescST, kk > 0 ? 1u : 0u);
          mid(kk);
        }
      };
      auto issue_dpt = [&](uint32_t adO) {
        const uint64_t dV0 = smem_desc_sw128(aV, 16, 1024), ddo = smem_desc_sw128(adO, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * C::kSubBytes + (kk & 3) * 32;
          mma_ss(tDP, desc_at(dV0, off), desc_at(ddo, off), C::kIdescST, kk > 0 ? 1u : 0u);
          mid(kk);
        }
      };
      // dV += P^T dO: A = P^T (shared memory, K-major over q), B = dO (MN-major over d)
      auto issue_dv = [&](uint32_t adO, bool first) {
        const uint64_t da = smem_desc_sw128(aP, 16, 1024);
        const uint64_t db = smem_desc_sw128(adO, C::kSubBytes, 1024);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          mma_ss(tDV, desc_at(da, (kk >> 2) * C::kSubBytes + (kk & 3) * 32), desc_at(db, kk * 2048),
                 C::kIdescAcc, (first && kk == 0) ? 0u : 1u);
          mid(kk);
        }
      };
      // dK += dS^T Q: A = dS^T (packed bf16 in TMEM), B = Q (MN-major over d)
      auto issue_dk = [&](uint32_t aQ, bool first) {
        const uint64_t db = smem_desc_sw128(aQ, C::kSubBytes, 1024);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ts(tDK, tDP + packed_kstep(kk), desc_at(db, kk * 2048), C::kIdescAcc,
                 (first && kk == 0) ? 0u : 1u);
      };
      auto q_full_of = [&](uint32_t cnt) { return &q_full[cnt % C::kStages]; };
      auto q_phase_of = [&](uint32_t cnt) { return (cnt / C::kStages) & 1; };
      // Per q tile t the order is S^T(t+1), dV(t), dK(t), dP^T(t+1): S^T(t+1)
      // is issued as soon as the elementwise warps have read S^T(t) out of
      // TMEM, so it runs under their exponential phase of t.
      for (int round = 0; ok; ++round) {
        const int w = snake_item(round, cta, grid);
        if (w >= P.n_items) break;
        int jt, bh;
        decode_item(P, w, false, jt, bh);
        QIter qi;
        qi.init(P, jt);
        int n = 0, qt, dg;
        while (qi.next(P, qt, dg)) ++n;
        const uint32_t base = q_cnt;
        q_cnt += n;
        if (!mbar_wait(kv_full, items & 1, abort_flag, P.err) ||
            !mbar_wait(q_full_of(base), q_phase_of(base), abort_flag, P.err))
          break;
        tc_fence_after();
        issue_st(q_addr(base));
        tc_commit(s_ready);
        if (n > 1) {
          pa.set(s_free, base & 1);
          pb.set(q_full_of(base + 1), q_phase_of(base + 1));
        }
        issue_dpt(q_addr(base) + C::kTileBytes);
        tc_commit(dp_ready);
        for (int t = 0; t < n; ++t) {
          const uint32_t cnt = base + t;
          const uint32_t aQ = q_addr(cnt), adO = aQ + C::kTileBytes;
          if (t + 1 < n) {
            if (!pa.finish(abort_flag, P.err) || !pb.finish(abort_flag, P.err)) {
              ok = false;
              break;
            }
            tc_fence_after();
            pa.set(pa_ready, cnt & 1);
            issue_st(q_addr(cnt + 1));
            tc_commit(s_ready);
          } else {
            pa.set(pa_ready, cnt & 1);
          }
          if (!pa.finish(abort_flag, P.err) ||
              (t == 0 && items > 0 && !mbar_wait(acc_free, (items - 1) & 1, abort_flag, P.err))) {
            ok = false;
            break;
          }
          tc_fence_after();
          pa.set(pb_ready, cnt & 1);
          issue_dv(adO, t == 0);
          tc_commit(p_free);
          if (!pa.finish(abort_flag, P.err)) { ok = false; break; }
          tc_fence_after();
          issue_dk(aQ, t == 0);
          tc_commit(&q_empty[cnt % C::kStages]);
          if (t + 1 < n) {
            if (t + 2 < n) {
              pa.set(s_free, (cnt + 1) & 1);
              pb.set(q_full_of(cnt + 2), q_phase_of(cnt + 2));
            }
            issue_dpt(q_addr(cnt + 1) + C::kTileBytes);
            tc_commit(dp_ready);
          }
        }
        if (!ok) break;
        tc_commit(kv_empty);
        tc_commit(kv_done);
        ++items;
      }
      tc_commit(drain);
      const unsigned long long t0 = globaltimer();
      while (!mbar_try_wait(drain, 0) && globaltimer() - t0 < kWaitLimitNs) {
      }
    }
    __syncwarp();
  }

  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

// delta_i = sum_d dO_id O_id and LSE_i * log2(e).  HBM-bound: each thread
// reads 16-byte pieces of O and dO (D/8 threads per row), two rows per thread
// so that four loads are in flight, and the row's partial sums meet through
// shuffles among its D/8 lanes.
template <int D>
__global__ void __launch_bounds__(256) bwd_pre_kernel(const __nv_bfloat16* __restrict__ o,
                                                      const __nv_bfloat16* __restrict__ dout,
                                                      const float* __restrict__ lse,
                                                      float* __restrict__ delta,
                                                      float* __restrict__ lse2, long rows) {
  constexpr int TPR = D / 8;                 // threads per row
  constexpr int RPB = 256 / TPR;             // rows per pass of the block
  const int sub = threadIdx.x % TPR, rl = threadIdx.x / TPR;
  const long r0 = (long)blockIdx.x * (2 * RPB) + rl, r1 = r0 + RPB;
  float acc[2] = {0.f, 0.f};
  uint4 a[2], b[2];
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const long row = k ? r1 : r0;
    if (row < rows) {
      a[k] = reinterpret_cast<const uint4*>(o + row * D)[sub];
      b[k] = reinterpret_cast<const uint4*>(dout + row * D)[sub];
    } else {
      a[k] = b[k] = make_uint4(0, 0, 0, 0);
    }
  }
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const uint32_t ua[4] = {a[k].x, a[k].y, a[k].z, a[k].w}, ub[4] = {b[k].x, b[k].y, b[k].z, b[k].w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const __nv_bfloat162 x = *reinterpret_cast<const __nv_bfloat162*>(&ua[e]);
      const __nv_bfloat162 y = *reinterpret_cast<const __nv_bfloat162*>(&ub[e]);
      acc[k] = fmaf(__low2float(x), __low2float(y), acc[k]);
      acc[k] = fmaf(__high2float(x), __high2float(y), acc[k]);
    }
#pragma unroll
    for (int off = TPR / 2; off > 0; off >>= 1) acc[k] += __shfl_xor_sync(0xffffffffu, acc[k], off);
  }
  if (sub == 0) {
    if (r0 < rows) {
      delta[r0] = acc[0];
      lse2[r0] = lse[r0] * kLog2e;
    }
    if (r1 < rows) {
      delta[r1] = acc[1];
      lse2[r1] = lse[r1] * kLog2e;
    }
  }
}

template <int D>
int launch_impl(const AttnShape& sh, const void* q, const void* k, const void* v, const void* o,
                const float* lse, const void* dout, void* dq, void* dk, void* dv, float* ws_delta,
                float* ws_lse2, int acc_f32, unsigned* err, cudaStream_t stream) {
  const long rows = (long)sh.B * sh.H * sh.S;
  CUtensorMap mq, mk, mv, mdo;
  if (!make_tmap_bf16_2d(&mq, q, rows, D, 64, 128) || !make_tmap_bf16_2d(&mk, k, rows, D, 64, 128) ||
      !make_tmap_bf16_2d(&mv, v, rows, D, 64, 128) || !make_tmap_bf16_2d(&mdo, dout, rows, D, 64, 128))
    return -1;
  prof_begin(kKDelta, stream);
  constexpr int kPreRows = 2 * 256 / (D / 8);  // rows per block of the preprocess
  bwd_pre_kernel<D><<<(unsigned)((rows + kPreRows - 1) / kPreRows), 256, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(dout), lse, ws_delta,
      ws_lse2, rows);
  prof_end(kKDelta, stream);
  if (cudaGetLastError() != cudaSuccess) return -1;

  BwdParams P;
  P.g = sh.g;
  P.BH = sh.B * sh.H;
  P.T = sh.g.c / 128;
  P.tiles = sh.S / 128;
  P.n_items = P.BH * P.tiles;
  P.G = (P.BH % 2 == 0) ? 2 : 1;
  P.sl2 = sh.scale * kLog2e;
  P.scale = sh.scale;
  P.lse2 = ws_lse2;
  P.delta = ws_delta;
  P.q = static_cast<const __nv_bfloat16*>(q);
  P.dout = static_cast<const __nv_bfloat16*>(dout);
  P.dq = static_cast<__nv_bfloat16*>(dq);
  P.dk = static_cast<__nv_bfloat16*>(dk);
  P.dv = static_cast<__nv_bfloat16*>(dv);
  P.acc_f32 = acc_f32;
  P.dq_acc = static_cast<float*>(dq);
  P.dk_acc = static_cast<float*>(dk);
  P.dv_acc = static_cast<float*>(dv);
  P.err = err;
  static std::atomic<unsigned long long> attr_done{0};
  if (!smem_attr_once(tc_dkdv_kernel<D>, DkdvCfg<D>::kSmemBytes, attr_done)) return -1;
  // One CTA per work item, items numbered longest first: the hardware block
  // scheduler hands them out in that order as SMs free up, a greedy
  // longest-first schedule.  (The kernels also run as a persistent grid --
  // fewer CTAs than items, a static snake assignment -- which balances worse:
  // 1-2% slower here.)
  const int grid = P.n_items;
  prof_begin(kKTcDkdv, stream);
  tc_dkdv_kernel<D><<<grid, 384, DkdvCfg<D>::kSmemBytes, stream>>>(mq, mk, mv, mdo, P);
  prof_end(kKTcDkdv, stream);
  if (cudaGetLastError() != cudaSuccess) return -1;
  if (tc_dq2_supported(P, D)) {
    if (launch_tc_dq2(P, k, v, rows, stream) < 0) return -1;
  } else if (launch_tc_dq<D>(P, mq, mk, mv, mdo, grid, stream) < 0) {
    return -1;
  }
  return 3;
}

}  // namespace
}  // namespace bwd

bool tc_bwd_supported(const AttnShape& sh) {
  if (!sh.bf16) return false;
  if (sh.D != 64 && sh.D != 128) return false;
  if (sh.g.c % 128 != 0) return false;
  if ((long long)sh.B * sh.H * sh.S >= (1LL << 31)) return false;
  return true;
}

int launch_tc_bwd(const AttnShape& sh, const void* q, const void* k, const void* v,
                  const void* o, const float* lse, const void* dout, void* dq, void* dk,
                  void* dv, float* ws_delta, float* ws_lse2, int acc_f32, unsigned* err,
                  cudaStream_t stream) {
  if (sh.D == 64)
    return bwd::launch_impl<64>(sh, q, k, v, o, lse, dout, dq, dk, dv, ws_delta, ws_lse2, acc_f32,
                                err, stream);
  return bwd::launch_impl<128>(sh, q, k, v, o, lse, dout, dq, dk, dv, ws_delta, ws_lse2, acc_f32,
                               err, stream);
}

}  // namespace cpattn
