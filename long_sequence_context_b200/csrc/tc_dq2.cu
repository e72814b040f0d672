// tc_dq2.cu -- two-SM (cta_group::2) tcgen05 dQ kernel of the recompute
// backward (bf16, D = 128, an even number of 128-row tiles per chunk).
//
// The computation is that of tc_dq.cu (S_j = Q K_j^T, dP_j = dO V_j^T,
// P_j = exp2(S_j scale log2 e - LSE log2 e), dS_j = P_j (dP_j - delta),
// dQ += dS_j K_j; sources: "Configuring RingAttention+FlashAttention for CP",
// section 3 code, note 2 and section 5 item 1; "Megatron-LM source analysis:
// Context Parallel", section 2), arranged over a cluster of two CTAs on the
// two SMs of one TPC:
//   - A work item is a pair of adjacent Q tiles of one chunk; CTA r of the
//     cluster owns tile 2p + r.  Both walk the K/V tiles of the later tile (the
//     earlier tile's extra diagonal tile is fully masked for it).
//   - One thread of CTA 0 issues every MMA as M = 256: each CTA's TMEM holds
//     its own Q and dO rows (the A operands), S, dP / dS and dQ for its 128
//     rows, and each CTA's shared memory holds half of every B operand: for S
//     and dP the K / V rows 64 r .. 64 r + 63, for dQ += dS K the K columns
//     64 r .. 64 r + 63.  So each SM loads and reads half of each K/V tile,
//     and one MMA instruction does both SMs' work.
//   - Both CTAs' TMA loads complete on CTA 0's barriers; CTA 0's MMA
//     completions arrive on the barriers of both CTAs; CTA 1's elementwise
//     warps arrive on CTA 0's barriers (one arrival per warp).
// Roles per CTA (384 threads): warps 0-7 elementwise (TMEM lane quarter w%4,
// score column half w/4; 208 registers via setmaxnreg), warp 8 TMA, warp 9 MMA
// issuer (CTA 0 only) and TMEM owner, warps 10-11 complete the third
// warpgroup (88 registers).
// TMEM (512 columns per CTA): Q [0,64) dO [64,128) (bf16 pairs), S [128,256),
// dP / dS [256,384), dQ [384,512).
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

struct Dq2Cfg {
  static constexpr int D = 128;
  static constexpr int kHalfRows = 64 * D * 2;        // 64 rows of a tile, both 64-column blocks: 16 KB
  static constexpr int kSub64 = 64 * 128;             // one 64-row x 64-column swizzled block: 8 KB
  static constexpr int kColBlock = 128 * 128;         // 128 rows x 64 columns: 16 KB
  // ring entry: K rows (64 r..) | K columns (64 r..) | V rows (64 r..)
  static constexpr int kOffKRows = 0, kOffKCols = kHalfRows, kOffVRows = kHalfRows + kColBlock;
  static constexpr int kEntryBytes = kOffVRows + kHalfRows;  // 48 KB
  static constexpr int kStages = 4;
  static constexpr int kOffBar = kStages * kEntryBytes;
  static constexpr int kSmemBytes = 1024 + kOffBar + 256;
  static constexpr uint32_t kColQ = 0, kColDO = 64, kColS = 128, kColDP = 256, kColDQ = 384;
  static constexpr uint32_t kIdescS = idesc_bf16_f32(256, 128, 0, 0);   // M = 256 over the pair
  static constexpr uint32_t kIdescDQ = idesc_bf16_f32(256, D, 0, 1);
  static constexpr int kArrivals = 16;                // 8 elementwise warps x 2 CTAs
  static_assert(kSmemBytes <= 232448, "shared memory per CTA");
};

__device__ __forceinline__ uint32_t packed_col2(int c) { return (c & 64) + ((c & 63) >> 1); }
__device__ __forceinline__ uint32_t packed_kstep2(int kk) { return (kk >= 4 ? 64 : 0) + (kk & 3) * 8; }

template <int D>
__device__ __forceinline__ void row_to_tmem2(const __nv_bfloat16* src, uint32_t taddr) {
  const uint4* s4 = reinterpret_cast<const uint4*>(src);
#pragma unroll
  for (int part = 0; part < D / 2; part += 32) {
    uint32_t w[32];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint4 u = s4[part / 4 + i];
      w[4 * i] = u.x;
      w[4 * i + 1] = u.y;
      w[4 * i + 2] = u.z;
      w[4 * i + 3] = u.w;
    }
    tmem_st32<0>(taddr + part, w);
  }
}

// pair index -> (head, later tile of the pair): heads G at a time, latest
// (longest) pairs first
__device__ __forceinline__ void decode_pair(const BwdParams& P, int w, int& qt1, int& bh) {
  const int pairs = P.tiles / 2;
  const int per_group = P.G * pairs;
  const int g = w / per_group, r = w % per_group;
  qt1 = 2 * (pairs - 1 - r / P.G) + 1;
  bh = g * P.G + r % P.G;
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(384, 1)
    tc_dq2_kernel(const __grid_constant__ CUtensorMap tmK64, const __grid_constant__ CUtensorMap tmK128,
                  const __grid_constant__ CUtensorMap tmV64, const BwdParams P) {
  using C = Dq2Cfg;
  constexpr int D = C::D;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* k_full = bars;                    // [kStages] (CTA 0's count both CTAs' bytes)
  uint64_t* v_full = bars + C::kStages;       // [kStages]
  uint64_t* kv_empty = bars + 2 * C::kStages;  // [kStages]
  uint64_t* q_ready = bars + 3 * C::kStages;  // Q, dO rows in TMEM (16 warp arrivals, CTA 0)
  uint64_t* s_ready = q_ready + 1;            // S_j in TMEM
  uint64_t* s_free = q_ready + 2;             // S_j read out (16 arrivals, CTA 0)
  uint64_t* dp_ready = q_ready + 3;           // dP_j in TMEM
  uint64_t* p_ready = q_ready + 4;            // dS_j in TMEM (16 arrivals, CTA 0)
  uint64_t* dq_done = q_ready + 5;
  uint64_t* acc_free = q_ready + 6;           // dQ read out (16 arrivals, CTA 0)
  uint64_t* drain = q_ready + 7;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(q_ready + 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    mbar_init(q_ready, C::kArrivals);
    mbar_init(s_ready, 1);
    mbar_init(s_free, C::kArrivals);
    mbar_init(dp_ready, 1);
    mbar_init(p_ready, C::kArrivals);
    mbar_init(dq_done, 1);
    mbar_init(acc_free, C::kArrivals);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 9) {
    tmem_alloc_pair(tmem_slot, 512);
    tmem_relinquish_pair();
  }
  if (warp == 8 && lane == 0) {
    prefetch_tensormap(&tmK64);
    prefetch_tensormap(&tmK128);
    prefetch_tensormap(&tmV64);
  }
  // both CTAs' barriers are initialised before either CTA touches the other's
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int S = P.g.S;
  // one arrival per warp on CTA 0's barrier (lane 0, after the warp's own
  // TMEM accesses are complete and fenced)
  auto arrive_leader = [&](uint64_t* bar) {
    __syncwarp();
    if (lane == 0) {
      if (rank == 0)
        mbar_arrive(bar);
      else
        mbar_arrive_remote(mapa_shared(smem_u32(bar), 0));
    }
  };

  if (warp < 8) {
    // ---------------------------------------------------------- elementwise --
    regs_inc<208>();
    const int quarter = warp & 3, half = warp >> 2;
    const int rloc = quarter * 32 + lane;  // query row within this CTA's Q tile
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const uint32_t tS = tmem_base + lane_off + C::kColS + half * 64;
    const uint32_t tDP = tmem_base + lane_off + C::kColDP + half * 64;
    uint32_t j_cnt = 0, items = 0;
    bool ok = true;
    for (int round = 0; ok; ++round) {
      const int w = snake_item(round, pair, npairs);
      if (w >= P.n_items / 2) break;
      int qt1, bh;
      decode_pair(P, w, qt1, bh);
      const int qt = qt1 - 1 + (int)rank;
      const long row = (long)bh * S + (long)qt * 128 + rloc;
      const float lse2 = P.lse2[row];
      const float dlt = P.delta[row];
      // this row of Q (column half 0's warps) or of dO (half 1's) into TMEM;
      // the previous item's MMAs have completed (its dQ was read out below)
      if (half == 0)
        row_to_tmem2<D>(P.q + row * D, tmem_base + lane_off + C::kColQ);
      else
        row_to_tmem2<D>(P.dout + row * D, tmem_base + lane_off + C::kColDO);
      tmem_wait_st();
      tc_fence_before();
      arrive_leader(q_ready);
      KIter<128> ki;
      ki.init(P, qt1);
      int kt, doff, nt = 0;
      while (ki.next(P, kt, doff)) {
        ++nt;
        // key tile offset from this CTA's own Q tile inside a DIAG block
        const int off = ki.diag ? kt - qt : -1;
        if (!mbar_wait_warp(s_ready, j_cnt & 1, abort_flag, P.err)) { ok = false; break; }
        tc_fence_after();
        uint32_t sv[64];
        tmem_ld32<0>(tS, sv);
        tmem_ld32<32>(tS + 32, sv);
        tmem_wait_ld();
        tc_fence_before();
        arrive_leader(s_free);
        float p[64];
#pragma unroll
        for (int c = 0; c < 64; c += 2) {
          const float2 x = ffma2(make_float2(__uint_as_float(sv[c]), __uint_as_float(sv[c + 1])),
                                 make_float2(P.sl2, P.sl2), make_float2(-lse2, -lse2));
          p[c] = ex2(x.x);
          p[c + 1] = ex2(x.y);
        }
        if (off >= 0) {
          // keys after the query are masked (a whole tile when off >= 1)
#pragma unroll
          for (int c = 0; c < 64; ++c)
            if (off * 128 + half * 64 + c > rloc) p[c] = 0.f;
        }
        if (!mbar_wait_warp(dp_ready, j_cnt & 1, abort_flag, P.err)) { ok = false; break; }
        ++j_cnt;
        tc_fence_after();
        uint32_t dpv[64];
        tmem_ld32<0>(tDP, dpv);
        tmem_ld32<32>(tDP + 32, dpv);
        tmem_wait_ld();
#pragma unroll
        for (int ch = 0; ch < 2; ++ch) {
          uint32_t dsk[16];
#pragma unroll
          for (int c = 0; c < 32; c += 2) {
            const int e = ch * 32 + c;
            const float2 ds = fmul2(make_float2(p[e], p[e + 1]),
                                    fsub2(make_float2(__uint_as_float(dpv[e]), __uint_as_float(dpv[e + 1])),
                                          make_float2(dlt, dlt)));
            dsk[c >> 1] = pack_bf16x2(ds.x, ds.y);
          }
          tmem_st16<0>(tmem_base + lane_off + C::kColDP + packed_col2(half * 64 + ch * 32), dsk);
        }
        tmem_wait_st();
        tc_fence_before();
        arrive_leader(p_ready);
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
        if (nt == 0) {
#pragma unroll
          for (int c = 0; c < 32; ++c) v[c] = 0u;
        }
        if (P.acc_f32)
          add_row32(P.dq_acc + row * D + col, v, P.scale);
        else
          store_row32(P.dq + row * D + col, v, P.scale);
      }
      tc_fence_before();
      arrive_leader(acc_free);
    }
  } else {
    regs_dec<88>();
  }
  if (warp == 8) {
    // ----------------------------------------------------------------- TMA --
    // Both CTAs load their halves; the bytes complete on CTA 0's barriers,
    // whose expected byte counts CTA 0 sets for the pair.
    if (lane == 0) {
      uint32_t kv_idx = 0;
      bool ok = true;
      for (int round = 0; ok; ++round) {
        const int w = snake_item(round, pair, npairs);
        if (w >= P.n_items / 2) break;
        int qt1, bh;
        decode_pair(P, w, qt1, bh);
        const int rowbase = bh * S;
        KIter<128> ki;
        ki.init(P, qt1);
        int kt, doff;
        while (ki.next(P, kt, doff)) {
          const int s = kv_idx % C::kStages;
          if (kv_idx >= (uint32_t)C::kStages &&
              !mbar_wait(&kv_empty[s], ((kv_idx / C::kStages) - 1) & 1, abort_flag, P.err)) {
            ok = false;
            break;
          }
          if (rank == 0) {
            mbar_expect_tx(&k_full[s], 2 * (C::kHalfRows + C::kColBlock));
            mbar_expect_tx(&v_full[s], 2 * C::kHalfRows);
          }
          const uint32_t kb = mapa_shared(smem_u32(&k_full[s]), 0);
          const uint32_t vb = mapa_shared(smem_u32(&v_full[s]), 0);
          uint8_t* e = smem + s * C::kEntryBytes;
          const int y0 = rowbase + kt * 128;
#pragma unroll
          for (int sb = 0; sb < D / 64; ++sb) {
            tma_load_2d_pair(e + C::kOffKRows + sb * C::kSub64, &tmK64, kb, sb * 64, y0 + 64 * (int)rank);
            tma_load_2d_pair(e + C::kOffVRows + sb * C::kSub64, &tmV64, vb, sb * 64, y0 + 64 * (int)rank);
          }
          tma_load_2d_pair(e + C::kOffKCols, &tmK128, kb, 64 * (int)rank, y0);
          ++kv_idx;
        }
      }
      if (*abort_flag && rank == 0) {
        // loads in flight land before the CTA's shared memory goes away
        const unsigned long long t0 = globaltimer();
        const uint32_t first = kv_idx > (uint32_t)C::kStages ? kv_idx - C::kStages : 0;
        for (uint32_t i = first; i < kv_idx; ++i) {
          while (!mbar_try_wait(&k_full[i % C::kStages], (i / C::kStages) & 1) &&
                 globaltimer() - t0 < kWaitLimitNs) {
          }
          while (!mbar_try_wait(&v_full[i % C::kStages], (i / C::kStages) & 1) &&
                 globaltimer() - t0 < kWaitLimitNs) {
          }
        }
      }
    }
    __syncwarp();
  } else if (warp == 9) {
    // --------------------------------------------------- MMA (CTA 0 only) --
    if (lane == 0 && rank == 0) {
      const uint32_t tQ = tmem_base + C::kColQ, tDO = tmem_base + C::kColDO;
      const uint32_t tS = tmem_base + C::kColS, tDP = tmem_base + C::kColDP, tDQ = tmem_base + C::kColDQ;
      const uint32_t a0 = smem_u32(smem);
      uint32_t kv_idx = 0, j_cnt = 0, items = 0;
      bool ok = true;
      auto slot_of = [&](uint32_t idx) { return idx % C::kStages; };
      auto phase_of = [&](uint32_t idx) { return (idx / C::kStages) & 1; };
      // S = Q K^T, dP = dO V^T: A from TMEM, B = 64 K / V rows per CTA (K-major)
      auto issue_rows = [&](uint32_t t_d, uint32_t t_a, uint32_t b_addr) {
        const uint64_t db = smem_desc_sw128(b_addr, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ts_pair(t_d, t_a + kk * 8, desc_at(db, (kk >> 2) * C::kSub64 + (kk & 3) * 32), C::kIdescS,
                      kk > 0 ? 1u : 0u);
      };
      for (int round = 0; ok; ++round) {
        const int w = snake_item(round, pair, npairs);
        if (w >= P.n_items / 2) break;
        int qt1, bh;
        decode_pair(P, w, qt1, bh);
        KIter<128> ki;
        ki.init(P, qt1);
        int n = 0, kt, doff;
        while (ki.next(P, kt, doff)) ++n;
        const uint32_t base = kv_idx;
        kv_idx += n;
        if (!mbar_wait(q_ready, items & 1, abort_flag, P.err)) break;
        if (n == 0) {  // no K/V tile (not reached by the ring walks): dQ stays zero
          tc_commit_pair(dq_done);
          ++items;
          continue;
        }
        if (!mbar_wait(&k_full[slot_of(base)], phase_of(base), abort_flag, P.err)) break;
        tc_fence_after();
        issue_rows(tS, tQ, a0 + slot_of(base) * C::kEntryBytes + C::kOffKRows);  // S_0
        tc_commit_pair(s_ready);
        if (!mbar_wait(&v_full[slot_of(base)], phase_of(base), abort_flag, P.err)) break;
        tc_fence_after();
        issue_rows(tDP, tDO, a0 + slot_of(base) * C::kEntryBytes + C::kOffVRows);  // dP_0
        tc_commit_pair(dp_ready);
        if (n > 1) {  // S_1 once S_0 has been read out
          if (!mbar_wait(s_free, j_cnt & 1, abort_flag, P.err) ||
              !mbar_wait(&k_full[slot_of(base + 1)], phase_of(base + 1), abort_flag, P.err))
            break;
          tc_fence_after();
          issue_rows(tS, tQ, a0 + slot_of(base + 1) * C::kEntryBytes + C::kOffKRows);
          tc_commit_pair(s_ready);
        }
        // Per K/V tile t: dQ(t), dP(t+1), S(t+2).  S(t+2) is issued right after
        // dP(t+1), so it is complete before the elementwise warps finish t+1.
        for (int t = 0; t < n; ++t) {
          const uint32_t cnt = j_cnt + t;
          const uint32_t e = a0 + slot_of(base + t) * C::kEntryBytes;
          if (!mbar_wait(p_ready, cnt & 1, abort_flag, P.err) ||
              (t == 0 && items > 0 && !mbar_wait(acc_free, (items - 1) & 1, abort_flag, P.err))) {
            ok = false;
            break;
          }
          tc_fence_after();
          {  // dQ += dS_t K_t: B = 64 K columns per CTA (MN-major)
            const uint64_t dk = smem_desc_sw128(e + C::kOffKCols, C::kColBlock, 1024);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              mma_ts_pair(tDQ, tDP + packed_kstep2(kk), desc_at(dk, kk * 2048), C::kIdescDQ,
                          (t == 0 && kk == 0) ? 0u : 1u);
            tc_commit_pair(&kv_empty[slot_of(base + t)]);
          }
          if (t + 1 < n) {  // dP_{t+1} into the columns dS_t occupied
            const uint32_t i1 = base + t + 1;
            if (!mbar_wait(&v_full[slot_of(i1)], phase_of(i1), abort_flag, P.err)) { ok = false; break; }
            tc_fence_after();
            issue_rows(tDP, tDO, a0 + slot_of(i1) * C::kEntryBytes + C::kOffVRows);
            tc_commit_pair(dp_ready);
          }
          if (t + 2 < n) {  // S_{t+2} once S_{t+1} has been read out
            const uint32_t i2 = base + t + 2;
            if (!mbar_wait(s_free, (cnt + 1) & 1, abort_flag, P.err) ||
                !mbar_wait(&k_full[slot_of(i2)], phase_of(i2), abort_flag, P.err)) {
              ok = false;
              break;
            }
            tc_fence_after();
            issue_rows(tS, tQ, a0 + slot_of(i2) * C::kEntryBytes + C::kOffKRows);
            tc_commit_pair(s_ready);
          }
        }
        if (!ok) break;
        j_cnt += n;
        tc_commit_pair(dq_done);
        ++items;
      }
      tc_commit_pair(drain);
    }
    __syncwarp();
    // every MMA writing this CTA's TMEM or reading its shared memory is done
    const unsigned long long t0 = globaltimer();
    while (!mbar_try_wait(drain, 0) && globaltimer() - t0 < kWaitLimitNs) {
    }
  }

  __syncthreads();
  // neither CTA leaves (or frees TMEM) while the other may still address it
  cluster_sync();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, 512);
  }
}

}  // namespace

// (kernel path 2 keeps every tcgen05 kernel on one SM, for tests that compare)
bool tc_dq2_supported(const BwdParams& P, int D) {
  return kernel_path() != 2 && D == 128 && P.T % 2 == 0 && P.tiles % 2 == 0;
}

int launch_tc_dq2(const BwdParams& P, const void* k, const void* v, long rows, cudaStream_t stream) {
  using C = Dq2Cfg;
  CUtensorMap mk64, mk128, mv64;
  if (!make_tmap_bf16_2d(&mk64, k, rows, C::D, 64, 64) || !make_tmap_bf16_2d(&mk128, k, rows, C::D, 64, 128) ||
      !make_tmap_bf16_2d(&mv64, v, rows, C::D, 64, 64))
    return -1;
  static std::atomic<unsigned long long> attr_done{0};
  if (!smem_attr_once(tc_dq2_kernel, C::kSmemBytes, attr_done)) return -1;
  // one cluster of two CTAs per pair of Q tiles, longest pairs first
  const int grid = P.n_items;  // = 2 x pairs
  prof_begin(kKTcDq, stream);
  tc_dq2_kernel<<<grid, 384, C::kSmemBytes, stream>>>(mk64, mk128, mv64, P);
  prof_end(kKTcDq, stream);
  return cudaGetLastError() == cudaSuccess ? 1 : -1;
}

}  // namespace bwd
}  // namespace cpattn
