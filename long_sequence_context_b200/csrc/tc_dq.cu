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
// Operands.  Q and dO are the same for every K/V tile of a work item, so the
// elementwise warps put their rows into TMEM once per item and both S and dP
// are TS MMAs (A from TMEM): only the K / V tile is read from shared memory,
// half the shared-memory operand traffic of two shared-memory operands.
//
// Overlap.  The elementwise work of a tile is split into an exponential phase
// that needs only S_j and a dS phase that needs dP_j.  S_j is read out of TMEM
// at once and released, so S_{j+1} is computed during the exponential phase of
// j; dS_j replaces dP_j in TMEM, and after it the MMA thread issues
// dQ += dS_j K_j and then dP_{j+1}, which run during the exponential phase of
// j+1.  The MMA thread tests the barriers of its next MMA group between the
// MMAs of the current one.
//
// TMEM (512 columns): Q [0,D/2) dO [D/2,D) (bf16, two per column), S [128,256)
// dP / dS [256,384) dQ [384,384+D).
// Roles (384 threads): warps 0-7 elementwise (warp w: TMEM lanes 32*(w%4)..,
// score columns 64*(w/4)..; 208 registers via setmaxnreg), warp 8 TMA (a ring
// of K / V tiles), warp 9 MMA issuer and TMEM owner, warps 10-11 only complete
// the third warpgroup (88 registers).  One CTA per Q tile, longest first.  dS
// of column half h is packed as bf16 into columns [64 h, 64 h + 32) of dP's
// range.
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
  static constexpr int kStages = D == 128 ? 6 : 12;   // K / V slots
  static constexpr int kOffKV = 0;
  static constexpr int kOffBar = kOffKV + kStages * kTileBytes;
  static constexpr int kSmemBytes = 1024 + kOffBar + 256;
  static constexpr int kRowWords = D / 2;             // TMEM columns of one bf16 row
  static constexpr uint32_t kColQ = 0, kColDO = kRowWords, kColS = 128, kColDP = 256, kColDQ = 384;
  static constexpr uint32_t kIdescS = idesc_bf16_f32(128, 128, 0, 0);
  static constexpr uint32_t kIdescDQ = idesc_bf16_f32(128, D, 0, 1);
  static_assert(kSmemBytes <= 232448, "shared memory per CTA");
};

// TMEM column of the packed bf16 pair for score columns (c, c+1): column half
// h = c / 64 packs into [64 h, 64 h + 32).
__device__ __forceinline__ uint32_t packed_col(int c) { return (c & 64) + ((c & 63) >> 1); }
// TMEM column of k-step kk (16 score columns) of the packed operand
__device__ __forceinline__ uint32_t packed_kstep(int kk) { return (kk >= 4 ? 64 : 0) + (kk & 3) * 8; }

// One bf16 row of D elements from global memory into TMEM columns
// [col, col + D/2) of this thread's lane (two elements per column).
template <int D>
__device__ __forceinline__ void row_to_tmem(const __nv_bfloat16* src, uint32_t taddr) {
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

template <int D>
__global__ void __launch_bounds__(384, 1)
    tc_dq_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                 const BwdParams P) {
  using C = DqCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sKV = smem + C::kOffKV;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* kv_full = bars;                  // [kStages]
  uint64_t* kv_empty = bars + C::kStages;    // [kStages]
  uint64_t* q_ready = bars + 2 * C::kStages;  // Q and dO rows in TMEM (256 arrivals)
  uint64_t* s_ready = q_ready + 1;           // S_j in TMEM
  uint64_t* s_free = q_ready + 2;            // S_j read out of TMEM (256 arrivals)
  uint64_t* dp_ready = q_ready + 3;          // dP_j in TMEM
  uint64_t* p_ready = q_ready + 4;           // dS_j written to TMEM (256 arrivals)
  uint64_t* dq_done = q_ready + 5;
  uint64_t* acc_free = q_ready + 6;
  uint64_t* drain = q_ready + 7;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(q_ready + 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    mbar_init(q_ready, 256);
    mbar_init(s_ready, 1);
    mbar_init(s_free, 256);
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
    prefetch_tensormap(&tmK);
    prefetch_tensormap(&tmV);
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
    const uint32_t tS = tmem_base + lane_off + C::kColS + half * 64;
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
      // the A operands of S = Q K^T and dP = dO V^T: this row of Q (column
      // half 0's warps) or of dO (half 1's) into TMEM; the previous item's
      // MMAs have completed (its dQ was read out below)
      if (half == 0)
        row_to_tmem<D>(P.q + row * D, tmem_base + lane_off + C::kColQ);
      else
        row_to_tmem<D>(P.dout + row * D, tmem_base + lane_off + C::kColDO);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(q_ready);
      KIter<128> ki;
      ki.init(P, qt);
      int kt, doff, nt = 0;
      while (ki.next(P, kt, doff)) {
        ++nt;
        // exponential phase: S_j is read out at once (S_{j+1} may then be
        // computed into the same columns)
        if (!mbar_wait_warp(s_ready, j_cnt & 1, abort_flag, P.err)) { ok = false; break; }
        tc_fence_after();
        uint32_t sv[64];
        tmem_ld32<0>(tS, sv);
        tmem_ld32<32>(tS + 32, sv);
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(s_free);
        float p[64];
#pragma unroll
        for (int c = 0; c < 64; c += 2) {
          const float2 x = ffma2(make_float2(__uint_as_float(sv[c]), __uint_as_float(sv[c + 1])),
                                 make_float2(P.sl2, P.sl2), make_float2(-lse2, -lse2));
          p[c] = ex2(x.x);
          p[c + 1] = ex2(x.y);
        }
        if (doff >= 0) {
          // diagonal tile: keys after the query are masked
#pragma unroll
          for (int c = 0; c < 64; ++c)
            if (half * 64 + c > rloc) p[c] = 0.f;
        }
        // dS phase: needs dP_j; dS_j replaces it in TMEM (A operand of dQ)
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
          tmem_st16<0>(tmem_base + lane_off + C::kColDP + packed_col(half * 64 + ch * 32), dsk);
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
      mbar_arrive(acc_free);
    }
  } else {
    regs_dec<88>();
  }
  if (warp == 8) {
    // ----------------------------------------------------------------- TMA --
    uint32_t kv_idx = 0;
    bool ok = true;
    for (int round = 0; ok; ++round) {
      const int w = snake_item(round, cta, grid);
      if (w >= P.n_items) break;
      int qt, bh;
      decode_item(P, w, true, qt, bh);
      const int rowbase = bh * S;
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
      const uint32_t first = kv_idx > (uint32_t)C::kStages ? kv_idx - C::kStages : 0;
      for (uint32_t i = first; i < kv_idx; ++i)
        while (!mbar_try_wait(&kv_full[i % C::kStages], (i / C::kStages) & 1) &&
               globaltimer() - t0 < kWaitLimitNs) {
        }
    }
  } else if (warp == 9) {
    // ----------------------------------------------------------------- MMA --
    if (lane == 0) {
      const uint32_t tQ = tmem_base + C::kColQ, tDO = tmem_base + C::kColDO;
      const uint32_t tS = tmem_base + C::kColS, tDP = tmem_base + C::kColDP, tDQ = tmem_base + C::kColDQ;
      const uint32_t aKV = smem_u32(sKV);
      uint32_t kv_idx = 0, j_cnt = 0, items = 0;
      bool ok = true;
      auto slot_of = [&](uint32_t idx) { return idx % C::kStages; };
      auto phase_of = [&](uint32_t idx) { return (idx / C::kStages) & 1; };
      // S = Q K^T and dP = dO V^T: A from TMEM, B (K / V tile) K-major.  The
      // barriers of the next MMA group are tested between the MMAs of the
      // current one (Probe), so that their latency overlaps queued tensor work.
      Probe pa, pb;
      auto issue_qk = [&](uint32_t t_d, uint32_t t_a, uint32_t slot) {
        const uint64_t db = smem_desc_sw128(aKV + slot * C::kTileBytes, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          mma_ts(t_d, t_a + kk * 8, desc_at(db, (kk >> 2) * C::kSubBytes + (kk & 3) * 32), C::kIdescS,
                 kk > 0 ? 1u : 0u);
          if (kk == 1 || kk == D / 16 - 2) {
            pa.test();
            pb.test();
          }
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
        if (n == 0) {  // no K/V tile (not reached by the ring walks): dQ stays zero
          if (!mbar_wait(q_ready, items & 1, abort_flag, P.err)) break;
          tc_commit(dq_done);
          ++items;
          continue;
        }
        if (!mbar_wait(q_ready, items & 1, abort_flag, P.err) ||
            !mbar_wait(&kv_full[slot_of(base)], phase_of(base), abort_flag, P.err)) break;
        tc_fence_after();
        pa.set(&kv_full[slot_of(base + 1)], phase_of(base + 1));
        issue_qk(tS, tQ, slot_of(base));  // S_0
        tc_commit(s_ready);
        if (!pa.finish(abort_flag, P.err)) break;
        tc_fence_after();
        if (n > 1) {
          pa.set(s_free, j_cnt & 1);
          pb.set(&kv_full[slot_of(base + 2)], phase_of(base + 2));
        }
        issue_qk(tDP, tDO, slot_of(base + 1));  // dP_0
        tc_commit(dp_ready);
        tc_commit(&kv_empty[slot_of(base + 1)]);
        for (int t = 0; t < n; ++t) {
          const uint32_t cnt = j_cnt + t;
          if (t + 1 < n) {  // S_{t+1} once S_t has been read out
            if (!pa.finish(abort_flag, P.err) || !pb.finish(abort_flag, P.err)) {
              ok = false;
              break;
            }
            tc_fence_after();
            pa.set(p_ready, cnt & 1);
            issue_qk(tS, tQ, slot_of(base + 2 * (t + 1)));
            tc_commit(s_ready);
          } else {
            pa.set(p_ready, cnt & 1);
          }
          // dS_t in TMEM (in dP's columns)
          if (!pa.finish(abort_flag, P.err) ||
              (t == 0 && items > 0 && !mbar_wait(acc_free, (items - 1) & 1, abort_flag, P.err))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t iv = base + 2 * (t + 1) + 1;
          if (t + 1 < n) pa.set(&kv_full[slot_of(iv)], phase_of(iv));
          {  // dQ += dS_t K_t
            const uint64_t dk = smem_desc_sw128(aKV + slot_of(base + 2 * t) * C::kTileBytes,
                                                C::kSubBytes, 1024);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              mma_ts(tDQ, tDP + packed_kstep(kk), desc_at(dk, kk * 2048), C::kIdescDQ,
                     (t == 0 && kk == 0) ? 0u : 1u);
              if (kk == 1 || kk == 6) pa.test();
            }
            tc_commit(&kv_empty[slot_of(base + 2 * t)]);
          }
          if (t + 1 < n) {  // dP_{t+1} into the columns dS_t occupied
            if (!pa.finish(abort_flag, P.err)) { ok = false; break; }
            tc_fence_after();
            if (t + 2 < n) {
              pa.set(s_free, (cnt + 1) & 1);
              pb.set(&kv_full[slot_of(base + 2 * (t + 2))], phase_of(base + 2 * (t + 2)));
            }
            issue_qk(tDP, tDO, slot_of(iv));
            tc_commit(dp_ready);
            tc_commit(&kv_empty[slot_of(iv)]);
          }
        }
        if (!ok) break;
        j_cnt += n;
        tc_commit(dq_done);
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

}  // namespace

template <int D>
int launch_tc_dq(const BwdParams& P, const CUtensorMap& mq, const CUtensorMap& mk,
                 const CUtensorMap& mv, const CUtensorMap& mdo, int grid, cudaStream_t stream) {
  using C = DqCfg<D>;
  static std::atomic<unsigned long long> attr_done{0};
  if (!smem_attr_once(tc_dq_kernel<D>, C::kSmemBytes, attr_done)) return -1;
  prof_begin(kKTcDq, stream);
  tc_dq_kernel<D><<<grid, 384, C::kSmemBytes, stream>>>(mk, mv, P);
  prof_end(kKTcDq, stream);
  return cudaGetLastError() == cudaSuccess ? 1 : -1;
}

template int launch_tc_dq<64>(const BwdParams&, const CUtensorMap&, const CUtensorMap&,
                              const CUtensorMap&, const CUtensorMap&, int, cudaStream_t);
template int launch_tc_dq<128>(const BwdParams&, const CUtensorMap&, const CUtensorMap&,
                               const CUtensorMap&, const CUtensorMap&, int, cudaStream_t);

}  // namespace bwd
}  // namespace cpattn
