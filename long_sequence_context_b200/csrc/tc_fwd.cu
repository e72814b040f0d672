// tc_fwd.cu -- tcgen05 tensor-core ring-attention forward for bf16, D in {64,128}.
//
// One kernel runs every virtual rank and every ring step.  A work item (one
// CTA, longest items first) is a pair of 128-row Q tiles of one chunk; its K/V
// tiles are walked in ring order (step t: the chunks of rank (r - t) mod N, SKIP blocks never
// visited, DIAG blocks stopping at the pair's diagonal), and the per-step
// partials are merged on chip by the online log-sum-exp rescale.  Sources:
// "Configuring RingAttention+FlashAttention for CP" (devpress.csdn.net),
// section 3 code (ring rule), note 2 (exact mask), section 5 item 1 (zigzag);
// "Megatron-LM source analysis: Context Parallel" (mieleap.com), section 5:
// the double-buffered ring loop, whose receive double buffer becomes here the
// TMA-filled multi-stage K/V ring in shared memory.
//
// CTA roles (384 threads, three warpgroups):
//   warps 0-3  softmax for Q tile 0 (thread = query row = TMEM lane)
//   warps 4-7  softmax for Q tile 1
//   warp  8    TMA producer: Q tiles, then K_j, V_j into an NSTAGE-slot ring
//   warp  9    MMA issuer (one thread) and TMEM owner
//   warps 10-11 idle (they hand their registers to the softmax warpgroups)
// TMEM (512 columns): S0 [0,128) S1 [128,256) O0 [256,256+D) O1 [384,384+D);
// P_i (bf16, two per column) overwrites the first 64 columns of S_i and feeds
// the P.V MMA straight from TMEM.
// Per K/V tile j the MMA thread issues PV0(j-1), S0(j), PV1(j-1), S1(j), so
// softmax of one Q tile overlaps the MMAs of the other.
//
// FP8 variant (F8 = true, D = 128; "Megatron-LM source analysis: Context
// Parallel", section 4: FP8 attention inputs under context parallelism): Q, K
// and V^T arrive as e4m3 codes with per-tensor scales (code = e4m3(x * s),
// s = 448 / max|x|), the two products run as kind::f8f6f4 MMAs (K = 32 per
// instruction), V is stored transposed per head ([d][key]) so that both
// operands of P.V are K-major, and P is written back to TMEM as e4m3 (four per
// column) scaled by 2^6.  The running maximum is then kept within 2^2 of the
// true one, so the scaled P stays <= 2^8 < 448; the row sum l is taken from
// the unrounded P.
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
constexpr float kLn2 = 0.6931471805599453f;
// keep a stale row maximum unless the new one exceeds it by more than 2^8
// (bf16 P) or 2^2 (e4m3 P, which must stay below 448 after its 2^6 scale)
constexpr float kRescaleThreshold = 8.0f;
constexpr float kRescaleThresholdF8 = 2.0f;
constexpr float kP8Log2Scale = 6.0f;  // e4m3 P holds 2^6 * P

template <int D, bool F8>
struct FwdCfg {
  static constexpr int kTile = 128;                       // rows per Q / K / V tile
  static constexpr int kElem = F8 ? 1 : 2;                // bytes per element
  static constexpr int kTileBytes = kTile * D * kElem;    // one Q / K / V tile
  static constexpr int kSubBytes = kTile * 128;           // one 128-byte-wide swizzled block
  static constexpr int kStages = F8 ? 10 : (D == 128 ? 5 : 8);  // K/V slots
  static constexpr int kThreads = 384;
  // setmaxnreg split of the 384 x 168 launch registers: 2*128*Rs + 128*Ro <= 64512
  // (e4m3: 216 / 72 leaves the packed softmax free of spills)
  static constexpr int kRegsSoftmax = F8 ? 216 : 208;
  static constexpr int kRegsOther = F8 ? 72 : 80;
  static constexpr int kBarOffset = 2 * kTileBytes + kStages * kTileBytes;
  static constexpr int kSmemBytes = 1024 + kBarOffset + 256;
  static constexpr uint32_t kIdescQK = F8 ? idesc_e4m3_f32(128, 128) : idesc_bf16_f32(128, 128, 0, 0);
  static constexpr uint32_t kIdescPV = F8 ? idesc_e4m3_f32(128, D) : idesc_bf16_f32(128, D, 0, 1);
  static_assert(!F8 || D == 128, "the e4m3 path takes D = 128 (one 128-byte swizzled row)");
};

struct FwdParams {
  RingGeom g;
  int BH;          // batch * heads
  int T;           // 128-row tiles per chunk
  int pairs;       // work items per chunk: ceil(T / 2)
  int n_items;     // BH * n_chunks * pairs
  int G;           // heads per scheduling group (divides BH)
  int t0, t1;      // ring steps [t0, t1)
  int out_f32;     // 1: fp32 normalised partial output, 0: bf16 output
  float sl2;       // scale * log2(e)
  void* o;
  float* lse;
  const float* amax;  // e4m3 path: device max|q|, max|k|, max|v| (the scales' source)
  unsigned* err;
  int stall;       // omit one K load in CTA 0 (failure-detection tests)
};

struct Item {
  int bh, a, qt0, qt1, single;
};

__device__ __forceinline__ void decode_item(const FwdParams& P, int w, Item& it) {
  // heads are taken G at a time (the CTAs busy at any moment share a few
  // heads' K / V in L2); inside a group, descending global tile position =
  // descending causal cost (longest first), heads interleaved
  const int per_group = P.G * P.g.n_chunks * P.pairs;
  const int grp = w / per_group, rem = w % per_group;
  const int u = rem / P.G;
  it.bh = grp * P.G + rem % P.G;
  const int a_rev = u / P.pairs, p_rev = u % P.pairs;
  it.a = P.g.n_chunks - 1 - a_rev;
  const int p = P.pairs - 1 - p_rev;
  it.qt0 = it.a * P.T + 2 * p;
  it.single = (2 * p + 1 >= P.T);
  it.qt1 = it.single ? it.qt0 : it.qt0 + 1;
}

// Walks the K/V tiles of one work item in ring order.  Only the mutable walk
// state lives in registers; the geometry is read from the kernel parameters.
struct KvIter {
  int a, rank, qt_hi, t, s, kt, kt_end, diag;
  __device__ __forceinline__ void init(const FwdParams& P, const Item& it) {
    a = it.a;
    rank = chunk_owner(P.g, a);
    qt_hi = it.qt1;
    t = P.t0;
    s = -1;
    kt = kt_end = 0;
    diag = 0;
  }
  __device__ __forceinline__ bool next_segment(const FwdParams& P) {
    while (true) {
      ++s;
      if (s >= slots(P.g)) {
        s = 0;
        ++t;
      }
      if (t >= P.t1) return false;
      const int src = step_src(P.g, rank, t);
      const int b = rank_chunk(P.g, src, s);
      const int kind = block_kind(P.g, a, b);
      if (kind == kSkip) continue;
      diag = kind == kDiag;
      kt = b * P.T;
      kt_end = diag ? qt_hi + 1 : kt + P.T;
      return true;
    }
  }
  // next global K/V tile index (within the head); false when exhausted
  __device__ __forceinline__ bool next(const FwdParams& P, int& tile, int& is_diag) {
    while (kt >= kt_end)
      if (!next_segment(P)) return false;
    tile = kt++;
    is_diag = diag;
    return true;
  }
};

// O row *= f for the D accumulator columns of this thread's TMEM lane
template <int D>
__device__ __noinline__ void rescale_rows(uint32_t tO, float f) {
#pragma unroll
  for (int cb = 0; cb < D; cb += 32) {
    uint32_t ov[32];
    tmem_ld32<0>(tO + cb, ov);
    tmem_wait_ld();
#pragma unroll
    for (int c = 0; c < 32; ++c) ov[c] = __float_as_uint(__uint_as_float(ov[c]) * f);
    tmem_st32<0>(tO + cb, ov);
  }
  tmem_wait_st();
}

__device__ __forceinline__ int snake_item(int round, int cta, int grid) {
  return round * grid + ((round & 1) ? (grid - 1 - cta) : cta);
}

// Per-tensor e4m3 scale 448 / amax (1 for an all-zero tensor), as the
// quantiser computes it.
__device__ __forceinline__ float e4m3_scale(float amax) {
  return amax > 0.f ? __fdiv_rn(448.f, amax) : 1.f;
}

template <int D, bool F8>
__global__ void __launch_bounds__(384, 1)
    tc_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const FwdParams P) {
  using C = FwdCfg<D, F8>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sQ[2] = {smem, smem + C::kTileBytes};
  uint8_t* sKV = smem + 2 * C::kTileBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOffset);
  uint64_t* kv_full = bars;
  uint64_t* kv_empty = bars + C::kStages;
  uint64_t* q_full = bars + 2 * C::kStages;
  uint64_t* q_empty = q_full + 1;
  uint64_t* s_ready = q_full + 2;  // [2]
  uint64_t* p_ready = q_full + 4;  // [2]
  uint64_t* o_ready = q_full + 6;  // [2]
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
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_ready[i], 1);
      mbar_init(&p_ready[i], 128);
      mbar_init(&o_ready[i], 1);
    }
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
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int grid = gridDim.x, cta = blockIdx.x;
  const int S = P.g.S;

  if (warp < 8) {
    // ------------------------------------------------------------ softmax --
    regs_inc<C::kRegsSoftmax>();
    // scores arrive as products of codes: undo the q and k scales; the output
    // undoes the v scale
    float sl2 = P.sl2, out_mul = 1.f;
    if constexpr (F8) {
      sl2 = P.sl2 / (e4m3_scale(P.amax[0]) * e4m3_scale(P.amax[1]));
      out_mul = 1.f / e4m3_scale(P.amax[2]);
    }
    constexpr float kThresh = F8 ? kRescaleThresholdF8 : kRescaleThreshold;
    constexpr float kPOff = F8 ? kP8Log2Scale : 0.f;
    const int wg = warp >> 2;               // which Q tile
    const int quarter = warp & 3;           // TMEM lane quarter of this warp
    const int rloc = quarter * 32 + lane;   // row within the 128-row tile
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const uint32_t tS = tmem_base + lane_off + wg * 128;
    const uint32_t tO = tmem_base + lane_off + 256 + wg * 128;
    uint32_t s_cnt = 0, o_cnt = 0;
    for (int round = 0;; ++round) {
      const int w = snake_item(round, cta, grid);
      if (w >= P.n_items) break;
      Item it;
      decode_item(P, w, it);
      const int qt = wg ? it.qt1 : it.qt0;
      const int qrow = qt * 128 + rloc;
      KvIter kv;
      kv.init(P, it);
      float m = -INFINITY, l = 0.f;
      int j = 0, tile, dg;
      bool ok = true;
      while (kv.next(P, tile, dg)) {
        if (!mbar_wait_warp(&s_ready[wg], s_cnt & 1, abort_flag, P.err)) { ok = false; break; }
        ++s_cnt;
        tc_fence_after();
        uint32_t r[128];
        tmem_ld32<0>(tS + 0, r);
        tmem_ld32<32>(tS + 32, r);
        tmem_ld32<64>(tS + 64, r);
        tmem_ld32<96>(tS + 96, r);
        tmem_wait_ld();
        if (dg && tile >= qt) {
          const int lim = (tile > qt) ? -1 : rloc;  // columns <= lim stay visible
#pragma unroll
          for (int c = 0; c < 128; ++c)
            if (c > lim) r[c] = __float_as_uint(-INFINITY);
        }
        // row maximum as 8 independent chains (a single chain of 127 dependent
        // max operations would put its full latency on every tile)
        float mp[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) mp[i] = fmaxf(__uint_as_float(r[i]), __uint_as_float(r[8 + i]));
#pragma unroll
        for (int c = 16; c < 128; c += 16)
#pragma unroll
          for (int i = 0; i < 8; ++i)
            mp[i] = fmax3(mp[i], __uint_as_float(r[c + i]), __uint_as_float(r[c + 8 + i]));
        const float mx = fmax3(fmax3(mp[0], mp[1], mp[2]), fmax3(mp[3], mp[4], mp[5]), fmaxf(mp[6], mp[7]));
        const float m_tile = mx * sl2;
        float m_new = m;
        if (m_tile > m + kThresh || m == -INFINITY) m_new = fmaxf(m, m_tile);
        const bool grow = (m != -INFINITY) && (m_new > m);
        const float f = grow ? ex2(m - m_new) : 1.f;
        l *= f;
        // TMEM loads / stores are warp-collective: the whole warp rescales
        // (factor 1 for rows whose maximum stayed) when any row needs it
        if (j > 0 && __any_sync(0xffffffffu, grow)) rescale_rows<D>(tO, f);
        m = m_new;
        const float base = ((m == -INFINITY) ? 0.f : m) - kPOff;
        // exponentials and row sum on packed pairs (the row sum as 4 chains)
        const float2 sl = make_float2(sl2, sl2), nb = make_float2(-base, -base);
        float2 ls2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
        if constexpr (F8) {
#pragma unroll
          for (int c = 0; c < 128; c += 4) {
            const float2 x01 = ffma2(make_float2(__uint_as_float(r[c]), __uint_as_float(r[c + 1])), sl, nb);
            const float2 x23 = ffma2(make_float2(__uint_as_float(r[c + 2]), __uint_as_float(r[c + 3])), sl, nb);
            const float2 p01 = make_float2(ex2(x01.x), ex2(x01.y));
            const float2 p23 = make_float2(ex2(x23.x), ex2(x23.y));
            ls2[0] = fadd2(ls2[0], p01);
            ls2[1] = fadd2(ls2[1], p23);
            r[c >> 2] = pack_e4m3x4(p01.x, p01.y, p23.x, p23.y);  // r[c/4] was read at or before this step
          }
        } else {
#pragma unroll
          for (int c = 0; c < 128; c += 2) {
            const float2 x = ffma2(make_float2(__uint_as_float(r[c]), __uint_as_float(r[c + 1])), sl, nb);
            const float2 p = make_float2(ex2(x.x), ex2(x.y));
            ls2[(c >> 1) & 1] = fadd2(ls2[(c >> 1) & 1], p);
            r[c >> 1] = pack_bf16x2(p.x, p.y);  // r[c/2] was read at or before this step
          }
        }
        const float ls[4] = {ls2[0].x, ls2[0].y, ls2[1].x, ls2[1].y};
        l += (ls[0] + ls[1]) + (ls[2] + ls[3]);
        tmem_st32<0>(tS + 0, r);
        if constexpr (!F8) tmem_st32<32>(tS + 32, r);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&p_ready[wg]);
        ++j;
      }
      if (!ok) break;
      const bool store = (wg == 0) || !it.single;
      const long orow = (long)it.bh * S + qrow;
      if (j == 0) {
        // no visible key at these steps: empty partial
        if (store) {
          if (P.out_f32) {
            float4* dst = reinterpret_cast<float4*>(static_cast<float*>(P.o) + orow * D);
#pragma unroll
            for (int c = 0; c < D / 4; ++c) dst[c] = make_float4(0.f, 0.f, 0.f, 0.f);
          } else {
            uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(P.o) + orow * D);
#pragma unroll
            for (int c = 0; c < D / 8; ++c) dst[c] = make_uint4(0, 0, 0, 0);
          }
          P.lse[orow] = -INFINITY;
        }
        continue;
      }
      if (!mbar_wait_warp(&o_ready[wg], o_cnt & 1, abort_flag, P.err)) break;
      ++o_cnt;
      tc_fence_after();
      const float inv = out_mul / l;
#pragma unroll
      for (int cb = 0; cb < D; cb += 32) {
        uint32_t ov[32];
        tmem_ld32<0>(tO + cb, ov);
        tmem_wait_ld();
        if (store) {
          if (P.out_f32) {
            float4* dst = reinterpret_cast<float4*>(static_cast<float*>(P.o) + orow * D + cb);
#pragma unroll
            for (int c = 0; c < 8; ++c)
              dst[c] = make_float4(__uint_as_float(ov[4 * c]) * inv, __uint_as_float(ov[4 * c + 1]) * inv,
                                   __uint_as_float(ov[4 * c + 2]) * inv, __uint_as_float(ov[4 * c + 3]) * inv);
          } else {
            uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(P.o) + orow * D + cb);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              uint4 u;
              u.x = pack_bf16x2(__uint_as_float(ov[8 * c + 0]) * inv, __uint_as_float(ov[8 * c + 1]) * inv);
              u.y = pack_bf16x2(__uint_as_float(ov[8 * c + 2]) * inv, __uint_as_float(ov[8 * c + 3]) * inv);
              u.z = pack_bf16x2(__uint_as_float(ov[8 * c + 4]) * inv, __uint_as_float(ov[8 * c + 5]) * inv);
              u.w = pack_bf16x2(__uint_as_float(ov[8 * c + 6]) * inv, __uint_as_float(ov[8 * c + 7]) * inv);
              dst[c] = u;
            }
          }
        }
      }
      if (store) P.lse[orow] = (m + __log2f(l) - kPOff) * kLn2;
      tc_fence_before();
    }
  } else {
    regs_dec<C::kRegsOther>();
  }
  if (warp == 8) {
    // -------------------------------------------------------- TMA producer --
    uint32_t kv_idx = 0, n_items = 0;
    bool stall = P.stall && cta == 0;
    bool ok = true;
    for (int round = 0; ok; ++round) {
      const int w = snake_item(round, cta, grid);
      if (w >= P.n_items) break;
      Item it;
      decode_item(P, w, it);
      KvIter kv;
      kv.init(P, it);
      int tile, dg;
      KvIter probe = kv;
      if (!probe.next(P, tile, dg)) continue;  // empty item: nothing to load
      if (n_items > 0 && !mbar_wait_warp(q_empty, (n_items - 1) & 1, abort_flag, P.err)) break;
      const int rowbase = it.bh * S;
      if (lane == 0) {
        mbar_expect_tx(q_full, 2 * C::kTileBytes);
        if constexpr (F8) {
          tma_load_2d(sQ[0], &tmQ, q_full, 0, rowbase + it.qt0 * 128);
          tma_load_2d(sQ[1], &tmQ, q_full, 0, rowbase + it.qt1 * 128);
        } else {
#pragma unroll
          for (int sb = 0; sb < D / 64; ++sb) {
            tma_load_2d(sQ[0] + sb * C::kSubBytes, &tmQ, q_full, sb * 64, rowbase + it.qt0 * 128);
            tma_load_2d(sQ[1] + sb * C::kSubBytes, &tmQ, q_full, sb * 64, rowbase + it.qt1 * 128);
          }
        }
      }
      ++n_items;
      while (kv.next(P, tile, dg)) {
        for (int which = 0; which < 2; ++which) {
          const int s = kv_idx % C::kStages;
          if (kv_idx >= (uint32_t)C::kStages &&
              !mbar_wait_warp(&kv_empty[s], ((kv_idx / C::kStages) - 1) & 1, abort_flag, P.err)) {
            ok = false;
            break;
          }
          if (lane == 0) {
            if (stall && which == 0) {
              stall = false;  // this K tile is never loaded: the consumer's wait runs out
            } else {
              mbar_expect_tx(&kv_full[s], C::kTileBytes);
              if constexpr (F8) {
                // K: [key rows][d] codes; V^T: [d rows][key] codes of this head
                if (which)
                  tma_load_2d(sKV + s * C::kTileBytes, &tmV, &kv_full[s], tile * 128, it.bh * D);
                else
                  tma_load_2d(sKV + s * C::kTileBytes, &tmK, &kv_full[s], 0, rowbase + tile * 128);
              } else {
                const CUtensorMap* map = which ? &tmV : &tmK;
#pragma unroll
                for (int sb = 0; sb < D / 64; ++sb)
                  tma_load_2d(sKV + s * C::kTileBytes + sb * C::kSubBytes, map, &kv_full[s],
                              sb * 64, rowbase + tile * 128);
              }
            }
          }
          __syncwarp();
          ++kv_idx;
        }
        if (!ok) break;
      }
    }
    if (*abort_flag) {
      // let loads already in flight land before the CTA's shared memory goes away
      const uint32_t first = kv_idx > (uint32_t)C::kStages ? kv_idx - C::kStages : 0;
      for (uint32_t i = first; i < kv_idx; ++i) {
        const unsigned long long t0 = globaltimer();
        while (!mbar_try_wait(&kv_full[i % C::kStages], (i / C::kStages) & 1) &&
               globaltimer() - t0 < kWaitLimitNs) {
        }
      }
    }
  } else if (warp == 9) {
    // ---------------------------------------------------------- MMA issuer --
    const uint32_t tS[2] = {tmem_base + 0, tmem_base + 128};
    const uint32_t tO[2] = {tmem_base + 256, tmem_base + 384};
    const uint32_t aQ[2] = {smem_u32(sQ[0]), smem_u32(sQ[1])};
    const uint32_t aKV = smem_u32(sKV);
    // one descriptor per operand tile; k-steps are constant offsets from it
    const uint64_t dQd[2] = {smem_desc_sw128(aQ[0], 16, 1024), smem_desc_sw128(aQ[1], 16, 1024)};
    // O += P V: A = P (bf16, two per TMEM column), B = V (MN-major over d);
    // e4m3: A = P (four per TMEM column), B = V^T (K-major over keys)
    auto issue_pv = [&](uint32_t t_o, uint32_t t_p, uint32_t slot_v, bool first) {
      if constexpr (F8) {
        const uint64_t dv = smem_desc_sw128(aKV + slot_v * C::kTileBytes, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_ts_f8(t_o, t_p + kk * 8, desc_at(dv, kk * 32), C::kIdescPV,
                    (first && kk == 0) ? 0u : 1u);
      } else {
        const uint64_t dv = smem_desc_sw128(aKV + slot_v * C::kTileBytes, C::kSubBytes, 1024);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ts(t_o, t_p + kk * 8, desc_at(dv, kk * 2048), C::kIdescPV, (first && kk == 0) ? 0u : 1u);
      }
    };
    // S = Q K^T: both operands K-major (bf16: 16 per k-step, e4m3: 32)
    auto issue_qk = [&](uint32_t t_s, uint64_t dq, uint32_t slot_k) {
      const uint64_t dk = smem_desc_sw128(aKV + slot_k * C::kTileBytes, 16, 1024);
      if constexpr (F8) {
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_ss_f8(t_s, desc_at(dq, kk * 32), desc_at(dk, kk * 32), C::kIdescQK, kk > 0 ? 1u : 0u);
      } else {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * C::kSubBytes + (kk & 3) * 32;
          mma_ss(t_s, desc_at(dq, off), desc_at(dk, off), C::kIdescQK, kk > 0 ? 1u : 0u);
        }
      }
    };
    uint32_t kv_idx = 0, p_cnt = 0, n_items = 0;
    bool ok = true;
    for (int round = 0; ok; ++round) {
      const int w = snake_item(round, cta, grid);
      if (w >= P.n_items) break;
      Item it;
      decode_item(P, w, it);
      KvIter kv;
      kv.init(P, it);
      int tile, dg;
      KvIter probe = kv;
      if (!probe.next(P, tile, dg)) continue;
      if (!mbar_wait_warp(q_full, n_items & 1, abort_flag, P.err)) break;
      ++n_items;
      tc_fence_after();
      bool has_prev = false, prev_first = true;
      uint32_t prev_sV = 0, prev_phV = 0;
      while (kv.next(P, tile, dg)) {
        const uint32_t sK = kv_idx % C::kStages, phK = (kv_idx / C::kStages) & 1;
        ++kv_idx;
        const uint32_t sV = kv_idx % C::kStages, phV = (kv_idx / C::kStages) & 1;
        ++kv_idx;
        if (!mbar_wait_warp(&kv_full[sK], phK, abort_flag, P.err)) { ok = false; break; }
        if (has_prev) {
          if (!mbar_wait_warp(&kv_full[prev_sV], prev_phV, abort_flag, P.err) ||
              !mbar_wait_warp(&p_ready[0], p_cnt & 1, abort_flag, P.err)) { ok = false; break; }
        }
        tc_fence_after();
        if (lane == 0) {
          if (has_prev) issue_pv(tO[0], tS[0], prev_sV, prev_first);
          issue_qk(tS[0], dQd[0], sK);
          tc_commit(&s_ready[0]);
        }
        __syncwarp();
        if (has_prev) {
          if (!mbar_wait_warp(&p_ready[1], p_cnt & 1, abort_flag, P.err)) { ok = false; break; }
          ++p_cnt;
          tc_fence_after();
        }
        if (lane == 0) {
          if (has_prev) {
            issue_pv(tO[1], tS[1], prev_sV, prev_first);
            tc_commit(&kv_empty[prev_sV]);
          }
          issue_qk(tS[1], dQd[1], sK);
          tc_commit(&s_ready[1]);
          tc_commit(&kv_empty[sK]);
        }
        __syncwarp();
        prev_first = !has_prev;
        has_prev = true;
        prev_sV = sV;
        prev_phV = phV;
      }
      if (!ok) break;
      if (lane == 0) tc_commit(q_empty);
      __syncwarp();
      // last tile's P.V for both Q tiles
      if (!mbar_wait_warp(&kv_full[prev_sV], prev_phV, abort_flag, P.err) ||
          !mbar_wait_warp(&p_ready[0], p_cnt & 1, abort_flag, P.err)) break;
      tc_fence_after();
      if (lane == 0) {
        issue_pv(tO[0], tS[0], prev_sV, prev_first);
        tc_commit(&o_ready[0]);
      }
      __syncwarp();
      if (!mbar_wait_warp(&p_ready[1], p_cnt & 1, abort_flag, P.err)) break;
      ++p_cnt;
      tc_fence_after();
      if (lane == 0) {
        issue_pv(tO[1], tS[1], prev_sV, prev_first);
        tc_commit(&o_ready[1]);
        tc_commit(&kv_empty[prev_sV]);
      }
      __syncwarp();
    }
    // every MMA issued by this thread completes before TMEM is released
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

template <int D, bool F8>
int launch_impl(const AttnShape& sh, const void* q, const void* k, const void* v, void* o,
                float* lse, const float* amax, unsigned* err, int stall, int t0, int t1,
                int out_f32, cudaStream_t stream) {
  using C = FwdCfg<D, F8>;
  CUtensorMap mq, mk, mv;
  const uint64_t rows = (uint64_t)sh.B * sh.H * sh.S;
  if constexpr (F8) {
    // q, k: [B*H*S][D] codes; v: V^T, [B*H*D][S] codes
    if (!make_tmap_u8_2d(&mq, q, rows, D, 128, 128) || !make_tmap_u8_2d(&mk, k, rows, D, 128, 128) ||
        !make_tmap_u8_2d(&mv, v, (uint64_t)sh.B * sh.H * D, sh.S, 128, 128))
      return -1;
  } else {
    if (!make_tmap_bf16_2d(&mq, q, rows, D, 64, 128) || !make_tmap_bf16_2d(&mk, k, rows, D, 64, 128) ||
        !make_tmap_bf16_2d(&mv, v, rows, D, 64, 128))
      return -1;
  }
  FwdParams P;
  P.g = sh.g;
  P.BH = sh.B * sh.H;
  P.T = sh.g.c / 128;
  P.pairs = (P.T + 1) / 2;
  P.n_items = P.BH * sh.g.n_chunks * P.pairs;
  P.G = (P.BH % 4 == 0) ? 4 : (P.BH % 2 == 0) ? 2 : 1;
  P.t0 = t0;
  P.t1 = t1;
  P.out_f32 = out_f32;
  P.sl2 = sh.scale * kLog2e;
  P.o = o;
  P.lse = lse;
  P.amax = amax;
  P.err = err;
  P.stall = stall;
  static std::atomic<unsigned long long> attr_done{0};
  if (!smem_attr_once(tc_fwd_kernel<D, F8>, C::kSmemBytes, attr_done)) return -1;
  // One CTA per work item, items numbered longest first (heads four at a
  // time): the hardware block scheduler hands them out in that order as SMs
  // free up, a greedy longest-first schedule.  A persistent grid with a static
  // snake assignment of the same order measured 4% slower at S = 32K and
  // balances far worse on small problems (S = 8K: a third of the SMs idle at
  // the end).
  const int grid = P.n_items;
  const int prof_id = F8 ? kKTcFwdFp8 : kKTcFwd;
  prof_begin(prof_id, stream);
  tc_fwd_kernel<D, F8><<<grid, C::kThreads, C::kSmemBytes, stream>>>(mq, mk, mv, P);
  prof_end(prof_id, stream);
  return cudaGetLastError() == cudaSuccess ? 1 : -1;
}

}  // namespace

bool tc_fwd_supported(const AttnShape& sh) {
  if (!sh.bf16) return false;
  if (sh.D != 64 && sh.D != 128) return false;
  if (sh.g.c % 128 != 0) return false;
  if ((long long)sh.B * sh.H * sh.S >= (1LL << 31)) return false;
  return true;
}

int launch_tc_fwd(const AttnShape& sh, const void* q, const void* k, const void* v, void* o,
                  float* lse, unsigned* err, int stall, cudaStream_t stream) {
  if (sh.D == 64)
    return launch_impl<64, false>(sh, q, k, v, o, lse, nullptr, err, stall, 0, sh.g.N, 0, stream);
  return launch_impl<128, false>(sh, q, k, v, o, lse, nullptr, err, stall, 0, sh.g.N, 0, stream);
}

int launch_tc_fwd_step(const AttnShape& sh, const void* q, const void* k, const void* v,
                       float* o_part, float* lse_part, int step, unsigned* err,
                       cudaStream_t stream) {
  if (sh.D == 64)
    return launch_impl<64, false>(sh, q, k, v, o_part, lse_part, nullptr, err, 0, step, step + 1, 1,
                                  stream);
  return launch_impl<128, false>(sh, q, k, v, o_part, lse_part, nullptr, err, 0, step, step + 1, 1,
                                 stream);
}

int launch_tc_fwd_fp8(const AttnShape& sh, const void* q8, const void* k8, const void* vt8,
                      const float* amax, void* o, float* lse, unsigned* err, cudaStream_t stream) {
  if (sh.D != 128) return -1;
  return launch_impl<128, true>(sh, q8, k8, vt8, o, lse, amax, err, 0, 0, sh.g.N, 0, stream);
}

}  // namespace cpattn
