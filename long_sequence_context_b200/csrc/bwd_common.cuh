// bwd_common.cuh -- shared pieces of the tcgen05 backward kernels: parameters,
// work-item order, the ring walks over q tiles (for a K/V tile) and over K/V
// tiles (for a q tile), and small epilogue helpers.
//
// Ring walks: "Configuring RingAttention+FlashAttention for CP" (devpress.csdn.net),
// section 3 code (step t reads rank (r - t) mod N), note 2 (exact causal mask)
// and section 5 item 1 (zigzag chunks); the walk over q tiles for a K/V tile is
// the mirror image ("Megatron-LM source analysis: Context Parallel", section 2).
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "ring.cuh"
#include "sm100.cuh"

namespace cpattn {
namespace bwd {

struct BwdParams {
  RingGeom g;
  int BH;
  int T;        // 128-row tiles per chunk
  int tiles;    // 128-row tiles per head (S / 128)
  int n_items;  // BH * tiles
  int G;        // heads per scheduling group (divides BH)
  float sl2;    // scale * log2(e)
  float scale;
  const float* lse2;   // LSE * log2(e), [BH][S]
  const float* delta;  // [BH][S]
  const __nv_bfloat16* q;
  const __nv_bfloat16* dout;
  __nv_bfloat16* dq;
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  // accumulate mode (acc_f32 != 0): the gradients are added in fp32 into
  // these [BH][S][D] arrays instead of being written to dq / dk / dv
  int acc_f32;
  float* dq_acc;
  float* dk_acc;
  float* dv_acc;
  unsigned* err;
};

// Work index -> (128-row tile, head).  Heads are taken G at a time so the CTAs
// busy at any moment share a few heads' operands in L2; inside a group tiles go
// longest first (ascending K/V position for dK/dV, descending Q position for dQ).
__device__ __forceinline__ void decode_item(const BwdParams& P, int w, bool descending, int& tile,
                                            int& bh) {
  const int per_group = P.G * P.tiles;
  const int g = w / per_group, r = w % per_group;
  tile = r / P.G;
  if (descending) tile = P.tiles - 1 - tile;
  bh = g * P.G + r % P.G;
}

__device__ __forceinline__ int snake_item(int round, int cta, int grid) {
  return round * grid + ((round & 1) ? (grid - 1 - cta) : cta);
}

// For K/V tile jt (128 rows): the q tiles that see it, in mirror ring order.
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
  __device__ __forceinline__ bool next(const BwdParams& P, int& qt, int& is_diag) {
    while (it >= it_end)
      if (!next_segment(P)) return false;
    qt = it++;
    is_diag = diag && qt == jt;
    return true;
  }
};

// For q tile qt (128 rows): its K/V tiles of KV_ROWS keys in forward ring order.
// diag_off (>= 0 when a mask is needed): key offset of the tile from the q
// tile's first row, in units of KV_ROWS.
template <int KV_ROWS>
struct KIter {
  static constexpr int kPer = 128 / KV_ROWS;  // K/V tiles per 128-row tile
  int a, rank, qt, t, s, kt, kt_end, diag;
  __device__ __forceinline__ void init(const BwdParams& P, int q_tile) {
    qt = q_tile;
    a = qt / P.T;
    rank = chunk_owner(P.g, a);
    t = 0;
    s = -1;
    kt = kt_end = 0;
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
      const int src = step_src(P.g, rank, t);
      const int b = rank_chunk(P.g, src, s);
      const int kind = block_kind(P.g, a, b);
      if (kind == kSkip) continue;
      diag = kind == kDiag;
      kt = b * P.T * kPer;
      kt_end = diag ? (qt + 1) * kPer : kt + P.T * kPer;  // DIAG: up to the q tile's own keys
      if (kt < kt_end) return true;
    }
  }
  __device__ __forceinline__ bool next(const BwdParams& P, int& tile, int& diag_off) {
    while (kt >= kt_end)
      if (!next_segment(P)) return false;
    tile = kt++;
    diag_off = (diag && tile >= qt * kPer) ? tile - qt * kPer : -1;
    return true;
  }
};

__device__ __forceinline__ uint32_t pack_scaled(uint32_t a, uint32_t b, float mul) {
  return sm100::pack_bf16x2(__uint_as_float(a) * mul, __uint_as_float(b) * mul);
}

// Write 32 fp32 TMEM values (scaled) as bf16 to global memory.
__device__ __forceinline__ void store_row32(__nv_bfloat16* dst, const uint32_t (&v)[32], float mul) {
  uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int c = 0; c < 4; ++c)
    d4[c] = make_uint4(pack_scaled(v[8 * c], v[8 * c + 1], mul), pack_scaled(v[8 * c + 2], v[8 * c + 3], mul),
                       pack_scaled(v[8 * c + 4], v[8 * c + 5], mul), pack_scaled(v[8 * c + 6], v[8 * c + 7], mul));
}

// Add 32 fp32 TMEM values (scaled) into an fp32 row of global memory.  Every
// output row belongs to one thread of one work item, so the read-modify-write
// needs no atomics; launches on one stream are ordered.
__device__ __forceinline__ void add_row32(float* dst, const uint32_t (&v)[32], float mul) {
  float4* d4 = reinterpret_cast<float4*>(dst);
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    float4 a = d4[c];
    a.x += __uint_as_float(v[4 * c]) * mul;
    a.y += __uint_as_float(v[4 * c + 1]) * mul;
    a.z += __uint_as_float(v[4 * c + 2]) * mul;
    a.w += __uint_as_float(v[4 * c + 3]) * mul;
    d4[c] = a;
  }
}

}  // namespace bwd
}  // namespace cpattn
