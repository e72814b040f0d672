// ring.cuh -- zigzag chunk ownership and the ring block rule, shared by the
// host planner (cpattn_plan) and every kernel, so the schedule the kernels
// walk is the one cpattn_plan reports.
//
// "Configuring RingAttention+FlashAttention for CP" (devpress.csdn.net):
//   section 5, item 1 -- causal: 2N chunks, rank r owns chunks r and 2N-1-r;
//   section 3 code    -- step t: rank r works on the K/V of rank (r - t) mod N;
//   section 3, note 2 -- exact mask: block (a, b) is SKIP if a < b, DIAG if
//                        a == b, FULL if a > b.
// Non-causal: N contiguous chunks, rank r owns chunk r, every block FULL.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#define CP_HD __host__ __device__ __forceinline__

namespace cpattn {

enum BlockKind : int { kSkip = 0, kFull = 1, kDiag = 2 };

struct RingGeom {
  int S;         // sequence length
  int N;         // cp_size (virtual ranks)
  int causal;    // 1: zigzag + causal mask, 0: contiguous, no mask
  int n_chunks;  // 2N causal, N non-causal
  int c;         // chunk length S / n_chunks
};

CP_HD RingGeom make_geom(int S, int N, int causal) {
  RingGeom g;
  g.S = S;
  g.N = N;
  g.causal = causal ? 1 : 0;
  g.n_chunks = causal ? 2 * N : N;
  g.c = (g.n_chunks > 0) ? S / g.n_chunks : 0;
  return g;
}

// number of chunks a rank owns
CP_HD int slots(const RingGeom& g) { return g.causal ? 2 : 1; }

// chunk held by rank r in slot s (s = 0: chunk r, s = 1: chunk 2N-1-r)
CP_HD int rank_chunk(const RingGeom& g, int r, int s) { return s == 0 ? r : 2 * g.N - 1 - r; }

// the rank owning chunk a
CP_HD int chunk_owner(const RingGeom& g, int a) {
  return (g.causal && a >= g.N) ? 2 * g.N - 1 - a : a;
}

// source rank of the K/V that rank r holds at ring step t
CP_HD int step_src(const RingGeom& g, int r, int t) {
  int s = (r - t) % g.N;
  return s < 0 ? s + g.N : s;
}

CP_HD int block_kind(const RingGeom& g, int a, int b) {
  if (!g.causal) return kFull;
  if (a < b) return kSkip;
  if (a == b) return kDiag;
  return kFull;
}

}  // namespace cpattn
