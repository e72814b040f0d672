// layer.cu -- the attention layer around the ring attention: Q/K/V and output
// projections (nn.Linear with bias) and the [B,S,E] <-> [B,H,S,D] head
// reshapes, forward and backward.  "Configuring RingAttention+FlashAttention
// for CP" (devpress.csdn.net), section 3 code: q/k/v_proj and out_proj of
// width E, q.view(B,S,H,D).transpose(1,2) before the ring loop, the inverse
// transpose and out_proj after it.
//
// The projections run on this library's tcgen05 GEMM (gemm.cu: bf16 in/out,
// fp32 accumulate; the forward bias fused into its epilogue).  The head
// reshapes and the bias gradients are this library's own kernels too; the
// attention in between is cpattn_fwd / cpattn_bwd.  Nothing here calls a
// vendor library.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <cmath>
#include <mutex>

#include "cpattn.h"
#include "kernels.h"

namespace cpattn {
namespace {

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Row-major C[M][N] = op(A) op(B) (+ bias[N]) on the tcgen05 GEMM.
// a_mn: A stored [K][M]; b_mn: B stored [K][N] (otherwise [M][K] / [N][K]).
bool gemm(cudaStream_t s, const void* A, const void* B, const void* bias, void* C, int M, int N,
          int K, int a_mn, int b_mn) {
  unsigned* err = device_error_word();
  if (!err || gemm_check(M, N, K) != 0) return false;
  const int n = launch_gemm(A, B, bias, C, M, N, K, a_mn, b_mn, err, s);
  if (n < 0) return false;
  add_launches(n);
  return true;
}

// Head reshapes, 16 bytes (8 bf16) per thread.
//   split (to_heads = 1): src [B][S][G][H][D] -> dst_g [B][H][S][D], g < G
//   merge (to_heads = 0): src_g [B][H][S][D] -> dst [B][S][G][H][D]
// `packed` is the [B][S][G][H][D] side, heads[g] the per-group [B][H][S][D] side.
__global__ void __launch_bounds__(256) heads_kernel(__nv_bfloat16* packed, __nv_bfloat16* h0,
                                                    __nv_bfloat16* h1, __nv_bfloat16* h2, int B,
                                                    int S, int G, int H, int D, int to_heads) {
  const long n_vec = (long)B * S * G * H * (D / 8);
  for (long i = (long)blockIdx.x * blockDim.x + threadIdx.x; i < n_vec; i += (long)gridDim.x * blockDim.x) {
    long r = i;
    const int dv = (int)(r % (D / 8));
    r /= D / 8;
    const int h = (int)(r % H);
    r /= H;
    const int g = (int)(r % G);
    r /= G;
    const int s = (int)(r % S);
    const int b = (int)(r / S);
    __nv_bfloat16* hd = g == 0 ? h0 : (g == 1 ? h1 : h2);
    uint4* p = reinterpret_cast<uint4*>(packed) + i;
    uint4* q = reinterpret_cast<uint4*>(hd + (((long)b * H + h) * S + s) * D) + dv;
    if (to_heads) *q = *p;
    else *p = *q;
  }
}

// db[n] = sum over rows of Y[rows][N] (fp32 accumulation, bf16 result), in
// two passes with a fixed order (deterministic): kColsumSplits row ranges give
// fp32 partials, then one thread per column adds them up.  Consecutive
// threads take consecutive columns (coalesced).
constexpr int kColsumSplits = 64;

__global__ void __launch_bounds__(256) colsum_partial_kernel(const __nv_bfloat16* __restrict__ Y,
                                                             float* __restrict__ part, long rows, int N) {
  const int n = blockIdx.x * blockDim.x + threadIdx.x;
  if (n >= N) return;
  const long per = (rows + kColsumSplits - 1) / kColsumSplits;
  const long r0 = blockIdx.y * per, r1 = r0 + per < rows ? r0 + per : rows;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  long r = r0;
  for (; r + 4 <= r1; r += 4)
#pragma unroll
    for (int u = 0; u < 4; ++u) acc[u] += __bfloat162float(Y[(r + u) * N + n]);
  for (; r < r1; ++r) acc[0] += __bfloat162float(Y[r * N + n]);
  part[(long)blockIdx.y * N + n] = (acc[0] + acc[1]) + (acc[2] + acc[3]);
}

__global__ void __launch_bounds__(256) colsum_final_kernel(const float* __restrict__ part,
                                                           __nv_bfloat16* __restrict__ db, int N) {
  const int n = blockIdx.x * blockDim.x + threadIdx.x;
  if (n >= N) return;
  float acc = 0.f;
  for (int k = 0; k < kColsumSplits; ++k) acc += part[(long)k * N + n];
  db[n] = __float2bfloat16_rn(acc);
}

bool heads(cudaStream_t s, void* packed, void* a, void* b, void* c, int B, int S, int G, int H, int D,
           int to_heads) {
  const long n_vec = (long)B * S * G * H * (D / 8);
  int dev = 0;
  cudaGetDevice(&dev);
  const long blocks = std::min<long>((n_vec + 255) / 256, (long)num_sms(dev) * 16);
  prof_begin(kKLayerHeads, s);
  heads_kernel<<<(unsigned)blocks, 256, 0, s>>>(
      static_cast<__nv_bfloat16*>(packed), static_cast<__nv_bfloat16*>(a),
      static_cast<__nv_bfloat16*>(b), static_cast<__nv_bfloat16*>(c), B, S, G, H, D, to_heads);
  prof_end(kKLayerHeads, s);
  add_launches(1);
  return cudaGetLastError() == cudaSuccess;
}

bool colsum(cudaStream_t s, const void* Y, void* db, long rows, int N, float* part) {
  prof_begin(kKLayerColsum, s);
  colsum_partial_kernel<<<dim3((N + 255) / 256, kColsumSplits), 256, 0, s>>>(
      static_cast<const __nv_bfloat16*>(Y), part, rows, N);
  colsum_final_kernel<<<(N + 255) / 256, 256, 0, s>>>(part, static_cast<__nv_bfloat16*>(db), N);
  prof_end(kKLayerColsum, s);
  add_launches(2);
  return cudaGetLastError() == cudaSuccess;
}

struct LayerWs {
  size_t qkv, om, dom, dq, dk, dv, dout, attn, part, total;
};

// Offsets of the layer workspace.  Forward: qkv [B*S][3E], om [B*S][E], lt.
// Backward: om, dom [B*S][E], dout, dq, dk, dv [B][H][S][D], dqkv (reuses qkv),
// the attention backward's workspace and the column-sum partials.
LayerWs layer_ws(int B, int S, int E, int H) {
  const size_t rows = (size_t)B * S, t = rows * E * 2;
  LayerWs w;
  size_t off = 0;
  w.qkv = off;  off += align256(3 * t);
  w.om = off;   off += align256(t);
  w.dom = off;  off += align256(t);
  w.dout = off; off += align256(t);
  w.dq = off;   off += align256(t);
  w.dk = off;   off += align256(t);
  w.dv = off;   off += align256(t);
  w.attn = off; off += align256(cpattn_bwd_workspace_bytes(B, H, S, E / H));
  w.part = off; off += align256((size_t)kColsumSplits * 3 * E * 4);
  w.total = off;
  return w;
}

int check_layer(int B, int S, int E, int H, int cp_size, int causal, float scale) {
  if (B < 1 || S < 1 || E < 1 || H < 1) return CPATTN_ERR_SHAPE;
  if (E % H != 0) return CPATTN_ERR_SHAPE;
  const int D = E / H;
  if (D != 64 && D != 128) return CPATTN_ERR_SHAPE;
  if ((long long)B * S * 3 * E >= (1LL << 31)) return CPATTN_ERR_SHAPE;  // GEMM dims and offsets
  if ((B * S) % 8 != 0 || E % 8 != 0) return CPATTN_ERR_SHAPE;           // GEMM row alignment
  (void)cp_size;
  (void)causal;
  if (!(scale > 0.f) || !std::isfinite(scale)) return CPATTN_ERR_ARG;
  return CPATTN_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace cpattn

using namespace cpattn;

extern "C" {

size_t cpattn_layer_workspace_bytes(int B, int S, int E, int H) {
  if (check_layer(B, S, E, H, 1, 1, 1.f) != CPATTN_OK) return 0;
  return layer_ws(B, S, E, H).total;
}

int cpattn_layer_fwd(const void* x, const void* w_qkv, const void* b_qkv, const void* w_o,
                     const void* b_o, void* y, void* q, void* k, void* v, void* o, float* lse,
                     int B, int S, int E, int H, int cp_size, int causal, float scale,
                     void* workspace, size_t ws_bytes, void* stream) {
  NvtxRange nv("cpattn_layer_fwd");
  int st = check_layer(B, S, E, H, cp_size, causal, scale);
  if (st != CPATTN_OK) return st;
  if (!x || !w_qkv || !b_qkv || !w_o || !b_o || !y || !q || !k || !v || !o || !lse) return CPATTN_ERR_ARG;
  const void* ptrs[] = {x, w_qkv, b_qkv, w_o, b_o, y, q, k, v, o, lse, workspace};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return CPATTN_ERR_ALIGN;
  const LayerWs w = layer_ws(B, S, E, H);
  if (!workspace || ws_bytes < w.total) return CPATTN_ERR_WORKSPACE;
  const int D = E / H;
  // the attention's own shape rules (chunking) are checked before any launch
  st = check_attention_shape(B, H, S, D, cp_size, causal, scale, CPATTN_BF16);
  if (st != CPATTN_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  void* qkv = ws + w.qkv;
  void* om = ws + w.om;
  const int rows = B * S;
  // q|k|v = x Wqkv^T + bqkv  ([B*S][3E], the three projections stacked)
  if (!gemm(s, x, w_qkv, b_qkv, qkv, rows, 3 * E, E, 0, 0)) return CPATTN_ERR_CUDA;
  if (!heads(s, qkv, q, k, v, B, S, 3, H, D, 1)) return CPATTN_ERR_CUDA;
  st = cpattn_fwd(q, k, v, o, lse, B, H, S, D, cp_size, causal, scale, CPATTN_BF16, stream);
  if (st != CPATTN_OK) return st;
  if (!heads(s, om, o, nullptr, nullptr, B, S, 1, H, D, 0)) return CPATTN_ERR_CUDA;
  if (!gemm(s, om, w_o, b_o, y, rows, E, E, 0, 0)) return CPATTN_ERR_CUDA;
  return CPATTN_OK;
}

int cpattn_layer_bwd(const void* x, const void* w_qkv, const void* w_o, const void* q, const void* k,
                     const void* v, const void* o, const float* lse, const void* dy, void* dx,
                     void* dw_qkv, void* db_qkv, void* dw_o, void* db_o, int B, int S, int E, int H,
                     int cp_size, int causal, float scale, void* workspace, size_t ws_bytes,
                     void* stream) {
  NvtxRange nv("cpattn_layer_bwd");
  int st = check_layer(B, S, E, H, cp_size, causal, scale);
  if (st != CPATTN_OK) return st;
  if (!x || !w_qkv || !w_o || !q || !k || !v || !o || !lse || !dy || !dx || !dw_qkv || !db_qkv ||
      !dw_o || !db_o)
    return CPATTN_ERR_ARG;
  const void* ptrs[] = {x, w_qkv, w_o, q, k, v, o, lse, dy, dx, dw_qkv, db_qkv, dw_o, db_o, workspace};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return CPATTN_ERR_ALIGN;
  const LayerWs w = layer_ws(B, S, E, H);
  if (!workspace || ws_bytes < w.total) return CPATTN_ERR_WORKSPACE;
  const int D = E / H;
  st = check_attention_shape(B, H, S, D, cp_size, causal, scale, CPATTN_BF16);
  if (st != CPATTN_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  void *dqkv = ws + w.qkv, *om = ws + w.om, *dom = ws + w.dom, *dout = ws + w.dout;
  void *dq = ws + w.dq, *dk = ws + w.dk, *dv = ws + w.dv, *attn = ws + w.attn;
  float* part = reinterpret_cast<float*>(ws + w.part);
  const int rows = B * S;
  // output projection: dWo = dY^T Om, dbo = colsum(dY), dOm = dY Wo
  if (!heads(s, om, const_cast<void*>(o), nullptr, nullptr, B, S, 1, H, D, 0)) return CPATTN_ERR_CUDA;
  if (!gemm(s, dy, om, nullptr, dw_o, E, E, rows, 1, 1)) return CPATTN_ERR_CUDA;
  if (!colsum(s, dy, db_o, rows, E, part)) return CPATTN_ERR_CUDA;
  if (!gemm(s, dy, w_o, nullptr, dom, rows, E, E, 0, 1)) return CPATTN_ERR_CUDA;
  // attention backward on the per-head view of dOm
  if (!heads(s, dom, dout, nullptr, nullptr, B, S, 1, H, D, 1)) return CPATTN_ERR_CUDA;
  st = cpattn_bwd(q, k, v, o, lse, dout, dq, dk, dv, B, H, S, D, cp_size, causal, scale, attn,
                  cpattn_bwd_workspace_bytes(B, H, S, D), CPATTN_BF16, stream);
  if (st != CPATTN_OK) return st;
  // input projection: dQKV = [dQ|dK|dV] per row, dWqkv = dQKV^T X,
  // dbqkv = colsum(dQKV), dX = dQKV Wqkv
  if (!heads(s, dqkv, dq, dk, dv, B, S, 3, H, D, 0)) return CPATTN_ERR_CUDA;
  if (!gemm(s, dqkv, x, nullptr, dw_qkv, 3 * E, E, rows, 1, 1)) return CPATTN_ERR_CUDA;
  if (!colsum(s, dqkv, db_qkv, rows, 3 * E, part)) return CPATTN_ERR_CUDA;
  if (!gemm(s, dqkv, w_qkv, nullptr, dx, rows, E, 3 * E, 0, 1)) return CPATTN_ERR_CUDA;
  return CPATTN_OK;
}

int cpattn_gemm(const void* A, const void* B, const void* bias, void* C, int M, int N, int K,
                int a_layout, int b_layout, void* stream) {
  NvtxRange nv("cpattn_gemm");
  if (gemm_check(M, N, K) != 0) return CPATTN_ERR_SHAPE;
  if ((a_layout != 0 && a_layout != 1) || (b_layout != 0 && b_layout != 1)) return CPATTN_ERR_ARG;
  if (!A || !B || !C) return CPATTN_ERR_ARG;
  if (!aligned16(A) || !aligned16(B) || !aligned16(C) || (bias && !aligned16(bias)))
    return CPATTN_ERR_ALIGN;
  return gemm(static_cast<cudaStream_t>(stream), A, B, bias, C, M, N, K, a_layout, b_layout)
             ? CPATTN_OK
             : CPATTN_ERR_CUDA;
}

}  // extern "C"
