// kernels.h -- internal launch interface between the C ABI (api.cu) and the
// kernel translation units.  Every launcher enqueues on `stream`, returns the
// number of kernels it enqueued (>= 0) or -1 when a launch failed.
#pragma once

#include <atomic>

#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>
#include <stddef.h>
#include <stdint.h>

#include "ring.cuh"

namespace cpattn {

struct AttnShape {
  int B, H, S, D;
  RingGeom g;
  float scale;
  int bf16;  // 1: bf16 tensors, 0: fp32 tensors
};

// ---- CUDA-core kernels (any dtype, D in {64,128}, chunk % 16 == 0) ----
// steps [t0, t1) of the ring; final=1 writes O in the input dtype, final=0
// writes the fp32 normalised partial.  lse always fp32.
int launch_simt_fwd(const AttnShape& sh, const void* q, const void* k, const void* v, void* o,
                    float* lse, int t0, int t1, int final_out, unsigned* err,
                    cudaStream_t stream);
int launch_merge(float* o_acc, float* lse_acc, const float* o_part, const float* lse_part,
                 long rows, int D, cudaStream_t stream);
int launch_finalize(const float* o_acc, void* o, long rows, int D, int bf16,
                    cudaStream_t stream);
// backward: delta = rowsum(dO * O) into ws_delta, then dK/dV (key-owned) and
// dQ (row-owned) kernels; no atomics.
// acc_f32 != 0: dq / dk / dv are fp32 accumulators the gradients are added to
int launch_simt_bwd(const AttnShape& sh, const void* q, const void* k, const void* v,
                    const void* o, const float* lse, const void* dout, void* dq, void* dk,
                    void* dv, float* ws_delta, int acc_f32, cudaStream_t stream);

// ---- tcgen05 tensor-core kernels (bf16, D in {64,128}, chunk % 128 == 0) ----
int launch_tc_fwd(const AttnShape& sh, const void* q, const void* k, const void* v, void* o,
                  float* lse, unsigned* err, int stall, cudaStream_t stream);
// one ring step, fp32 normalised partial O and partial LSE (-inf where empty)
int launch_tc_fwd_step(const AttnShape& sh, const void* q, const void* k, const void* v,
                       float* o_part, float* lse_part, int step, unsigned* err,
                       cudaStream_t stream);
// workspace: per-row delta and LSE * log2(e), fp32 [B*H*S] each;
// acc_f32 != 0: dq / dk / dv are fp32 accumulators the gradients are added to
int launch_tc_bwd(const AttnShape& sh, const void* q, const void* k, const void* v,
                  const void* o, const float* lse, const void* dout, void* dq, void* dk,
                  void* dv, float* ws_delta, float* ws_lse2, int acc_f32, unsigned* err,
                  cudaStream_t stream);
// e4m3 forward (D = 128): q8, k8 [B*H*S][D] codes, vt8 [B*H*D][S] codes (V
// transposed per head), amax: device max|q|, max|k|, max|v|; o bf16.
int launch_tc_fwd_fp8(const AttnShape& sh, const void* q8, const void* k8, const void* vt8,
                      const float* amax, void* o, float* lse, unsigned* err, cudaStream_t stream);
bool tc_fwd_supported(const AttnShape& sh);
bool tc_bwd_supported(const AttnShape& sh);

int num_sms(int device);

// Device address of the library's error word on the current device (looked up
// once per device), or null when the lookup failed.
unsigned* device_error_word();

// Kernel family selected by cpattn_set_path: 0 automatic, 1 CUDA cores only,
// 2 tcgen05 kernels on one SM each (no two-SM kernels).
int kernel_path();

// ---- tcgen05 GEMM (gemm.cu): C[M][N] = op(A) op(B) (+ bias[N]), bf16, fp32 accumulation.
// a_mn: A stored [K][M] (else [M][K]); b_mn: B stored [K][N] (else [N][K]).
// gemm_check: 0 when the sizes are supported (M, N, K >= 1, multiples of 8).
int gemm_check(int M, int N, int K);
int launch_gemm(const void* A, const void* B, const void* bias, void* C, int M, int N, int K,
                int a_mn, int b_mn, unsigned* err, cudaStream_t stream);

// The attention entry points' shape and argument rules (CPATTN_OK or the
// status cpattn_fwd / cpattn_bwd would return), for callers that compose them.
int check_attention_shape(int B, int H, int S, int D, int cp_size, int causal, float scale,
                          int dtype);
// Adds n kernels to the library's launch counter (cpattn_launch_count).
void add_launches(int n);

// Raises `func`'s dynamic shared-memory limit to `bytes` on the current
// device, once per device (the attribute belongs to the device's copy of the
// kernel); `done` holds one bit per device already set.
template <typename Kernel>
bool smem_attr_once(Kernel* func, int bytes, std::atomic<unsigned long long>& done) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
  const unsigned long long bit = 1ull << dev;
  if (done.load() & bit) return true;
  if (cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
    return false;
  done.fetch_or(bit);
  return true;
}

// Per-kernel timing for diagnostics: when enabled (cpattn_profile), every
// launcher brackets each kernel with prof_begin / prof_end, which record a
// pair of CUDA events on the launch stream.
enum KernelId : int {
  kKTcFwd = 0,
  kKSimtFwd = 1,
  kKMerge = 2,
  kKFinalize = 3,
  kKDelta = 4,
  kKSimtDkdv = 5,
  kKSimtDq = 6,
  kKTcDkdv = 7,
  kKTcDq = 8,
  kKLayerHeads = 9,   // head split / merge of the attention layer
  kKLayerColsum = 10, // bias gradients of the attention layer
  kKAccumulate = 11,  // fp32 gradient sums of the multi-rank ring backward
  kKGemm = 12,        // projection GEMMs of the attention layer (cpattn_gemm)
  kKTcFwdFp8 = 13,    // tcgen05 forward on e4m3 inputs (cpattn_fwd_fp8)
  kKQuant = 14,       // max|x| and e4m3 quantisation (cpattn_amax, cpattn_quantize_e4m3)
  kKNumKernels = 15
};
void prof_begin(int kernel_id, cudaStream_t stream);
void prof_end(int kernel_id, cudaStream_t stream);

// An NVTX range named after the entry point, open for the duration of one C
// ABI call (host side: argument checks and enqueueing), so that a timeline
// profiler can attribute each kernel and copy to the call that issued it.
// Without an attached tool the push / pop are no-ops.
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

}  // namespace cpattn
