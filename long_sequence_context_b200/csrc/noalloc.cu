// noalloc.cu -- cpattn_bwd_noalloc: the recompute backward for callers that
// cannot allocate device memory.
//
// Who needs it: code that runs where cudaMalloc is not allowed or not safe --
// inside a custom allocator's own callbacks, in a process whose memory pool is
// owned by another framework and must not be touched, or in real-time paths
// where an allocation's synchronisation or failure cannot be tolerated.  Such
// callers can pass their inputs and outputs but cannot hand cpattn_bwd a
// workspace.
//
// What it does: the backward's scratch -- two fp32 values per row, delta_i =
// dO_i . O_i and LSE_i * log2(e) -- lives in one fixed array in device global
// memory, declared below.  The
// driver creates it when this library's module is loaded on a device, and
// every device that loads the library keeps it until the process exits.  This
// file never calls cudaMalloc, cudaFree or any allocating routine; it looks up
// the array's device address and passes it to cpattn_bwd as the workspace.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "cpattn.h"

namespace {

// The shared scratch.  Host code may not use this name as a device address
// (on the host it names a shadow variable); cudaGetSymbolAddress gives the
// device address.
static __device__ __align__(256) unsigned char g_noalloc_scratch[CPATTN_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {nullptr};

// Device address of the scratch array on the current device, looked up once
// per device (the first call on a device does this set-up) and kept for the
// process: the address belongs to the device's primary context, so the
// library is not used across a cudaDeviceReset.
int scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return CPATTN_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
      return CPATTN_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return CPATTN_OK;
}

}  // namespace

extern "C" int cpattn_bwd_noalloc(const void* q, const void* k, const void* v, const void* o,
                                  const float* lse, const void* dout, void* dq, void* dk,
                                  void* dv, int B, int H, int S, int D, int cp_size, int causal,
                                  float scale, int dtype, void* stream) {
  const size_t need = cpattn_bwd_workspace_bytes(B, H, S, D);
  if (need == 0) return CPATTN_ERR_SHAPE;
  if (need > (size_t)CPATTN_NOALLOC_SCRATCH_BYTES) return CPATTN_ERR_WORKSPACE;
  void* scratch = nullptr;
  const int st = scratch_address(&scratch);
  if (st != CPATTN_OK) return st;
  // cpattn_bwd treats its workspace as uninitialised: its preprocess kernel
  // writes delta and LSE * log2(e) for every row of this call before the
  // gradient kernels read them, so the previous call's leftovers are never used.
  return cpattn_bwd(q, k, v, o, lse, dout, dq, dk, dv, B, H, S, D, cp_size, causal, scale,
                    scratch, (size_t)CPATTN_NOALLOC_SCRATCH_BYTES, dtype, stream);
}
