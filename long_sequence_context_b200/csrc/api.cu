// api.cu -- the C ABI of libcpattn.so (declared in include/cpattn.h):
// argument checks, the host planner, kernel-family dispatch and the device
// error word.  No device memory is allocated here or anywhere in the library.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#include <atomic>
#include <mutex>

#include "cpattn.h"
#include "kernels.h"

using namespace cpattn;

// Error word written by kernels whose bounded waits ran out (one per device;
// every device that loads the library holds its own copy of this variable).
__device__ unsigned int g_cpattn_error = 0;

namespace {

std::atomic<long long> g_launches{0};
std::atomic<int> g_path{0};
std::atomic<int> g_last_path{-1};
std::atomic<int> g_stall{0};

constexpr int kMaxDevices = 64;
std::mutex g_err_mu;
unsigned* g_err_ptr[kMaxDevices] = {nullptr};

// Device address of g_cpattn_error for the current device (looked up once).
unsigned* err_word() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_err_mu);
  if (!g_err_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_cpattn_error) != cudaSuccess) return nullptr;
    g_err_ptr[dev] = static_cast<unsigned*>(p);
  }
  return g_err_ptr[dev];
}

// ---- optional per-kernel event timing ----
struct ProfRec {
  int id;
  cudaEvent_t a, b;
};
constexpr int kProfPool = 8192;
std::mutex g_prof_mu;
bool g_prof_on = false;
cudaEvent_t g_prof_events[2 * kProfPool];
int g_prof_created = 0;
int g_prof_used = 0;
ProfRec g_prof_recs[kProfPool];
int g_prof_open_id = -1;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int count(int n) {
  if (n < 0) return CPATTN_ERR_CUDA;
  g_launches += n;
  return CPATTN_OK;
}

// Shape / argument validation shared by fwd, fwd_step and bwd.
int check_shape(int B, int H, int S, int D, int cp_size, int causal, float scale, int dtype,
                AttnShape* sh) {
  if (dtype != CPATTN_BF16 && dtype != CPATTN_FP32) return CPATTN_ERR_DTYPE;
  if (!(scale > 0.f) || !isfinite(scale)) return CPATTN_ERR_ARG;
  if (B < 1 || H < 1 || S < 1 || cp_size < 1) return CPATTN_ERR_SHAPE;
  if (D != 64 && D != 128) return CPATTN_ERR_SHAPE;
  const int n_chunks = causal ? 2 * cp_size : cp_size;
  if (S % n_chunks != 0) return CPATTN_ERR_SHAPE;
  if ((long long)B * H * S * D > (1LL << 40)) return CPATTN_ERR_SHAPE;
  if ((long long)B * H > 65535LL) return CPATTN_ERR_SHAPE;  // grid.y of the CUDA-core kernels
  sh->B = B;
  sh->H = H;
  sh->S = S;
  sh->D = D;
  sh->g = make_geom(S, cp_size, causal);
  sh->scale = scale;
  sh->bf16 = dtype == CPATTN_BF16;
  return CPATTN_OK;
}

}  // namespace

namespace cpattn {
int check_attention_shape(int B, int H, int S, int D, int cp_size, int causal, float scale,
                          int dtype) {
  AttnShape sh;
  return check_shape(B, H, S, D, cp_size, causal, scale, dtype, &sh);
}

void add_launches(int n) { g_launches += n; }

unsigned* device_error_word() { return err_word(); }
int kernel_path() { return g_path.load(); }
}  // namespace cpattn

namespace {

bool use_tc_fwd(const AttnShape& sh) { return g_path.load() != 1 && tc_fwd_supported(sh); }
bool use_tc_bwd(const AttnShape& sh) { return g_path.load() != 1 && tc_bwd_supported(sh); }

}  // namespace

extern "C" {

const char* cpattn_status_str(int s) {
  switch (s) {
    case CPATTN_OK: return "ok";
    case CPATTN_ERR_ARG: return "invalid argument";
    case CPATTN_ERR_SHAPE: return "unsupported shape";
    case CPATTN_ERR_DTYPE: return "unsupported dtype";
    case CPATTN_ERR_ALIGN: return "pointer not 16-byte aligned";
    case CPATTN_ERR_CUDA: return "CUDA error";
    case CPATTN_ERR_TIMEOUT: return "in-kernel wait timed out";
    case CPATTN_ERR_WORKSPACE: return "workspace missing or too small";
    default: return "unknown status";
  }
}

long long cpattn_launch_count(void) { return g_launches.load(); }
int cpattn_set_path(int path) { return g_path.exchange(path == 1 || path == 2 ? path : 0); }
int cpattn_last_path(void) { return g_last_path.load(); }
int cpattn_debug_stall(int n) { return g_stall.exchange(n < 0 ? 0 : n); }

int cpattn_plan(int S, int cp_size, int causal, int32_t* out, int capacity, int* n_rows) {
  NvtxRange nv("cpattn_plan");
  if (!n_rows) return CPATTN_ERR_ARG;
  *n_rows = 0;
  if (cp_size < 1 || S < 1) return CPATTN_ERR_SHAPE;
  const RingGeom g = make_geom(S, cp_size, causal);
  if (S % g.n_chunks != 0) return CPATTN_ERR_SHAPE;
  const long long need = (long long)cp_size * cp_size * slots(g) * slots(g);
  if (need > 0x7fffffffLL) return CPATTN_ERR_SHAPE;
  *n_rows = (int)need;
  if (!out || capacity < need) return CPATTN_ERR_ARG;
  int32_t* p = out;
  for (int r = 0; r < cp_size; ++r)
    for (int t = 0; t < cp_size; ++t) {
      const int src = step_src(g, r, t);
      for (int sa = 0; sa < slots(g); ++sa)
        for (int sb = 0; sb < slots(g); ++sb) {
          const int a = rank_chunk(g, r, sa), b = rank_chunk(g, src, sb);
          p[0] = r;
          p[1] = t;
          p[2] = a;
          p[3] = b;
          p[4] = src;
          p[5] = block_kind(g, a, b);
          p += CPATTN_PLAN_FIELDS;
        }
    }
  return CPATTN_OK;
}

int cpattn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
               int S, int D, int cp_size, int causal, float scale, int dtype, void* stream) {
  NvtxRange nv("cpattn_fwd");
  AttnShape sh;
  int st = check_shape(B, H, S, D, cp_size, causal, scale, dtype, &sh);
  if (st) return st;
  if (!q || !k || !v || !o || !lse) return CPATTN_ERR_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
    return CPATTN_ERR_ALIGN;
  unsigned* err = err_word();
  if (!err) return CPATTN_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (use_tc_fwd(sh)) {
    int stall = 0;
    int cur = g_stall.load();
    while (cur > 0 && !g_stall.compare_exchange_weak(cur, cur - 1)) {
    }
    if (cur > 0) stall = 1;
    g_last_path = 0;
    return count(launch_tc_fwd(sh, q, k, v, o, lse, err, stall, s));
  }
  g_last_path = 1;
  return count(launch_simt_fwd(sh, q, k, v, o, lse, 0, cp_size, 1, err, s));
}

int cpattn_fwd_step(const void* q, const void* k, const void* v, float* o_part,
                    float* lse_part, int B, int H, int S, int D, int cp_size, int causal,
                    float scale, int step, int dtype, void* stream) {
  NvtxRange nv("cpattn_fwd_step");
  AttnShape sh;
  int st = check_shape(B, H, S, D, cp_size, causal, scale, dtype, &sh);
  if (st) return st;
  if (step < 0 || step >= cp_size) return CPATTN_ERR_ARG;
  if (!q || !k || !v || !o_part || !lse_part) return CPATTN_ERR_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o_part) ||
      !aligned16(lse_part))
    return CPATTN_ERR_ALIGN;
  unsigned* err = err_word();
  if (!err) return CPATTN_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (use_tc_fwd(sh)) {
    g_last_path = 0;
    return count(launch_tc_fwd_step(sh, q, k, v, o_part, lse_part, step, err, s));
  }
  g_last_path = 1;
  return count(launch_simt_fwd(sh, q, k, v, o_part, lse_part, step, step + 1, 0, err, s));
}

int cpattn_merge(float* o_acc, float* lse_acc, const float* o_part, const float* lse_part,
                 long rows, int D, void* stream) {
  NvtxRange nv("cpattn_merge");
  if (rows < 0) return CPATTN_ERR_SHAPE;
  if (D != 64 && D != 128) return CPATTN_ERR_SHAPE;
  if (rows == 0) return CPATTN_OK;
  if (!o_acc || !lse_acc || !o_part || !lse_part) return CPATTN_ERR_ARG;
  if (!aligned16(o_acc) || !aligned16(o_part)) return CPATTN_ERR_ALIGN;
  return count(launch_merge(o_acc, lse_acc, o_part, lse_part, rows, D,
                            static_cast<cudaStream_t>(stream)));
}

int cpattn_finalize(const float* o_acc, void* o, long rows, int D, int dtype, void* stream) {
  NvtxRange nv("cpattn_finalize");
  if (dtype != CPATTN_BF16 && dtype != CPATTN_FP32) return CPATTN_ERR_DTYPE;
  if (rows < 0) return CPATTN_ERR_SHAPE;
  if (D != 64 && D != 128) return CPATTN_ERR_SHAPE;
  if (rows == 0) return CPATTN_OK;
  if (!o_acc || !o) return CPATTN_ERR_ARG;
  if (!aligned16(o_acc) || !aligned16(o)) return CPATTN_ERR_ALIGN;
  return count(launch_finalize(o_acc, o, rows, D, dtype == CPATTN_BF16,
                               static_cast<cudaStream_t>(stream)));
}

size_t cpattn_bwd_workspace_bytes(int B, int H, int S, int D) {
  if (B < 1 || H < 1 || S < 1 || (D != 64 && D != 128)) return 0;
  // two fp32 per row (delta, LSE * log2 e), each array 256-byte aligned
  const size_t rows = (size_t)B * H * S;
  const size_t one = (rows * sizeof(float) + 255) & ~(size_t)255;
  return 2 * one;
}

}  // extern "C"

namespace {

// cpattn_bwd and cpattn_bwd_accumulate: the same backward; acc_f32 != 0 adds
// the gradients into fp32 accumulators instead of writing them.
int bwd_impl(const void* q, const void* k, const void* v, const void* o, const float* lse,
             const void* dout, void* dq, void* dk, void* dv, int B, int H, int S, int D,
             int cp_size, int causal, float scale, void* workspace, size_t ws_bytes, int dtype,
             int acc_f32, void* stream) {
  AttnShape sh;
  int st = check_shape(B, H, S, D, cp_size, causal, scale, dtype, &sh);
  if (st) return st;
  if (!q || !k || !v || !o || !lse || !dout || !dq || !dk || !dv) return CPATTN_ERR_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse) ||
      !aligned16(dout) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
    return CPATTN_ERR_ALIGN;
  const size_t need = cpattn_bwd_workspace_bytes(B, H, S, D);
  if (!workspace || ws_bytes < need) return CPATTN_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return CPATTN_ERR_ALIGN;
  unsigned* err = err_word();
  if (!err) return CPATTN_ERR_CUDA;
  const size_t rows = (size_t)B * H * S;
  const size_t one = (rows * sizeof(float) + 255) & ~(size_t)255;
  float* ws_delta = static_cast<float*>(workspace);
  float* ws_lse2 = reinterpret_cast<float*>(static_cast<char*>(workspace) + one);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (use_tc_bwd(sh)) {
    g_last_path = 0;
    return count(
        launch_tc_bwd(sh, q, k, v, o, lse, dout, dq, dk, dv, ws_delta, ws_lse2, acc_f32, err, s));
  }
  g_last_path = 1;
  return count(launch_simt_bwd(sh, q, k, v, o, lse, dout, dq, dk, dv, ws_delta, acc_f32, s));
}

}  // namespace

extern "C" {

int cpattn_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
               const void* dout, void* dq, void* dk, void* dv, int B, int H, int S, int D,
               int cp_size, int causal, float scale, void* workspace, size_t ws_bytes,
               int dtype, void* stream) {
  NvtxRange nv("cpattn_bwd");
  return bwd_impl(q, k, v, o, lse, dout, dq, dk, dv, B, H, S, D, cp_size, causal, scale,
                  workspace, ws_bytes, dtype, 0, stream);
}

int cpattn_bwd_accumulate(const void* q, const void* k, const void* v, const void* o,
                          const float* lse, const void* dout, float* dq_acc, float* dk_acc,
                          float* dv_acc, int B, int H, int S, int D, int cp_size, int causal,
                          float scale, void* workspace, size_t ws_bytes, int dtype,
                          void* stream) {
  NvtxRange nv("cpattn_bwd_accumulate");
  return bwd_impl(q, k, v, o, lse, dout, dq_acc, dk_acc, dv_acc, B, H, S, D, cp_size, causal,
                  scale, workspace, ws_bytes, dtype, 1, stream);
}

int cpattn_sync_status(void* stream) {
  NvtxRange nv("cpattn_sync_status");
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return CPATTN_ERR_CUDA;
  unsigned* err = err_word();
  if (!err) return CPATTN_ERR_CUDA;
  unsigned h = 0;
  if (cudaMemcpyFromSymbol(&h, g_cpattn_error, sizeof(h)) != cudaSuccess) return CPATTN_ERR_CUDA;
  if (h) {
    unsigned zero = 0;
    if (cudaMemcpyToSymbol(g_cpattn_error, &zero, sizeof(zero)) != cudaSuccess)
      return CPATTN_ERR_CUDA;
    return CPATTN_ERR_TIMEOUT;
  }
  return CPATTN_OK;
}

int cpattn_profile(int on) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  const int prev = g_prof_on ? 1 : 0;
  g_prof_on = on != 0;
  if (g_prof_on) g_prof_used = 0;
  return prev;
}

int cpattn_profile_read(int kernel_id, double* total_ms, long long* launches) {
  if (!total_ms || !launches) return CPATTN_ERR_ARG;
  *total_ms = 0.0;
  *launches = 0;
  std::lock_guard<std::mutex> lk(g_prof_mu);
  for (int i = 0; i < g_prof_used; ++i) {
    if (g_prof_recs[i].id != kernel_id) continue;
    if (cudaEventSynchronize(g_prof_recs[i].b) != cudaSuccess) return CPATTN_ERR_CUDA;
    float ms = 0.f;
    if (cudaEventElapsedTime(&ms, g_prof_recs[i].a, g_prof_recs[i].b) != cudaSuccess)
      return CPATTN_ERR_CUDA;
    *total_ms += ms;
    *launches += 1;
  }
  return CPATTN_OK;
}

}  // extern "C"

namespace cpattn {
void prof_begin(int kernel_id, cudaStream_t stream) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  if (!g_prof_on || g_prof_used >= kProfPool) return;
  const int need = 2 * (g_prof_used + 1);
  while (g_prof_created < need) {
    if (cudaEventCreate(&g_prof_events[g_prof_created]) != cudaSuccess) return;
    ++g_prof_created;
  }
  ProfRec& r = g_prof_recs[g_prof_used];
  r.id = kernel_id;
  r.a = g_prof_events[2 * g_prof_used];
  r.b = g_prof_events[2 * g_prof_used + 1];
  cudaEventRecord(r.a, stream);
  g_prof_open_id = kernel_id;
}
void prof_end(int kernel_id, cudaStream_t stream) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  if (!g_prof_on || g_prof_open_id != kernel_id || g_prof_used >= kProfPool) return;
  cudaEventRecord(g_prof_recs[g_prof_used].b, stream);
  ++g_prof_used;
  g_prof_open_id = -1;
}
int num_sms(int device) {
  static int cache[kMaxDevices] = {0};
  if (device < 0 || device >= kMaxDevices) return 148;
  if (!cache[device]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, device) != cudaSuccess || n <= 0)
      n = 148;
    cache[device] = n;
  }
  return cache[device];
}
}  // namespace cpattn
