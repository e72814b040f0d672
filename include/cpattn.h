/*
 * cpattn.h -- C ABI of libcpattn.so: causal scaled-dot-product attention
 * evaluated the ring way (context parallel / RingAttention) on one GPU.
 *
 * What is computed.  For every (batch b, head h) and query row i,
 *     O_i = sum_{j in A_i} softmax_j(scale * q_i . k_j) v_j,
 *     LSE_i = log sum_{j in A_i} exp(scale * q_i . k_j)      (natural log)
 * with A_i = { j <= i } when causal, all j otherwise.  "Configuring
 * RingAttention+FlashAttention for CP" (devpress.csdn.net), section 1: each
 * rank's Q takes turns against the K/V blocks of every rank and the results
 * are aggregated; section 3, note 2: the mask is exact, nothing leaks.
 *
 * How it is evaluated.  The sequence is split over cp_size virtual ranks.
 *   causal:     2*cp_size chunks of c = S / (2*cp_size) rows; rank r owns
 *               chunks r and 2*cp_size-1-r (the zigzag of the same page,
 *               section 5, item 1);
 *   non-causal: cp_size contiguous chunks of c = S / cp_size rows.
 * At ring step t rank r attends to the K/V of rank (r - t) mod cp_size (same
 * page, section 3 code).  A (q chunk a, kv chunk b) block is SKIP when a < b,
 * DIAG (masked j <= i) when a == b, FULL otherwise.  Each step yields a partial
 * (O, LSE) per row; partials are combined by the log-sum-exp merge
 *     L = max(La,Lb) + log(exp(La-M) + exp(Lb-M)),  O = e^(La-L) Oa + e^(Lb-L) Ob.
 * "Megatron-LM source analysis: Context Parallel" (mieleap.com), section 5:
 * the per-step attention call of the double-buffered ring loop.
 *
 * Conventions for every entry point.
 *   - Tensors are caller-owned DEVICE pointers, contiguous, layout [B][H][S][D]
 *     (LSE and per-row vectors [B][H][S]).  The library keeps no pointer after
 *     the call returns and allocates no device memory on any call.
 *   - dtype is cpattn_dtype: CPATTN_BF16 (bf16 in/out, fp32 accumulate) or
 *     CPATTN_FP32 (fp32 in/out, fp32 arithmetic throughout).
 *   - stream is a cudaStream_t (NULL = legacy default stream).  Work is
 *     enqueued asynchronously; argument and shape errors are returned before
 *     anything is enqueued.  In-kernel failures (a bounded wait that ran out)
 *     are recorded on the device and reported by cpattn_sync_status().
 *   - Preconditions (CPATTN_ERR_SHAPE otherwise): B, H >= 1; S >= 1;
 *     cp_size >= 1; D is 64 or 128; causal: S % (2*cp_size) == 0, non-causal:
 *     S % cp_size == 0 (any chunk length c).  bf16 problems with c % 128 == 0
 *     run on the tcgen05 tensor-core kernels, the rest (every fp32 problem,
 *     bf16 chunks of other lengths) on the CUDA-core kernels.
 *   - Pointers must be 16-byte aligned (CPATTN_ERR_ALIGN); scale must be
 *     finite and > 0 (CPATTN_ERR_ARG).
 *   - Sizes are not visible through plain pointers: every buffer must hold the
 *     elements its stated layout implies (the Python binding checks shapes and
 *     dtypes before calling).
 *   - Each entry point opens an NVTX range named after itself for the host
 *     side of the call (no-op without an attached profiler).
 */
#ifndef CPATTN_H
#define CPATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    CPATTN_OK = 0,
    CPATTN_ERR_ARG = 1,       /* null pointer, bad scale, bad step, bad capacity */
    CPATTN_ERR_SHAPE = 2,     /* sizes violate the preconditions above */
    CPATTN_ERR_DTYPE = 3,     /* unknown dtype */
    CPATTN_ERR_ALIGN = 4,     /* a pointer is not 16-byte aligned */
    CPATTN_ERR_CUDA = 5,      /* a CUDA runtime call or launch failed */
    CPATTN_ERR_TIMEOUT = 6,   /* a bounded in-kernel wait ran out (reported later) */
    CPATTN_ERR_WORKSPACE = 7  /* workspace missing or smaller than required */
} cpattn_status;

typedef enum { CPATTN_BF16 = 0, CPATTN_FP32 = 1 } cpattn_dtype;

/* Block kinds in a plan row. */
enum { CPATTN_SKIP = 0, CPATTN_FULL = 1, CPATTN_DIAG = 2 };

/* Number of int32 fields in one plan row. */
#define CPATTN_PLAN_FIELDS 6

/*
 * cpattn_plan -- host only, no GPU needed.
 * Writes the ring schedule: one row of CPATTN_PLAN_FIELDS int32 per
 * (rank r, step t, q slot, kv slot) in lexicographic order, SKIP rows included:
 *     (r, t, q_chunk a, kv_chunk b, src_rank, kind)
 * with src_rank = (r - t) mod cp_size, a the q slot's chunk of rank r and b
 * the kv slot's chunk of rank src_rank.  Rows: cp_size*cp_size*4 causal,
 * cp_size*cp_size non-causal.  out: host buffer of capacity rows
 * (capacity*CPATTN_PLAN_FIELDS int32).  *n_rows is always set to the number of
 * rows needed; CPATTN_ERR_ARG if capacity is too small (nothing written) or a
 * pointer is null, CPATTN_ERR_SHAPE if S is not a multiple of the chunk count.
 * Sources: ring rule and zigzag as cited at the top of this file.
 */
int cpattn_plan(int S, int cp_size, int causal, int32_t* out, int capacity, int* n_rows);

/*
 * cpattn_fwd -- the whole ring forward in one launch: every virtual rank, every
 * step, partials merged on chip by the online (log-sum-exp) rescale, SKIP
 * blocks never computed.
 *   q, k, v : [B][H][S][D] input dtype (read)
 *   o       : [B][H][S][D] input dtype (written)
 *   lse     : [B][H][S] fp32, natural-log LSE of scale*q.k (written)
 */
int cpattn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
               int S, int D, int cp_size, int causal, float scale, int dtype, void* stream);

/*
 * cpattn_fwd_step -- ring step `step` (0 <= step < cp_size) for all virtual
 * ranks at once: each row's partial against the K/V that its rank holds at
 * that step (both kv chunks of the source rank, SKIP blocks omitted).
 *   o_part  : [B][H][S][D] fp32, normalised partial output (written)
 *   lse_part: [B][H][S] fp32, partial LSE; -inf (and o_part = 0) where every
 *             block of the row is SKIP at this step (written)
 */
int cpattn_fwd_step(const void* q, const void* k, const void* v, float* o_part,
                    float* lse_part, int B, int H, int S, int D, int cp_size, int causal,
                    float scale, int step, int dtype, void* stream);

/*
 * cpattn_merge -- in place: (o_acc, lse_acc) <- merge((o_acc, lse_acc),
 * (o_part, lse_part)) for `rows` rows of D fp32 values, by the log-sum-exp
 * rule at the top of this file.  A side with LSE = -inf contributes nothing
 * (both -inf: o_acc and lse_acc unchanged).  The merge the pages leave
 * unwritten: their listing adds partial outputs, which is wrong; this is the
 * exact combination.  rows >= 0, D in {64, 128}.
 */
int cpattn_merge(float* o_acc, float* lse_acc, const float* o_part, const float* lse_part,
                 long rows, int D, void* stream);

/*
 * cpattn_finalize -- o[rows][D] (dtype) <- o_acc[rows][D] (fp32), rounding to
 * nearest-even for bf16.
 */
int cpattn_finalize(const float* o_acc, void* o, long rows, int D, int dtype, void* stream);

/*
 * cpattn_bwd_workspace_bytes -- bytes of device workspace cpattn_bwd needs for
 * this shape (two fp32 values per row: delta_i = dO_i . O_i and LSE_i in base
 * 2).  0 on bad sizes.
 */
size_t cpattn_bwd_workspace_bytes(int B, int H, int S, int D);

/*
 * cpattn_bwd -- recompute backward from (O, LSE): for every non-SKIP block,
 * P = exp(scale q.k - LSE) (DIAG masked), dV += P^T dO, dP = dO V^T,
 * dS = P (dP - delta) with delta_i = dO_i . O_i, dK += scale dS^T Q,
 * dQ += scale dS K.  The gradient is that of the same function the forward
 * computes ("Megatron-LM source analysis: Context Parallel", section 2: the
 * backward mirrors the forward's communication).
 *   q, k, v, o, dout : [B][H][S][D] dtype (read); lse: [B][H][S] fp32 from
 *                      cpattn_fwd (read)
 *   dq, dk, dv       : [B][H][S][D] dtype (written)
 *   workspace        : caller-owned device buffer of ws_bytes >=
 *                      cpattn_bwd_workspace_bytes(B, H, S, D), 256-byte aligned;
 *                      contents on entry are ignored
 */
int cpattn_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
               const void* dout, void* dq, void* dk, void* dv, int B, int H, int S, int D,
               int cp_size, int causal, float scale, void* workspace, size_t ws_bytes,
               int dtype, void* stream);

/*
 * cpattn_bwd_accumulate -- the same backward as cpattn_bwd, but the block's
 * gradients are ADDED, in fp32 and without rounding to the input dtype, into
 * caller-owned fp32 accumulators:
 *     dq_acc += dQ,  dk_acc += dK,  dv_acc += dV      ([B][H][S][D] fp32 each)
 * For the multi-rank ring and all-gather drivers, which call the backward once
 * per (q chunk, kv chunk) block and sum the blocks' terms for every chunk
 * ("Megatron-LM source analysis: Context Parallel", section 2: the backward
 * mirrors the forward's exchange, every block adding to the gradients of its q
 * and kv chunks).  With bf16 inputs the sums then carry one rounding at the
 * end (the caller's cast) instead of one per block term.
 *   Arguments, workspace, preconditions and errors: as cpattn_bwd.  The
 *   accumulators must not alias each other or any input.  Every element of
 *   every accumulator is read and written exactly once per call (no atomics), so
 *   calls on one stream compose; calls that overlap on the GPU and share an
 *   accumulator race.
 */
int cpattn_bwd_accumulate(const void* q, const void* k, const void* v, const void* o,
                          const float* lse, const void* dout, float* dq_acc, float* dk_acc,
                          float* dv_acc, int B, int H, int S, int D, int cp_size, int causal,
                          float scale, void* workspace, size_t ws_bytes, int dtype,
                          void* stream);

/*
 * FP8 (e4m3) forward.  "Megatron-LM source analysis: Context Parallel",
 * section 4: FP8 attention inputs combined with context parallelism, to save
 * memory.  The pages fix neither the format nor the scaling; this library
 * uses e4m3 ("fn": largest finite 448, no infinities) with one scale per
 * tensor:
 *     s = 448 / max|x|  (fp32; 1 for an all-zero tensor),
 *     code = e4m3(fp32(x * s)), round to nearest even, saturating to +-448,
 * and the value a code stands for is code / s.  The attention computed is the
 * attention of those values, with P = softmax rounded to e4m3 (scaled by 2^6)
 * before the P.V product; O is bf16, LSE fp32 as in cpattn_fwd.
 *
 * cpattn_amax -- *amax (device fp32) = max_i |x[i]| over n elements of dtype.
 *   amax must be 4-byte aligned; the call zeroes it first (cudaMemsetAsync on
 *   `stream`), so it needs no initialisation.
 * cpattn_quantize_e4m3 -- codes of x ([BH][S][D], dtype) with the scale
 *   derived from *amax (device, as written by cpattn_amax):
 *     transpose = 0: out [BH][S][D] bytes (the layout of q and k)
 *     transpose = 1: out [BH][D][S] bytes (V transposed per head); S % 64 == 0
 *   D in {64, 128}; x and out 16-byte aligned.
 * cpattn_fwd_fp8 -- the ring forward of cpattn_fwd on e4m3 inputs:
 *     q8, k8 : [B][H][S][D] codes;  vt8: [B][H][D][S] codes (V transposed)
 *     amax   : device float[3] = max|q|, max|k|, max|v| (the scales' source)
 *     o      : [B][H][S][D] bf16;   lse: [B][H][S] fp32 (written)
 *   Preconditions: those of cpattn_fwd, and D == 128 and a chunk length that
 *   is a multiple of 128 (CPATTN_ERR_SHAPE).  Pointers 16-byte aligned (amax:
 *   4).  One tcgen05 launch (kind::f8f6f4 MMAs).
 */
int cpattn_amax(const void* x, long n, int dtype, float* amax, void* stream);
int cpattn_quantize_e4m3(const void* x, int dtype, int BH, int S, int D, int transpose,
                         const float* amax, uint8_t* out, void* stream);
int cpattn_fwd_fp8(const uint8_t* q8, const uint8_t* k8, const uint8_t* vt8, const float* amax,
                   void* o, float* lse, int B, int H, int S, int D, int cp_size, int causal,
                   float scale, void* stream);

/* Size of the fixed device scratch array used by cpattn_bwd_noalloc (64 MiB). */
#define CPATTN_NOALLOC_SCRATCH_BYTES (64u << 20)

/*
 * cpattn_bwd_noalloc -- the same backward as cpattn_bwd, for callers that
 * cannot allocate device memory (code running inside an allocator's own
 * callbacks, in a process whose memory pool belongs to another framework, or on
 * a path that cannot afford an allocation's synchronisation or failure).  The
 * pages have no counterpart: this is an interface convenience, not part of the
 * method.
 *   Arguments: as cpattn_bwd, minus the workspace.  The caller still passes
 *   every input and output.
 *   Scratch: a fixed CPATTN_NOALLOC_SCRATCH_BYTES array in device global
 *   memory that every device loading this library holds until the process
 *   exits.  The function itself allocates and frees nothing.
 *   Limits: shapes whose cpattn_bwd_workspace_bytes(B, H, S, D) exceeds
 *   CPATTN_NOALLOC_SCRATCH_BYTES are rejected with CPATTN_ERR_WORKSPACE before
 *   anything is enqueued (CPATTN_ERR_SHAPE for invalid sizes).
 *   Set-up: the first call on a device looks up the array's device address
 *   (with that device current) and keeps it for the life of the process;
 *   make that first call before any stream capture begins.  The address
 *   belongs to the device's current context: do not use the library across a
 *   cudaDeviceReset (or any other teardown of the primary context) in the same
 *   process.
 *   Sharing: all calls on a device use the same array, which keeps the last
 *   call's contents.  It holds two fp32 values per row, delta_i = dO_i . O_i
 *   and LSE_i * log2(e); the backward's preprocess kernel rewrites both for
 *   every row of the call before anything reads them, so leftovers of earlier
 *   calls are never used (dQ, dK and dV go straight to the caller's outputs).
 *   Calls that can overlap on the GPU -- on different streams, or from
 *   different host threads -- race on the array; serialise them.
 */
int cpattn_bwd_noalloc(const void* q, const void* k, const void* v, const void* o,
                       const float* lse, const void* dout, void* dq, void* dk, void* dv, int B,
                       int H, int S, int D, int cp_size, int causal, float scale, int dtype,
                       void* stream);

/*
 * cpattn_accumulate -- acc[i] += x[i] for i < n, acc fp32, x of `dtype`: the
 * running gradient sums of the multi-rank ring backward, where every (q chunk,
 * kv chunk) block adds its dQ, dK, dV terms ("Megatron-LM source analysis:
 * Context Parallel", section 2: the backward mirrors the forward's exchange).
 * n must be a multiple of 4 (CPATTN_ERR_SHAPE), both pointers 16-byte aligned
 * (CPATTN_ERR_ALIGN); n = 0 does nothing.
 */
int cpattn_accumulate(float* acc, const void* x, long n, int dtype, void* stream);

/*
 * The attention layer around the ring attention ("Configuring
 * RingAttention+FlashAttention for CP", section 3 code): Q, K, V projections
 * of width E (nn.Linear with bias), the [B,S,E] -> [B,H,S,D] head split, the
 * ring attention (cpattn_fwd), the head merge and the output projection.
 * bf16 only; D = E / H must be 64 or 128 and the attention's own
 * preconditions apply to (B, H, S, D, cp_size, causal).
 *   Layouts (row-major, caller-owned device memory, 16-byte aligned):
 *     x, y, dy, dx           [B][S][E]
 *     w_qkv, dw_qkv          [3E][E]   rows = the q, k and v projection weights
 *                                      stacked (out features x in features)
 *     b_qkv, db_qkv          [3E]
 *     w_o, dw_o              [E][E];   b_o, db_o [E]
 *     q, k, v, o             [B][H][S][D] (bf16), lse [B][H][S] (fp32): saved
 *                                      by the forward for the backward
 *   The projections run on this library's tcgen05 GEMM (cpattn_gemm below:
 *   bf16, fp32 accumulation, the bias added in the GEMM epilogue); the head
 *   reshapes and the bias gradients are this library's kernels too.  B*S and E
 *   must be multiples of 8 (CPATTN_ERR_SHAPE).
 *   Workspace: cpattn_layer_workspace_bytes(B, S, E, H) bytes (0 for invalid
 *   sizes), used by both calls; its contents need not survive between them.
 *   Errors: CPATTN_ERR_SHAPE / ARG / ALIGN / WORKSPACE before anything is
 *   enqueued; CPATTN_ERR_CUDA when a launch fails.
 */
size_t cpattn_layer_workspace_bytes(int B, int S, int E, int H);

/* y = out_proj(merge_heads(attention(split_heads(x w_qkv^T + b_qkv)))) */
int cpattn_layer_fwd(const void* x, const void* w_qkv, const void* b_qkv, const void* w_o,
                     const void* b_o, void* y, void* q, void* k, void* v, void* o, float* lse,
                     int B, int S, int E, int H, int cp_size, int causal, float scale,
                     void* workspace, size_t ws_bytes, void* stream);

/*
 * Gradients of the layer for upstream gradient dy, from the forward's saved
 * q, k, v, o, lse: dx, dw_qkv, db_qkv, dw_o, db_o (all overwritten).
 */
int cpattn_layer_bwd(const void* x, const void* w_qkv, const void* w_o, const void* q,
                     const void* k, const void* v, const void* o, const float* lse,
                     const void* dy, void* dx, void* dw_qkv, void* db_qkv, void* dw_o,
                     void* db_o, int B, int S, int E, int H, int cp_size, int causal,
                     float scale, void* workspace, size_t ws_bytes, void* stream);

/*
 * cpattn_gemm -- the layer's projection GEMM on the tcgen05 tensor cores:
 *     C[M][N] = op(A) op(B) (+ bias[n] added to every row),
 * bf16 operands, bias and result (round to nearest even), fp32 accumulation,
 * all row-major and caller-owned device memory.  The products of the
 * attention layer's nn.Linear projections and their gradients ("Configuring
 * RingAttention+FlashAttention for CP", section 3 code: q/k/v_proj, out_proj).
 *   a_layout 0: A stored [M][K];   1: A stored [K][M] (A is its transpose)
 *   b_layout 0: B stored [N][K] (the nn.Linear weight layout, C = A B^T);
 *            1: B stored [K][N] (C = A B)
 *   bias: [N] or NULL.  C must not alias A, B or bias.
 *   M, N, K >= 1 and multiples of 8 (CPATTN_ERR_SHAPE); pointers 16-byte
 *   aligned (CPATTN_ERR_ALIGN); layouts other than 0 / 1: CPATTN_ERR_ARG.
 *   In-kernel bounded-wait failures are reported by cpattn_sync_status().
 */
int cpattn_gemm(const void* A, const void* B, const void* bias, void* C, int M, int N, int K,
                int a_layout, int b_layout, void* stream);

/*
 * cpattn_sync_status -- synchronises `stream`, then returns and clears the
 * device-side error word of the current device (CPATTN_OK, CPATTN_ERR_TIMEOUT)
 * or CPATTN_ERR_CUDA if the synchronisation itself failed.  The word's device
 * address is looked up once per device and kept: as for cpattn_bwd_noalloc,
 * do not use the library across a cudaDeviceReset in the same process.
 */
int cpattn_sync_status(void* stream);

/* Human-readable name of a status code (static string). */
const char* cpattn_status_str(int status);

/*
 * Diagnostics.
 * cpattn_launch_count: number of kernels this library has enqueued so far in
 *   this process (all devices).
 * cpattn_set_path: 0 = automatic (tcgen05 kernels where the shape allows),
 *   1 = force the CUDA-core kernels, 2 = tcgen05 kernels on one SM each (the
 *   two-SM dQ kernel off); any other value means 0.  Returns the previous
 *   setting.  For tests that compare the kernel families.
 * cpattn_last_path: kernel family used by the last fwd/bwd call
 *   (0 tcgen05, 1 CUDA cores).
 * cpattn_debug_stall: n > 0 makes the next n tcgen05 forward launches omit one
 *   K/V tile load, so the bounded waits run out and the call reports
 *   CPATTN_ERR_TIMEOUT through cpattn_sync_status; the device stays usable.
 *   For failure-detection tests only.
 */
long long cpattn_launch_count(void);
/*
 * cpattn_profile: on != 0 starts per-kernel timing (a CUDA event pair recorded
 *   on the launch stream around every kernel the library enqueues, up to 8192
 *   kernels) and discards earlier records; 0 stops recording.  Returns the
 *   previous setting.
 * cpattn_profile_read: total milliseconds and launch count of one kernel kind
 *   since the last cpattn_profile(1); waits for those events.  Kernel kinds:
 *   0 tcgen05 forward, 1 CUDA-core forward, 2 merge, 3 finalize, 4 backward
 *   preprocess (delta), 5 CUDA-core dK/dV, 6 CUDA-core dQ, 7 tcgen05 dK/dV,
 *   8 tcgen05 dQ, 9 layer head split / merge, 10 layer bias gradients,
 *   11 gradient accumulation (cpattn_accumulate), 12 GEMM (cpattn_gemm and
 *   the layer's projections), 13 tcgen05 e4m3 forward (cpattn_fwd_fp8),
 *   14 max|x| and e4m3 quantisation.
 */
int cpattn_profile(int on);
int cpattn_profile_read(int kernel_kind, double* total_ms, long long* launches);
int cpattn_set_path(int path);
int cpattn_last_path(void);
int cpattn_debug_stall(int n);

#ifdef __cplusplus
}
#endif

#endif /* CPATTN_H */
