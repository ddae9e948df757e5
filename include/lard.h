/*
 * lard.h -- C ABI of liblard: the linear-memory relation-KL kernel of
 * LinearARD (relation distillation for RoPE-scaled students), for NVIDIA
 * B200 (sm_100a).
 *
 * Method, as defined on the pages this library follows:
 *   "LinearARD: Linear-Memory Attention Distillation for RoPE Restoration"
 *   (papernotes.org notes), 方法详解 / 关键设计 1: for a head, teacher (m = t)
 *   and student (m = s) projections X_m, Y_m in R^{n x d} give relation
 *   logits Z_m = tau * X_m Y_m^T under a causal mask M; R_m is their
 *   row-wise softmax; the loss is the row-averaged forward KL(R_t || R_s),
 *   summed over the Q/Q, K/K and V/V relations (lambda = 1, section
 *   损失函数 / 训练策略).
 *   Same page, 关键设计 3: Phase 1 streams tiles and keeps only the per-row
 *   statistic LSE_m(i) = log sum_k exp Z_m(i,k) in HBM (O(BHn) memory);
 *   Phase 2 recomputes 128 x 128 tiles of Z_s and Z_t on chip, rebuilds
 *   R = exp(Z - LSE), forms dZ = (R_s - R_t)/n and contracts it with the
 *   projections into dX_s and dY_s, never storing an n x n map.
 *   LinearARD abstract (fugumt.com page): the kernel computes the exact KL
 *   divergence and gradients from per-token log-sum-exp statistics.
 *
 * Readings this library takes where the pages are silent:
 *   - tau is a parameter (1/sqrt(d) in the usual setting), tau > 0;
 *   - the causal mask keeps j <= i (diagonal included); causal = 0 gives the
 *     plain full-row softmax;
 *   - the loss of one (batch, head) is (1/n) sum_i KL_i; heads and batch
 *     entries are summed; a caller sums the three relations;
 *   - gradients carry the chain-rule factor tau of Z = tau X Y^T:
 *     dX_s = tau dZ Y_s, dY_s = tau dZ^T X_s; the teacher gets none;
 *   - for a self-relation (Y = X) the student gradient is the sum of the two
 *     partials; lard_kl_bwd returns them apart, lard_kl_bwd_self (and
 *     lard_kl_bwd_multi with dYs = NULL) adds them on the device.
 *
 * Conventions for every entry point:
 *   - Tensors are row-major [B, H, n, d], contiguous, in device memory of
 *     the GPU that runs the call, base addresses 16-byte aligned.  Inputs
 *     are bf16 (LARD_DTYPE_BF16) or fp32 (LARD_DTYPE_FP32); every output is
 *     fp32, except the gradients of the two _bf16 Phase-2 calls.  The caller
 *     allocates and owns every buffer (and the workspace of
 *     lard_kl_bwd_multi_bf16); the library allocates no device memory (the
 *     no-allocation variant uses a fixed array that the library holds).
 *   - Work is enqueued asynchronously on `stream` (0 = legacy default
 *     stream); results are valid once the stream reaches that point.
 *   - Argument errors are reported synchronously, before anything is
 *     enqueued, and nothing is written.  Launch errors map to LARD_ERR_CUDA.
 *   - Every wait inside the kernels has a time limit; a wait that runs out
 *     makes the kernel stop early and sets a device-side fault word that
 *     lard_device_status() reports as LARD_ERR_TIMEOUT.
 *   - Supported: d in {64, 128} for bf16, d a multiple of 32 up to 256 for
 *     fp32; any n from 1 to 2^31 - 128 (ragged last tile handled);
 *     B*H*n*d < 2^40.
 *   - Calls are thread-safe (lard_kl_bwd_multi_bf16_noalloc: see its note on
 *     overlapping calls).  Inputs may alias each other (Y = X).
 */
#ifndef LARD_H
#define LARD_H

#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define LARD_API __attribute__((visibility("default")))
#else
#define LARD_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    LARD_OK = 0,
    LARD_ERR_INVALID_ARG = 1, /* null/misaligned pointer, bad size, non-finite scalar, aliasing */
    LARD_ERR_UNSUPPORTED = 2, /* head dim or dtype not built, or a GPU other than sm_100 */
    LARD_ERR_CUDA = 3,        /* a CUDA runtime call or kernel launch failed */
    LARD_ERR_TIMEOUT = 4,     /* a kernel wait ran out of time (see lard_device_status) */
    LARD_ERR_TOO_LARGE = 5    /* the problem needs more than the fixed workspace of
                                 lard_kl_bwd_multi_bf16_noalloc */
} lard_status;

typedef enum { LARD_DTYPE_BF16 = 0, LARD_DTYPE_FP32 = 1 } lard_dtype;

/*
 * Phase 1 (LinearARD notes, 关键设计 3, first phase): per-row log-sum-exp of
 * the teacher and student relation logits and the row KL, streamed over
 * 128 x 128 tiles without materialising Z.
 *
 *   Xt, Yt, Xs, Ys  inputs [B, H, n, d] (teacher X, teacher Y, student X,
 *                   student Y).  Yt may equal Xt and Ys may equal Xs.
 *   tau             logit scale, finite and > 0.
 *   causal          1: mask j > i; 0: no mask.
 *   lse_t, lse_s    out [B, H, n]: LSE_m(i) = log sum_{j allowed} exp Z_m(i,j).
 *   row_kl          out [B, H, n]: KL(R_t(i,.) || R_s(i,.)).
 *   loss_bh         out [B*H] or NULL: (1/n) sum_i row_kl.
 *   loss_total      out [1] or NULL: sum of loss_bh (requires loss_bh).
 * Extra device memory beyond the caller's buffers: none.  The HBM state
 * kept between the phases is lse_t and lse_s, 8 bytes per row.
 */
LARD_API lard_status lard_kl_fwd(const void* Xt, const void* Yt, const void* Xs, const void* Ys,
                        lard_dtype dtype, int B, int H, int n, int d, float tau, int causal,
                        float* lse_t, float* lse_s, float* row_kl,
                        float* loss_bh, float* loss_total, cudaStream_t stream);

/*
 * Phase 2 (LinearARD notes, 关键设计 3, second phase): recompute Z_t and Z_s
 * tile by tile, rebuild R from the Phase-1 LSEs, form dZ = (R_s - R_t)/n and
 * contract it into the student gradients.
 *
 *   Xt, Yt, Xs, Ys, dtype, B, H, n, d, tau, causal: as for lard_kl_fwd
 *                   (must be the same values that produced lse_t / lse_s).
 *   lse_t, lse_s    in [B, H, n], written by lard_kl_fwd.
 *   grad_scale      g, finite: upstream gradient of the summed loss.
 *   dXs, dYs        out [B, H, n, d] fp32, overwritten:
 *                   dXs = g * dL/dXs = g * tau * dZ Y_s,
 *                   dYs = g * dL/dYs = g * tau * dZ^T X_s,
 *                   with L = sum over (b, h) of the row-averaged KL.
 *                   They must not overlap each other or any input.
 * The bf16 path accumulates dXs with fp32 reduce-adds in L2, so its last
 * bits depend on the order in which tiles finish; the fp32 path is
 * deterministic.
 */
LARD_API lard_status lard_kl_bwd(const void* Xt, const void* Yt, const void* Xs, const void* Ys,
                        lard_dtype dtype, int B, int H, int n, int d, float tau, int causal,
                        const float* lse_t, const float* lse_s, float grad_scale,
                        float* dXs, float* dYs, cudaStream_t stream);

/*
 * Phase 2 for a self-relation (Y_t = X_t, Y_s = X_s, as for the Q/Q, K/K and
 * V/V maps of LinearARD notes, 关键设计 1), returning the total student
 * gradient: X_s enters the logits as both the row and the column factor, so
 * dL/dX_s = tau dZ X_s + tau dZ^T X_s, the sum of lard_kl_bwd's dXs and dYs.
 *
 *   Xt, Xs, dtype, B, H, n, d, tau, causal, lse_t, lse_s, grad_scale: as for
 *                   lard_kl_bwd with Yt = Xt and Ys = Xs.
 *   dXs             out [B, H, n, d] fp32, overwritten with g * dL/dX_s (both
 *                   paths); must not overlap any input.
 * Both partials are added into dXs on the device (one n x d fp32 buffer and
 * no separate sum).  LARD_ERR_UNSUPPORTED for fp32 inputs: call lard_kl_bwd
 * and add dXs + dYs instead.
 */
LARD_API lard_status lard_kl_bwd_self(const void* Xt, const void* Xs, lard_dtype dtype, int B, int H, int n,
                             int d, float tau, int causal, const float* lse_t, const float* lse_s,
                             float grad_scale, float* dXs, cudaStream_t stream);

/*
 * Several relations in one launch per phase.  LinearARD distils three
 * self-relations per layer (Q/Q, K/K, V/V; LinearARD notes, 关键设计 1), and a
 * GQA model has fewer K/V heads than Q heads; one launch over all of them
 * replaces a launch (and its tail) per relation.  Each relation is:
 *
 *   Xt, Yt, Xs, Ys  in [B, H, n, d] (as for lard_kl_fwd; Yt may equal Xt and
 *                   Ys may equal Xs).
 *   H               its head count (>= 1).
 *   lse_t, lse_s    [B, H, n]: written by lard_kl_fwd_multi, read by
 *                   lard_kl_bwd_multi.
 *   row_kl          [B, H, n]: written by lard_kl_fwd_multi.
 *   loss_bh         [B*H] or NULL: written by lard_kl_fwd_multi.
 *   dXs             [B, H, n, d] fp32: written by lard_kl_bwd_multi.
 *   dYs             [B, H, n, d] fp32, written by lard_kl_bwd_multi; or NULL
 *                   for a self-relation (Yt == Xt, Ys == Xs, bf16 only), whose
 *                   total student gradient is then written to dXs, as by
 *                   lard_kl_bwd_self.
 * Fields a phase does not use may be NULL.
 */
#define LARD_MAX_RELATIONS 4
typedef struct lard_relation {
    const void* Xt;
    const void* Yt;
    const void* Xs;
    const void* Ys;
    int H;
    float* lse_t;
    float* lse_s;
    float* row_kl;
    float* loss_bh;
    float* dXs;
    float* dYs;
} lard_relation;

/*
 * Phase 1 of nrel (1 .. LARD_MAX_RELATIONS) relations sharing dtype, B, n, d,
 * tau and causal.  Each relation's outputs are what lard_kl_fwd writes for
 * it.  loss_total (or NULL; requires every loss_bh) is the sum of all
 * relations' losses.  No output may overlap another buffer of the call; all
 * buffers live on one GPU.  Errors as for lard_kl_fwd.
 */
LARD_API lard_status lard_kl_fwd_multi(const lard_relation* rel, int nrel, lard_dtype dtype, int B, int n,
                              int d, float tau, int causal, float* loss_total, cudaStream_t stream);

/*
 * Phase 2 of nrel relations (as for lard_kl_fwd_multi, with the same inputs
 * and the lse_t / lse_s it wrote).  Each relation's dXs (and dYs) are what
 * lard_kl_bwd (or, with dYs == NULL, lard_kl_bwd_self) writes for it.
 */
LARD_API lard_status lard_kl_bwd_multi(const lard_relation* rel, int nrel, lard_dtype dtype, int B, int n,
                              int d, float tau, int causal, float grad_scale, cudaStream_t stream);

/*
 * bf16 gradient outputs (Phase 2).  A bf16 training step consumes bf16
 * gradients; writing them directly halves the gradient bytes the call writes
 * and a caller copies out.  dY_s[J] is complete in the kernel and is rounded
 * once; dX_s receives contributions from every column block of a row, so it
 * is accumulated in fp32 in a caller-provided workspace and rounded once
 * (round-to-nearest-even) by a final pass of the same call.  For a fused
 * self-relation (dYs == NULL) both partials accumulate in the workspace and
 * dXs receives the rounded total gradient.  This follows LinearARD notes,
 * 关键设计 3 (gradients accumulated into dX_s and dY_s) with the rounding the
 * pages leave open placed after the accumulation.
 *
 *   dXs, dYs   bf16 [B, H, n, d] outputs of one relation, 16-byte aligned;
 *              dYs == NULL for a fused self-relation (Yt == Xt, Ys == Xs).
 */
typedef struct lard_grads_bf16 {
    void* dXs;
    void* dYs;
} lard_grads_bf16;

/*
 * Bytes of fp32 workspace lard_kl_bwd_multi_bf16 needs for these relations:
 * the sum over relations of B * H * n * d * 4.  Returns 0 if the description
 * is invalid (rel NULL, nrel outside 1 .. LARD_MAX_RELATIONS, a size < 1).
 */
LARD_API size_t lard_kl_bwd_bf16_workspace_bytes(const lard_relation* rel, int nrel, int B, int n, int d);

/*
 * Phase 2 of nrel relations (as lard_kl_bwd_multi) with bf16 gradient outputs.
 *   rel        as for lard_kl_bwd_multi, with every dXs and dYs field NULL (the
 *              gradients go to `out`).
 *   out        [nrel] bf16 output buffers, overwritten with what
 *              lard_kl_bwd_multi writes in fp32, rounded once to bf16.
 *   workspace  device memory on the call's GPU, 16-byte aligned, at least
 *              lard_kl_bwd_bf16_workspace_bytes(rel, nrel, B, n, d) bytes
 *              (workspace_bytes); its contents are overwritten and have no
 *              meaning after the call; it must not overlap any other buffer.
 * bf16 inputs only (LARD_ERR_UNSUPPORTED for fp32 inputs, whose path is the
 * full-precision one).  Other errors as for lard_kl_bwd_multi.  The
 * workspace is the only memory the call uses beyond its inputs and outputs;
 * the library allocates none.
 */
LARD_API lard_status lard_kl_bwd_multi_bf16(const lard_relation* rel, const lard_grads_bf16* out, int nrel,
                                   lard_dtype dtype, int B, int n, int d, float tau, int causal,
                                   float grad_scale, void* workspace, size_t workspace_bytes,
                                   cudaStream_t stream);

/*
 * lard_kl_bwd_multi_bf16 for callers that cannot allocate device memory.
 *
 * Some callers cannot call cudaMalloc at the point where they run Phase 2:
 * code inside another framework's training step whose memory pool owns the
 * whole device, or a runtime that forbids device allocation once it has
 * started.  Such a caller cannot provide the fp32 workspace that
 * lard_kl_bwd_multi_bf16 asks for.  This entry point takes the same
 * arguments without the workspace and uses instead a fixed array in the
 * library's device memory of LARD_NOALLOC_WORKSPACE_BYTES (64 MiB): every
 * GPU that loads the library holds that array until the process exits.
 * The pages that define the method have no counterpart of this entry point.
 *
 *   rel, out, nrel, dtype, B, n, d, tau, causal, grad_scale, stream: as for
 *              lard_kl_bwd_multi_bf16.
 * Limit: lard_kl_bwd_bf16_workspace_bytes(rel, nrel, B, n, d) must not exceed
 * LARD_NOALLOC_WORKSPACE_BYTES (for example B * H * n * d summed over the
 * relations <= 16 Mi elements: 32 heads of n = 4096, d = 128); a larger
 * problem returns LARD_ERR_TOO_LARGE before anything is enqueued.
 * The call allocates nothing: it looks up the array's device address on the
 * first call on each GPU (so that first call should come before any stream
 * capture), clears the part it uses on `stream`, and accumulates there.
 * Every call on a GPU shares the one array, which keeps the last call's
 * contents: calls whose work can overlap on the GPU (on different streams
 * without ordering between them, or from several host threads) race on it
 * and give wrong gradients.  Order such calls, for example on one stream.
 */
#define LARD_NOALLOC_WORKSPACE_BYTES (64u << 20)
LARD_API lard_status lard_kl_bwd_multi_bf16_noalloc(const lard_relation* rel, const lard_grads_bf16* out,
                                           int nrel, lard_dtype dtype, int B, int n, int d, float tau,
                                           int causal, float grad_scale, cudaStream_t stream);

/* Human-readable name of a status code (static storage, never NULL). */
LARD_API const char* lard_status_string(lard_status s);

/*
 * Synchronises `stream`, then reads and clears the device-side fault word of
 * the GPU that `stream` belongs to (for the legacy default stream 0, the
 * current device).  Returns LARD_ERR_TIMEOUT if a kernel wait ran out of
 * time since the last check (and stores the fault bits in *fault_bits if it
 * is not NULL), LARD_ERR_CUDA if synchronisation failed, else LARD_OK.
 * Bits: 0x1-0x4 a Phase-1 role, 0x10-0x80 a Phase-2 role, 0x100 a block
 * that left before its own copies or tensor-core work had finished (its
 * exit wait ran out), 0x8000 the self-test below.
 */
LARD_API lard_status lard_device_status(cudaStream_t stream, unsigned int* fault_bits);

/*
 * Failure-detection self-test: enqueues one small kernel whose wait (an
 * mbarrier that nothing arrives at) runs out after `limit_us` microseconds
 * (1 .. 5e6) and sets its bit (0x8000) in the device fault word; an exit
 * wait on the same barrier then runs out after as long again and sets the
 * exit-wait bit (0x100).  The kernel returns normally, so that a following
 * lard_device_status() reports LARD_ERR_TIMEOUT with both bits while the
 * CUDA context stays usable.  The pages define no counterpart; this checks
 * the bounded waits every kernel of this library relies on.
 */
LARD_API lard_status lard_selftest_timeout(unsigned int limit_us, cudaStream_t stream);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
LARD_API int lard_version(void);

#ifdef __cplusplus
}
#endif

#endif /* LARD_H */
