/*
 * lard_probe.h -- C ABI of liblard_probe: a throughput probe of the
 * exponential units, for sm_100a.
 *
 * The relation-KL kernels (lard.h) compute two exponentials per relation
 * logit in each phase; the special-function (MUFU) unit that evaluates them
 * is, with the tensor cores, what bounds them.  This probe measures the
 * exponential rate a B200 sustains, so that a benchmark reports the kernels
 * against a measured peak.  The pages that define the method have no
 * counterpart; it is a measuring instrument, not part of the computation.
 */
#ifndef LARD_PROBE_H
#define LARD_PROBE_H

#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define LARD_PROBE_API __attribute__((visibility("default")))
#else
#define LARD_PROBE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/*
 * Runs one probe kernel on the current device, on `stream`, and waits for it.
 *   kind    0: ex2.approx.ftz.f32 (one exponential per instruction);
 *           1: ex2.approx.f16x2 (two half-precision exponentials per instruction);
 *           2: the FMA-pipe exp2 of the kernels (range reduction and a degree-5
 *              polynomial on packed fp32 pairs);
 *           3: kind 1 between fp32 values (two fp32 packed to half precision,
 *              one ex2.approx.f16x2, the results widened back to fp32).
 *   blocks  grid size (256 threads per block), >= 1.
 *   iters   chain steps per thread (8 independent chains per thread), >= 1.
 *   ms      out: elapsed time of the kernel (CUDA events on `stream`).
 *   exps    out: exponentials computed.
 * Returns 0 on success, 1 for a bad argument, 3 if a CUDA call failed.
 * Allocates no device memory.
 */
LARD_PROBE_API int lard_probe_exp_rate(int kind, int blocks, int iters, float* ms, double* exps,
                                       cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* LARD_PROBE_H */
