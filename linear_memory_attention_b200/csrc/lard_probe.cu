// lard_probe.cu -- throughput probe of the exponential units the relation-KL
// kernels are bound by (declared in include/lard_probe.h).  Not part of the
// relation-KL computation: the benchmark calls it to measure the peak against
// which the Phase-1 kernel's exponential rate is reported, instead of
// assuming one.
#include <cstdint>

#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "lard_exp2.cuh"
#include "lard_probe.h"

namespace {

__device__ float g_probe_sink[1024];

__device__ __forceinline__ float ex2f(float x) {
    float y;
    asm volatile("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ uint32_t ex2h2(uint32_t x) {
    uint32_t y;
    asm volatile("ex2.approx.f16x2 %0, %1;" : "=r"(y) : "r"(x));
    return y;
}

// Each thread runs 8 independent chains x = -0.5 * 2^x (bounded in
// [-0.5, -0.35]); the multiply runs on the FMA pipe, which has 8x the MUFU
// unit's rate, so the exponentials set the pace.
__global__ void __launch_bounds__(256) probe_ex2_f32(int iters) {
    float a[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) a[k] = -0.25f - 0.01f * static_cast<float>((threadIdx.x + k) & 7);
    for (int it = 0; it < iters; ++it) {
#pragma unroll
        for (int k = 0; k < 8; ++k) a[k] = -0.5f * ex2f(a[k]);
    }
    float s = 0.f;
#pragma unroll
    for (int k = 0; k < 8; ++k) s += a[k];
    if (s == 1.0f) g_probe_sink[threadIdx.x & 1023] = s;  // never true; keeps the chains live
}

// The same with two half-precision exponentials per instruction.
__global__ void __launch_bounds__(256) probe_ex2_f16x2(int iters) {
    __half2 a[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) a[k] = __float2half2_rn(-0.25f - 0.01f * static_cast<float>((threadIdx.x + k) & 7));
    const __half2 m = __float2half2_rn(-0.5f);
    for (int it = 0; it < iters; ++it) {
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            uint32_t v = ex2h2(*reinterpret_cast<uint32_t*>(&a[k]));
            a[k] = __hmul2(*reinterpret_cast<__half2*>(&v), m);
        }
    }
    float s = 0.f;
#pragma unroll
    for (int k = 0; k < 8; ++k) s += __low2float(a[k]) + __high2float(a[k]);
    if (s == 1.0f) g_probe_sink[threadIdx.x & 1023] = s;
}

// The FMA-pipe exponential of the kernels (range reduction + degree-5
// polynomial on fp32 pairs), 8 independent pair chains per thread.
__global__ void __launch_bounds__(256) probe_exp2_fma2(int iters) {
    float2 a[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) a[k] = lard::splat2(-0.25f - 0.01f * static_cast<float>((threadIdx.x + k) & 7));
    for (int it = 0; it < iters; ++it) {
#pragma unroll
        for (int k = 0; k < 8; ++k) a[k] = lard::mul2(lard::exp2_fma2(a[k]), lard::splat2(-0.5f));
    }
    float s = 0.f;
#pragma unroll
    for (int k = 0; k < 8; ++k) s += a[k].x + a[k].y;
    if (s == 1.0f) g_probe_sink[threadIdx.x & 1023] = s;
}

// Two fp32 exponents packed to half precision, one ex2.approx.f16x2, and the
// two results widened back to fp32: the round trip a kernel keeping its sums
// in fp32 would pay for half-precision exponentials.
__global__ void __launch_bounds__(256) probe_ex2_f16x2_via_f32(int iters) {
    float a[8], b[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        a[k] = -0.25f - 0.01f * static_cast<float>((threadIdx.x + k) & 7);
        b[k] = a[k] - 0.125f;
    }
    for (int it = 0; it < iters; ++it) {
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            __half2 h = __floats2half2_rn(a[k], b[k]);
            uint32_t v = ex2h2(*reinterpret_cast<uint32_t*>(&h));
            const float2 e = __half22float2(*reinterpret_cast<__half2*>(&v));
            a[k] = -0.5f * e.x;
            b[k] = -0.5f * e.y;
        }
    }
    float s = 0.f;
#pragma unroll
    for (int k = 0; k < 8; ++k) s += a[k] + b[k];
    if (s == 1.0f) g_probe_sink[threadIdx.x & 1023] = s;
}

}  // namespace

extern "C" {

LARD_PROBE_API int lard_probe_exp_rate(int kind, int blocks, int iters, float* ms, double* exps, cudaStream_t stream) {
    if (!ms || !exps || blocks < 1 || iters < 1 || kind < 0 || kind > 3) return 1;
    cudaEvent_t a, b;
    if (cudaEventCreate(&a) != cudaSuccess) return 3;
    if (cudaEventCreate(&b) != cudaSuccess) {
        cudaEventDestroy(a);
        return 3;
    }
    cudaEventRecord(a, stream);
    if (kind == 0) probe_ex2_f32<<<blocks, 256, 0, stream>>>(iters);
    else if (kind == 1) probe_ex2_f16x2<<<blocks, 256, 0, stream>>>(iters);
    else if (kind == 2) probe_exp2_fma2<<<blocks, 256, 0, stream>>>(iters);
    else probe_ex2_f16x2_via_f32<<<blocks, 256, 0, stream>>>(iters);
    cudaEventRecord(b, stream);
    int rc = 0;
    if (cudaGetLastError() != cudaSuccess || cudaEventSynchronize(b) != cudaSuccess ||
        cudaEventElapsedTime(ms, a, b) != cudaSuccess)
        rc = 3;
    cudaEventDestroy(a);
    cudaEventDestroy(b);
    const double per_instr = (kind == 0) ? 1.0 : 2.0;  // f16x2 and pairs: two per chain step
    *exps = static_cast<double>(blocks) * 256.0 * iters * 8.0 * per_instr;
    return rc;
}

}  // extern "C"
