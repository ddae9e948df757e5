// lard_kernel_common.cuh -- state shared by the kernels of liblard.
#pragma once

#include "sm100_ptx.cuh"

namespace lard {

// Device-side fault word, one per GPU that loads the library.  A kernel wait
// that runs out of time ORs its role's bit in; lard_device_status() reads and
// clears it.
__device__ unsigned int g_lard_fault;

constexpr unsigned int kFaultFwdProducer = 1u << 0;
constexpr unsigned int kFaultFwdMma = 1u << 1;
constexpr unsigned int kFaultFwdSoftmax = 1u << 2;
constexpr unsigned int kFaultBwdProducer = 1u << 4;
constexpr unsigned int kFaultBwdMma = 1u << 5;
constexpr unsigned int kFaultBwdSoftmax = 1u << 6;
constexpr unsigned int kFaultBwdEpilogue = 1u << 7;
constexpr unsigned int kFaultSelfTest = 1u << 15;

// Exercises the bounded wait: one thread waits, with a short limit, on an
// mbarrier that nothing arrives at; the wait runs out, raises the fault word
// and the kernel returns normally.
__global__ void lard_selftest_timeout_kernel(unsigned long long limit_ns) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        abort_flag = 0;
        ptx::mbar_init(&bar, 1);
        ptx::fence_mbar_init();
        ptx::mbar_wait(&bar, 0, &abort_flag, limit_ns, &g_lard_fault, kFaultSelfTest);
    }
}

}  // namespace lard
