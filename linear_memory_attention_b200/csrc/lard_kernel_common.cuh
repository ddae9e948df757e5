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
constexpr unsigned int kFaultDrain = 1u << 8;  // a block exited before its own copies or MMAs finished
constexpr unsigned int kFaultSelfTest = 1u << 15;

// Wait on the way out for copies and MMAs this block started (ptx::mbar_drain,
// which ignores the abort flag).  A drain that runs out of time means the
// block may leave while the hardware still writes its shared memory or TMEM,
// so it is reported on its own bit.
__device__ __forceinline__ void drain(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
    if (!ptx::mbar_drain(bar, parity, limit_ns)) atomicOr(&g_lard_fault, kFaultDrain);
}

// Relations (X/Y pairs of equal n and d, any head counts) that one launch of a
// tensor-core kernel may cover; their blocks are laid out one relation after
// the other in the grid.
constexpr int kMaxRelations = 4;

// Relation of a grid block: the last r whose first block is <= blockIdx.x.
template <typename Rel>
__device__ __forceinline__ int relation_of_block(const Rel (&rel)[kMaxRelations], int nrel) {
    int r = 0;
#pragma unroll
    for (int k = 1; k < kMaxRelations; ++k)
        if (k < nrel && static_cast<int>(blockIdx.x) >= rel[k].block0) r = k;
    return r;
}

// Exercises the bounded waits: one thread waits, with a short limit, on an
// mbarrier that nothing arrives at; the wait runs out and raises its bit in
// the fault word.  Then the exit wait of a block (drain) runs out on the same
// barrier and raises the drain bit, and the kernel returns normally.
__global__ void lard_selftest_timeout_kernel(unsigned long long limit_ns) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        abort_flag = 0;
        ptx::mbar_init(&bar, 1);
        ptx::fence_mbar_init();
        ptx::mbar_wait(&bar, 0, &abort_flag, limit_ns, &g_lard_fault, kFaultSelfTest);
        drain(&bar, 0, limit_ns);
    }
}

}  // namespace lard
