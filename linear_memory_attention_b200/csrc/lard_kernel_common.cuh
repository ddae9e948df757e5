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

}  // namespace lard
