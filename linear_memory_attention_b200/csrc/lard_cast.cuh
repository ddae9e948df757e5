// lard_cast.cuh -- the last step of Phase 2 with bf16 gradient outputs: the
// gradients are accumulated in fp32 (dX_s by reduce-adds in L2, across the
// column blocks that contribute to a row) and rounded to bf16 once, here,
// round-to-nearest-even.
#pragma once

#include <cuda_bf16.h>

#include "lard_kernel_common.cuh"

namespace lard {

// The fp32 accumulators of the relations of one call and their bf16 outputs.
// Each relation's element count is a multiple of 8 (d is).
struct CastSet {
    const float* src[kMaxRelations];
    __nv_bfloat16* dst[kMaxRelations];
    long long start8[kMaxRelations + 1];  // prefix sums of (elements / 8); start8[nrel] = total
    int nrel;
};

// Grid-stride over 8-element groups: two 16-byte fp32 loads, one 16-byte bf16
// store per group.  The loads bypass L1 and are marked as last use.
__global__ void __launch_bounds__(256) lard_cast_bf16_kernel(const __grid_constant__ CastSet s) {
    const long long total = s.start8[s.nrel];
    for (long long q = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; q < total;
         q += static_cast<long long>(gridDim.x) * blockDim.x) {
        int r = 0;
#pragma unroll
        for (int k = 1; k < kMaxRelations; ++k)
            if (k < s.nrel && q >= s.start8[k]) r = k;
        const long long g = q - s.start8[r];
        const float4* src = reinterpret_cast<const float4*>(s.src[r]) + 2 * g;
        const float4 a = __ldcs(src), b = __ldcs(src + 1);
        uint4 o;
        o.x = ptx::pack_bf16x2(a.x, a.y);
        o.y = ptx::pack_bf16x2(a.z, a.w);
        o.z = ptx::pack_bf16x2(b.x, b.y);
        o.w = ptx::pack_bf16x2(b.z, b.w);
        reinterpret_cast<uint4*>(s.dst[r])[g] = o;
    }
}

}  // namespace lard
