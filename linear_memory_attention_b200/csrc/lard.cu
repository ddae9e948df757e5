// lard.cu -- the C ABI of liblard (declared in include/lard.h): argument
// checks, per-device setup, TMA tensor maps and kernel launches.  Every step
// of the relation-KL computation runs in the kernels of the included headers.
#include <cuda.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include <climits>
#include <cmath>
#include <cstdint>
#include <mutex>

#include "lard.h"
#include "lard_kernel_common.cuh"
#include "lard_bwd_tc.cuh"
#include "lard_cast.cuh"
#include "lard_fp32.cuh"
#include "lard_fwd_tc.cuh"

namespace {

constexpr int kVersion = 200;                          // 0.2.0
constexpr unsigned long long kWaitLimitNs = 2000000000ull;   // 2 s per wait
constexpr unsigned long long kDrainLimitNs = 8000000000ull;  // 8 s per drain on the way out
constexpr int kMaxDevices = 64;
constexpr long long kMaxElems = 1LL << 40;

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// Workspace of lard_kl_bwd_multi_bf16_noalloc, for callers that cannot
// allocate device memory: a file-scope device array, present on every GPU
// that loads the library, shared by every call of that entry point on that
// GPU.  Host code reaches it only through the device address that
// cudaGetSymbolAddress returns (g_static_ws_ptr, set once per device).
constexpr size_t kStaticWorkspaceBytes = size_t(64) << 20;  // 64 MiB
static_assert(kStaticWorkspaceBytes == LARD_NOALLOC_WORKSPACE_BYTES, "workspace size differs from the header");
static __device__ __align__(256) unsigned char g_lard_static_ws[kStaticWorkspaceBytes];

std::mutex g_mu;
bool g_ready[kMaxDevices];
void* g_static_ws_ptr[kMaxDevices];
lard_status g_dev_status[kMaxDevices];
EncodeTiledFn g_encode = nullptr;

// Restores the caller's current device when a call returns.
struct DeviceGuard {
    int prev = -1;
    DeviceGuard() {
        if (cudaGetDevice(&prev) != cudaSuccess) {
            prev = -1;
            cudaGetLastError();
        }
    }
    ~DeviceGuard() {
        if (prev >= 0) cudaSetDevice(prev);
    }
};

// NVTX range over one call (a profiler that records NVTX shows each phase's
// enqueue, and correlates the kernels it launched; without one it costs nothing).
struct NvtxRange {
    explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
};

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool overlap(const void* a, size_t na, const void* b, size_t nb) {
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x < y + nb && y < x + na;
}

bool d_supported(lard_dtype dt, int d) {
    if (dt == LARD_DTYPE_BF16) return d == 64 || d == 128;
    return d >= 32 && d <= 256 && d % 32 == 0;
}

template <typename K>
cudaError_t set_smem(K kernel, int bytes) {
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

// The warp-specialised kernels move registers between warpgroups with
// setmaxnreg; that only terminates if the block's launch allocation covers
// every warpgroup's share.  Checks the built kernel's register count.
template <typename K>
bool split_fits(K kernel, int threads, int split_total) {
    cudaFuncAttributes a;
    if (cudaFuncGetAttributes(&a, kernel) != cudaSuccess) return false;
    const int per_thread = (a.numRegs + 7) / 8 * 8;
    return per_thread * threads >= split_total;
}

// One-time setup of device `dev` (made current by the caller).
lard_status setup_device(int dev) {
    std::lock_guard<std::mutex> lk(g_mu);
    if (dev < 0 || dev >= kMaxDevices) return LARD_ERR_UNSUPPORTED;
    if (g_ready[dev]) return g_dev_status[dev];
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
        return LARD_ERR_CUDA;
    lard_status st = LARD_OK;
    if (major != 10 || minor != 0) st = LARD_ERR_UNSUPPORTED;  // built for sm_100a only
    if (st == LARD_OK && !g_encode) {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault,
                                             &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess || !fn)
            st = LARD_ERR_CUDA;
        else
            g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    }
    if (st == LARD_OK) {
        bool ok = set_smem(lard::lard_fwd_tc_kernel<64>, lard::FwdLayout<64>::SMEM_BYTES) == cudaSuccess &&
                  set_smem(lard::lard_fwd_tc_kernel<128>, lard::FwdLayout<128>::SMEM_BYTES) == cudaSuccess &&
                  set_smem(lard::lard_bwd_tc_kernel<64>, lard::BwdLayout<64>::SMEM_BYTES) == cudaSuccess &&
                  set_smem(lard::lard_bwd_tc_kernel<128>, lard::BwdLayout<128>::SMEM_BYTES) == cudaSuccess;
        if (!ok) st = LARD_ERR_CUDA;
    }
    if (st == LARD_OK) {
        const bool fits = split_fits(lard::lard_fwd_tc_kernel<64>, lard::kFwdThreads, lard::kFwdRegsSplitTotal) &&
                          split_fits(lard::lard_fwd_tc_kernel<128>, lard::kFwdThreads, lard::kFwdRegsSplitTotal) &&
                          split_fits(lard::lard_bwd_tc_kernel<64>, 512, lard::kBwdRegsSplitTotal) &&
                          split_fits(lard::lard_bwd_tc_kernel<128>, 512, lard::kBwdRegsSplitTotal);
        if (!fits) st = LARD_ERR_UNSUPPORTED;  // a build whose register count cannot host the split
    }
    g_dev_status[dev] = st;
    g_ready[dev] = true;
    return st;
}

// Finds the GPU that holds `ptr`, makes it current and sets it up.
lard_status select_device(const void* ptr) {
    cudaPointerAttributes at;
    if (cudaPointerGetAttributes(&at, ptr) != cudaSuccess) {
        cudaGetLastError();
        return LARD_ERR_INVALID_ARG;
    }
    if (at.type != cudaMemoryTypeDevice && at.type != cudaMemoryTypeManaged) return LARD_ERR_INVALID_ARG;
    if (cudaSetDevice(at.device) != cudaSuccess) return LARD_ERR_CUDA;
    return setup_device(at.device);
}

// 3-D tensor map over [BH, n, d] bf16 with 64 x 128 boxes, 128-byte swizzle.
// Rows past n read as zeros.
bool make_map(CUtensorMap* m, const void* base, long long BH, int n, int d) {
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(n),
                          static_cast<cuuint64_t>(BH)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(n) * d * 2};
    cuuint32_t box[3] = {64, 128, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
                    estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D tensor map over the fp32 gradient [BH, n, d] with 32 x 32 boxes
// (128-byte rows), 128-byte swizzle, for the TMA reduce-adds of Phase 2.
bool make_grad_map(CUtensorMap* m, void* base, long long BH, int n, int d) {
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(n),
                          static_cast<cuuint64_t>(BH)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 4, static_cast<cuuint64_t>(n) * d * 4};
    cuuint32_t box[3] = {32, 32, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return g_encode(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, base, dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Checks shared by both phases.
lard_status check_common(const void* Xt, const void* Yt, const void* Xs, const void* Ys, lard_dtype dtype,
                         int B, int H, int n, int d, float tau, int causal, long long* BH_out) {
    if (!Xt || !Yt || !Xs || !Ys) return LARD_ERR_INVALID_ARG;
    if (B < 1 || H < 1 || n < 1 || d < 1) return LARD_ERR_INVALID_ARG;
    if (n > INT_MAX - 127) return LARD_ERR_INVALID_ARG;  // row and tile indices stay in int
    if (!(std::isfinite(tau) && tau > 0.f)) return LARD_ERR_INVALID_ARG;
    if (causal != 0 && causal != 1) return LARD_ERR_INVALID_ARG;
    if (dtype != LARD_DTYPE_BF16 && dtype != LARD_DTYPE_FP32) return LARD_ERR_UNSUPPORTED;
    if (!d_supported(dtype, d)) return LARD_ERR_UNSUPPORTED;
    const long long BH = static_cast<long long>(B) * H;
    if (BH > INT_MAX / 2 || BH * n > kMaxElems / d) return LARD_ERR_INVALID_ARG;
    const long long T = (static_cast<long long>(n) + 127) / 128;
    if (BH * T > INT_MAX) return LARD_ERR_INVALID_ARG;
    for (const void* p : {Xt, Yt, Xs, Ys})
        if (!aligned(p, 16)) return LARD_ERR_INVALID_ARG;
    *BH_out = BH;
    return LARD_OK;
}

size_t in_bytes(lard_dtype dt, long long BH, int n, int d) {
    return static_cast<size_t>(BH) * n * d * (dt == LARD_DTYPE_BF16 ? 2 : 4);
}

template <int E>
void launch_fwd_fp32(const float* Xt, const float* Yt, const float* Xs, const float* Ys,
                     const lard::Fp32Params& p, float* lse_t, float* lse_s, float* row_kl, cudaStream_t s) {
    const long long warps = static_cast<long long>(p.BH) * p.n;
    const unsigned blocks = static_cast<unsigned>((warps + 7) / 8);
    lard::lard_fwd_fp32_kernel<E><<<blocks, 256, 0, s>>>(Xt, Yt, Xs, Ys, p, lse_t, lse_s, row_kl);
}

template <int E>
void launch_bwd_fp32(const float* Xt, const float* Yt, const float* Xs, const float* Ys,
                     const lard::Fp32Params& p, const float* lse_t, const float* lse_s, float* dXs,
                     float* dYs, cudaStream_t s) {
    const long long warps = static_cast<long long>(p.BH) * p.n;
    const unsigned blocks = static_cast<unsigned>((warps + 7) / 8);
    lard::lard_bwd_rownorm_fp32_kernel<E><<<blocks, 256, 0, s>>>(Xt, Yt, Xs, Ys, p, lse_t, lse_s, dXs);
    lard::lard_bwd_dy_fp32_kernel<E><<<blocks, 256, 0, s>>>(Xt, Yt, Xs, Ys, p, lse_t, lse_s, dXs, dYs);
    lard::lard_bwd_dx_fp32_kernel<E><<<blocks, 256, 0, s>>>(Xt, Yt, Xs, Ys, p, lse_t, lse_s, dXs);
}

#define LARD_DISPATCH_E(d, F, ...)                   \
    switch ((d) / 32) {                              \
        case 1: F<1>(__VA_ARGS__); break;            \
        case 2: F<2>(__VA_ARGS__); break;            \
        case 3: F<3>(__VA_ARGS__); break;            \
        case 4: F<4>(__VA_ARGS__); break;            \
        case 5: F<5>(__VA_ARGS__); break;            \
        case 6: F<6>(__VA_ARGS__); break;            \
        case 7: F<7>(__VA_ARGS__); break;            \
        default: F<8>(__VA_ARGS__); break;           \
    }

}  // namespace

namespace {

// Byte ranges of one call's buffers: outputs may overlap nothing else.
struct Ranges {
    const void* p[64];
    size_t n[64];
    bool out[64];
    int k = 0;
    void add(const void* ptr, size_t bytes, bool is_out) {
        if (!ptr || k >= 64) return;
        p[k] = ptr;
        n[k] = bytes;
        out[k] = is_out;
        ++k;
    }
    bool outputs_disjoint() const {
        for (int a = 0; a < k; ++a)
            for (int b = a + 1; b < k; ++b)
                if ((out[a] || out[b]) && overlap(p[a], n[a], p[b], n[b])) return false;
        return true;
    }
};

// Makes the GPU of the first relation current (and set up); every other
// buffer of the call (`extra`, then each relation's fields) must be device or
// managed memory on it.
lard_status select_call_device(const lard_relation* rel, int nrel, const void* extra,
                               const lard_grads_bf16* out16 = nullptr) {
    lard_status st = select_device(rel[0].Xt);
    if (st != LARD_OK) return st;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return LARD_ERR_CUDA;
    auto on_dev = [&](const void* q) {
        if (!q) return true;
        cudaPointerAttributes at;
        if (cudaPointerGetAttributes(&at, q) != cudaSuccess) {
            cudaGetLastError();
            return false;
        }
        return (at.type == cudaMemoryTypeDevice || at.type == cudaMemoryTypeManaged) && at.device == dev;
    };
    if (!on_dev(extra)) return LARD_ERR_INVALID_ARG;
    for (int r = 0; r < nrel; ++r) {
        const lard_relation& R = rel[r];
        for (const void* q : {R.Xt, R.Yt, R.Xs, R.Ys, (const void*)R.lse_t, (const void*)R.lse_s,
                              (const void*)R.row_kl, (const void*)R.loss_bh, (const void*)R.dXs,
                              (const void*)R.dYs})
            if (!on_dev(q)) return LARD_ERR_INVALID_ARG;
        if (out16 && (!on_dev(out16[r].dXs) || !on_dev(out16[r].dYs))) return LARD_ERR_INVALID_ARG;
    }
    return LARD_OK;
}

// Σ over relations of B * H * n * d * 4 bytes: the fp32 dX_s accumulators of a
// Phase-2 call with bf16 outputs (0 for an invalid description).
size_t bf16_workspace_bytes(const lard_relation* rel, int nrel, int B, int n, int d) {
    if (!rel || nrel < 1 || nrel > lard::kMaxRelations || B < 1 || n < 1 || d < 1) return 0;
    size_t total = 0;
    for (int r = 0; r < nrel; ++r) {
        if (rel[r].H < 1) return 0;
        total += static_cast<size_t>(B) * rel[r].H * n * d * 4;
    }
    return total;
}

lard_status kl_fwd(const lard_relation* rel, int nrel, lard_dtype dtype, int B, int n, int d, float tau,
                   int causal, float* loss_total, cudaStream_t stream) {
    NvtxRange range("lard Phase 1 (LSE, row KL, losses)");
    if (!rel || nrel < 1 || nrel > lard::kMaxRelations) return LARD_ERR_INVALID_ARG;
    long long BH[lard::kMaxRelations];
    Ranges rg;
    for (int r = 0; r < nrel; ++r) {
        const lard_relation& R = rel[r];
        lard_status st = check_common(R.Xt, R.Yt, R.Xs, R.Ys, dtype, B, R.H, n, d, tau, causal, &BH[r]);
        if (st != LARD_OK) return st;
        if (!R.lse_t || !R.lse_s || !R.row_kl) return LARD_ERR_INVALID_ARG;
        if (loss_total && !R.loss_bh) return LARD_ERR_INVALID_ARG;
        for (const void* q : {(const void*)R.lse_t, (const void*)R.lse_s, (const void*)R.row_kl,
                              (const void*)R.loss_bh})
            if (q && !aligned(q, 4)) return LARD_ERR_INVALID_ARG;
        const size_t nin = in_bytes(dtype, BH[r], n, d), nrow = static_cast<size_t>(BH[r]) * n * 4;
        for (const void* in : {R.Xt, R.Yt, R.Xs, R.Ys}) rg.add(in, nin, false);
        rg.add(R.lse_t, nrow, true);
        rg.add(R.lse_s, nrow, true);
        rg.add(R.row_kl, nrow, true);
        rg.add(R.loss_bh, static_cast<size_t>(BH[r]) * 4, true);
    }
    if (loss_total && !aligned(loss_total, 4)) return LARD_ERR_INVALID_ARG;
    rg.add(loss_total, 4, true);
    if (!rg.outputs_disjoint()) return LARD_ERR_INVALID_ARG;

    DeviceGuard guard;
    lard_status st = select_call_device(rel, nrel, loss_total);
    if (st != LARD_OK) return st;

    const int T = (n + 127) / 128;
    if (dtype == LARD_DTYPE_BF16) {
        lard::TcFwdGroup g;
        long long blocks = 0;
        for (int r = 0; r < nrel; ++r) {
            if (!make_map(&g.yt[r], rel[r].Yt, BH[r], n, d) || !make_map(&g.ys[r], rel[r].Ys, BH[r], n, d))
                return LARD_ERR_INVALID_ARG;
            g.rel[r].Xt = static_cast<const __nv_bfloat16*>(rel[r].Xt);
            g.rel[r].Xs = static_cast<const __nv_bfloat16*>(rel[r].Xs);
            g.rel[r].lse_t = rel[r].lse_t;
            g.rel[r].lse_s = rel[r].lse_s;
            g.rel[r].row_kl = rel[r].row_kl;
            g.rel[r].block0 = static_cast<int>(blocks);
            blocks += BH[r] * T;
        }
        if (blocks > INT_MAX) return LARD_ERR_INVALID_ARG;
        g.nrel = nrel;
        g.n = n;
        g.T = T;
        g.causal = causal;
        g.tau = tau;
        g.cfac = static_cast<float>(static_cast<double>(tau) * 1.4426950408889634);
        g.wait_ns = kWaitLimitNs;
        g.drain_ns = kDrainLimitNs;
        const unsigned grid = static_cast<unsigned>(blocks);
        if (d == 128)
            lard::lard_fwd_tc_kernel<128><<<grid, lard::kFwdThreads, lard::FwdLayout<128>::SMEM_BYTES, stream>>>(g);
        else
            lard::lard_fwd_tc_kernel<64><<<grid, lard::kFwdThreads, lard::FwdLayout<64>::SMEM_BYTES, stream>>>(g);
    } else {
        for (int r = 0; r < nrel; ++r) {
            lard::Fp32Params p;
            p.BH = static_cast<int>(BH[r]);
            p.n = n;
            p.causal = causal;
            p.tau = tau;
            p.dz_scale = 0.0;
            LARD_DISPATCH_E(d, launch_fwd_fp32, static_cast<const float*>(rel[r].Xt),
                            static_cast<const float*>(rel[r].Yt), static_cast<const float*>(rel[r].Xs),
                            static_cast<const float*>(rel[r].Ys), p, rel[r].lse_t, rel[r].lse_s, rel[r].row_kl,
                            stream);
        }
    }
    // Per-head losses of every relation that asked for them, in one launch.
    lard::LossRowsSet rows;
    long long row_blocks = 0;
    int k = 0;
    for (int r = 0; r < nrel; ++r) {
        if (!rel[r].loss_bh) continue;
        rows.row_kl[k] = rel[r].row_kl;
        rows.loss_bh[k] = rel[r].loss_bh;
        rows.block0[k] = static_cast<int>(row_blocks);
        row_blocks += BH[r];
        ++k;
    }
    rows.nrel = k;
    rows.n = n;
    if (k > 0) lard::lard_loss_rows_kernel<<<static_cast<unsigned>(row_blocks), 256, 0, stream>>>(rows);
    if (loss_total) {
        lard::LossSet ls;
        for (int r = 0; r < nrel; ++r) {
            ls.loss_bh[r] = rel[r].loss_bh;
            ls.BH[r] = static_cast<int>(BH[r]);
        }
        ls.nrel = nrel;
        lard::lard_loss_total_kernel<<<1, 256, 0, stream>>>(ls, loss_total);
    }
    return cudaGetLastError() == cudaSuccess ? LARD_OK : LARD_ERR_CUDA;
}

// bf16 gradient outputs of a Phase-2 call: where they go and the fp32
// workspace that accumulates dX_s (and, fused, dY_s) before the rounding.
struct Bf16Grads {
    const lard_grads_bf16* out;
    void* ws;
    size_t ws_bytes;
};

lard_status kl_bwd(const lard_relation* rel, int nrel, lard_dtype dtype, int B, int n, int d, float tau,
                   int causal, float grad_scale, cudaStream_t stream, const Bf16Grads* b16 = nullptr) {
    NvtxRange range(b16 ? "lard Phase 2 (gradients, bf16 outputs)" : "lard Phase 2 (gradients)");
    if (!rel || nrel < 1 || nrel > lard::kMaxRelations) return LARD_ERR_INVALID_ARG;
    if (!std::isfinite(grad_scale)) return LARD_ERR_INVALID_ARG;
    if (b16 && !b16->out) return LARD_ERR_INVALID_ARG;
    long long BH[lard::kMaxRelations];
    Ranges rg;
    bool fused_any = false;
    size_t ws_need = 0;
    for (int r = 0; r < nrel; ++r) {
        const lard_relation& R = rel[r];
        lard_status st = check_common(R.Xt, R.Yt, R.Xs, R.Ys, dtype, B, R.H, n, d, tau, causal, &BH[r]);
        if (st != LARD_OK) return st;
        if (!R.lse_t || !R.lse_s) return LARD_ERR_INVALID_ARG;
        // The gradient buffers: fp32 in the relation, or bf16 in b16->out.
        const void* gx = b16 ? b16->out[r].dXs : static_cast<const void*>(R.dXs);
        const void* gy = b16 ? b16->out[r].dYs : static_cast<const void*>(R.dYs);
        if (b16 && (R.dXs || R.dYs)) return LARD_ERR_INVALID_ARG;  // outputs are given once
        if (!gx) return LARD_ERR_INVALID_ARG;
        const bool fuse = gy == nullptr;
        if (fuse && (R.Yt != R.Xt || R.Ys != R.Xs)) return LARD_ERR_INVALID_ARG;
        fused_any = fused_any || fuse;
        if (!aligned(R.lse_t, 4) || !aligned(R.lse_s, 4) || !aligned(gx, 16) || (!fuse && !aligned(gy, 16)))
            return LARD_ERR_INVALID_ARG;
        const size_t nin = in_bytes(dtype, BH[r], n, d);
        const size_t ngrad = static_cast<size_t>(BH[r]) * n * d * (b16 ? 2 : 4);
        const size_t nrow = static_cast<size_t>(BH[r]) * n * 4;
        for (const void* in : {R.Xt, R.Yt, R.Xs, R.Ys}) rg.add(in, nin, false);
        rg.add(R.lse_t, nrow, false);
        rg.add(R.lse_s, nrow, false);
        rg.add(gx, ngrad, true);
        rg.add(gy, ngrad, true);
        ws_need += static_cast<size_t>(BH[r]) * n * d * 4;
    }
    if (b16) {
        if (!b16->ws || !aligned(b16->ws, 16) || b16->ws_bytes < ws_need) return LARD_ERR_INVALID_ARG;
        rg.add(b16->ws, ws_need, true);
    }
    if (!rg.outputs_disjoint()) return LARD_ERR_INVALID_ARG;
    // The fp32 path parks per-row corrections in the dXs rows while it builds
    // dYs, so it has no place to add dYs into dXs; and it is the full-precision
    // path, which bf16 outputs would defeat.
    if ((fused_any || b16) && dtype != LARD_DTYPE_BF16) return LARD_ERR_UNSUPPORTED;

    DeviceGuard guard;
    lard_status st = select_call_device(rel, nrel, b16 ? b16->ws : nullptr, b16 ? b16->out : nullptr);
    if (st != LARD_OK) return st;

    const int T = (n + 127) / 128;
    const double dz_scale = static_cast<double>(tau) * grad_scale / n;
    if (dtype == LARD_DTYPE_BF16) {
        lard::TcBwdGroup g;
        lard::CastSet cast;
        long long blocks = 0;
        float* acc[lard::kMaxRelations];  // fp32 dX_s accumulator of each relation
        size_t ws_off = 0;
        cast.start8[0] = 0;
        for (int r = 0; r < nrel; ++r) {
            const lard_relation& R = rel[r];
            const size_t elems = static_cast<size_t>(BH[r]) * n * d;
            acc[r] = b16 ? reinterpret_cast<float*>(static_cast<char*>(b16->ws) + ws_off) : R.dXs;
            ws_off += elems * 4;
            if (!make_map(&g.xt[r], R.Xt, BH[r], n, d) || !make_map(&g.yt[r], R.Yt, BH[r], n, d) ||
                !make_map(&g.xs[r], R.Xs, BH[r], n, d) || !make_map(&g.ys[r], R.Ys, BH[r], n, d) ||
                !make_grad_map(&g.dx[r], acc[r], BH[r], n, d))
                return LARD_ERR_INVALID_ARG;
            g.rel[r].lse_t = R.lse_t;
            g.rel[r].lse_s = R.lse_s;
            g.rel[r].dYs = b16 ? nullptr : R.dYs;
            g.rel[r].dYs_bf16 = b16 ? static_cast<__nv_bfloat16*>(b16->out[r].dYs) : nullptr;
            g.rel[r].fuse_dy = (b16 ? b16->out[r].dYs : static_cast<void*>(R.dYs)) == nullptr;
            g.rel[r].block0 = static_cast<int>(blocks);
            blocks += BH[r] * T;
            if (b16) {
                cast.src[r] = acc[r];
                cast.dst[r] = static_cast<__nv_bfloat16*>(b16->out[r].dXs);
                cast.start8[r + 1] = cast.start8[r] + static_cast<long long>(elems / 8);
            }
        }
        if (blocks > INT_MAX) return LARD_ERR_INVALID_ARG;
        for (int r = 0; r < nrel; ++r)
            if (cudaMemsetAsync(acc[r], 0, static_cast<size_t>(BH[r]) * n * d * 4, stream) != cudaSuccess)
                return LARD_ERR_CUDA;
        g.nrel = nrel;
        g.n = n;
        g.T = T;
        g.causal = causal;
        g.cfac = static_cast<float>(static_cast<double>(tau) * 1.4426950408889634);
        g.dz_scale = static_cast<float>(dz_scale);
        g.wait_ns = kWaitLimitNs;
        g.drain_ns = kDrainLimitNs;
        const unsigned grid = static_cast<unsigned>(blocks);
        if (d == 128)
            lard::lard_bwd_tc_kernel<128><<<grid, 512, lard::BwdLayout<128>::SMEM_BYTES, stream>>>(g);
        else
            lard::lard_bwd_tc_kernel<64><<<grid, 512, lard::BwdLayout<64>::SMEM_BYTES, stream>>>(g);
        if (b16) {
            cast.nrel = nrel;
            int dev = 0, sms = 148;
            if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
            const long long groups = cast.start8[nrel];
            const long long want = (groups + 255) / 256;
            const unsigned cgrid = static_cast<unsigned>(want < 8LL * sms ? (want > 0 ? want : 1) : 8LL * sms);
            lard::lard_cast_bf16_kernel<<<cgrid, 256, 0, stream>>>(cast);
        }
    } else {
        for (int r = 0; r < nrel; ++r) {
            lard::Fp32Params p;
            p.BH = static_cast<int>(BH[r]);
            p.n = n;
            p.causal = causal;
            p.tau = tau;
            p.dz_scale = dz_scale;
            LARD_DISPATCH_E(d, launch_bwd_fp32, static_cast<const float*>(rel[r].Xt),
                            static_cast<const float*>(rel[r].Yt), static_cast<const float*>(rel[r].Xs),
                            static_cast<const float*>(rel[r].Ys), p, rel[r].lse_t, rel[r].lse_s, rel[r].dXs,
                            rel[r].dYs, stream);
        }
    }
    return cudaGetLastError() == cudaSuccess ? LARD_OK : LARD_ERR_CUDA;
}

lard_relation one_relation(const void* Xt, const void* Yt, const void* Xs, const void* Ys, int H) {
    lard_relation R;
    R.Xt = Xt;
    R.Yt = Yt;
    R.Xs = Xs;
    R.Ys = Ys;
    R.H = H;
    R.lse_t = R.lse_s = R.row_kl = R.loss_bh = R.dXs = R.dYs = nullptr;
    return R;
}

}  // namespace

extern "C" {

lard_status lard_kl_fwd(const void* Xt, const void* Yt, const void* Xs, const void* Ys, lard_dtype dtype,
                        int B, int H, int n, int d, float tau, int causal, float* lse_t, float* lse_s,
                        float* row_kl, float* loss_bh, float* loss_total, cudaStream_t stream) {
    lard_relation R = one_relation(Xt, Yt, Xs, Ys, H);
    R.lse_t = lse_t;
    R.lse_s = lse_s;
    R.row_kl = row_kl;
    R.loss_bh = loss_bh;
    return kl_fwd(&R, 1, dtype, B, n, d, tau, causal, loss_total, stream);
}

lard_status lard_kl_bwd(const void* Xt, const void* Yt, const void* Xs, const void* Ys, lard_dtype dtype,
                        int B, int H, int n, int d, float tau, int causal, const float* lse_t,
                        const float* lse_s, float grad_scale, float* dXs, float* dYs, cudaStream_t stream) {
    if (!dYs) return LARD_ERR_INVALID_ARG;
    lard_relation R = one_relation(Xt, Yt, Xs, Ys, H);
    R.lse_t = const_cast<float*>(lse_t);
    R.lse_s = const_cast<float*>(lse_s);
    R.dXs = dXs;
    R.dYs = dYs;
    return kl_bwd(&R, 1, dtype, B, n, d, tau, causal, grad_scale, stream);
}

lard_status lard_kl_bwd_self(const void* Xt, const void* Xs, lard_dtype dtype, int B, int H, int n, int d,
                             float tau, int causal, const float* lse_t, const float* lse_s, float grad_scale,
                             float* dXs, cudaStream_t stream) {
    lard_relation R = one_relation(Xt, Xt, Xs, Xs, H);
    R.lse_t = const_cast<float*>(lse_t);
    R.lse_s = const_cast<float*>(lse_s);
    R.dXs = dXs;
    return kl_bwd(&R, 1, dtype, B, n, d, tau, causal, grad_scale, stream);
}

lard_status lard_kl_fwd_multi(const lard_relation* rel, int nrel, lard_dtype dtype, int B, int n, int d,
                              float tau, int causal, float* loss_total, cudaStream_t stream) {
    return kl_fwd(rel, nrel, dtype, B, n, d, tau, causal, loss_total, stream);
}

lard_status lard_kl_bwd_multi(const lard_relation* rel, int nrel, lard_dtype dtype, int B, int n, int d,
                              float tau, int causal, float grad_scale, cudaStream_t stream) {
    return kl_bwd(rel, nrel, dtype, B, n, d, tau, causal, grad_scale, stream);
}

size_t lard_kl_bwd_bf16_workspace_bytes(const lard_relation* rel, int nrel, int B, int n, int d) {
    return bf16_workspace_bytes(rel, nrel, B, n, d);
}

lard_status lard_kl_bwd_multi_bf16_noalloc(const lard_relation* rel, const lard_grads_bf16* out, int nrel,
                                           lard_dtype dtype, int B, int n, int d, float tau, int causal,
                                           float grad_scale, cudaStream_t stream) {
    if (!rel || !out || nrel < 1 || nrel > lard::kMaxRelations || !rel[0].Xt) return LARD_ERR_INVALID_ARG;
    const size_t need = bf16_workspace_bytes(rel, nrel, B, n, d);
    if (need == 0) return LARD_ERR_INVALID_ARG;
    if (need > kStaticWorkspaceBytes) return LARD_ERR_TOO_LARGE;
    // The device address of this GPU's copy of the array, looked up once per
    // device with that device current.
    DeviceGuard guard;
    lard_status st = select_device(rel[0].Xt);
    if (st != LARD_OK) return st;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return LARD_ERR_CUDA;
    void* ws = nullptr;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        if (!g_static_ws_ptr[dev]) {
            void* p = nullptr;
            if (cudaGetSymbolAddress(&p, g_lard_static_ws) != cudaSuccess || !p) {
                cudaGetLastError();
                return LARD_ERR_CUDA;
            }
            g_static_ws_ptr[dev] = p;
        }
        ws = g_static_ws_ptr[dev];
    }
    const Bf16Grads b16{out, ws, kStaticWorkspaceBytes};
    return kl_bwd(rel, nrel, dtype, B, n, d, tau, causal, grad_scale, stream, &b16);
}

lard_status lard_kl_bwd_multi_bf16(const lard_relation* rel, const lard_grads_bf16* out, int nrel,
                                   lard_dtype dtype, int B, int n, int d, float tau, int causal,
                                   float grad_scale, void* workspace, size_t workspace_bytes,
                                   cudaStream_t stream) {
    if (!out) return LARD_ERR_INVALID_ARG;
    const Bf16Grads b16{out, workspace, workspace_bytes};
    return kl_bwd(rel, nrel, dtype, B, n, d, tau, causal, grad_scale, stream, &b16);
}

const char* lard_status_string(lard_status s) {
    switch (s) {
        case LARD_OK: return "LARD_OK";
        case LARD_ERR_INVALID_ARG: return "LARD_ERR_INVALID_ARG";
        case LARD_ERR_UNSUPPORTED: return "LARD_ERR_UNSUPPORTED";
        case LARD_ERR_CUDA: return "LARD_ERR_CUDA";
        case LARD_ERR_TIMEOUT: return "LARD_ERR_TIMEOUT";
        case LARD_ERR_TOO_LARGE: return "LARD_ERR_TOO_LARGE";
    }
    return "LARD_ERR_UNKNOWN";
}

lard_status lard_device_status(cudaStream_t stream, unsigned int* fault_bits) {
    if (cudaStreamSynchronize(stream) != cudaSuccess) return LARD_ERR_CUDA;
    // The fault word to read is the one on the stream's GPU, which need not be
    // the current device.
    int dev = 0;
    if (cudaStreamGetDevice(stream, &dev) != cudaSuccess) return LARD_ERR_CUDA;
    DeviceGuard guard;
    if (cudaSetDevice(dev) != cudaSuccess) return LARD_ERR_CUDA;
    unsigned int v = 0;
    if (cudaMemcpyFromSymbol(&v, lard::g_lard_fault, sizeof(v)) != cudaSuccess) return LARD_ERR_CUDA;
    if (fault_bits) *fault_bits = v;
    if (v) {
        const unsigned int zero = 0;
        if (cudaMemcpyToSymbol(lard::g_lard_fault, &zero, sizeof(zero)) != cudaSuccess) return LARD_ERR_CUDA;
        return LARD_ERR_TIMEOUT;
    }
    return LARD_OK;
}

lard_status lard_selftest_timeout(unsigned int limit_us, cudaStream_t stream) {
    if (limit_us == 0 || limit_us > 5000000u) return LARD_ERR_INVALID_ARG;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return LARD_ERR_CUDA;
    lard_status st = setup_device(dev);
    if (st != LARD_OK) return st;
    lard::lard_selftest_timeout_kernel<<<1, 32, 0, stream>>>(1000ull * limit_us);
    return cudaGetLastError() == cudaSuccess ? LARD_OK : LARD_ERR_CUDA;
}

int lard_version(void) { return kVersion; }

}  // extern "C"
