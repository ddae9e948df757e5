// lard_fp32.cuh -- the fp32-input path (CUDA cores, fp64 arithmetic).
//
// Same two phases as the tensor-core path (LinearARD notes, 关键设计 3), for
// inputs given in fp32.  The bf16 tensor cores would round the inputs and
// tf32 keeps too few mantissa bits, so this path runs on the CUDA cores.  It
// forms logits, statistics, probabilities and dZ in fp64: dZ = R_s - R_t
// cancels when student and teacher agree, and fp32 logits would lose the
// relative accuracy this path is for.  Outputs are rounded to fp32 once.
// One warp owns one row (Phase 1, dX) or one column (dY); its 32 lanes split
// the head dimension and a shuffle reduction forms each logit.  Nothing is
// accumulated with atomics, so results are deterministic.
#pragma once

#include "lard_kernel_common.cuh"

namespace lard {

struct Fp32Params {
    int BH, n, causal;
    double tau;
    double dz_scale;  // tau * grad_scale / n
};

__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Phase 1: online LSE of both relations and the row KL, one warp per row.
template <int E>  // head dim = 32 * E
__global__ void __launch_bounds__(256) lard_fwd_fp32_kernel(const float* __restrict__ Xt,
                                                            const float* __restrict__ Yt,
                                                            const float* __restrict__ Xs,
                                                            const float* __restrict__ Ys,
                                                            const Fp32Params p, float* lse_t,
                                                            float* lse_s, float* row_kl) {
    constexpr int D = 32 * E;
    const long long gw = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (gw >= static_cast<long long>(p.BH) * p.n) return;
    const int bh = static_cast<int>(gw / p.n);
    const int i = static_cast<int>(gw % p.n);
    const size_t head = static_cast<size_t>(bh) * p.n * D;
    double xt[E], xs[E];
#pragma unroll
    for (int e = 0; e < E; ++e) {
        xt[e] = Xt[head + static_cast<size_t>(i) * D + lane + 32 * e];
        xs[e] = Xs[head + static_cast<size_t>(i) * D + lane + 32 * e];
    }
    double m_t = -INFINITY, l_t = 0.0, m_s = -INFINITY, l_s = 0.0, a = 0.0;
    const int jend = p.causal ? i + 1 : p.n;
    for (int j = 0; j < jend; ++j) {
        double dt = 0.0, ds = 0.0;
#pragma unroll
        for (int e = 0; e < E; ++e) {
            dt = fma(xt[e], static_cast<double>(Yt[head + static_cast<size_t>(j) * D + lane + 32 * e]), dt);
            ds = fma(xs[e], static_cast<double>(Ys[head + static_cast<size_t>(j) * D + lane + 32 * e]), ds);
        }
        const double zt = p.tau * warp_sum(dt);
        const double zs = p.tau * warp_sum(ds);
        if (zt > m_t) {
            const double sc = exp(m_t - zt);
            l_t = l_t * sc + 1.0;
            a = a * sc + (zt - zs);
            m_t = zt;
        } else {
            const double pt = exp(zt - m_t);
            l_t += pt;
            a = fma(pt, zt - zs, a);
        }
        if (zs > m_s) {
            l_s = l_s * exp(m_s - zs) + 1.0;
            m_s = zs;
        } else {
            l_s += exp(zs - m_s);
        }
    }
    if (lane == 0) {
        const size_t o = static_cast<size_t>(bh) * p.n + i;
        lse_t[o] = static_cast<float>(m_t + log(l_t));
        lse_s[o] = static_cast<float>(m_s + log(l_s));
        row_kl[o] = static_cast<float>(a / l_t - (m_t - m_s) - log(l_t / l_s));
    }
}

// Phase 2 reads the fp32 LSEs of the API, whose rounding (up to half an ulp,
// about 5e-7 at LSE ~ 10) would scale every R of a row by e^{+-5e-7}; the
// cancellation in R_s - R_t can amplify that past the fp32 path's accuracy
// target.  So each row's normaliser is made exact again in fp64:
//   pass 1 (rows)    c_m(i) = log sum_j exp(z_m(i,j) - LSE_m(i)), parked in
//                    the first 16 bytes of the caller's dX_s row i;
//   pass 2 (columns) dY_s[j] = dz_scale * sum_i (R_s - R_t)(i,j) X_s[i] with
//                    R_m = exp(z_m - LSE_m - c_m);
//   pass 3 (rows)    dX_s[i] = dz_scale * (sum_j r_s y_j / sum_j r_s
//                    - sum_j r_t y_j / sum_j r_t), normalised in the same
//                    pass, overwriting the parked values.

// Pass 1: exact row-normaliser corrections, one warp per row.
template <int E>
__global__ void __launch_bounds__(256) lard_bwd_rownorm_fp32_kernel(
    const float* __restrict__ Xt, const float* __restrict__ Yt, const float* __restrict__ Xs,
    const float* __restrict__ Ys, const Fp32Params p, const float* __restrict__ lse_t,
    const float* __restrict__ lse_s, float* dXs) {
    constexpr int D = 32 * E;
    const long long gw = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (gw >= static_cast<long long>(p.BH) * p.n) return;
    const int bh = static_cast<int>(gw / p.n);
    const int i = static_cast<int>(gw % p.n);
    const size_t head = static_cast<size_t>(bh) * p.n * D;
    double xt[E], xs[E];
#pragma unroll
    for (int e = 0; e < E; ++e) {
        xt[e] = Xt[head + static_cast<size_t>(i) * D + lane + 32 * e];
        xs[e] = Xs[head + static_cast<size_t>(i) * D + lane + 32 * e];
    }
    const double bt = lse_t[static_cast<size_t>(bh) * p.n + i];
    const double bs = lse_s[static_cast<size_t>(bh) * p.n + i];
    double st = 0.0, ss = 0.0;
    const int jend = p.causal ? i + 1 : p.n;
    for (int j = 0; j < jend; ++j) {
        double dt = 0.0, ds = 0.0;
#pragma unroll
        for (int e = 0; e < E; ++e) {
            dt = fma(xt[e], static_cast<double>(Yt[head + static_cast<size_t>(j) * D + lane + 32 * e]), dt);
            ds = fma(xs[e], static_cast<double>(Ys[head + static_cast<size_t>(j) * D + lane + 32 * e]), ds);
        }
        st += exp(p.tau * warp_sum(dt) - bt);
        ss += exp(p.tau * warp_sum(ds) - bs);
    }
    if (lane == 0) {
        double* park = reinterpret_cast<double*>(dXs + head + static_cast<size_t>(i) * D);
        park[0] = log(st);
        park[1] = log(ss);
    }
}

// Pass 3: dX_s with the row normalised in the same pass, one warp per row.
template <int E>
__global__ void __launch_bounds__(256) lard_bwd_dx_fp32_kernel(
    const float* __restrict__ Xt, const float* __restrict__ Yt, const float* __restrict__ Xs,
    const float* __restrict__ Ys, const Fp32Params p, const float* __restrict__ lse_t,
    const float* __restrict__ lse_s, float* dXs) {
    constexpr int D = 32 * E;
    const long long gw = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (gw >= static_cast<long long>(p.BH) * p.n) return;
    const int bh = static_cast<int>(gw / p.n);
    const int i = static_cast<int>(gw % p.n);
    const size_t head = static_cast<size_t>(bh) * p.n * D;
    double xt[E], xs[E], at[E], as[E];
#pragma unroll
    for (int e = 0; e < E; ++e) {
        xt[e] = Xt[head + static_cast<size_t>(i) * D + lane + 32 * e];
        xs[e] = Xs[head + static_cast<size_t>(i) * D + lane + 32 * e];
        at[e] = 0.0;
        as[e] = 0.0;
    }
    const double bt = lse_t[static_cast<size_t>(bh) * p.n + i];
    const double bs = lse_s[static_cast<size_t>(bh) * p.n + i];
    double st = 0.0, ss = 0.0;
    const int jend = p.causal ? i + 1 : p.n;
    for (int j = 0; j < jend; ++j) {
        double dt = 0.0, ds = 0.0, ys[E];
#pragma unroll
        for (int e = 0; e < E; ++e) {
            ys[e] = Ys[head + static_cast<size_t>(j) * D + lane + 32 * e];
            dt = fma(xt[e], static_cast<double>(Yt[head + static_cast<size_t>(j) * D + lane + 32 * e]), dt);
            ds = fma(xs[e], ys[e], ds);
        }
        const double rt = exp(p.tau * warp_sum(dt) - bt);
        const double rs = exp(p.tau * warp_sum(ds) - bs);
        st += rt;
        ss += rs;
#pragma unroll
        for (int e = 0; e < E; ++e) {
            at[e] = fma(rt, ys[e], at[e]);
            as[e] = fma(rs, ys[e], as[e]);
        }
    }
    const double ist = 1.0 / st, iss = 1.0 / ss;
#pragma unroll
    for (int e = 0; e < E; ++e)
        dXs[head + static_cast<size_t>(i) * D + lane + 32 * e] =
            static_cast<float>(p.dz_scale * (as[e] * iss - at[e] * ist));
}

// Pass 2: dY_s, one warp per column, with the parked row corrections.
template <int E>
__global__ void __launch_bounds__(256) lard_bwd_dy_fp32_kernel(
    const float* __restrict__ Xt, const float* __restrict__ Yt, const float* __restrict__ Xs,
    const float* __restrict__ Ys, const Fp32Params p, const float* __restrict__ lse_t,
    const float* __restrict__ lse_s, const float* __restrict__ parked, float* dYs) {
    constexpr int D = 32 * E;
    const long long gw = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (gw >= static_cast<long long>(p.BH) * p.n) return;
    const int bh = static_cast<int>(gw / p.n);
    const int j = static_cast<int>(gw % p.n);
    const size_t head = static_cast<size_t>(bh) * p.n * D;
    double yt[E], ys[E], acc[E];
#pragma unroll
    for (int e = 0; e < E; ++e) {
        yt[e] = Yt[head + static_cast<size_t>(j) * D + lane + 32 * e];
        ys[e] = Ys[head + static_cast<size_t>(j) * D + lane + 32 * e];
        acc[e] = 0.0;
    }
    const int ibeg = p.causal ? j : 0;
    for (int i = ibeg; i < p.n; ++i) {
        double dt = 0.0, ds = 0.0, xs[E];
#pragma unroll
        for (int e = 0; e < E; ++e) {
            xs[e] = Xs[head + static_cast<size_t>(i) * D + lane + 32 * e];
            dt = fma(static_cast<double>(Xt[head + static_cast<size_t>(i) * D + lane + 32 * e]), yt[e], dt);
            ds = fma(xs[e], ys[e], ds);
        }
        const double* c = reinterpret_cast<const double*>(parked + head + static_cast<size_t>(i) * D);
        const size_t o = static_cast<size_t>(bh) * p.n + i;
        const double rt = exp(p.tau * warp_sum(dt) - static_cast<double>(lse_t[o]) - c[0]);
        const double rs = exp(p.tau * warp_sum(ds) - static_cast<double>(lse_s[o]) - c[1]);
        const double dz = (rs - rt) * p.dz_scale;
#pragma unroll
        for (int e = 0; e < E; ++e) acc[e] = fma(dz, xs[e], acc[e]);
    }
#pragma unroll
    for (int e = 0; e < E; ++e) dYs[head + static_cast<size_t>(j) * D + lane + 32 * e] = static_cast<float>(acc[e]);
}

// Per-row KL arrays of the relations of one call, one grid block per (relation,
// batch, head), relations one after the other.
struct LossRowsSet {
    const float* row_kl[kMaxRelations];
    float* loss_bh[kMaxRelations];
    int block0[kMaxRelations];  // first block of each relation
    int nrel, n;
};

// loss_bh[bh] = (1/n) sum_i row_kl[bh, i] (LinearARD notes, 关键设计 1: the
// row-averaged KL), summed in fp64.
__global__ void __launch_bounds__(256) lard_loss_rows_kernel(const __grid_constant__ LossRowsSet s) {
    int r = 0;
#pragma unroll
    for (int k = 1; k < kMaxRelations; ++k)
        if (k < s.nrel && static_cast<int>(blockIdx.x) >= s.block0[k]) r = k;
    const int bh = static_cast<int>(blockIdx.x) - s.block0[r];
    const float* row_kl = s.row_kl[r];
    const int n = s.n;
    double acc = 0.0;
    for (int i = threadIdx.x; i < n; i += blockDim.x) acc += row_kl[static_cast<size_t>(bh) * n + i];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    __shared__ double part[8];
    if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = acc;
    __syncthreads();
    if (threadIdx.x == 0) {
        double t = 0.0;
        for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) t += part[w];
        s.loss_bh[r][bh] = static_cast<float>(t / n);
    }
}

// Per-head losses of the relations of one call.
struct LossSet {
    const float* loss_bh[kMaxRelations];
    int BH[kMaxRelations];
    int nrel;
};

// loss_total = sum over relations and (batch, head) of loss_bh (the relations'
// losses add with weight 1, LinearARD notes, 损失函数), summed in fp64.
__global__ void __launch_bounds__(256) lard_loss_total_kernel(const __grid_constant__ LossSet s, float* loss_total) {
    double acc = 0.0;
    for (int r = 0; r < s.nrel; ++r)
        for (int b = threadIdx.x; b < s.BH[r]; b += blockDim.x) acc += s.loss_bh[r][b];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    __shared__ double part[8];
    if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = acc;
    __syncthreads();
    if (threadIdx.x == 0) {
        double t = 0.0;
        for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) t += part[w];
        *loss_total = static_cast<float>(t);
    }
}

}  // namespace lard
