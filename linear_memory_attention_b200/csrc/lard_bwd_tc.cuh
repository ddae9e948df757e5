// lard_bwd_tc.cuh -- Phase 2 on the 5th-generation tensor cores (bf16 inputs).
//
// LinearARD notes (papernotes.org), 关键设计 3, second phase: per T_r x T_c =
// 128 x 128 tile, recompute the student and teacher logits on chip, rebuild
// R = exp(Z - LSE) from the Phase-1 statistics, form dZ = (R_s - R_t)/n and
// contract it with the projections into dX_s and dY_s.  Fully masked tiles
// (J > I) are never visited.
//
// One CTA owns a 128-column block J of one (batch, head) of one relation (a
// launch covers up to kMaxRelations relations, TcBwdGroup); its dY_s[J]
// accumulator stays in TMEM for the whole sweep over the row blocks I >= J
// (all I without the mask).  Each tile's dX_s[I] contribution is staged in
// shared memory and added to HBM with TMA bulk reduce-adds (fp32 adds in L2,
// whole 128-byte lines, rows past n clipped by the tensor map).  For a fused
// self-relation the finished dY_s[J] is added into the same buffer the same
// way; otherwise it is stored to dY_s, in fp32 or rounded once to bf16.  With
// bf16 gradient outputs the dX_s reduce-adds go to a caller-provided fp32
// workspace, which lard_cast_bf16_kernel rounds to bf16 after this kernel.
// The kernel is bound by shared-memory bandwidth: per tile the four SS GEMMs
// read 256 KB of operands, and TMA writes, dZ stores and the dX staging add
// another 224 KB; the GEMMs share the SM's shared-memory bandwidth with them.
// TMEM (512 columns): dY [0, D), S_t [128, 256), S_s [256, 384), dX [384, 384 + D).
// Shared memory: Y_t[J], Y_s[J] resident; a 2-stage ring for X_s[I]; one
// buffer for X_t[I] (only the first GEMM of a tile reads it, so the next one
// has a whole tile of softmax work to land); one 128 x 128 bf16 dZ tile,
// 128B-swizzled, read by both gradient GEMMs:
//   GEMM 3  dY[J] += dZ^T X_s[I]   (A = dZ as MN-major, B = X_s as MN-major)
//   GEMM 4  dX[I]  = dZ  Y_s[J]    (A = dZ as K-major,  B = Y_s as MN-major)
// and 2 x 4 KB of dX staging per drain warp.
// Roles (512 threads):
//   warp 0       TMA producer          warp 1   TMEM owner, MMA issuer
//   warps 4-11   dZ: one row per thread, one 64-column half per warpgroup
//   warps 12-15  dX drain (TMEM -> smem -> TMA reduce-add), final dY store or add
#pragma once

#include "lard_exp2.cuh"
#include "lard_kernel_common.cuh"

namespace lard {

// One relation of a launch.
struct TcBwdRel {
    const float* lse_t;
    const float* lse_s;
    float* dYs;               // fp32 dY_s output, or
    __nv_bfloat16* dYs_bf16;  // bf16 dY_s output (rounded once from the TMEM accumulator)
    int fuse_dy;  // 1: add dY_s into the dX_s accumulator (self-relation total gradient), no dY_s output
    int block0;   // first grid block of this relation (its B*H*T blocks follow)
};

// A launch: up to kMaxRelations relations of equal n and d in one grid.
struct TcBwdGroup {
    CUtensorMap xt[kMaxRelations], yt[kMaxRelations], xs[kMaxRelations], ys[kMaxRelations];
    CUtensorMap dx[kMaxRelations];  // fp32 dX_s accumulator (the output, or a workspace), for the reduce-adds
    TcBwdRel rel[kMaxRelations];
    int nrel, n, T, causal;
    float cfac;      // tau * log2(e)
    float dz_scale;  // tau * grad_scale / n: dZ and the chain-rule tau in one factor
    unsigned long long wait_ns;   // limit of each wait inside the loops
    unsigned long long drain_ns;  // limit of each drain on the way out (longer)
};

template <int D>
struct BwdLayout {
    static constexpr int KC = D / 64;
    static constexpr int TILE = KC * 16384;
    static constexpr int OFF_YT = 0;
    static constexpr int OFF_YS = TILE;
    static constexpr int OFF_XS = 2 * TILE;  // 2 stages
    static constexpr int OFF_XT = 4 * TILE;  // 1 stage
    static constexpr int OFF_DZ = 5 * TILE;
    static constexpr int OFF_STG = OFF_DZ + 32768;  // 4 drain warps x 2 x 4 KB
    static constexpr int OFF_CTRL = OFF_STG + 32768;
    static constexpr int CTRL_BYTES = 1024;
    static constexpr int SMEM_BYTES = OFF_CTRL + CTRL_BYTES + 1024;
};

struct BwdCtrl {
    uint64_t y_full;
    uint64_t xs_full[2];
    uint64_t xs_empty[2];
    uint64_t xt_full, xt_empty;
    uint64_t s_full, s_free, dz_full, dz_free, dx_full, dx_free, dy_full, mma_done;
    uint32_t tmem_base;
    int abort_flag;
};
static_assert(sizeof(BwdCtrl) <= 1024, "control block too large");

constexpr uint32_t kTmemDY = 0, kTmemSt = 128, kTmemSs = 256, kTmemDX = 384;

// Register split (per thread): launched at 128; the control warpgroup and the
// drain warpgroup give registers to the two dZ warpgroups.  The shares must
// not add up to more than the launch allocation, or setmaxnreg.inc would wait
// for ever; the host checks the built kernel's register count against
// kBwdRegsSplitTotal before the first launch.
constexpr int kBwdRegsLaunch = 128, kBwdRegsCtl = 72, kBwdRegsDz = 184, kBwdRegsDrain = 64;
constexpr int kBwdRegsSplitTotal = 128 * (kBwdRegsCtl + kBwdRegsDrain + 2 * kBwdRegsDz);
static_assert(kBwdRegsSplitTotal <= 512 * kBwdRegsLaunch, "register split exceeds the launch allocation");

template <int D>
__global__ void __launch_bounds__(512, 1)
    lard_bwd_tc_kernel(const __grid_constant__ TcBwdGroup g) {
    using L = BwdLayout<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (ptx::smem_u32(smem_raw) & 1023u)) & 1023u);
    BwdCtrl* ctrl = reinterpret_cast<BwdCtrl*>(smem + L::OFF_CTRL);
    volatile int* abort_flag = &ctrl->abort_flag;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    // This block's relation; then head-major order within it, longest column
    // blocks first within a head: the blocks resident at any time share one
    // head's X tiles and dX rows in L2.
    const int rel = relation_of_block(g.rel, g.nrel);
    const CUtensorMap* tm_xt = &g.xt[rel];
    const CUtensorMap* tm_yt = &g.yt[rel];
    const CUtensorMap* tm_xs = &g.xs[rel];
    const CUtensorMap* tm_ys = &g.ys[rel];
    const CUtensorMap* tm_dx = &g.dx[rel];
    const struct {
        int n, T, causal;
        float cfac, dz_scale;
        const float *lse_t, *lse_s;
        float* dYs;
        __nv_bfloat16* dYs_bf16;
        int fuse_dy;
        unsigned long long wait_ns, drain_ns;
    } p = {g.n, g.T, g.causal, g.cfac, g.dz_scale, g.rel[rel].lse_t, g.rel[rel].lse_s, g.rel[rel].dYs,
           g.rel[rel].dYs_bf16, g.rel[rel].fuse_dy, g.wait_ns, g.drain_ns};
    const int local = static_cast<int>(blockIdx.x) - g.rel[rel].block0;
    const int bh = local / p.T;
    const int J = local % p.T;
    const int K = p.causal ? (p.T - J) : p.T;
    auto row_block = [&](int k) { return p.causal ? (J + k) : k; };

    if (threadIdx.x == 0) {
        ptx::mbar_init(&ctrl->y_full, 1);
        for (int s = 0; s < 2; ++s) {
            ptx::mbar_init(&ctrl->xs_full[s], 1);
            ptx::mbar_init(&ctrl->xs_empty[s], 1);
        }
        ptx::mbar_init(&ctrl->xt_full, 1);
        ptx::mbar_init(&ctrl->xt_empty, 1);
        ptx::mbar_init(&ctrl->s_full, 1);
        ptx::mbar_init(&ctrl->s_free, 8);
        ptx::mbar_init(&ctrl->dz_full, 8);
        ptx::mbar_init(&ctrl->dz_free, 1);
        ptx::mbar_init(&ctrl->dx_full, 1);
        ptx::mbar_init(&ctrl->dx_free, 4);
        ptx::mbar_init(&ctrl->dy_full, 1);
        ptx::mbar_init(&ctrl->mma_done, 1);
        ctrl->abort_flag = 0;
        ptx::fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        ptx::prefetch_tensormap(tm_xt);
        ptx::prefetch_tensormap(tm_yt);
        ptx::prefetch_tensormap(tm_xs);
        ptx::prefetch_tensormap(tm_ys);
        ptx::prefetch_tensormap(tm_dx);
    }
    if (warp == 1) {
        ptx::tmem_alloc(&ctrl->tmem_base, 512);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = ctrl->tmem_base;
    const uint64_t lim = p.wait_ns, dlim = p.drain_ns;
    if (warp < 4) {
      ptx::regs_dec<kBwdRegsCtl>();
      if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            ptx::mbar_arrive_expect_tx(&ctrl->y_full, 2 * L::TILE);
            for (int c = 0; c < L::KC; ++c) {
                ptx::tma_load_3d(smem + L::OFF_YT + c * 16384, tm_yt, &ctrl->y_full, c * 64, J * 128, bh);
                ptx::tma_load_3d(smem + L::OFF_YS + c * 16384, tm_ys, &ctrl->y_full, c * 64, J * 128, bh);
            }
        }
        __syncwarp();
        int issued_t = 0, issued_s = 0;
        for (int k = 0; k < K; ++k) {
            const int I = row_block(k);
            // X_t(k) may land once S_t(k-1) has been computed ...
            bool ok = ptx::mbar_wait(&ctrl->xt_empty, (k & 1) ^ 1, abort_flag, lim, &g_lard_fault,
                                     kFaultBwdProducer);
            if (!__all_sync(0xffffffffu, ok)) break;
            if (lane == 0) {
                ptx::mbar_arrive_expect_tx(&ctrl->xt_full, L::TILE);
                for (int c = 0; c < L::KC; ++c)
                    ptx::tma_load_3d(smem + L::OFF_XT + c * 16384, tm_xt, &ctrl->xt_full, c * 64, I * 128, bh);
            }
            __syncwarp();
            ++issued_t;
            // ... and X_s(k) once GEMM 3 of tile k-2 has released its stage.
            const int s = k & 1;
            ok = ptx::mbar_wait(&ctrl->xs_empty[s], ((k >> 1) & 1) ^ 1, abort_flag, lim, &g_lard_fault,
                                kFaultBwdProducer);
            if (!__all_sync(0xffffffffu, ok)) break;
            if (lane == 0) {
                ptx::mbar_arrive_expect_tx(&ctrl->xs_full[s], L::TILE);
                for (int c = 0; c < L::KC; ++c)
                    ptx::tma_load_3d(smem + L::OFF_XS + s * L::TILE + c * 16384, tm_xs, &ctrl->xs_full[s],
                                     c * 64, I * 128, bh);
            }
            __syncwarp();
            ++issued_s;
        }
        // Let every copy this warp started land before the block can exit.
        drain(&ctrl->y_full, 0, dlim);
        if (issued_t > 0) drain(&ctrl->xt_full, (issued_t - 1) & 1, dlim);
        for (int s = 0; s < 2 && s < issued_s; ++s) {
            const int last = s + 2 * ((issued_s - 1 - s) / 2);
            drain(&ctrl->xs_full[s], (last >> 1) & 1, dlim);
        }
      } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        constexpr uint32_t kIdescS = ptx::idesc_bf16(128, 128, 0, 0);
        constexpr uint32_t kIdescDY = ptx::idesc_bf16(128, D, 1, 1);
        constexpr uint32_t kIdescDX = ptx::idesc_bf16(128, D, 0, 1);
        constexpr uint32_t kHi = ptx::sdesc_hi(1024);
        // Descriptor low words, fixed for the CTA's life: K-major (leading offset
        // 16 B) for the logit GEMMs and dZ as GEMM 4's A; MN-major (leading offset
        // = one 64-column chunk) for dZ^T, X_s and Y_s in the gradient GEMMs.
        const uint32_t yt_k = ptx::sdesc_lo(ptx::smem_u32(smem + L::OFF_YT), 16);
        const uint32_t ys_k = ptx::sdesc_lo(ptx::smem_u32(smem + L::OFF_YS), 16);
        const uint32_t ys_mn = ptx::sdesc_lo(ptx::smem_u32(smem + L::OFF_YS), 16384);
        const uint32_t xt_k = ptx::sdesc_lo(ptx::smem_u32(smem + L::OFF_XT), 16);
        const uint32_t xs_k0 = ptx::sdesc_lo(ptx::smem_u32(smem + L::OFF_XS), 16);
        const uint32_t xs_mn0 = ptx::sdesc_lo(ptx::smem_u32(smem + L::OFF_XS), 16384);
        const uint32_t dz_k = ptx::sdesc_lo(ptx::smem_u32(smem + L::OFF_DZ), 16);
        const uint32_t dz_mn = ptx::sdesc_lo(ptx::smem_u32(smem + L::OFF_DZ), 16384);
        constexpr uint32_t kStage = L::TILE >> 4;  // one X_s stage, in descriptor units
        const uint32_t t_ss = tmem + kTmemSs, t_st = tmem + kTmemSt, t_dy = tmem + kTmemDY, t_dx = tmem + kTmemDX;
        auto issue_ss = [&](int k) {
            const uint32_t a = xs_k0 + (k & 1) * kStage;
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                if (kk == 0) ptx::umma_ss<0>(t_ss, a, ys_k, kHi, kIdescS);
                else ptx::umma_ss<1>(t_ss, a + ptx::desc_step_k(kk), ys_k + ptx::desc_step_k(kk), kHi, kIdescS);
            }
        };
        auto issue_st = [&]() {
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                if (kk == 0) ptx::umma_ss<0>(t_st, xt_k, yt_k, kHi, kIdescS);
                else ptx::umma_ss<1>(t_st, xt_k + ptx::desc_step_k(kk), yt_k + ptx::desc_step_k(kk), kHi, kIdescS);
            }
            ptx::umma_commit(&ctrl->xt_empty);
            ptx::umma_commit(&ctrl->s_full);
        };
        // S(k) for k = 0: S_s first (X_s(0) is loaded before X_t(0) is needed).
        bool ok = ptx::mbar_wait(&ctrl->y_full, 0, abort_flag, lim, &g_lard_fault, kFaultBwdMma) &&
                  ptx::mbar_wait(&ctrl->xs_full[0], 0, abort_flag, lim, &g_lard_fault, kFaultBwdMma) &&
                  ptx::mbar_wait(&ctrl->xt_full, 0, abort_flag, lim, &g_lard_fault, kFaultBwdMma);
        ok = __all_sync(0xffffffffu, ok);
        if (ok) {
            ptx::tc_fence_after();
            if (lane == 0) {
                issue_ss(0);
                issue_st();
            }
            __syncwarp();
        }
        for (int k = 0; ok && k < K; ++k) {
            if (k + 1 < K) {
                // S(k+1) as soon as the dZ warps have read S(k) out of TMEM.
                ok = ptx::mbar_wait(&ctrl->xs_full[(k + 1) & 1], ((k + 1) >> 1) & 1, abort_flag, lim,
                                    &g_lard_fault, kFaultBwdMma) &&
                     ptx::mbar_wait(&ctrl->s_free, k & 1, abort_flag, lim, &g_lard_fault, kFaultBwdMma);
                if (!__all_sync(0xffffffffu, ok)) break;
                ptx::tc_fence_after();
                if (lane == 0) issue_ss(k + 1);
                __syncwarp();
                ok = ptx::mbar_wait(&ctrl->xt_full, (k + 1) & 1, abort_flag, lim, &g_lard_fault, kFaultBwdMma);
                if (!__all_sync(0xffffffffu, ok)) break;
                ptx::tc_fence_after();
                if (lane == 0) issue_st();
                __syncwarp();
            }
            ok = ptx::mbar_wait(&ctrl->dz_full, k & 1, abort_flag, lim, &g_lard_fault, kFaultBwdMma) &&
                 ptx::mbar_wait(&ctrl->dx_free, (k & 1) ^ 1, abort_flag, lim, &g_lard_fault, kFaultBwdMma);
            if (!__all_sync(0xffffffffu, ok)) break;
            ptx::tc_fence_after();
            if (lane == 0) {
                const uint32_t b3 = xs_mn0 + (k & 1) * kStage;
                // GEMM 3: dY[J] (+)= dZ^T X_s[I]; K runs over the 128 rows i, 16 per step.
                ptx::umma_ss_acc(t_dy, dz_mn, b3, kHi, kIdescDY, k > 0 ? 1u : 0u);
#pragma unroll
                for (int kk = 1; kk < 8; ++kk)
                    ptx::umma_ss<1>(t_dy, dz_mn + ptx::desc_step_mn(kk), b3 + ptx::desc_step_mn(kk), kHi, kIdescDY);
                // GEMM 4: dX[I] = dZ Y_s[J]; K runs over the 128 columns j.
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    if (kk == 0) ptx::umma_ss<0>(t_dx, dz_k, ys_mn, kHi, kIdescDX);
                    else ptx::umma_ss<1>(t_dx, dz_k + ptx::desc_step_k(kk), ys_mn + ptx::desc_step_mn(kk), kHi, kIdescDX);
                }
                ptx::umma_commit(&ctrl->dz_free);
                ptx::umma_commit(&ctrl->xs_empty[k & 1]);
                ptx::umma_commit(&ctrl->dx_full);
            }
            __syncwarp();
        }
        if (lane == 0) {
            if (ok) ptx::umma_commit(&ctrl->dy_full);
            ptx::umma_commit(&ctrl->mma_done);
        }
        __syncwarp();
        drain(&ctrl->mma_done, 0, dlim);
      }
    } else if (warp < 12) {
        ptx::regs_inc<kBwdRegsDz>();
        // ------------------------------------------------------------ dZ
        const int q = warp & 3;
        const int hcol = (warp - 4) >> 2;
        const int r = q * 32 + lane;
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(q * 32) << 16);
        const uint32_t sdz_row = ptx::smem_u32(smem + L::OFF_DZ) + hcol * 16384 + r * 128;
        const float cf = p.cfac;
        const float dzs = p.dz_scale;
        const float kLog2e = 1.4426950408889634f;
        // The row's LSEs for tile k are loaded one tile ahead, off the critical path.
        auto load_lse = [&](int k, float& t, float& s) {
            const int i = row_block(k) * 128 + r;
            const size_t o = static_cast<size_t>(bh) * p.n + (i < p.n ? i : 0);
            t = p.lse_t[o];
            s = p.lse_s[o];
        };
        float nlt = 0.f, nls = 0.f;
        load_lse(0, nlt, nls);
        for (int k = 0; k < K; ++k) {
            const int I = row_block(k);
            const int i = I * 128 + r;
            const bool row_ok = i < p.n;
            const float bt = row_ok ? nlt * kLog2e : 0.f;
            const float bs = row_ok ? nls * kLog2e : 0.f;
            if (k + 1 < K) load_lse(k + 1, nlt, nls);
            int jlim = 128;  // columns [0, jlim) of this tile are allowed for row i
            if (!row_ok) jlim = 0;
            else if (p.causal) { if (I == J) jlim = r + 1; }
            else if (J == p.T - 1) jlim = p.n - J * 128;

            const float2 cf2 = splat2(cf), nbt2 = splat2(-bt), nbs2 = splat2(-bs), dzs2 = splat2(dzs);
            bool ok = ptx::mbar_wait(&ctrl->s_full, k & 1, abort_flag, lim, &g_lard_fault, kFaultBwdSoftmax);
            if (!__all_sync(0xffffffffu, ok)) break;
            ptx::tc_fence_after();
            // Read this thread's 64 columns of S_t and S_s at once and hand the
            // TMEM back, so that S(k+1) can be computed under this tile's math.
            float st0[32], ss0[32], st1[32], ss1[32];
            __syncwarp();
            ptx::tmem_ld32(lane_base + kTmemSt + hcol * 64, st0);
            ptx::tmem_ld32(lane_base + kTmemSs + hcol * 64, ss0);
            ptx::tmem_ld32(lane_base + kTmemSt + hcol * 64 + 32, st1);
            ptx::tmem_ld32(lane_base + kTmemSs + hcol * 64 + 32, ss1);
            ptx::tmem_ld_wait(st0);
            ptx::reg_dep(ss0);
            ptx::reg_dep(st1);
            ptx::reg_dep(ss1);
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&ctrl->s_free);
#pragma unroll
            for (int round = 0; round < 2; ++round) {
                const int cb = hcol * 64 + round * 32;
                const float* st = round ? st1 : st0;
                const float* ss = round ? ss1 : ss0;
                uint32_t pk[16];
                const bool masked = cb + 32 > jlim;  // only diagonal and tail tiles
#pragma unroll
                for (int c = 0; c < 32; c += 2) {
                    const float2 ut = fma2(make_float2(st[c], st[c + 1]), cf2, nbt2);
                    const float2 us = fma2(make_float2(ss[c], ss[c + 1]), cf2, nbs2);
                    const float2 rt = make_float2(ptx::ex2(ut.x), ptx::ex2(ut.y));
                    const float2 rs = make_float2(ptx::ex2(us.x), ptx::ex2(us.y));
                    float2 d = mul2(sub2(rs, rt), dzs2);
                    if (masked) {
                        if (cb + c >= jlim) d.x = 0.f;
                        if (cb + c + 1 >= jlim) d.y = 0.f;
                    }
                    pk[c >> 1] = ptx::pack_bf16x2(d.x, d.y);
                }
                if (round == 0) {  // the dZ tile of k-1 must have been consumed by GEMMs 3 and 4
                    ok = ptx::mbar_wait(&ctrl->dz_free, (k & 1) ^ 1, abort_flag, lim, &g_lard_fault,
                                        kFaultBwdSoftmax);
                    if (!__all_sync(0xffffffffu, ok)) break;
                }
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int unit = round * 4 + u;
                    ptx::st_shared_v4(sdz_row + ((unit ^ (r & 7)) << 4), pk[4 * u], pk[4 * u + 1],
                                      pk[4 * u + 2], pk[4 * u + 3]);
                }
            }
            if (!ok) break;
            ptx::fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&ctrl->dz_full);
        }
    } else {
        ptx::regs_dec<kBwdRegsDrain>();
        // ------------------------------------------------------------ dX drain, dY store
        const int q = warp & 3;
        const int r = q * 32 + lane;
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(q * 32) << 16);
        uint8_t* stage = smem + L::OFF_STG + q * 8192;  // this warp's two 4 KB boxes
        const uint32_t stage_u32 = ptx::smem_u32(stage);
        int nchunk = 0;
        // Stage this warp's 32 x 32 box of fp32 values (one row per lane) in shared
        // memory and add it into the gradient buffer at (column c * 32, row y0).
        auto reduce_box = [&](const float (&v)[32], int c, int y0) {
            const int b = nchunk & 1;
            ++nchunk;
            if (lane == 0) ptx::bulk_wait_read<1>();  // box b's previous reduce has read it
            __syncwarp();
            const uint32_t row = stage_u32 + b * 4096 + lane * 128;
            const uint32_t* w = reinterpret_cast<const uint32_t*>(v);
#pragma unroll
            for (int u = 0; u < 8; ++u)
                ptx::st_shared_v4(row + ((u ^ (lane & 7)) << 4), w[4 * u], w[4 * u + 1], w[4 * u + 2], w[4 * u + 3]);
            ptx::fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                ptx::tma_reduce_add_3d(tm_dx, stage + b * 4096, c * 32, y0, bh);
                ptx::bulk_commit();
            }
        };
        bool ok = true;
        for (int k = 0; k < K; ++k) {
            const int y0 = row_block(k) * 128 + q * 32;  // first dX row of this warp's box
            ok = ptx::mbar_wait(&ctrl->dx_full, k & 1, abort_flag, lim, &g_lard_fault, kFaultBwdEpilogue);
            if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
            ptx::tc_fence_after();
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                float v[32];
                __syncwarp();
                ptx::tmem_ld32(lane_base + kTmemDX + c * 32, v);
                ptx::tmem_ld_wait(v);
                if (c == D / 32 - 1) {  // the dX accumulator is free for the next tile
                    ptx::tc_fence_before();
                    __syncwarp();
                    if (lane == 0) ptx::mbar_arrive(&ctrl->dx_free);
                }
                if (y0 < p.n) reduce_box(v, c, y0);  // warp-uniform: a box wholly past n is skipped
            }
        }
        if (ok) {
            ok = ptx::mbar_wait(&ctrl->dy_full, 0, abort_flag, lim, &g_lard_fault, kFaultBwdEpilogue);
            ok = __all_sync(0xffffffffu, ok);
        }
        if (ok) {
            ptx::tc_fence_after();
            const int j = J * 128 + r;
            const int y0 = J * 128 + q * 32;
            const size_t row = (static_cast<size_t>(bh) * p.n + (j < p.n ? j : 0)) * D;
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                float v[32];
                __syncwarp();
                ptx::tmem_ld32(lane_base + kTmemDY + c * 32, v);
                ptx::tmem_ld_wait(v);
                if (p.fuse_dy) {
                    if (y0 < p.n) reduce_box(v, c, y0);
                } else if (j < p.n) {
                    if (p.dYs_bf16) {  // dY_s[J] is complete here: round it once
                        uint4* dst = reinterpret_cast<uint4*>(p.dYs_bf16 + row + c * 32);
#pragma unroll
                        for (int u = 0; u < 4; ++u)
                            dst[u] = make_uint4(ptx::pack_bf16x2(v[8 * u], v[8 * u + 1]),
                                                ptx::pack_bf16x2(v[8 * u + 2], v[8 * u + 3]),
                                                ptx::pack_bf16x2(v[8 * u + 4], v[8 * u + 5]),
                                                ptx::pack_bf16x2(v[8 * u + 6], v[8 * u + 7]));
                    } else {
                        float* dst = p.dYs + row + c * 32;
#pragma unroll
                        for (int u = 0; u < 8; ++u)
                            *reinterpret_cast<float4*>(dst + 4 * u) =
                                make_float4(v[4 * u], v[4 * u + 1], v[4 * u + 2], v[4 * u + 3]);
                    }
                }
            }
        }
        if (lane == 0) ptx::bulk_wait<0>();
        __syncwarp();
    }

    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    if (warp == 1) ptx::tmem_dealloc(tmem, 512);
}

}  // namespace lard
