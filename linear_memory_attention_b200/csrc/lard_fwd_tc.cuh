// lard_fwd_tc.cuh -- Phase 1 on the 5th-generation tensor cores (bf16 inputs).
//
// LinearARD notes (papernotes.org), 关键设计 3, first phase: stream the
// relation tiles and keep only per-row log-sum-exp statistics of the teacher
// and the student, so that HBM holds O(BHn) scalars instead of the n x n map.
// This kernel also forms the row KL online from the same tiles (a
// reading: the pages give no place for it; it needs no extra exponential).
//
// One CTA owns a 128-row block I of one (batch, head) of one relation and
// streams the column blocks J it may attend to (J <= I under the causal mask),
// diagonal first.  A launch covers up to kMaxRelations relations (TcFwdGroup:
// Q/Q, K/K and V/V with their own head counts); their blocks follow one
// another in the grid.
// X_t[I] and X_s[I] are the A operands of every GEMM of the CTA, so they are
// kept in tensor memory (two bf16 per 32-bit column, row i in lane i): the
// GEMMs then read only B = Y[J] from shared memory, which leaves shared-memory
// bandwidth to the TMA stream of Y tiles, and all of shared memory holds a
// 3-deep ring of (Y_t[J], Y_s[J]) tiles.
// TMEM (512 columns): X_t [0, 64), X_s [64, 128), S_s [128, 256),
//                     S_t buffer b at [256 + 128 b, 384 + 128 b).
// Roles (640 threads):
//   warp 0      TMA producer of the Y ring.
//   warp 1      TMEM owner and MMA issuer: S_t = X_t Y_t^T, S_s = X_s Y_s^T
//               (M = N = 128, K = d, A from TMEM).  S_t is double-buffered,
//               S_s single-buffered: the statistics warps read a tile's S out
//               of TMEM at the start of their work on it.
//   warps 4-19  X_t / X_s rows into TMEM (prologue), then row statistics in
//               four warpgroups: each thread owns one row (its TMEM lane) and
//               one 32-column quarter of every tile; it keeps, in the log2
//               domain, the running maxima m_t, m_s, the sums l_t, l_s and the
//               teacher-weighted logit gap a = sum 2^(u_t - m_t) (S_t - S_s).
//               The four quarters of a row are merged at the end.  Four
//               warps per scheduler keep the MUFU and FMA pipes busy while
//               others wait on TMEM loads.
// Every wait is bounded (see ptx::mbar_wait).
#pragma once

#include "lard_exp2.cuh"
#include "lard_kernel_common.cuh"

namespace lard {

// One relation of a launch.
struct TcFwdRel {
    const __nv_bfloat16* Xt;  // row sources of the TMEM-resident A operands
    const __nv_bfloat16* Xs;
    float* lse_t;
    float* lse_s;
    float* row_kl;
    int block0;  // first grid block of this relation (its B*H*T blocks follow)
};

// A launch: up to kMaxRelations relations of equal n and d (for example the
// Q/Q, K/K and V/V maps, with their own head counts) in one grid.
struct TcFwdGroup {
    CUtensorMap yt[kMaxRelations];  // Y_t and Y_s of each relation, {d, n, B*H}
    CUtensorMap ys[kMaxRelations];
    TcFwdRel rel[kMaxRelations];
    int nrel, n, T, causal;
    float cfac;  // tau * log2(e): S -> log2-domain logit
    float tau;
    unsigned long long wait_ns;   // limit of each wait inside the loops
    unsigned long long drain_ns;  // limit of each drain on the way out (longer)
};

template <int D>
struct FwdLayout {
    static constexpr int KC = D / 64;        // 64-column (128-byte) chunks per row
    static constexpr int TILE = KC * 16384;  // one 128 x D bf16 operand tile
    static constexpr int NS = (D == 128) ? 3 : 6;
    static constexpr int OFF_Y = 0;  // stage s: Y_t at OFF_Y + 2*s*TILE, Y_s after it
    static constexpr int OFF_CTRL = OFF_Y + NS * 2 * TILE;
    static constexpr int CTRL_BYTES = 8192;
    static constexpr int SMEM_BYTES = OFF_CTRL + CTRL_BYTES + 1024;  // + alignment slack
};

// Register split (per thread): launched at 96; the control warpgroup gives
// registers to the four statistics warpgroups.  The shares must not add up to
// more than the launch allocation, or setmaxnreg.inc would wait for ever; the
// host checks the built kernel's register count against kFwdRegsSplitTotal
// before the first launch.
constexpr int kFwdThreads = 640, kFwdStatGroups = 4;
constexpr int kFwdRegsLaunch = 96, kFwdRegsCtl = 48, kFwdRegsStat = 104;
constexpr int kFwdRegsSplitTotal = 128 * (kFwdRegsCtl + kFwdStatGroups * kFwdRegsStat);
static_assert(kFwdRegsSplitTotal <= kFwdThreads * kFwdRegsLaunch, "register split exceeds the launch allocation");

constexpr uint32_t kFwdTmemXt = 0, kFwdTmemXs = 64, kFwdTmemSs = 128, kFwdTmemSt = 256;

struct FwdCtrl {
    uint64_t y_full[6];
    uint64_t y_empty[6];
    uint64_t x_ready;      // X_t, X_s written to TMEM (16 warps)
    uint64_t s_full[2];    // S_t(k) and S_s(k) computed (by S_t buffer)
    uint64_t st_empty[2];  // S_t buffer read out (16 warps)
    uint64_t ss_empty;     // S_s read out (16 warps)
    uint64_t mma_done;
    uint32_t tmem_base;
    int abort_flag;
    float merge[3][128][5];
};
static_assert(sizeof(FwdCtrl) <= 8192, "control block too large");

template <int D>
__global__ void __launch_bounds__(kFwdThreads, 1)
    lard_fwd_tc_kernel(const __grid_constant__ TcFwdGroup g) {
    using L = FwdLayout<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (ptx::smem_u32(smem_raw) & 1023u)) & 1023u);
    FwdCtrl* ctrl = reinterpret_cast<FwdCtrl*>(smem + L::OFF_CTRL);
    volatile int* abort_flag = &ctrl->abort_flag;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    // This block's relation; then head-major order within it, longest row
    // blocks first within a head: the blocks resident at any time share one
    // head's Y tiles, which stay in L2.
    const int rel = relation_of_block(g.rel, g.nrel);
    const CUtensorMap* tm_yt = &g.yt[rel];
    const CUtensorMap* tm_ys = &g.ys[rel];
    const struct {
        int n, T, causal;
        float cfac, tau;
        const __nv_bfloat16 *Xt, *Xs;
        float *lse_t, *lse_s, *row_kl;
        unsigned long long wait_ns, drain_ns;
    } p = {g.n, g.T, g.causal, g.cfac, g.tau, g.rel[rel].Xt, g.rel[rel].Xs, g.rel[rel].lse_t,
           g.rel[rel].lse_s, g.rel[rel].row_kl, g.wait_ns, g.drain_ns};
    const int local = static_cast<int>(blockIdx.x) - g.rel[rel].block0;
    const int bh = local / p.T;
    const int I = p.T - 1 - local % p.T;
    const int numJ = p.causal ? (I + 1) : p.T;
    auto col_block = [&](int jt) { return p.causal ? (I - jt) : ((I - jt + p.T) % p.T); };

    if (threadIdx.x == 0) {
        for (int s = 0; s < L::NS; ++s) {
            ptx::mbar_init(&ctrl->y_full[s], 1);
            ptx::mbar_init(&ctrl->y_empty[s], 1);
        }
        ptx::mbar_init(&ctrl->x_ready, 4 * kFwdStatGroups);
        for (int b = 0; b < 2; ++b) {
            ptx::mbar_init(&ctrl->s_full[b], 1);
            ptx::mbar_init(&ctrl->st_empty[b], 4 * kFwdStatGroups);
        }
        ptx::mbar_init(&ctrl->ss_empty, 4 * kFwdStatGroups);
        ptx::mbar_init(&ctrl->mma_done, 1);
        ctrl->abort_flag = 0;
        ptx::fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        ptx::prefetch_tensormap(tm_yt);
        ptx::prefetch_tensormap(tm_ys);
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
      ptx::regs_dec<kFwdRegsCtl>();
      if (warp == 0) {
        // ------------------------------------------------------------ producer
        int issued = 0;
        for (int jt = 0; jt < numJ; ++jt) {
            const int s = jt % L::NS, rnd = jt / L::NS;
            bool ok = ptx::mbar_wait(&ctrl->y_empty[s], (rnd & 1) ^ 1, abort_flag, lim, &g_lard_fault,
                                     kFaultFwdProducer);
            if (!__all_sync(0xffffffffu, ok)) break;
            if (lane == 0) {
                const int J = col_block(jt);
                uint8_t* yt = smem + L::OFF_Y + 2 * s * L::TILE;
                ptx::mbar_arrive_expect_tx(&ctrl->y_full[s], 2 * L::TILE);
                for (int c = 0; c < L::KC; ++c) {
                    ptx::tma_load_3d(yt + c * 16384, tm_yt, &ctrl->y_full[s], c * 64, J * 128, bh);
                    ptx::tma_load_3d(yt + L::TILE + c * 16384, tm_ys, &ctrl->y_full[s], c * 64, J * 128, bh);
                }
            }
            __syncwarp();
            ++issued;
        }
        // Let every copy this warp started land before the block can exit.
        for (int s = 0; s < L::NS && s < issued; ++s) {
            const int last = s + L::NS * ((issued - 1 - s) / L::NS);
            drain(&ctrl->y_full[s], (last / L::NS) & 1, dlim);
        }
      } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        constexpr uint32_t kIdesc = ptx::idesc_bf16(128, 128, 0, 0);
        constexpr uint32_t kHi = ptx::sdesc_hi(1024);
        // Descriptor low words of stage 0's Y_t; stage s and Y_s are fixed offsets.
        const uint32_t y0_lo = ptx::sdesc_lo(ptx::smem_u32(smem + L::OFF_Y), 16);
        const uint32_t st0 = tmem + kFwdTmemSt, ss = tmem + kFwdTmemSs;
        const uint32_t xt = tmem + kFwdTmemXt, xs = tmem + kFwdTmemXs;
        bool ok = ptx::mbar_wait(&ctrl->x_ready, 0, abort_flag, lim, &g_lard_fault, kFaultFwdMma);
        ok = __all_sync(0xffffffffu, ok);
        for (int jt = 0; ok && jt < numJ; ++jt) {
            const int s = jt % L::NS, rnd = jt / L::NS;
            const int buf = jt & 1, use = jt >> 1;
            ok = ptx::mbar_wait(&ctrl->y_full[s], rnd & 1, abort_flag, lim, &g_lard_fault, kFaultFwdMma) &&
                 ptx::mbar_wait(&ctrl->st_empty[buf], (use & 1) ^ 1, abort_flag, lim, &g_lard_fault,
                                kFaultFwdMma);
            if (!__all_sync(0xffffffffu, ok)) break;
            ptx::tc_fence_after();
            const uint32_t yt_lo = y0_lo + s * (2 * L::TILE >> 4);
            const uint32_t ys_lo = yt_lo + (L::TILE >> 4);
            if (lane == 0) {
                const uint32_t dt = st0 + buf * 128;
#pragma unroll
                for (int k = 0; k < D / 16; ++k) {
                    if (k == 0) ptx::umma_ts<0>(dt, xt, yt_lo, kHi, kIdesc);
                    else ptx::umma_ts<1>(dt, xt + k * 8, yt_lo + ptx::desc_step_k(k), kHi, kIdesc);
                }
            }
            __syncwarp();
            // S_s is single-buffered: wait until S_s(jt - 1) has been read out.
            ok = ptx::mbar_wait(&ctrl->ss_empty, (jt & 1) ^ 1, abort_flag, lim, &g_lard_fault, kFaultFwdMma);
            if (!__all_sync(0xffffffffu, ok)) break;
            ptx::tc_fence_after();
            if (lane == 0) {
#pragma unroll
                for (int k = 0; k < D / 16; ++k) {
                    if (k == 0) ptx::umma_ts<0>(ss, xs, ys_lo, kHi, kIdesc);
                    else ptx::umma_ts<1>(ss, xs + k * 8, ys_lo + ptx::desc_step_k(k), kHi, kIdesc);
                }
                ptx::umma_commit(&ctrl->y_empty[s]);
                ptx::umma_commit(&ctrl->s_full[buf]);
            }
            __syncwarp();
        }
        if (lane == 0) ptx::umma_commit(&ctrl->mma_done);
        __syncwarp();
        drain(&ctrl->mma_done, 0, dlim);
      }
    } else {
        ptx::regs_inc<kFwdRegsStat>();
        // ------------------------------------------------------------ row statistics
        const int q = warp & 3;
        const int grp = (warp - 4) >> 2;  // column quarter [32 grp, 32 grp + 32)
        const int r = q * 32 + lane;
        const int i = I * 128 + r;
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(q * 32) << 16);
        const float cf = p.cfac;

        // Prologue: the A operands into TMEM, one row per thread, rows past n as
        // zeros.  Quarter g writes half g & 1 of X_t (g < 2) or of X_s (g >= 2).
        {
            const int half = grp & 1;
            const size_t row = static_cast<size_t>(bh) * p.n + (i < p.n ? i : 0);
            const uint4* src = reinterpret_cast<const uint4*>((grp < 2 ? p.Xt : p.Xs) + row * D) + half * (D / 16);
            const uint32_t dst = lane_base + (grp < 2 ? kFwdTmemXt : kFwdTmemXs) + half * (D / 4);
#pragma unroll
            for (int c = 0; c < D / 128; ++c) {
                uint32_t w[32];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    uint4 v = make_uint4(0u, 0u, 0u, 0u);
                    if (i < p.n) v = __ldg(src + c * 8 + u);
                    w[4 * u] = v.x;
                    w[4 * u + 1] = v.y;
                    w[4 * u + 2] = v.z;
                    w[4 * u + 3] = v.w;
                }
                __syncwarp();
                ptx::tmem_st32(dst + c * 32, w);
            }
            if (D == 64) {  // a quarter is 16 columns: one x16 store through the x32 form's first half
                uint32_t w[32];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    uint4 v = make_uint4(0u, 0u, 0u, 0u);
                    if (u < 4 && i < p.n) v = __ldg(src + u);
                    w[4 * u] = v.x;
                    w[4 * u + 1] = v.y;
                    w[4 * u + 2] = v.z;
                    w[4 * u + 3] = v.w;
                }
                __syncwarp();
                ptx::tmem_st16(dst, w);
            }
            ptx::tmem_st_wait();
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&ctrl->x_ready);
        }

        float m_t = -INFINITY, l_t = 0.f, m_s = -INFINITY, l_s = 0.f, acc = 0.f;
        const int cb = grp * 32;
        for (int jt = 0; jt < numJ; ++jt) {
            const int buf = jt & 1, use = jt >> 1;
            bool ok = ptx::mbar_wait(&ctrl->s_full[buf], use & 1, abort_flag, lim, &g_lard_fault,
                                     kFaultFwdSoftmax);
            if (!__all_sync(0xffffffffu, ok)) break;
            ptx::tc_fence_after();
            const int J = col_block(jt);
            int jlim = 128;  // columns [0, jlim) of this tile are allowed for row i
            if (p.causal) {
                if (J == I) jlim = r + 1;
            } else if (J == p.T - 1) {
                jlim = p.n - J * 128;
            }
            // Read this thread's 32 columns of S_t and S_s and hand the TMEM back
            // before the exponentials.
            float st[32], ss[32];
            __syncwarp();
            ptx::tmem_ld32(lane_base + kFwdTmemSt + buf * 128 + cb, st);
            ptx::tmem_ld32(lane_base + kFwdTmemSs + cb, ss);
            ptx::tmem_ld_wait(st);
            ptx::reg_dep(ss);
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                ptx::mbar_arrive(&ctrl->ss_empty);
                ptx::mbar_arrive(&ctrl->st_empty[buf]);
            }
            if (cb < jlim) {
                if (cb + 32 > jlim) {
#pragma unroll
                    for (int c = 0; c < 32; ++c)
                        if (cb + c >= jlim) { st[c] = -1e30f; ss[c] = -1e30f; }
                }
                float mt = st[0], ms = ss[0];
#pragma unroll
                for (int c = 1; c < 31; c += 2) {
                    mt = ptx::fmax3(mt, st[c], st[c + 1]);
                    ms = ptx::fmax3(ms, ss[c], ss[c + 1]);
                }
                mt = fmaxf(mt, st[31]);
                ms = fmaxf(ms, ss[31]);
                const float nmt = mt * cf, nms = ms * cf;
                if (nmt > m_t) {
                    const float sc = ptx::ex2(m_t - nmt);
                    l_t *= sc;
                    acc *= sc;
                    m_t = nmt;
                }
                if (nms > m_s) {
                    l_s *= ptx::ex2(m_s - nms);
                    m_s = nms;
                }
                // Column pairs in packed fp32x2 arithmetic; 2 of every 16 pairs
                // take the FMA-pipe exponential, which relieves the MUFU unit
                // (16 exponentials per clock per SM).  More than that costs more
                // than it saves: the polynomial takes 14 issue slots per pair
                // against 2, and under the power cap the clock pays for them.
                const float2 cf2 = splat2(cf), nmt2 = splat2(-m_t), nms2 = splat2(-m_s);
                float2 LT = splat2(0.f), LS = splat2(0.f), AC = splat2(0.f);
#pragma unroll
                for (int c = 0; c < 32; c += 2) {
                    const float2 St = make_float2(st[c], st[c + 1]);
                    const float2 Ss = make_float2(ss[c], ss[c + 1]);
                    const float2 ut = fma2(St, cf2, nmt2);
                    const float2 us = fma2(Ss, cf2, nms2);
                    const int pr = c >> 1;
                    const bool on_fma = (pr == 0) || (pr == 8);
                    const float2 pt = on_fma ? exp2_fma2(ut) : make_float2(ptx::ex2(ut.x), ptx::ex2(ut.y));
                    const float2 ps = on_fma ? exp2_fma2(us) : make_float2(ptx::ex2(us.x), ptx::ex2(us.y));
                    LT = add2(LT, pt);
                    LS = add2(LS, ps);
                    AC = fma2(pt, sub2(St, Ss), AC);
                }
                l_t += LT.x + LT.y;
                l_s += LS.x + LS.y;
                acc += AC.x + AC.y;
            }
        }
        // Merge the four column quarters of each row.
        if (grp > 0) {
            float* m = ctrl->merge[grp - 1][r];
            m[0] = m_t;
            m[1] = l_t;
            m[2] = m_s;
            m[3] = l_s;
            m[4] = acc;
        }
        ptx::named_bar_sync(1, 128 * kFwdStatGroups);
        if (grp == 0 && i < p.n && !*abort_flag) {
            float M_t = m_t, M_s = m_s;
#pragma unroll
            for (int g = 0; g < kFwdStatGroups - 1; ++g) {
                M_t = fmaxf(M_t, ctrl->merge[g][r][0]);
                M_s = fmaxf(M_s, ctrl->merge[g][r][2]);
            }
            float f = ptx::ex2(m_t - M_t), gs = ptx::ex2(m_s - M_s);
            float L_t = l_t * f, A = acc * f, L_s = l_s * gs;
#pragma unroll
            for (int g = 0; g < kFwdStatGroups - 1; ++g) {
                const float* m = ctrl->merge[g][r];
                const float fg = ptx::ex2(m[0] - M_t);
                L_t += m[1] * fg;
                A += m[4] * fg;
                L_s += m[3] * ptx::ex2(m[2] - M_s);
            }
            const float kLn2 = 0.6931471805599453f;
            const size_t o = static_cast<size_t>(bh) * p.n + i;
            p.lse_t[o] = (M_t + log2f(L_t)) * kLn2;
            p.lse_s[o] = (M_s + log2f(L_s)) * kLn2;
            // KL_i = E_t[Z_t - Z_s] - LSE_t + LSE_s, with the maxima cancelled
            // analytically so that only small quantities are subtracted.
            p.row_kl[o] = p.tau * A / L_t - kLn2 * ((M_t - M_s) + log2f(L_t / L_s));
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    if (warp == 1) ptx::tmem_dealloc(tmem, 512);
}

}  // namespace lard
