// lard_fwd_tc.cuh -- Phase 1 on the 5th-generation tensor cores (bf16 inputs).
//
// LinearARD notes (papernotes.org), 关键设计 3, first phase: stream the
// relation tiles and keep only per-row log-sum-exp statistics of the teacher
// and the student, so that HBM holds O(BHn) scalars instead of the n x n map.
// This kernel also forms the row KL online from the same tiles (a
// reading: the pages give no place for it; it needs no extra exponential).
//
// One CTA owns a 128-row block I of one (batch, head) and streams the column
// blocks J it may attend to (J <= I under the causal mask), diagonal first.
// Roles (384 threads):
//   warp 0      TMA producer: X_t[I], X_s[I] once, then Y_t[J], Y_s[J] per
//               tile into an NS-deep ring of 128B-swizzled shared tiles.
//   warp 1      TMEM owner and MMA issuer: S_t = X_t Y_t^T and S_s = X_s Y_s^T
//               (M = N = 128, K = d) into a double-buffered pair of TMEM
//               accumulators (4 x 128 fp32 columns).
//   warps 4-11  row statistics: each thread owns one row (its TMEM lane) and
//               one 64-column half of every tile; it keeps, in the log2
//               domain, the running maxima m_t, m_s, the sums l_t, l_s and
//               the teacher-weighted logit gap a = sum 2^(u_t - m_t) (S_t - S_s).
//               The two halves of a row are merged at the end.
// Every wait is bounded (see ptx::mbar_wait).
#pragma once

#include "lard_kernel_common.cuh"

namespace lard {

struct TcFwdParams {
    int BH, n, T, causal;
    float cfac;  // tau * log2(e): S -> log2-domain logit
    float tau;
    float* lse_t;
    float* lse_s;
    float* row_kl;
    unsigned long long wait_ns;
};

template <int D>
struct FwdLayout {
    static constexpr int KC = D / 64;        // 64-column (128-byte) chunks per row
    static constexpr int TILE = KC * 16384;  // one 128 x D bf16 operand tile
    static constexpr int NS = (D == 128) ? 2 : 4;
    static constexpr int OFF_XT = 0;
    static constexpr int OFF_XS = TILE;
    static constexpr int OFF_Y = 2 * TILE;  // stage s: Y_t at OFF_Y + 2*s*TILE, Y_s after it
    static constexpr int OFF_CTRL = OFF_Y + NS * 2 * TILE;
    static constexpr int CTRL_BYTES = 4096;
    static constexpr int SMEM_BYTES = OFF_CTRL + CTRL_BYTES + 1024;  // + alignment slack
};

// Register split (per thread): launched at 168; the control warpgroup gives
// registers to the two statistics warpgroups.  The shares must not add up to
// more than the launch allocation, or setmaxnreg.inc would wait for ever; the
// host checks the built kernel's register count against kFwdRegsSplitTotal
// before the first launch.
constexpr int kFwdRegsLaunch = 168, kFwdRegsCtl = 40, kFwdRegsStat = 232;
constexpr int kFwdRegsSplitTotal = 128 * (kFwdRegsCtl + 2 * kFwdRegsStat);
static_assert(kFwdRegsSplitTotal <= 384 * kFwdRegsLaunch, "register split exceeds the launch allocation");

struct FwdCtrl {
    uint64_t x_full;
    uint64_t y_full[4];
    uint64_t y_empty[4];
    uint64_t s_full[2];
    uint64_t s_empty[2];
    uint64_t mma_done;
    uint32_t tmem_base;
    int abort_flag;
    float merge[128][5];
};
static_assert(sizeof(FwdCtrl) <= 4096, "control block too large");

template <int D>
__global__ void __launch_bounds__(384, 1)
    lard_fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_xt,
                       const __grid_constant__ CUtensorMap tm_yt,
                       const __grid_constant__ CUtensorMap tm_xs,
                       const __grid_constant__ CUtensorMap tm_ys, const TcFwdParams p) {
    using L = FwdLayout<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (ptx::smem_u32(smem_raw) & 1023u)) & 1023u);
    FwdCtrl* ctrl = reinterpret_cast<FwdCtrl*>(smem + L::OFF_CTRL);
    volatile int* abort_flag = &ctrl->abort_flag;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    // Head-major order, longest row blocks first within a head: the blocks
    // resident at any time then share one head's Y tiles, which stay in L2.
    const int bh = static_cast<int>(blockIdx.x) / p.T;
    const int I = p.T - 1 - static_cast<int>(blockIdx.x) % p.T;
    const int numJ = p.causal ? (I + 1) : p.T;
    auto col_block = [&](int jt) { return p.causal ? (I - jt) : ((I - jt + p.T) % p.T); };

    if (threadIdx.x == 0) {
        ptx::mbar_init(&ctrl->x_full, 1);
        for (int s = 0; s < L::NS; ++s) {
            ptx::mbar_init(&ctrl->y_full[s], 1);
            ptx::mbar_init(&ctrl->y_empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            ptx::mbar_init(&ctrl->s_full[b], 1);
            ptx::mbar_init(&ctrl->s_empty[b], 8);
        }
        ptx::mbar_init(&ctrl->mma_done, 1);
        ctrl->abort_flag = 0;
        ptx::fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        ptx::prefetch_tensormap(&tm_xt);
        ptx::prefetch_tensormap(&tm_yt);
        ptx::prefetch_tensormap(&tm_xs);
        ptx::prefetch_tensormap(&tm_ys);
    }
    if (warp == 1) {
        ptx::tmem_alloc(&ctrl->tmem_base, 512);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = ctrl->tmem_base;
    const uint64_t lim = p.wait_ns;
    if (warp < 4) {
      ptx::regs_dec<kFwdRegsCtl>();
      if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            ptx::mbar_arrive_expect_tx(&ctrl->x_full, 2 * L::TILE);
            for (int c = 0; c < L::KC; ++c) {
                ptx::tma_load_3d(smem + L::OFF_XT + c * 16384, &tm_xt, &ctrl->x_full, c * 64, I * 128, bh);
                ptx::tma_load_3d(smem + L::OFF_XS + c * 16384, &tm_xs, &ctrl->x_full, c * 64, I * 128, bh);
            }
        }
        __syncwarp();
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
                    ptx::tma_load_3d(yt + c * 16384, &tm_yt, &ctrl->y_full[s], c * 64, J * 128, bh);
                    ptx::tma_load_3d(yt + L::TILE + c * 16384, &tm_ys, &ctrl->y_full[s], c * 64, J * 128, bh);
                }
            }
            __syncwarp();
            ++issued;
        }
        // Let every copy this warp started land before the block can exit.
        ptx::mbar_drain(&ctrl->x_full, 0, lim);
        for (int s = 0; s < L::NS && s < issued; ++s) {
            const int last = s + L::NS * ((issued - 1 - s) / L::NS);
            ptx::mbar_drain(&ctrl->y_full[s], (last / L::NS) & 1, lim);
        }
      } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        constexpr uint32_t kIdesc = ptx::idesc_bf16(128, 128, 0, 0);
        const uint32_t sxt = ptx::smem_u32(smem + L::OFF_XT);
        const uint32_t sxs = ptx::smem_u32(smem + L::OFF_XS);
        bool ok = ptx::mbar_wait(&ctrl->x_full, 0, abort_flag, lim, &g_lard_fault, kFaultFwdMma);
        ok = __all_sync(0xffffffffu, ok);
        for (int jt = 0; ok && jt < numJ; ++jt) {
            const int s = jt % L::NS, rnd = jt / L::NS;
            const int buf = jt & 1, use = jt >> 1;
            ok = ptx::mbar_wait(&ctrl->y_full[s], rnd & 1, abort_flag, lim, &g_lard_fault, kFaultFwdMma);
            if (!__all_sync(0xffffffffu, ok)) break;
            ok = ptx::mbar_wait(&ctrl->s_empty[buf], (use & 1) ^ 1, abort_flag, lim, &g_lard_fault,
                                kFaultFwdMma);
            if (!__all_sync(0xffffffffu, ok)) break;
            ptx::tc_fence_after();
            if (lane == 0) {
                const uint32_t syt = ptx::smem_u32(smem + L::OFF_Y + 2 * s * L::TILE);
                const uint32_t sys = syt + L::TILE;
                const uint32_t dt = tmem + buf * 256;
                const uint32_t ds = dt + 128;
#pragma unroll
                for (int k = 0; k < D / 16; ++k) {
                    const uint32_t koff = (k >> 2) * 16384 + (k & 3) * 32;
                    ptx::umma_bf16(dt, ptx::sdesc_sw128(sxt + koff, 16, 1024),
                                   ptx::sdesc_sw128(syt + koff, 16, 1024), kIdesc, k > 0);
                }
#pragma unroll
                for (int k = 0; k < D / 16; ++k) {
                    const uint32_t koff = (k >> 2) * 16384 + (k & 3) * 32;
                    ptx::umma_bf16(ds, ptx::sdesc_sw128(sxs + koff, 16, 1024),
                                   ptx::sdesc_sw128(sys + koff, 16, 1024), kIdesc, k > 0);
                }
                ptx::umma_commit(&ctrl->y_empty[s]);
                ptx::umma_commit(&ctrl->s_full[buf]);
            }
            __syncwarp();
        }
        if (lane == 0) ptx::umma_commit(&ctrl->mma_done);
        __syncwarp();
        ptx::mbar_drain(&ctrl->mma_done, 0, lim);
      }
    } else {
        ptx::regs_inc<kFwdRegsStat>();
        // ------------------------------------------------------------ row statistics
        const int q = warp & 3;
        const int hcol = (warp - 4) >> 2;
        const int r = q * 32 + lane;
        const int i = I * 128 + r;
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(q * 32) << 16);
        const float cf = p.cfac;
        float m_t = -INFINITY, l_t = 0.f, m_s = -INFINITY, l_s = 0.f, acc = 0.f;

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
            // Read this thread's 64 columns of S_t and S_s at once and hand the
            // TMEM buffer back before the exponentials.
            float st0[32], ss0[32], st1[32], ss1[32];
            __syncwarp();
            ptx::tmem_ld32(lane_base + buf * 256 + hcol * 64, st0);
            ptx::tmem_ld32(lane_base + buf * 256 + 128 + hcol * 64, ss0);
            ptx::tmem_ld32(lane_base + buf * 256 + hcol * 64 + 32, st1);
            ptx::tmem_ld32(lane_base + buf * 256 + 128 + hcol * 64 + 32, ss1);
            ptx::tmem_ld_wait(st0);
            ptx::reg_dep(ss0);
            ptx::reg_dep(st1);
            ptx::reg_dep(ss1);
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&ctrl->s_empty[buf]);
#pragma unroll
            for (int round = 0; round < 2; ++round) {
                const int cb = hcol * 64 + round * 32;
                float* st = round ? st1 : st0;
                float* ss = round ? ss1 : ss0;
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
                    float lt0 = 0.f, lt1 = 0.f, ls0 = 0.f, ls1 = 0.f, a0 = 0.f, a1 = 0.f;
#pragma unroll
                    for (int c = 0; c < 32; c += 2) {
                        const float pt0 = ptx::ex2(fmaf(st[c], cf, -m_t));
                        const float ps0 = ptx::ex2(fmaf(ss[c], cf, -m_s));
                        const float pt1 = ptx::ex2(fmaf(st[c + 1], cf, -m_t));
                        const float ps1 = ptx::ex2(fmaf(ss[c + 1], cf, -m_s));
                        lt0 += pt0;
                        ls0 += ps0;
                        lt1 += pt1;
                        ls1 += ps1;
                        a0 = fmaf(pt0, st[c] - ss[c], a0);
                        a1 = fmaf(pt1, st[c + 1] - ss[c + 1], a1);
                    }
                    l_t += lt0 + lt1;
                    l_s += ls0 + ls1;
                    acc += a0 + a1;
                }
            }
        }
        // Merge the two column halves of each row.
        if (hcol == 1) {
            ctrl->merge[r][0] = m_t;
            ctrl->merge[r][1] = l_t;
            ctrl->merge[r][2] = m_s;
            ctrl->merge[r][3] = l_s;
            ctrl->merge[r][4] = acc;
        }
        ptx::named_bar_sync(1, 256);
        if (hcol == 0 && i < p.n && !*abort_flag) {
            const float pm_t = ctrl->merge[r][0], pl_t = ctrl->merge[r][1];
            const float pm_s = ctrl->merge[r][2], pl_s = ctrl->merge[r][3];
            const float pa = ctrl->merge[r][4];
            const float M_t = fmaxf(m_t, pm_t), M_s = fmaxf(m_s, pm_s);
            const float f0 = ptx::ex2(m_t - M_t), f1 = ptx::ex2(pm_t - M_t);
            const float g0 = ptx::ex2(m_s - M_s), g1 = ptx::ex2(pm_s - M_s);
            const float L_t = l_t * f0 + pl_t * f1;
            const float L_s = l_s * g0 + pl_s * g1;
            const float A = acc * f0 + pa * f1;
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
