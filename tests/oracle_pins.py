"""Pins for the fp64 oracle: checks that tie it to something other than itself.

The pages print no worked values (no loss, LSE or gradient for any input),
so every pin here comes from mathematics or from an independent library:

* central finite differences of the oracle's own loss (gradients, the tau
  factor, the 1/n, the X/Y orientation);
* torch.autograd through torch's log_softmax / kl_div (a library routine,
  float64) for loss, row KL, LSE and both gradients;
* scipy.special.logsumexp / softmax and scipy.stats.entropy (KL) row by row;
* closed forms: constant rows give LSE = tau*|v|^2 + ln|A_i| and uniform R;
  n = 2 reduces to the binary (logistic) KL and its sigmoid gradient;
* invariants: student == teacher gives exactly zero loss and gradients;
  causal row 0 has KL = 0 and LSE = Z(0,0); KL_i >= 0 (Gibbs); rows of R
  sum to one (seen as dX_s = 0 when all student key rows are equal);
  sum_i <dX_s[i], X_s[i]> = sum_j <dY_s[j], Y_s[j]>.

Each pin takes an ``Oracle`` instance and raises AssertionError on failure,
so the same checks run against planted mistakes (test_oracle_mutants.py).
"""
import math

import numpy as np
import torch
from scipy import special, stats


def _rng(seed):
    return np.random.default_rng(seed)


def _rand(rng, *shape, scale=1.0):
    return rng.standard_normal(shape) * scale


def _close(a, b, rtol, atol, what):
    a, b = np.asarray(a, dtype=np.float64), np.asarray(b, dtype=np.float64)
    err = np.abs(a - b)
    bound = atol + rtol * np.abs(b)
    if not np.all(err <= bound):
        k = int(np.argmax(err - bound))
        raise AssertionError(f"{what}: max violation at flat index {k}: got {a.flat[k]!r} "
                             f"want {b.flat[k]!r} (|err| {err.flat[k]:.3e})")


# ---------------------------------------------------------------- finite differences

def pin_finite_differences(orc):
    """Central differences (h = 1e-6) of the oracle loss vs its analytic
    gradients, n in {1,2,3,5,8}, d in {2,4}, causal and not, X != Y and X = Y."""
    h = 1e-6
    rng = _rng(11)
    for causal in (True, False):
        for n in (1, 2, 3, 5, 8):
            for d in (2, 4):
                tau = 1.0 / math.sqrt(d)
                Xt, Yt, Xs, Ys = (_rand(rng, 1, n, d) for _ in range(4))
                out = orc.relation(Xt, Yt, Xs, Ys, tau, causal)
                gscale = max(np.abs(out["dXs"]).max(), np.abs(out["dYs"]).max(), 1e-3)

                def loss(xs, ys):
                    return orc.relation(Xt, Yt, xs, ys, tau, causal)["loss"]

                for which in ("X", "Y"):
                    fd = np.zeros((n, d))
                    for i in range(n):
                        for k in range(d):
                            xp, xm = Xs.copy(), Xs.copy()
                            yp, ym = Ys.copy(), Ys.copy()
                            if which == "X":
                                xp[0, i, k] += h
                                xm[0, i, k] -= h
                            else:
                                yp[0, i, k] += h
                                ym[0, i, k] -= h
                            fd[i, k] = (loss(xp, yp) - loss(xm, ym)) / (2 * h)
                    ana = out["dXs"][0] if which == "X" else out["dYs"][0]
                    _close(ana, fd, 0.0, 1e-6 * gscale + 1e-10,
                           f"FD d{which} causal={causal} n={n} d={d}")

                # self-relation: one tensor plays X and Y, gradient = dXs + dYs
                Xt2, Xs2 = _rand(rng, 1, n, d), _rand(rng, 1, n, d)
                out2 = orc.relation(Xt2, Xt2, Xs2, Xs2, tau, causal)
                fd = np.zeros((n, d))
                for i in range(n):
                    for k in range(d):
                        xp, xm = Xs2.copy(), Xs2.copy()
                        xp[0, i, k] += h
                        xm[0, i, k] -= h
                        fd[i, k] = (orc.relation(Xt2, Xt2, xp, xp, tau, causal)["loss"]
                                    - orc.relation(Xt2, Xt2, xm, xm, tau, causal)["loss"]) / (2 * h)
                g2 = out2["dXs"][0] + out2["dYs"][0]
                _close(g2, fd, 0.0, 1e-6 * max(np.abs(g2).max(), 1e-3) + 1e-10,
                       f"FD self-relation causal={causal} n={n} d={d}")


# ---------------------------------------------------------------- torch.autograd

def _torch_reference(Xt, Yt, Xs, Ys, tau, causal):
    """Loss through torch's own log_softmax / kl_div (float64) and its autograd."""
    Xt, Yt = torch.tensor(Xt), torch.tensor(Yt)
    Xs = torch.tensor(Xs, requires_grad=True)
    Ys = torch.tensor(Ys, requires_grad=True)
    n = Xt.shape[-2]
    keep = torch.ones(n, n, dtype=torch.bool)
    if causal:
        keep = torch.tril(keep)
    big = -1e300
    zt = (tau * Xt @ Yt.transpose(-1, -2)).masked_fill(~keep, big)
    zs = (tau * Xs @ Ys.transpose(-1, -2)).masked_fill(~keep, big)
    lt = torch.nn.functional.log_softmax(zt, dim=-1)
    ls = torch.nn.functional.log_softmax(zs, dim=-1)
    kl_rows = torch.nn.functional.kl_div(ls, lt, log_target=True, reduction="none").sum(-1)
    loss_bh = kl_rows.mean(-1)
    loss = loss_bh.sum()
    loss.backward()
    return {
        "loss": loss.item(), "loss_bh": loss_bh.detach().numpy(),
        "row_kl": kl_rows.detach().numpy(),
        "lse_t": torch.logsumexp(zt, -1).numpy(), "lse_s": torch.logsumexp(zs, -1).detach().numpy(),
        "dXs": Xs.grad.numpy(), "dYs": Ys.grad.numpy(),
    }


def pin_torch_autograd(orc):
    """Loss, row KL, LSE and both gradients vs torch autograd (float64)."""
    rng = _rng(12)
    for causal in (True, False):
        for (BH, n, d) in ((1, 1, 3), (2, 7, 4), (3, 40, 8)):
            tau = 1.0 / math.sqrt(d)
            Xt, Yt, Xs, Ys = (_rand(rng, BH, n, d, scale=1.5) for _ in range(4))
            for self_rel in (False, True):
                yt, ys = (Xt, Xs) if self_rel else (Yt, Ys)
                o = orc.relation(Xt, yt, Xs, ys, tau, causal)
                r = _torch_reference(Xt, yt, Xs, ys, tau, causal)
                tag = f"autograd causal={causal} BH={BH} n={n} d={d} self={self_rel}"
                _close(o["loss"], r["loss"], 1e-12, 1e-14, tag + " loss")
                _close(o["loss_bh"], r["loss_bh"], 1e-12, 1e-14, tag + " loss_bh")
                _close(o["row_kl"], r["row_kl"], 1e-10, 1e-13, tag + " row_kl")
                _close(o["lse_t"], r["lse_t"], 1e-13, 1e-13, tag + " lse_t")
                _close(o["lse_s"], r["lse_s"], 1e-13, 1e-13, tag + " lse_s")
                # with self_rel torch still holds one leaf per operand, so its two
                # gradients are the partials dXs and dYs the oracle reports
                _close(o["dXs"], r["dXs"], 1e-10, 1e-14, tag + " dXs")
                _close(o["dYs"], r["dYs"], 1e-10, 1e-14, tag + " dYs")


# ---------------------------------------------------------------- scipy, row by row

def pin_scipy_rows(orc):
    """Per-row LSE (scipy.special.logsumexp) and KL (scipy.stats.entropy)."""
    rng = _rng(13)
    n, d = 37, 8
    tau = 1.0 / math.sqrt(d)
    for causal in (True, False):
        Xt, Yt, Xs, Ys = (_rand(rng, n, d, scale=2.0) for _ in range(4))
        o = orc.relation(Xt[None], Yt[None], Xs[None], Ys[None], tau, causal)
        zt = tau * (Xt @ Yt.T)
        zs = tau * (Xs @ Ys.T)
        for i in range(n):
            cols = slice(0, i + 1) if causal else slice(0, n)
            _close(o["lse_t"][0, i], special.logsumexp(zt[i, cols]), 1e-13, 1e-13, f"lse_t row {i}")
            _close(o["lse_s"][0, i], special.logsumexp(zs[i, cols]), 1e-13, 1e-13, f"lse_s row {i}")
            pt = special.softmax(zt[i, cols])
            ps = special.softmax(zs[i, cols])
            _close(o["row_kl"][0, i], stats.entropy(pt, ps), 1e-9, 1e-13, f"KL row {i}")


# ---------------------------------------------------------------- invariants and closed forms

def pin_identical_student(orc):
    """Student == teacher: KL and both gradients are exactly zero."""
    rng = _rng(14)
    for causal in (True, False):
        Xt, Yt = _rand(rng, 2, 50, 16), _rand(rng, 2, 50, 16)
        o = orc.relation(Xt, Yt, Xt.copy(), Yt.copy(), 0.25, causal)
        assert np.all(o["row_kl"] == 0.0), "KL must be exactly 0 when student == teacher"
        assert o["loss"] == 0.0
        assert np.all(o["dXs"] == 0.0) and np.all(o["dYs"] == 0.0), "zero gradient expected"


def pin_causal_row0(orc):
    """Causal row 0 has one entry: R(0,0) = 1, KL_0 = 0, LSE(0) = Z(0,0)."""
    rng = _rng(15)
    d = 16
    tau = 0.25
    Xt, Yt, Xs, Ys = (_rand(rng, 1, 20, d) for _ in range(4))
    o = orc.relation(Xt, Yt, Xs, Ys, tau, True)
    assert o["row_kl"][0, 0] == 0.0
    _close(o["lse_t"][0, 0], tau * math.fsum(Xt[0, 0] * Yt[0, 0]), 1e-14, 1e-14, "lse_t(0)")
    _close(o["lse_s"][0, 0], tau * math.fsum(Xs[0, 0] * Ys[0, 0]), 1e-14, 1e-14, "lse_s(0)")


def pin_constant_rows(orc):
    """All rows equal (Y = X): Z is constant, so LSE(i) = tau|v|^2 + ln|A_i| and
    R is uniform; a different constant teacher then gives KL = 0 and zero grads."""
    n, d = 30, 6
    v = np.linspace(-1.0, 1.3, d)
    u = np.linspace(0.7, -0.4, d)
    X = np.tile(v, (1, n, 1))
    T = np.tile(u, (1, n, 1))
    tau = 0.4
    for causal in (True, False):
        o = orc.relation(T, T, X, X, tau, causal)
        cnt = np.arange(1, n + 1) if causal else np.full(n, n)
        _close(o["lse_s"][0], tau * float(v @ v) + np.log(cnt), 1e-13, 1e-13, "constant-row LSE_s")
        _close(o["lse_t"][0], tau * float(u @ u) + np.log(cnt), 1e-13, 1e-13, "constant-row LSE_t")
        _close(o["row_kl"][0], np.zeros(n), 0.0, 1e-14, "uniform vs uniform KL")
        _close(o["dXs"], np.zeros_like(X), 0.0, 1e-15, "uniform vs uniform dX")
        _close(o["dYs"], np.zeros_like(X), 0.0, 1e-15, "uniform vs uniform dY")


def pin_binary_closed_form(orc):
    """n = 2, d = 1, causal: row 1 is a two-way softmax, so KL_1 is the binary
    KL of sigmoids and the student gradient is the logistic one."""
    tau = 0.7
    xt, yt, xs, ys = np.array([0.3, -1.1]), np.array([0.9, 0.4]), np.array([1.2, 0.5]), \
        np.array([-0.6, 1.5])
    o = orc.relation(xt[None, :, None], yt[None, :, None], xs[None, :, None], ys[None, :, None],
                     tau, True)
    # row 1 logits: a = Z(1,0), b = Z(1,1); p = P(j=0) = sigmoid(a - b)
    at, bt = tau * xt[1] * yt[0], tau * xt[1] * yt[1]
    as_, bs = tau * xs[1] * ys[0], tau * xs[1] * ys[1]
    p = 1.0 / (1.0 + math.exp(-(at - bt)))
    q = 1.0 / (1.0 + math.exp(-(as_ - bs)))
    kl1 = p * math.log(p / q) + (1 - p) * math.log((1 - p) / (1 - q))
    _close(o["row_kl"][0], [0.0, kl1], 1e-12, 1e-15, "binary KL")
    _close(o["loss"], kl1 / 2, 1e-12, 1e-15, "binary loss (mean over 2 rows)")
    # dL/d(a_s - b_s) = (q - p)/2 ; a_s - b_s = tau * xs1 * (ys0 - ys1)
    g = (q - p) / 2.0
    want_dx = np.array([0.0, g * tau * (ys[0] - ys[1])])
    want_dy = np.array([0.0 + g * tau * xs[1], -g * tau * xs[1]])
    _close(o["dXs"][0, :, 0], want_dx, 1e-12, 1e-15, "binary dX_s")
    _close(o["dYs"][0, :, 0], want_dy, 1e-12, 1e-15, "binary dY_s")


def pin_gibbs_rowsum_duality(orc):
    """KL_i >= 0; rows of R_s and R_t each sum to one (equal student key rows
    make dX_s vanish); sum_i <dX_s[i], X_s[i]> = sum_j <dY_s[j], Y_s[j]>."""
    rng = _rng(16)
    n, d = 45, 8
    tau = 1.0 / math.sqrt(d)
    for causal in (True, False):
        Xt, Yt, Xs, Ys = (_rand(rng, 1, n, d, scale=1.7) for _ in range(4))
        o = orc.relation(Xt, Yt, Xs, Ys, tau, causal)
        assert np.all(o["row_kl"] >= -1e-15), "Gibbs: KL must be non-negative"
        assert o["loss"] > 1e-3, "random teacher/student must disagree"
        lhs = float(np.sum(o["dXs"] * Xs))
        rhs = float(np.sum(o["dYs"] * Ys))
        _close(lhs, rhs, 1e-11, 1e-15, "duality <dX,X> = <dY,Y>")
        Ys_eq = np.tile(Ys[:, :1, :], (1, n, 1))
        o2 = orc.relation(Xt, Yt, Xs, Ys_eq, tau, causal)
        scale = np.abs(o2["dYs"]).max()
        _close(o2["dXs"], np.zeros_like(Xs), 0.0, 1e-13 * max(scale, 1.0), "row sums (dX = 0)")


def pin_self_relation_total_gradient(orc):
    """A self-relation (Y = X, as Q/Q, K/K, V/V): torch autograd through one
    tied student leaf gives the total gradient, which must be the sum of the
    oracle's two partials dXs + dYs (the quantity lard_kl_bwd_self returns)."""
    rng = _rng(17)
    for causal in (True, False):
        for (BH, n, d) in ((1, 5, 4), (2, 23, 8)):
            tau = 1.0 / math.sqrt(d)
            Xt, Xs = _rand(rng, BH, n, d, scale=1.3), _rand(rng, BH, n, d, scale=1.3)
            o = orc.relation(Xt, Xt, Xs, Xs, tau, causal)
            xt = torch.tensor(Xt)
            xs = torch.tensor(Xs, requires_grad=True)
            keep = torch.ones(n, n, dtype=torch.bool)
            if causal:
                keep = torch.tril(keep)
            zt = (tau * xt @ xt.transpose(-1, -2)).masked_fill(~keep, -1e300)
            zs = (tau * xs @ xs.transpose(-1, -2)).masked_fill(~keep, -1e300)
            kl = torch.nn.functional.kl_div(torch.log_softmax(zs, -1), torch.log_softmax(zt, -1),
                                            log_target=True, reduction="none").sum(-1)
            kl.mean(-1).sum().backward()
            _close(o["dXs"] + o["dYs"], xs.grad.numpy(), 1e-10, 1e-14,
                   f"self-relation total gradient causal={causal} n={n}")


PINS = [pin_finite_differences, pin_torch_autograd, pin_scipy_rows, pin_identical_student,
        pin_causal_row0, pin_constant_rows, pin_binary_closed_form, pin_gibbs_rowsum_duality,
        pin_self_relation_total_gradient]
