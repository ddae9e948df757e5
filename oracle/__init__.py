"""fp64 CPU oracle for the LinearARD relation-KL loss (test infrastructure).

Only ``tests/``, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg import this package.  It wraps ``lard_oracle.c`` through ctypes and shares
nothing with the CUDA implementation.

Definitions followed (LinearARD notes, papernotes.org, 关键设计 1 and 3;
LinearARD abstract, fugumt.com):
    Z_m = tau * X_m Y_m^T, causal mask j <= i, R_m = row softmax,
    loss per (batch, head) = (1/n) sum_i KL(R_t(i,.) || R_s(i,.)),
    dZ = (R_s - R_t)/n, dX_s = tau dZ Y_s, dY_s = tau dZ^T X_s.
"""
import ctypes

import numpy as np

from . import build as _build

_DP = ctypes.POINTER(ctypes.c_double)


def _f64(a):
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(_DP)


class Oracle:
    """ctypes handle on one build of ``lard_oracle.c``."""

    def __init__(self, libpath: str):
        lib = ctypes.CDLL(libpath)
        lib.lard_oracle_rows.restype = ctypes.c_int
        lib.lard_oracle_rows.argtypes = [_DP, _DP, _DP, _DP, ctypes.c_long, ctypes.c_long,
                                         ctypes.c_double, ctypes.c_int, ctypes.c_long,
                                         ctypes.c_long, _DP, _DP, _DP, _DP, _DP]
        lib.lard_oracle_relation.restype = ctypes.c_double
        lib.lard_oracle_relation.argtypes = [_DP, _DP, _DP, _DP, ctypes.c_long, ctypes.c_long,
                                             ctypes.c_long, ctypes.c_double, ctypes.c_int,
                                             _DP, _DP, _DP, _DP, _DP, _DP]
        lib.lard_oracle_num_threads.restype = ctypes.c_int
        lib.lard_oracle_num_threads.argtypes = []
        self._lib = lib
        self.path = libpath

    def num_threads(self) -> int:
        """Threads the oracle's OpenMP loops use (OMP_NUM_THREADS, else all cores)."""
        return int(self._lib.lard_oracle_num_threads())

    def relation(self, Xt, Yt, Xs, Ys, tau, causal=True):
        """Full relation over a batch of heads.

        Inputs are arrays of shape [..., n, d] (leading dims are flattened into
        heads) holding the exact values the device sees, converted to float64.
        Returns a dict with lse_t, lse_s, row_kl [..., n], loss_bh [...],
        loss (sum over heads), dXs, dYs [..., n, d].
        """
        Xt, Yt, Xs, Ys = (_f64(a) for a in (Xt, Yt, Xs, Ys))
        shape = Xt.shape
        n, d = shape[-2], shape[-1]
        BH = int(np.prod(shape[:-2])) if len(shape) > 2 else 1
        for a in (Yt, Xs, Ys):
            if a.shape != shape:
                raise ValueError("all four inputs must have the same shape")
        lse_t, lse_s, row_kl = np.empty((BH, n)), np.empty((BH, n)), np.empty((BH, n))
        loss_bh = np.empty(BH)
        dXs, dYs = np.empty((BH, n, d)), np.empty((BH, n, d))
        total = self._lib.lard_oracle_relation(_ptr(Xt), _ptr(Yt), _ptr(Xs), _ptr(Ys), BH, n, d,
                                               float(tau), int(bool(causal)), _ptr(lse_t),
                                               _ptr(lse_s), _ptr(row_kl), _ptr(loss_bh),
                                               _ptr(dXs), _ptr(dYs))
        if not np.isfinite(total):
            raise MemoryError("oracle failed (argument error or out of host memory)")
        lead = shape[:-2]
        return {
            "lse_t": lse_t.reshape(*lead, n), "lse_s": lse_s.reshape(*lead, n),
            "row_kl": row_kl.reshape(*lead, n), "loss_bh": loss_bh.reshape(lead),
            "loss": float(total), "dXs": dXs.reshape(shape), "dYs": dYs.reshape(shape),
        }

    def rows(self, Xt, Yt, Xs, Ys, tau, causal, r0, r1, want_dY=False):
        """Rows [r0, r1) of one head ([n, d] inputs).

        Returns lse_t, lse_s, row_kl [r1-r0], dXs [r1-r0, d] and, if want_dY,
        the contribution of these rows to dY_s, [n, d].  Under the causal mask
        rows [r0, n) give the exact dY_s for every column >= r0.
        """
        Xt, Yt, Xs, Ys = (_f64(a) for a in (Xt, Yt, Xs, Ys))
        n, d = Xt.shape
        m = r1 - r0
        lse_t, lse_s, kl = np.empty(m), np.empty(m), np.empty(m)
        dX = np.empty((m, d))
        dY = np.zeros((n, d)) if want_dY else None
        rc = self._lib.lard_oracle_rows(_ptr(Xt), _ptr(Yt), _ptr(Xs), _ptr(Ys), n, d, float(tau),
                                        int(bool(causal)), int(r0), int(r1), _ptr(lse_t),
                                        _ptr(lse_s), _ptr(kl), _ptr(dX), _ptr(dY))
        if rc == 1:
            raise ValueError("oracle: bad arguments")
        if rc == 2:
            raise MemoryError("oracle: out of host memory for the explicit maps")
        out = {"lse_t": lse_t, "lse_s": lse_s, "row_kl": kl, "dXs": dX}
        if want_dY:
            out["dYs"] = dY
        return out


def map_bytes(rows_, n) -> int:
    """Host bytes the explicit maps of ``rows_`` rows need (five double maps)."""
    return 5 * 8 * int(rows_) * int(n)


_default = None


def default() -> Oracle:
    global _default
    if _default is None:
        _default = Oracle(_build.build())
    return _default


def relation(*a, **k):
    return default().relation(*a, **k)


def rows(*a, **k):
    return default().rows(*a, **k)


def num_threads() -> int:
    return default().num_threads()


__all__ = ["Oracle", "default", "relation", "rows", "num_threads", "map_bytes"]
