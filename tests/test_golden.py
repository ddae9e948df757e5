"""Stored fixtures under tests/golden/ (written by make_golden.py from the oracle).

CPU: the oracle still reproduces the stored values (any change to its
arithmetic must come with a re-run of make_golden.py).
GPU: the CUDA path on the same exact inputs, zero-padded from d to a kernel
head size (padding columns add nothing to any dot product, and their
gradients are exactly zero), matches the stored values.
"""
import glob
import json
import os

import numpy as np
import pytest

import oracle
from parity_util import compare_full

GOLDEN = sorted(glob.glob(os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "*.json")))


def _load(path):
    with open(path) as f:
        c = json.load(f)
    arr = {k: np.array(c[k], dtype=np.float64) for k in ("Xt", "Yt", "Xs", "Ys")}
    exp = {k: (np.array(v) if isinstance(v, list) else v) for k, v in c["expected"].items()}
    return c, arr, exp


def test_golden_present():
    assert len(GOLDEN) >= 3


@pytest.mark.parametrize("path", GOLDEN, ids=os.path.basename)
def test_oracle_reproduces_golden(path):
    c, a, e = _load(path)
    r = oracle.relation(a["Xt"], a["Yt"], a["Xs"], a["Ys"], c["tau"], c["causal"])
    for k in ("lse_t", "lse_s", "row_kl", "dXs", "dYs"):
        np.testing.assert_allclose(r[k], e[k], rtol=1e-12, atol=1e-14, err_msg=k)
    assert abs(r["loss"] - e["loss"]) <= 1e-13


@pytest.mark.parametrize("path", GOLDEN, ids=os.path.basename)
def test_golden_inputs_exact_in_bf16(path):
    import torch
    _, a, _ = _load(path)
    for k, v in a.items():
        t = torch.from_numpy(v)
        assert torch.equal(t.to(torch.bfloat16).to(torch.float64), t), k


@pytest.mark.gpu
@pytest.mark.parametrize("dtype,d_pad", [("bf16", 64), ("bf16", 128), ("fp32", 64)])
@pytest.mark.parametrize("path", GOLDEN, ids=os.path.basename)
def test_device_matches_golden(path, dtype, d_pad):
    import torch
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from linear_memory_attention_b200 import lard
    from parity_util import gpu_relation
    c, a, e = _load(path)
    n, d = c["n"], c["d"]
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32

    def pad(v):
        t = torch.zeros((1, 1, n, d_pad), dtype=torch.float64)
        t[0, 0, :, :d] = torch.from_numpy(v)
        return t.to(tdt)

    Xt, Xs = pad(a["Xt"]), pad(a["Xs"])
    Yt = Xt if c["self_relation"] else pad(a["Yt"])
    Ys = Xs if c["self_relation"] else pad(a["Ys"])
    g = gpu_relation(lard, Xt, Yt, Xs, Ys, c["tau"], int(c["causal"]))
    assert np.all(g["dXs"][..., d:] == 0) and np.all(g["dYs"][..., d:] == 0)
    want = {"lse_t": e["lse_t"][None], "lse_s": e["lse_s"][None], "row_kl": e["row_kl"][None],
            "loss": e["loss"], "loss_bh": np.array([e["loss"]]),
            "dXs": e["dXs"][None], "dYs": e["dYs"][None]}
    got = dict(g)
    got["dXs"] = g["dXs"][0, :, :, :d]
    got["dYs"] = g["dYs"][0, :, :, :d]
    got["lse_t"], got["lse_s"], got["row_kl"] = g["lse_t"][0], g["lse_s"][0], g["row_kl"][0]
    compare_full(got, want, dtype, f"golden {c['name']} {dtype} d={d_pad}")
