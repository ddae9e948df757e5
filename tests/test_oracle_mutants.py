"""Plant plausible mistakes in a copy of the oracle's source, on the CPU, and
check that the pins catch every one.  This shows the pins constrain each part
of the oracle: the mask, the LSE, the KL direction and its normalisation, the
sign and scale of dZ, the tau of the chain rule and the operands of both
contractions."""
import os
import subprocess

import pytest

import oracle
import oracle_pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "lard_oracle.c")

MUTANTS = {
    "mask drops the diagonal": ("return causal ? (j <= i) : 1;", "return causal ? (j < i) : 1;"),
    "mask is anti-causal": ("return causal ? (j <= i) : 1;", "return causal ? (j >= i) : 1;"),
    "LSE forgets the max": ("lse[i - r0] = mx + log(s);", "lse[i - r0] = log(s);"),
    "KL direction reversed": ("kl += Rt[o + j] * (log_rt - log_rs);",
                              "kl += Rs[o + j] * (log_rs - log_rt);"),
    "KL drops the student LSE": ("const double log_rs = Zs[o + j] - Ls[i - r0];",
                                 "const double log_rs = Zs[o + j];"),
    "dZ sign flipped": ("(Rs[(i - r0) * n + j] - Rt[(i - r0) * n + j]) / (double)n",
                        "(Rt[(i - r0) * n + j] - Rs[(i - r0) * n + j]) / (double)n"),
    "dZ misses 1/n": ("(Rs[(i - r0) * n + j] - Rt[(i - r0) * n + j]) / (double)n",
                      "(Rs[(i - r0) * n + j] - Rt[(i - r0) * n + j])"),
    "dZ row-count normalisation": ("(Rs[(i - r0) * n + j] - Rt[(i - r0) * n + j]) / (double)n",
                                   "(Rs[(i - r0) * n + j] - Rt[(i - r0) * n + j]) / (double)(i + 1)"),
    "loss not row-averaged": ("const double lbh = s / (double)n;", "const double lbh = s;"),
    "dX drops tau": ("dXs_rows[(i - r0) * d + k] = tau * acc;", "dXs_rows[(i - r0) * d + k] = acc;"),
    "dY drops tau": ("dYs_accum[j * d + k] += tau * acc;", "dYs_accum[j * d + k] += acc;"),
    "dX uses teacher keys": ("acc += dZ[(i - r0) * n + j] * Ys[j * d + k];",
                             "acc += dZ[(i - r0) * n + j] * Yt[j * d + k];"),
    "dY uses wrong operand": ("acc += dZ[(i - r0) * n + j] * Xs[i * d + k];",
                              "acc += dZ[(i - r0) * n + j] * Ys[i * d + k];"),
    "dY uses untransposed dZ": ("acc += dZ[(i - r0) * n + j] * Xs[i * d + k];",
                                "acc += dZ[(j - r0) * n + i] * Xs[i * d + k];"),
    "student map uses teacher keys": ("relation_logits(Xs, Ys, n, d, tau, r0, r1, Zs);",
                                      "relation_logits(Xs, Yt, n, d, tau, r0, r1, Zs);"),
    "logits miss tau": ("Z[(i - r0) * n + j] = tau * dot;", "Z[(i - r0) * n + j] = dot;"),
}


@pytest.fixture(scope="module")
def source():
    with open(SRC) as f:
        return f.read()


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, source, tmp_path):
    old, new = MUTANTS[name]
    assert source.count(old) == 1, f"mutation site for '{name}' not unique in the oracle"
    src = tmp_path / "mutant.c"
    src.write_text(source.replace(old, new))
    lib = tmp_path / "libmutant.so"
    subprocess.run(["gcc", "-O2", "-fno-fast-math", "-ffp-contract=off", "-fopenmp", "-fPIC",
                    "-shared", "-std=c11", "-o", str(lib), str(src), "-lm"], check=True)
    mutant = oracle.Oracle(str(lib))
    caught = []
    for pin in oracle_pins.PINS:
        try:
            pin(mutant)
        except Exception as e:  # noqa: BLE001 - any failure counts as caught
            caught.append(f"{pin.__name__}: {type(e).__name__}")
    assert caught, f"no pin caught the planted mistake '{name}'"
