"""Write the small stored fixtures of this folder from the fp64 oracle.

Only `oracle/` computes anything here.  The inputs are fixed integer patterns
scaled by 1/8, so every value is exact in bf16, fp32 and fp64 and the same
numbers reach the oracle and the device.  The fixtures freeze the oracle's
results: a later change to its arithmetic makes `tests/test_golden.py` fail
until this script is re-run.  That run must be justified by the passage of the
LinearARD pages (or the reading of it) that the change follows.

    python tests/golden/make_golden.py
"""
import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))


def pattern(n, d, a, b, c):
    """x[i, k] = (((a*i + b*k + c) mod 17) - 8) / 8: values in [-1, 1], exact in bf16."""
    i = np.arange(n)[:, None]
    k = np.arange(d)[None, :]
    return (((a * i + b * k + c) % 17) - 8) / 8.0


CASES = [
    # name, n, d, tau, causal, self-relation
    ("causal_self_n6_d4", 6, 4, 0.5, True, True),
    ("full_cross_n5_d4", 5, 4, 0.5, False, False),
    ("causal_cross_n9_d8", 9, 8, 1.0 / np.sqrt(8.0), True, False),
]


def build_case(name, n, d, tau, causal, self_rel):
    Xt = pattern(n, d, 3, 5, 1)
    Xs = pattern(n, d, 3, 5, 2)          # student: the teacher pattern shifted by one step
    if self_rel:
        Yt, Ys = Xt, Xs
    else:
        Yt = pattern(n, d, 7, 2, 4)
        Ys = pattern(n, d, 7, 2, 6)
    return {"name": name, "n": n, "d": d, "tau": float(tau), "causal": bool(causal),
            "self_relation": bool(self_rel),
            "Xt": Xt.tolist(), "Yt": Yt.tolist(), "Xs": Xs.tolist(), "Ys": Ys.tolist()}


def main():
    sys.path.insert(0, ROOT)
    import oracle
    for name, n, d, tau, causal, self_rel in CASES:
        case = build_case(name, n, d, tau, causal, self_rel)
        arr = {k: np.array(case[k]) for k in ("Xt", "Yt", "Xs", "Ys")}
        r = oracle.relation(arr["Xt"], arr["Yt"], arr["Xs"], arr["Ys"], tau, causal)
        case["expected"] = {
            "lse_t": r["lse_t"].tolist(), "lse_s": r["lse_s"].tolist(),
            "row_kl": r["row_kl"].tolist(), "loss": r["loss"],
            "dXs": r["dXs"].tolist(), "dYs": r["dYs"].tolist(),
        }
        path = os.path.join(HERE, name + ".json")
        with open(path, "w") as f:
            json.dump(case, f, indent=1)
            f.write("\n")
        print("wrote", path)


if __name__ == "__main__":
    main()
