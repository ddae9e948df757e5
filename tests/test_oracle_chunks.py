"""CPU check of the chunked whole-head oracle the full-size parity tests use:
the oracle's rows mode over row chunks (dY_s summed over the chunks) gives
what one whole-relation call gives."""
import numpy as np
import pytest

import oracle
from parity_util import oracle_head


@pytest.mark.parametrize("causal", [True, False], ids=["causal", "full"])
def test_chunked_head_equals_whole_relation(causal):
    rng = np.random.default_rng(3)
    n, d = 157, 16
    xt = rng.standard_normal((n, d))
    xs = xt + 0.3 * rng.standard_normal((n, d))
    tau = 1 / np.sqrt(d)
    whole = oracle.relation(xt, xt, xs, xs, tau, causal)
    # maps of 23 rows at a time: seven chunks, the last one ragged
    chunked = oracle_head(xt, xs, tau, causal, max_map_bytes=oracle.map_bytes(23, n))
    for k in ("lse_t", "lse_s", "row_kl", "dXs", "dYs"):
        np.testing.assert_allclose(chunked[k], whole[k], rtol=1e-12, atol=1e-15, err_msg=k)
    assert abs(chunked["loss"] - whole["loss"]) <= 1e-12 * abs(whole["loss"])
