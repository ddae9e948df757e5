"""CPU checks of the C ABI: the library loads, exports every entry point that
include/lard.h declares, and rejects bad arguments before touching CUDA."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "lard.h")
PROBE_HEADER = os.path.join(ROOT, "include", "lard_probe.h")


def declared_entry_points(header=HEADER, api="LARD_API"):
    text = open(header).read()
    return re.findall(api + r"\s+[\w\s\*]+?\b(lard_\w+)\s*\(", text)


@pytest.fixture(scope="module")
def lib():
    from linear_memory_attention_b200 import build
    build.build()
    from linear_memory_attention_b200 import lard
    return lard._lib


def test_header_declares_the_boundary():
    names = declared_entry_points()
    for n in ("lard_kl_fwd", "lard_kl_bwd", "lard_kl_bwd_self", "lard_status_string",
              "lard_device_status", "lard_selftest_timeout", "lard_version"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_entry_points():
        assert hasattr(lib, name), f"{name} declared in include/lard.h but not exported"


def test_binding_lists_every_export():
    from linear_memory_attention_b200 import lard
    assert set(declared_entry_points()) == set(lard.EXPORTS)


def test_probe_library_exports_its_header():
    """The exponential-unit probe library (used by the benchmark) exports what
    include/lard_probe.h declares; no compute call without a GPU."""
    from linear_memory_attention_b200 import build, probe
    build.build()
    names = declared_entry_points(PROBE_HEADER, "LARD_PROBE_API")
    assert names and set(names) == set(probe.EXPORTS)
    for name in names:
        assert hasattr(probe._lib, name)
    # argument errors return before any CUDA call
    ms, ex = ctypes.c_float(), ctypes.c_double()
    assert probe._lib.lard_probe_exp_rate(7, 1, 1, ctypes.byref(ms), ctypes.byref(ex), None) == 1
    assert probe._lib.lard_probe_exp_rate(0, 0, 1, ctypes.byref(ms), ctypes.byref(ex), None) == 1


def test_status_strings_and_version(lib):
    from linear_memory_attention_b200 import lard
    assert [lard.lard_status_string(c) for c in range(6)] == [
        "LARD_OK", "LARD_ERR_INVALID_ARG", "LARD_ERR_UNSUPPORTED", "LARD_ERR_CUDA",
        "LARD_ERR_TIMEOUT", "LARD_ERR_TOO_LARGE"]
    assert lard.lard_status_string(99) == "LARD_ERR_UNKNOWN"
    assert lard.lard_version() >= 100


# Aligned fake device addresses: every case below must be rejected by the
# argument checks, which run before any CUDA call.
A, B_, C, D_ = 0x100000, 0x200000, 0x300000, 0x400000
O1, O2, O3, O4, O5 = 0x10000000, 0x11000000, 0x12000000, 0x13000000, 0x14000000


def fwd(lib, *, xt=A, yt=B_, xs=C, ys=D_, dtype=0, B=1, H=2, n=300, d=128, tau=0.088, causal=1,
        lse_t=O1, lse_s=O2, kl=O3, loss_bh=O4, loss=O5):
    f = ctypes.c_float
    return lib.lard_kl_fwd(xt, yt, xs, ys, dtype, B, H, n, d, f(tau), causal, lse_t, lse_s, kl,
                           loss_bh, loss, None)


def bwd(lib, *, dtype=0, n=300, d=128, tau=0.088, causal=1, g=1.0, dx=O3, dy=O4, lse_t=O1,
        lse_s=O2):
    f = ctypes.c_float
    return lib.lard_kl_bwd(A, B_, C, D_, dtype, 1, 2, n, d, f(tau), causal, lse_t, lse_s, f(g), dx,
                           dy, None)


@pytest.mark.parametrize("kw,code", [
    (dict(xt=None), 1), (dict(ys=None), 1), (dict(lse_t=None), 1), (dict(kl=None), 1),
    (dict(n=0), 1), (dict(B=0), 1), (dict(H=-1), 1), (dict(tau=float("nan")), 1),
    (dict(tau=-0.5), 1), (dict(tau=0.0), 1), (dict(causal=2), 1), (dict(dtype=7), 2),
    (dict(d=96), 2), (dict(d=256), 2), (dict(dtype=1, d=48), 2), (dict(dtype=1, d=288), 2),
    (dict(xs=C + 8), 1), (dict(loss_bh=None), 1), (dict(lse_s=O1), 1), (dict(kl=A), 1),
])
def test_fwd_rejects_bad_arguments(lib, kw, code):
    if kw == dict(loss_bh=None):
        # loss_total requires loss_bh
        assert fwd(lib, loss_bh=None) == code
    else:
        assert fwd(lib, **kw) == code


@pytest.mark.parametrize("kw,code", [
    (dict(dx=None), 1), (dict(lse_s=None), 1), (dict(g=float("inf")), 1),
    (dict(dy=O3 + 16), 1), (dict(dx=A), 1), (dict(dy=O1), 1), (dict(dx=O3 + 4), 1),
    (dict(d=32), 2), (dict(n=-3), 1),
])
def test_bwd_rejects_bad_arguments(lib, kw, code):
    assert bwd(lib, **kw) == code


def bwd_self(lib, *, dtype=0, n=300, d=128, tau=0.088, causal=1, g=1.0, dx=O3, lse_t=O1, lse_s=O2):
    f = ctypes.c_float
    return lib.lard_kl_bwd_self(A, C, dtype, 1, 2, n, d, f(tau), causal, lse_t, lse_s, f(g), dx, None)


@pytest.mark.parametrize("kw,code", [
    (dict(dx=None), 1), (dict(lse_t=None), 1), (dict(g=float("nan")), 1), (dict(dx=A), 1),
    (dict(dx=O1), 1), (dict(dx=O3 + 4), 1), (dict(d=32), 2), (dict(tau=0.0), 1),
    (dict(dtype=1), 2),
])
def test_bwd_self_rejects_bad_arguments(lib, kw, code):
    assert bwd_self(lib, **kw) == code


def relations(specs):
    from linear_memory_attention_b200.lard import _Relation
    arr = (_Relation * max(1, len(specs)))()
    for k, sp in enumerate(specs):
        for name, v in sp.items():
            setattr(arr[k], name, v)
    return arr


REL0 = dict(Xt=A, Yt=B_, Xs=C, Ys=D_, H=2, lse_t=O1, lse_s=O2, row_kl=O3, loss_bh=O4, dXs=O5,
            dYs=0x1c000000)
REL1 = dict(Xt=0x500000, Yt=0x500000, Xs=0x600000, Ys=0x600000, H=1, lse_t=0x15000000,
            lse_s=0x16000000, row_kl=0x17000000, loss_bh=0x18000000, dXs=0x19000000, dYs=0x1a000000)


def fwd_multi(lib, specs, nrel=None, dtype=0, n=300, d=128, loss=0x1b000000):
    arr = relations(specs)
    return lib.lard_kl_fwd_multi(arr, len(specs) if nrel is None else nrel, dtype, 1, n, d,
                                 ctypes.c_float(0.088), 1, loss, None)


def bwd_multi(lib, specs, nrel=None, dtype=0, n=300, d=128, g=1.0):
    arr = relations(specs)
    return lib.lard_kl_bwd_multi(arr, len(specs) if nrel is None else nrel, dtype, 1, n, d,
                                 ctypes.c_float(0.088), 1, ctypes.c_float(g), None)


@pytest.mark.parametrize("specs,nrel,code", [
    ([REL0], 0, 1), ([REL0] * 5, 5, 1),
    ([REL0, dict(REL1, row_kl=O3)], None, 1),          # two relations write one buffer
    ([REL0, dict(REL1, lse_t=A)], None, 1),            # an output over another relation's input
    ([REL0, dict(REL1, loss_bh=None)], None, 1),       # loss_total needs every loss_bh
    ([REL0, dict(REL1, H=0)], None, 1),
    ([REL0, dict(REL1, Xs=0x600008)], None, 1),        # misaligned input
])
def test_fwd_multi_rejects_bad_arguments(lib, specs, nrel, code):
    assert fwd_multi(lib, specs, nrel) == code


# A fused relation with fp32 inputs is refused (2) only after every range and
# pointer check has passed, so a case that should fail those checks must give 1.
FUSED1 = dict(REL1, dYs=None)


def test_bwd_multi_valid_ranges_reach_the_dtype_check(lib):
    assert bwd_multi(lib, [REL0, FUSED1], dtype=1) == 2


@pytest.mark.parametrize("specs,kw,code", [
    ([REL0, dict(FUSED1, dXs=O5)], {}, 1),             # two relations write one gradient
    ([dict(REL0, dYs=0x600000), FUSED1], {}, 1),       # gradient over an input
    ([dict(REL0, dYs=O1), FUSED1], {}, 1),             # gradient over an LSE input
    ([dict(REL0, dYs=None), FUSED1], {}, 1),           # fused gradient needs Y = X
    ([REL0, dict(FUSED1, lse_s=None)], {}, 1),
    ([REL0, dict(FUSED1, dXs=0x19000004)], {}, 1),     # misaligned gradient
    ([REL0, FUSED1], dict(g=float("inf")), 1),
    ([REL0, FUSED1], dict(d=48), 2),                   # unsupported head size for fp32 (d % 32)
])
def test_bwd_multi_rejects_bad_arguments(lib, specs, kw, code):
    kw = dict(dict(dtype=1), **kw)
    assert bwd_multi(lib, specs, **kw) == code


def test_binding_marshalling_errors():
    """The Python binding's own checks, before any call into the library."""
    import torch
    from linear_memory_attention_b200 import lard
    a = torch.zeros((1, 2, 64, 128), dtype=torch.bfloat16)
    b = torch.zeros((1, 2, 64, 64), dtype=torch.bfloat16)
    f = torch.zeros((1, 2, 64, 128), dtype=torch.float16)
    with pytest.raises(ValueError):
        lard._relations([], "fwd")                                   # no relation
    with pytest.raises(ValueError):
        lard._relations([dict(Xt=a, Xs=a)] * 5, "fwd")               # more than LARD_MAX_RELATIONS
    with pytest.raises(ValueError):
        lard._relations([dict(Xt=a, Xs=a), dict(Xt=b, Xs=b)], "fwd")  # relations of different d
    with pytest.raises(ValueError):
        lard._relations([dict(Xt=a, Xs=b)], "fwd")                   # X_t and X_s of different shapes
    with pytest.raises(ValueError):
        lard._shape(f)                                               # unsupported dtype
    with pytest.raises(ValueError):
        lard._shape(a[0])                                            # not [B, H, n, d]
    a1 = a[:, :1].contiguous()
    outs = lambda H: dict(lse_t=torch.empty(1, H, 64), lse_s=torch.empty(1, H, 64),  # noqa: E731
                          row_kl=torch.empty(1, H, 64), loss_bh=torch.empty(H),
                          dXs=torch.empty(1, H, 64, 128), dYs=torch.empty(1, H, 64, 128))
    arr, dt, B, n, d = lard._relations([dict(Xt=a, Xs=a, **outs(2)), dict(Xt=a1, Xs=a1, **outs(1))],
                                       "fwd")
    assert (dt, B, n, d) == (lard.LARD_DTYPE_BF16, 1, 64, 128)
    assert arr[0].H == 2 and arr[1].H == 1 and arr[0].Yt == arr[0].Xt
    assert arr[1].dXs is None and arr[1].dYs is None                 # a phase passes only its outputs
    arr, *_ = lard._relations([dict(Xt=a, Xs=a, **dict(outs(2), dYs=None))], "bwd")
    assert arr[0].dYs is None and arr[0].row_kl is None and arr[0].dXs is not None


@pytest.mark.parametrize("field,bad", [
    ("dXs", lambda: torch_zeros((1, 2, 64, 128), "bfloat16")),     # wrong dtype
    ("dXs", lambda: torch_zeros((1, 2, 64, 64), "float32")),       # short
    ("dYs", lambda: torch_zeros((1, 2, 128, 64), "float32")[:, :, ::2]),  # right size, not contiguous
    ("lse_t", lambda: torch_zeros((1, 2, 63), "float32")),         # short
    ("lse_s", lambda: torch_zeros((1, 2, 64), "float64")),         # wrong dtype
    ("row_kl", lambda: None),                                      # missing
    ("loss_bh", lambda: torch_zeros((3,), "float32")),             # wrong length
])
def test_binding_checks_every_output(field, bad):
    """Every output buffer is checked for dtype, size, contiguity and device: the
    library cannot see buffer sizes, so a short or wrong-typed buffer would be
    written past its end."""
    import torch
    from linear_memory_attention_b200 import lard
    a = torch.zeros((1, 2, 64, 128), dtype=torch.bfloat16)
    good = dict(lse_t=torch.empty(1, 2, 64), lse_s=torch.empty(1, 2, 64), row_kl=torch.empty(1, 2, 64),
                loss_bh=torch.empty(2), dXs=torch.empty(1, 2, 64, 128), dYs=torch.empty(1, 2, 64, 128))
    rel = dict(Xt=a, Xs=a, **dict(good, **{field: bad()}))
    phase = "bwd" if field in ("dXs", "dYs") else "fwd"
    with pytest.raises(ValueError):
        lard._relations([rel], phase)
    if field in ("dXs",):
        with pytest.raises(ValueError):
            lard.lard_kl_bwd(a, a, a, a, 0.1, True, good["lse_t"], good["lse_s"], 1.0, rel["dXs"],
                             good["dYs"])
        with pytest.raises(ValueError):
            lard.lard_kl_bwd_self(a, a, 0.1, True, good["lse_t"], good["lse_s"], 1.0, rel["dXs"])
    if field in ("lse_t", "row_kl", "loss_bh"):
        kw = dict(good)
        kw[field] = rel[field]
        with pytest.raises(ValueError):
            lard.lard_kl_fwd(a, a, a, a, 0.1, True, kw["lse_t"], kw["lse_s"], kw["row_kl"], kw["loss_bh"])
    with pytest.raises(ValueError):
        lard.lard_kl_fwd_multi([dict(Xt=a, Xs=a, **good)], 0.1, True, loss_total=torch.empty(2))


def torch_zeros(shape, dtype):
    import torch
    return torch.zeros(shape, dtype=getattr(torch, dtype))


def bwd_multi_bf16(lib, specs, outs, ws=0x1d000000, ws_bytes=None, dtype=0, n=300, d=128, g=1.0):
    from linear_memory_attention_b200.lard import _Bf16Grads
    arr = relations(specs)
    o = (_Bf16Grads * max(1, len(outs)))()
    for k, (x, y) in enumerate(outs):
        o[k].dXs, o[k].dYs = x, y
    if ws_bytes is None:
        ws_bytes = lib.lard_kl_bwd_bf16_workspace_bytes(arr, len(specs), 1, n, d)
    return lib.lard_kl_bwd_multi_bf16(arr, o, len(specs), dtype, 1, n, d, ctypes.c_float(0.088), 1,
                                      ctypes.c_float(g), ws, ws_bytes, None)


BF0 = dict(REL0, dXs=None, dYs=None)
BF1 = dict(REL1, dXs=None, dYs=None)
OUT0, OUT1 = (0x20000000, 0x21000000), (0x22000000, None)


def test_bf16_workspace_bytes(lib):
    assert lib.lard_kl_bwd_bf16_workspace_bytes(relations([BF0, BF1]), 2, 1, 300, 128) == (2 + 1) * 300 * 128 * 4
    assert lib.lard_kl_bwd_bf16_workspace_bytes(relations([BF0]), 1, 3, 300, 64) == 3 * 2 * 300 * 64 * 4
    assert lib.lard_kl_bwd_bf16_workspace_bytes(relations([BF0]), 0, 1, 300, 128) == 0
    assert lib.lard_kl_bwd_bf16_workspace_bytes(relations([dict(BF0, H=0)]), 1, 1, 300, 128) == 0
    assert lib.lard_kl_bwd_bf16_workspace_bytes(None, 1, 1, 300, 128) == 0


@pytest.mark.parametrize("specs,outs,kw,code", [
    ([BF0, BF1], [OUT0, OUT1], dict(dtype=1), 2),                     # fp32 inputs: full-precision path only
    ([BF0, BF1], [OUT0, OUT1], dict(ws_bytes=100), 1),                # workspace too small
    ([BF0, BF1], [OUT0, OUT1], dict(ws=0x1d000008), 1),               # misaligned workspace
    ([BF0, BF1], [OUT0, OUT1], dict(ws=0), 1),                        # no workspace
    ([BF0, BF1], [OUT0, OUT1], dict(ws=0x20000000), 1),               # workspace over an output
    ([BF0, BF1], [OUT0, (0x20000000 + 4096, None)], {}, 1),           # two outputs overlap
    ([BF0, BF1], [(None, 0x21000000), OUT1], {}, 1),                  # dXs missing
    ([dict(BF0, dXs=O5), BF1], [OUT0, OUT1], {}, 1),                  # fp32 field set as well
    ([BF0, BF1], [(0x20000008, 0x21000000), OUT1], {}, 1),            # misaligned bf16 output
    ([BF0, dict(BF1, Ys=0x700000)], [OUT0, OUT1], {}, 1),             # fused needs Y = X
    ([BF0, BF1], [OUT0, OUT1], dict(g=float("nan")), 1),
    ([BF0, BF1], [OUT0, OUT1], dict(d=96), 2),
])
def test_bwd_multi_bf16_rejects_bad_arguments(lib, specs, outs, kw, code):
    assert bwd_multi_bf16(lib, specs, outs, **kw) == code


def test_sizes_beyond_the_limits_are_refused(lib):
    """B*H*n*d must stay below 2^40 and the grid below 2^31 blocks: refused
    synchronously, before any CUDA call (the pointers are fake)."""
    assert fwd(lib, B=1 << 12, H=1 << 12, n=1 << 13, d=128) == 1   # 2^44 elements
    assert bwd(lib, n=(1 << 31) - 1) == 1                          # row indices past int
    assert fwd(lib, n=(1 << 31) - 127, B=1, H=1, d=64) == 1         # its last tile's rows past int
    assert fwd(lib, B=1 << 16, H=1 << 15, n=1) == 1                 # B*H past the 2^30 head limit


@pytest.mark.parametrize("module", ["lard.py", "probe.py"])
def test_binding_without_its_library_fails_loudly(tmp_path, module):
    """The bindings have no fallback: a copy of a binding module with no built
    library beside it refuses to import, naming the missing library."""
    import subprocess
    import sys
    src = os.path.join(ROOT, "linear_memory_attention_b200", module)
    dst = tmp_path / module
    dst.write_text(open(src).read())
    out = subprocess.run([sys.executable, "-c", f"import {module[:-3]}"], cwd=tmp_path,
                         capture_output=True, text=True, timeout=300)
    assert out.returncode != 0
    assert "ImportError" in out.stderr and "is not built" in out.stderr
