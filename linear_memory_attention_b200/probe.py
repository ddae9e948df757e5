"""ctypes binding of liblard_probe (include/lard_probe.h): the throughput probe
of the exponential units that the benchmark measures its Phase-1 peak with."""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "liblard_probe.so")
EXPORTS = ("lard_probe_exp_rate",)
KINDS = {"ex2_f32": 0, "ex2_f16x2": 1, "exp2_fma_pair": 2, "ex2_f16x2_via_f32": 3}


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"liblard_probe.so is not built ({LIB_PATH}); build it with "
                          "`python -m linear_memory_attention_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    lib.lard_probe_exp_rate.restype = ctypes.c_int
    lib.lard_probe_exp_rate.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                        ctypes.POINTER(ctypes.c_float), ctypes.POINTER(ctypes.c_double),
                                        ctypes.c_void_p]
    return lib


_lib = _load()


def exp_rate(kind: str, blocks: int, iters: int, stream=None):
    """Run one probe kernel; returns (elapsed ms, exponentials computed)."""
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    ms, exps = ctypes.c_float(0.0), ctypes.c_double(0.0)
    rc = _lib.lard_probe_exp_rate(KINDS[kind], int(blocks), int(iters), ctypes.byref(ms), ctypes.byref(exps),
                                  ctypes.c_void_p(stream.cuda_stream))
    if rc != 0:
        raise RuntimeError(f"lard_probe_exp_rate({kind}) failed with {rc}")
    return float(ms.value), float(exps.value)
