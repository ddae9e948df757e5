"""ctypes binding of liblard (the C ABI declared in include/lard.h).

Argument marshalling only: tensors are passed as raw device pointers with
their sizes and the current CUDA stream; every step of the computation runs
in the library's kernels.  Importing this module fails loudly if the library
has not been built.

Functions keep the C names:
    lard_kl_fwd(Xt, Yt, Xs, Ys, tau, causal, lse_t, lse_s, row_kl,
                loss_bh=None, loss_total=None, stream=None)
    lard_kl_bwd(Xt, Yt, Xs, Ys, tau, causal, lse_t, lse_s, grad_scale,
                dXs, dYs, stream=None)
    lard_kl_bwd_self(Xt, Xs, tau, causal, lse_t, lse_s, grad_scale, dXs,
                     stream=None)
    lard_kl_fwd_multi(relations, tau, causal, loss_total=None, stream=None)
    lard_kl_bwd_multi(relations, tau, causal, grad_scale, stream=None)
    lard_kl_bwd_multi_bf16(relations, tau, causal, grad_scale, workspace, stream=None)
    lard_kl_bwd_bf16_workspace_bytes(relations) -> bytes
    lard_kl_bwd_multi_bf16_noalloc(relations, tau, causal, grad_scale, stream=None)
    lard_device_status(stream=None) -> fault bits (raises on timeout)
    lard_status_string(code), lard_version()
Tensors are torch tensors [B, H, n, d] (inputs bf16 or fp32, outputs fp32 except
the bf16 gradients of lard_kl_bwd_multi_bf16), contiguous, on the GPU that runs the call.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "liblard.so")

LARD_OK, LARD_ERR_INVALID_ARG, LARD_ERR_UNSUPPORTED, LARD_ERR_CUDA, LARD_ERR_TIMEOUT, LARD_ERR_TOO_LARGE = range(6)
LARD_NOALLOC_WORKSPACE_BYTES = 64 << 20
LARD_DTYPE_BF16, LARD_DTYPE_FP32 = 0, 1

EXPORTS = ("lard_kl_fwd", "lard_kl_bwd", "lard_kl_bwd_self", "lard_kl_fwd_multi",
           "lard_kl_bwd_multi", "lard_kl_bwd_bf16_workspace_bytes", "lard_kl_bwd_multi_bf16",
           "lard_kl_bwd_multi_bf16_noalloc",
           "lard_status_string", "lard_device_status", "lard_selftest_timeout", "lard_version")
LARD_MAX_RELATIONS = 4


class _Relation(ctypes.Structure):
    """struct lard_relation of include/lard.h."""
    _fields_ = [("Xt", ctypes.c_void_p), ("Yt", ctypes.c_void_p), ("Xs", ctypes.c_void_p),
                ("Ys", ctypes.c_void_p), ("H", ctypes.c_int), ("lse_t", ctypes.c_void_p),
                ("lse_s", ctypes.c_void_p), ("row_kl", ctypes.c_void_p), ("loss_bh", ctypes.c_void_p),
                ("dXs", ctypes.c_void_p), ("dYs", ctypes.c_void_p)]


class _Bf16Grads(ctypes.Structure):
    """struct lard_grads_bf16 of include/lard.h."""
    _fields_ = [("dXs", ctypes.c_void_p), ("dYs", ctypes.c_void_p)]


class LardError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {_status_name(status)}")


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"liblard.so is not built ({LIB_PATH}); build it with "
            "`python -m linear_memory_attention_b200.build` (nvcc, sm_100a)")
    lib = ctypes.CDLL(LIB_PATH)
    vp, f32p, i, f = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    lib.lard_kl_fwd.restype = i
    lib.lard_kl_fwd.argtypes = [vp, vp, vp, vp, i, i, i, i, i, f, i, f32p, f32p, f32p, f32p, f32p, vp]
    lib.lard_kl_bwd.restype = i
    lib.lard_kl_bwd.argtypes = [vp, vp, vp, vp, i, i, i, i, i, f, i, f32p, f32p, f, f32p, f32p, vp]
    lib.lard_kl_bwd_self.restype = i
    lib.lard_kl_bwd_self.argtypes = [vp, vp, i, i, i, i, i, f, i, f32p, f32p, f, f32p, vp]
    rp = ctypes.POINTER(_Relation)
    lib.lard_kl_fwd_multi.restype = i
    lib.lard_kl_fwd_multi.argtypes = [rp, i, i, i, i, i, f, i, f32p, vp]
    lib.lard_kl_bwd_multi.restype = i
    lib.lard_kl_bwd_multi.argtypes = [rp, i, i, i, i, i, f, i, f, vp]
    g16p = ctypes.POINTER(_Bf16Grads)
    lib.lard_kl_bwd_bf16_workspace_bytes.restype = ctypes.c_size_t
    lib.lard_kl_bwd_bf16_workspace_bytes.argtypes = [rp, i, i, i, i]
    lib.lard_kl_bwd_multi_bf16.restype = i
    lib.lard_kl_bwd_multi_bf16.argtypes = [rp, g16p, i, i, i, i, i, f, i, f, vp, ctypes.c_size_t, vp]
    lib.lard_kl_bwd_multi_bf16_noalloc.restype = i
    lib.lard_kl_bwd_multi_bf16_noalloc.argtypes = [rp, g16p, i, i, i, i, i, f, i, f, vp]
    lib.lard_status_string.restype = ctypes.c_char_p
    lib.lard_status_string.argtypes = [i]
    lib.lard_device_status.restype = i
    lib.lard_device_status.argtypes = [vp, ctypes.POINTER(ctypes.c_uint)]
    lib.lard_selftest_timeout.restype = i
    lib.lard_selftest_timeout.argtypes = [ctypes.c_uint, vp]
    lib.lard_version.restype = i
    lib.lard_version.argtypes = []
    return lib


_lib = _load()


def _status_name(code: int) -> str:
    return _lib.lard_status_string(int(code)).decode()


def lard_status_string(code: int) -> str:
    return _status_name(code)


def lard_version() -> int:
    return int(_lib.lard_version())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream, like=None):
    """The CUDA stream handle to enqueue on: ``stream`` if given, else the current
    stream of the GPU that holds ``like`` (the call's first input)."""
    import torch
    if stream is None:
        dev = like.device if like is not None and like.is_cuda else None
        stream = torch.cuda.current_stream(dev)
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _shape(Xt):
    import torch
    if Xt.dim() != 4:
        raise ValueError("inputs must be [B, H, n, d]")
    if Xt.dtype == torch.bfloat16:
        dt = LARD_DTYPE_BF16
    elif Xt.dtype == torch.float32:
        dt = LARD_DTYPE_FP32
    else:
        raise ValueError(f"unsupported input dtype {Xt.dtype}")
    B, H, n, d = Xt.shape
    return dt, int(B), int(H), int(n), int(d)


def _check_inputs(Xt, Yt, Xs, Ys):
    for t in (Xt, Yt, Xs, Ys):
        if t.shape != Xt.shape or t.dtype != Xt.dtype or not t.is_contiguous():
            raise ValueError("inputs must share one shape and dtype and be contiguous")
        if t.device != Xt.device:
            raise ValueError("inputs must be on one device")


def _check_out(t, numel, like, name, dtype=None, optional=False):
    """An output buffer the library writes: the C side cannot see its size, so a
    wrong dtype or a short buffer would be written past its end.  Requires a
    contiguous tensor of ``numel`` elements of ``dtype`` (float32 by default) on
    the device of ``like``."""
    import torch
    if t is None:
        if optional:
            return
        raise ValueError(f"{name}: output buffer required")
    dtype = torch.float32 if dtype is None else dtype
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name}: expected a torch tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name}: expected {dtype}, got {t.dtype}")
    if t.numel() != numel:
        raise ValueError(f"{name}: expected {numel} elements, got {t.numel()}")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")
    if t.device != like.device:
        raise ValueError(f"{name}: on {t.device}, inputs on {like.device}")


def _check_fwd_outs(Xt, H, lse_t, lse_s, row_kl, loss_bh, loss_total=None, total_optional=True):
    B, n = Xt.shape[0], Xt.shape[2]
    for name, t in (("lse_t", lse_t), ("lse_s", lse_s), ("row_kl", row_kl)):
        _check_out(t, B * H * n, Xt, name)
    _check_out(loss_bh, B * H, Xt, "loss_bh", optional=True)
    _check_out(loss_total, 1, Xt, "loss_total", optional=total_optional)


def _check_grad(t, Xt, H, name, optional=False, dtype=None):
    B, n, d = Xt.shape[0], Xt.shape[2], Xt.shape[3]
    _check_out(t, B * H * n * d, Xt, name, dtype=dtype, optional=optional)


def lard_kl_fwd(Xt, Yt, Xs, Ys, tau, causal, lse_t, lse_s, row_kl, loss_bh=None, loss_total=None,
                stream=None):
    """Phase 1: writes lse_t, lse_s, row_kl [B,H,n] and optionally loss_bh [B*H], loss_total [1]."""
    _check_inputs(Xt, Yt, Xs, Ys)
    dt, B, H, n, d = _shape(Xt)
    _check_fwd_outs(Xt, H, lse_t, lse_s, row_kl, loss_bh, loss_total)
    st = _lib.lard_kl_fwd(_ptr(Xt), _ptr(Yt), _ptr(Xs), _ptr(Ys), dt, B, H, n, d, float(tau),
                          int(bool(causal)), _ptr(lse_t), _ptr(lse_s), _ptr(row_kl), _ptr(loss_bh),
                          _ptr(loss_total), _stream(stream, Xt))
    if st != LARD_OK:
        raise LardError(st, "lard_kl_fwd")


def lard_kl_bwd(Xt, Yt, Xs, Ys, tau, causal, lse_t, lse_s, grad_scale, dXs, dYs, stream=None):
    """Phase 2: overwrites dXs, dYs [B,H,n,d] fp32 with grad_scale * dL/dXs, dL/dYs."""
    _check_inputs(Xt, Yt, Xs, Ys)
    dt, B, H, n, d = _shape(Xt)
    for name, t in (("lse_t", lse_t), ("lse_s", lse_s)):
        _check_out(t, B * H * n, Xt, name)
    _check_grad(dXs, Xt, H, "dXs")
    _check_grad(dYs, Xt, H, "dYs")
    st = _lib.lard_kl_bwd(_ptr(Xt), _ptr(Yt), _ptr(Xs), _ptr(Ys), dt, B, H, n, d, float(tau),
                          int(bool(causal)), _ptr(lse_t), _ptr(lse_s), float(grad_scale),
                          _ptr(dXs), _ptr(dYs), _stream(stream, Xt))
    if st != LARD_OK:
        raise LardError(st, "lard_kl_bwd")


def lard_kl_bwd_self(Xt, Xs, tau, causal, lse_t, lse_s, grad_scale, dXs, stream=None):
    """Phase 2 of a self-relation: overwrites dXs [B,H,n,d] fp32 with grad_scale * dL/dXs
    through both of Xs's roles (the sum of lard_kl_bwd's dXs and dYs).  bf16 inputs only."""
    for t in (Xt, Xs):
        if t.shape != Xt.shape or t.dtype != Xt.dtype or not t.is_contiguous():
            raise ValueError("inputs must share one shape and dtype and be contiguous")
    if Xs.device != Xt.device:
        raise ValueError("inputs must be on one device")
    dt, B, H, n, d = _shape(Xt)
    for name, t in (("lse_t", lse_t), ("lse_s", lse_s)):
        _check_out(t, B * H * n, Xt, name)
    _check_grad(dXs, Xt, H, "dXs")
    st = _lib.lard_kl_bwd_self(_ptr(Xt), _ptr(Xs), dt, B, H, n, d, float(tau), int(bool(causal)),
                               _ptr(lse_t), _ptr(lse_s), float(grad_scale), _ptr(dXs),
                               _stream(stream, Xt))
    if st != LARD_OK:
        raise LardError(st, "lard_kl_bwd_self")


def _relations(rels, phase):
    """ctypes array of lard_relation from dicts with the field names (tensors or None).
    ``phase`` ("fwd" or "bwd") selects which output buffers are checked and passed;
    fields the phase does not use are passed as NULL."""
    if not 1 <= len(rels) <= LARD_MAX_RELATIONS:
        raise ValueError(f"1 to {LARD_MAX_RELATIONS} relations per call")
    arr = (_Relation * len(rels))()
    B = n = d = dt = None
    for k, r in enumerate(rels):
        Xt, Xs = r["Xt"], r["Xs"]
        Yt, Ys = r.get("Yt", Xt), r.get("Ys", Xs)
        _check_inputs(Xt, Yt, Xs, Ys)
        dtk, Bk, Hk, nk, dk = _shape(Xt)
        if B is None:
            dt, B, n, d = dtk, Bk, nk, dk
        elif (dtk, Bk, nk, dk) != (dt, B, n, d):
            raise ValueError("relations of one call must share dtype, B, n and d")
        arr[k].Xt, arr[k].Yt, arr[k].Xs, arr[k].Ys = (t.data_ptr() for t in (Xt, Yt, Xs, Ys))
        if Xt.device != rels[0]["Xt"].device:
            raise ValueError("relations of one call must be on one device")
        arr[k].H = Hk
        for name in ("lse_t", "lse_s"):
            _check_out(r.get(name), Bk * Hk * nk, Xt, name)
        if phase == "fwd":
            _check_out(r.get("row_kl"), Bk * Hk * nk, Xt, "row_kl")
            _check_out(r.get("loss_bh"), Bk * Hk, Xt, "loss_bh", optional=True)
            used = ("lse_t", "lse_s", "row_kl", "loss_bh")
        elif phase == "bwd_outputs_elsewhere":  # the gradients are passed apart (bf16 outputs)
            used = ("lse_t", "lse_s")
        else:
            _check_grad(r.get("dXs"), Xt, Hk, "dXs")
            _check_grad(r.get("dYs"), Xt, Hk, "dYs", optional=True)
            used = ("lse_t", "lse_s", "dXs", "dYs")
        for name in used:
            t = r.get(name)
            setattr(arr[k], name, None if t is None else t.data_ptr())
    return arr, dt, B, n, d


def lard_kl_fwd_multi(relations, tau, causal, loss_total=None, stream=None):
    """Phase 1 of up to 4 relations in one launch.  ``relations``: dicts with Xt, Xs (and
    optionally Yt, Ys; default Y = X), lse_t, lse_s, row_kl and optionally loss_bh."""
    arr, dt, B, n, d = _relations(relations, "fwd")
    Xt0 = relations[0]["Xt"]
    _check_out(loss_total, 1, Xt0, "loss_total", optional=True)
    if loss_total is not None and any(r.get("loss_bh") is None for r in relations):
        raise ValueError("loss_total needs every relation's loss_bh")
    st = _lib.lard_kl_fwd_multi(arr, len(relations), dt, B, n, d, float(tau), int(bool(causal)),
                                _ptr(loss_total), _stream(stream, Xt0))
    if st != LARD_OK:
        raise LardError(st, "lard_kl_fwd_multi")


def lard_kl_bwd_multi(relations, tau, causal, grad_scale, stream=None):
    """Phase 2 of up to 4 relations in one launch.  ``relations``: dicts as for
    lard_kl_fwd_multi with lse_t, lse_s, dXs and dYs; dYs None for a self-relation adds
    both gradient paths into dXs."""
    arr, dt, B, n, d = _relations(relations, "bwd")
    st = _lib.lard_kl_bwd_multi(arr, len(relations), dt, B, n, d, float(tau), int(bool(causal)),
                                float(grad_scale), _stream(stream, relations[0]["Xt"]))
    if st != LARD_OK:
        raise LardError(st, "lard_kl_bwd_multi")


def lard_kl_bwd_bf16_workspace_bytes(relations) -> int:
    """Bytes of fp32 workspace lard_kl_bwd_multi_bf16 needs for these relations."""
    arr = (_Relation * len(relations))()
    for k, r in enumerate(relations):
        arr[k].H = int(r["Xt"].shape[1])
    B, _, n, d = relations[0]["Xt"].shape
    return int(_lib.lard_kl_bwd_bf16_workspace_bytes(arr, len(relations), int(B), int(n), int(d)))


def lard_kl_bwd_multi_bf16(relations, tau, causal, grad_scale, workspace, stream=None):
    """Phase 2 of up to 4 relations with bf16 gradient outputs: each relation dict
    holds dXs (bf16 [B,H,n,d]) and dYs (bf16, or None for a self-relation, whose
    total gradient then goes to dXs).  ``workspace`` is a device tensor of at least
    lard_kl_bwd_bf16_workspace_bytes(relations) bytes, overwritten."""
    import torch
    arr, dt, B, n, d = _relations([{k: v for k, v in r.items() if k not in ("dXs", "dYs")}
                                   for r in relations], "bwd_outputs_elsewhere")
    out = (_Bf16Grads * len(relations))()
    for k, r in enumerate(relations):
        H = int(r["Xt"].shape[1])
        _check_grad(r.get("dXs"), r["Xt"], H, "dXs", dtype=torch.bfloat16)
        _check_grad(r.get("dYs"), r["Xt"], H, "dYs", dtype=torch.bfloat16, optional=True)
        out[k].dXs = r["dXs"].data_ptr()
        out[k].dYs = None if r.get("dYs") is None else r["dYs"].data_ptr()
    Xt0 = relations[0]["Xt"]
    need = lard_kl_bwd_bf16_workspace_bytes(relations)
    if not isinstance(workspace, torch.Tensor) or not workspace.is_contiguous() or workspace.device != Xt0.device:
        raise ValueError("workspace: a contiguous device tensor on the inputs' device")
    nbytes = workspace.numel() * workspace.element_size()
    if nbytes < need:
        raise ValueError(f"workspace: {nbytes} bytes, {need} needed")
    st = _lib.lard_kl_bwd_multi_bf16(arr, out, len(relations), dt, B, n, d, float(tau), int(bool(causal)),
                                     float(grad_scale), ctypes.c_void_p(workspace.data_ptr()), nbytes,
                                     _stream(stream, Xt0))
    if st != LARD_OK:
        raise LardError(st, "lard_kl_bwd_multi_bf16")


def lard_kl_bwd_multi_bf16_noalloc(relations, tau, causal, grad_scale, stream=None):
    """lard_kl_bwd_multi_bf16 without a workspace argument, for callers that cannot
    allocate device memory: the library's fixed LARD_NOALLOC_WORKSPACE_BYTES array
    is used instead.  Calls that can overlap on the GPU race on that array."""
    import torch
    arr, dt, B, n, d = _relations([{k: v for k, v in r.items() if k not in ("dXs", "dYs")}
                                   for r in relations], "bwd_outputs_elsewhere")
    out = (_Bf16Grads * len(relations))()
    for k, r in enumerate(relations):
        H = int(r["Xt"].shape[1])
        _check_grad(r.get("dXs"), r["Xt"], H, "dXs", dtype=torch.bfloat16)
        _check_grad(r.get("dYs"), r["Xt"], H, "dYs", dtype=torch.bfloat16, optional=True)
        out[k].dXs = r["dXs"].data_ptr()
        out[k].dYs = None if r.get("dYs") is None else r["dYs"].data_ptr()
    st = _lib.lard_kl_bwd_multi_bf16_noalloc(arr, out, len(relations), dt, B, n, d, float(tau),
                                             int(bool(causal)), float(grad_scale),
                                             _stream(stream, relations[0]["Xt"]))
    if st != LARD_OK:
        raise LardError(st, "lard_kl_bwd_multi_bf16_noalloc")


def relations_kl(pairs, tau, causal=True, grad_scale=1.0, backward=True, fused_self=False,
                 grad_dtype="fp32", stream=None):
    """Both phases for several self-relations [(Xt, Xs), ...] in one launch per phase.

    Returns (outputs per relation, loss): each output dict holds lse_t, lse_s, row_kl,
    loss_bh and, if ``backward``, dXs (the total gradient if ``fused_self``) and dYs
    (absent if ``fused_self``), in ``grad_dtype`` ("fp32" or "bf16"); loss is the
    summed loss of all relations (1 element).
    """
    import torch
    gdt = {"fp32": torch.float32, "bf16": torch.bfloat16}[grad_dtype]
    outs, rels = [], []
    for Xt, Xs in pairs:
        B, H, n, d = Xt.shape
        f32 = dict(device=Xt.device, dtype=torch.float32)
        o = {"lse_t": torch.empty((B, H, n), **f32), "lse_s": torch.empty((B, H, n), **f32),
             "row_kl": torch.empty((B, H, n), **f32), "loss_bh": torch.empty((B * H,), **f32)}
        if backward:
            o["dXs"] = torch.empty((B, H, n, d), device=Xt.device, dtype=gdt)
            if not fused_self:
                o["dYs"] = torch.empty((B, H, n, d), device=Xt.device, dtype=gdt)
        outs.append(o)
        rels.append(dict(Xt=Xt, Xs=Xs, **o))
    loss = torch.empty((1,), device=pairs[0][0].device, dtype=torch.float32)
    lard_kl_fwd_multi(rels, tau, causal, loss, stream)
    if backward:
        if grad_dtype == "fp32":
            lard_kl_bwd_multi(rels, tau, causal, grad_scale, stream)
        else:
            ws = torch.empty((lard_kl_bwd_bf16_workspace_bytes(rels),), device=pairs[0][0].device,
                             dtype=torch.uint8)
            lard_kl_bwd_multi_bf16(rels, tau, causal, grad_scale, ws, stream)
    return outs, loss


def lard_device_status(stream=None) -> int:
    """Synchronise the stream and check the kernels' fault word; raises on a timed-out wait."""
    bits = ctypes.c_uint(0)
    st = _lib.lard_device_status(_stream(stream), ctypes.byref(bits))
    if st != LARD_OK:
        err = LardError(st, f"lard_device_status (fault bits 0x{bits.value:x})")
        err.fault_bits = bits.value
        raise err
    return bits.value


def lard_selftest_timeout(limit_us: int, stream=None) -> None:
    """Enqueue the bounded-wait self-test kernel (its wait runs out after limit_us)."""
    st = _lib.lard_selftest_timeout(int(limit_us), _stream(stream))
    if st != LARD_OK:
        raise LardError(st, "lard_selftest_timeout")


def relation_kl(Xt, Xs, tau, causal=True, Yt=None, Ys=None, grad_scale=1.0, backward=True,
                stream=None):
    """Allocate the outputs and run both phases for one relation.

    Returns a dict with lse_t, lse_s, row_kl, loss_bh, loss (a 1-element
    tensor) and, if ``backward``, dXs and dYs.  Y defaults to X (self-relation).
    """
    import torch
    Yt = Xt if Yt is None else Yt
    Ys = Xs if Ys is None else Ys
    B, H, n, d = Xt.shape
    dev = Xt.device
    f32 = dict(device=dev, dtype=torch.float32)
    out = {"lse_t": torch.empty((B, H, n), **f32), "lse_s": torch.empty((B, H, n), **f32),
           "row_kl": torch.empty((B, H, n), **f32), "loss_bh": torch.empty((B * H,), **f32),
           "loss": torch.empty((1,), **f32)}
    lard_kl_fwd(Xt, Yt, Xs, Ys, tau, causal, out["lse_t"], out["lse_s"], out["row_kl"],
                out["loss_bh"], out["loss"], stream)
    if backward:
        out["dXs"] = torch.empty((B, H, n, d), **f32)
        out["dYs"] = torch.empty((B, H, n, d), **f32)
        lard_kl_bwd(Xt, Yt, Xs, Ys, tau, causal, out["lse_t"], out["lse_s"], grad_scale,
                    out["dXs"], out["dYs"], stream)
    return out
