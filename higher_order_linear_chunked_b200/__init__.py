"""B200 (sm_100a) masked Higher-order Linear Attention forward.

A thin ctypes binding over the C ABI of ``libhla.so`` (declared in
``include/hla.h``).  This module only marshals arguments: every step of the
computation runs in the library's CUDA kernels, on the tensors' device, on the
current torch stream.  PyTorch supplies device memory and streams.  There is no
CPU implementation here and no fallback: if the library is missing or the
tensors are not CUDA tensors, the calls raise.

Operations ("Higher-order Linear Attention" summary, gist.science 2510.27258):

* :func:`hla2` - second-order masked output (Metodología 1), optional per-head
  decay ``gamma`` (Contribuciones 2);
* :func:`hla2_normalized` - the ratio-normalised variant (Metodología 1);
* :func:`ahla` - asymmetric AHLA (Metodología 2);
* :func:`hla3` - third-order masked output (Metodología 3).

Inputs are ``[B, H, T, d]`` (``v``: ``[B, H, T, dv]``) contiguous fp32 or
bf16 tensors; the output is fp32 ``[B, H, T, dv]``.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libhla.so")

HLA_OK = 0
HLA_F32, HLA_BF16 = 0, 1
OP_HLA2, OP_HLA2_NORM, OP_AHLA, OP_HLA3, OP_HLA2_UNMASKED, OP_AHLA_NORM, OP_HLA3_NORM = 0, 1, 2, 3, 4, 5, 6

STATUS_NAMES = {0: "HLA_OK", 1: "HLA_ERR_NULL", 2: "HLA_ERR_SHAPE", 3: "HLA_ERR_ALIGN", 4: "HLA_ERR_DTYPE",
                5: "HLA_ERR_UNSUPPORTED", 6: "HLA_ERR_WORKSPACE", 7: "HLA_ERR_CUDA", 8: "HLA_ERR_TIMEOUT"}

# Every symbol include/hla.h declares.
EXPORTS = ("hla_abi_version", "hla_status_str", "hla_workspace_bytes", "hla2_forward", "hla2_forward_normalized",
           "ahla_forward", "hla3_forward", "hla_forward_profiled", "hla_kernel_launches", "hla_uses_tensor_cores", "hla_set_segment_chunks", "hla_read_device_status", "hla_selftest_umma", "hla_selftest_wait_timeout",
           "hla2_forward_normalized_noalloc", "hla_state_floats", "hla_state_workspace_bytes",
           "hla_state_kernel_launches", "hla_state", "hla_step", "hla2_forward_unmasked",
           "ahla_forward_normalized", "hla3_forward_normalized", "hla_noalloc_read_device_status",
           "hla_backward_workspace_bytes", "hla_backward_kernel_launches", "hla2_backward",
           "hla2_backward_normalized", "ahla_backward")


class HLAError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {STATUS_NAMES.get(status, status)}")


_lib = None


def load_library(path: Optional[str] = None):
    """Load ``libhla.so`` (raises OSError when it has not been built)."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise OSError(f"libhla.so not found at {p}: run higher_order_linear_chunked_b200.build.build() first")
    lib = ctypes.CDLL(p)
    vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    lib.hla_abi_version.argtypes, lib.hla_abi_version.restype = [], i
    lib.hla_status_str.argtypes, lib.hla_status_str.restype = [i], ctypes.c_char_p
    lib.hla_workspace_bytes.argtypes = [i, i, i, i, i, i, i, i]
    lib.hla_workspace_bytes.restype = sz
    common = [vp, vp, vp, vp, i, i, i, i, i, i, vp]
    for name in ("hla2_forward", "ahla_forward", "hla3_forward", "hla2_forward_unmasked"):
        fn = getattr(lib, name)
        fn.argtypes = common + [vp, sz, vp]
        fn.restype = i
    for name in ("hla2_forward_normalized", "ahla_forward_normalized", "hla3_forward_normalized"):
        fn = getattr(lib, name)
        fn.argtypes = common + [f, vp, sz, vp]
        fn.restype = i
    lib.hla_forward_profiled.argtypes = [i] + common + [f, vp, sz, vp, vp]
    lib.hla_forward_profiled.restype = i
    lib.hla_kernel_launches.argtypes = [i, i, i, i, i, i, i, i]
    lib.hla_kernel_launches.restype = i
    lib.hla_uses_tensor_cores.argtypes = [i, i, i, i, i, i, i, i]
    lib.hla_uses_tensor_cores.restype = i
    lib.hla_set_segment_chunks.argtypes = [i]
    lib.hla_set_segment_chunks.restype = i
    lib.hla_read_device_status.argtypes = [vp, vp, ctypes.POINTER(i)]
    lib.hla_read_device_status.restype = i
    lib.hla2_forward_normalized_noalloc.argtypes = common + [f, vp]
    lib.hla2_forward_normalized_noalloc.restype = i
    lib.hla_backward_workspace_bytes.argtypes = [i, i, i, i, i, i, i]
    lib.hla_backward_workspace_bytes.restype = sz
    lib.hla_backward_kernel_launches.argtypes = [i, i, i, i, i, i, i]
    lib.hla_backward_kernel_launches.restype = i
    lib.hla2_backward.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, vp, vp, sz, vp]
    lib.hla2_backward.restype = i
    lib.ahla_backward.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, vp, vp, sz, vp]
    lib.ahla_backward.restype = i
    lib.hla2_backward_normalized.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, vp, f, vp, sz, vp]
    lib.hla2_backward_normalized.restype = i
    lib.hla_noalloc_read_device_status.argtypes = [vp, ctypes.POINTER(i)]
    lib.hla_noalloc_read_device_status.restype = i
    lib.hla_selftest_umma.argtypes = [i, vp, vp, vp, i, i, vp]
    lib.hla_selftest_umma.restype = i
    lib.hla_selftest_wait_timeout.argtypes = [vp, sz, ctypes.c_uint, vp]
    lib.hla_selftest_wait_timeout.restype = i
    lib.hla_state_floats.argtypes, lib.hla_state_floats.restype = [i, i, i, i], sz
    lib.hla_state_workspace_bytes.argtypes = [i, i, i, i, i, i, i, i]
    lib.hla_state_workspace_bytes.restype = sz
    lib.hla_state_kernel_launches.argtypes = [i, i, i, i, i, i, i, i]
    lib.hla_state_kernel_launches.restype = i
    lib.hla_state.argtypes = [i, vp, vp, vp, vp, i, i, i, i, i, i, vp, vp, sz, vp]
    lib.hla_state.restype = i
    lib.hla_step.argtypes = [i, vp, vp, vp, vp, vp, i, i, i, i, i, vp, f, vp]
    lib.hla_step.restype = i
    if path is None:
        _lib = lib
    return lib


def _torch():
    import torch
    return torch


def _dtype_code(t) -> int:
    torch = _torch()
    if t.dtype == torch.float32:
        return HLA_F32
    if t.dtype == torch.bfloat16:
        return HLA_BF16
    raise TypeError(f"q, k, v must be float32 or bfloat16, got {t.dtype}")


def _check(q, k, v):
    for name, t in (("q", q), ("k", k), ("v", v)):
        if not t.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor (this library has no CPU path)")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
        if t.dim() != 4:
            raise ValueError(f"{name} must be [B, H, T, d]")
    if not (q.dtype == k.dtype == v.dtype):
        raise TypeError("q, k, v must share one dtype")
    if q.shape != k.shape or q.shape[:3] != v.shape[:3]:
        raise ValueError("shape mismatch: q, k [B,H,T,d], v [B,H,T,dv]")


def workspace_bytes(op: int, dtype_code: int, decayed: bool, B: int, H: int, T: int, d: int, dv: int) -> int:
    return int(load_library().hla_workspace_bytes(op, dtype_code, int(bool(decayed)), B, H, T, d, dv))


def kernel_launches(op: int, dtype_code: int, decayed: bool, B: int, H: int, T: int, d: int, dv: int) -> int:
    return int(load_library().hla_kernel_launches(op, dtype_code, int(bool(decayed)), B, H, T, d, dv))


def uses_tensor_cores(op: int, dtype_code: int, decayed: bool, B: int, H: int, T: int, d: int, dv: int) -> int:
    """1: the whole forward on tcgen05; 2: its output kernel only; 0: CUDA cores (hla_uses_tensor_cores)."""
    return int(load_library().hla_uses_tensor_cores(op, dtype_code, int(bool(decayed)), B, H, T, d, dv))


def set_segment_chunks(chunks: int) -> None:
    """Tensor-core path tuning: 128-token chunks per segment (0 = automatic)."""
    rc = load_library().hla_set_segment_chunks(int(chunks))
    if rc != HLA_OK:
        raise HLAError(rc, "hla_set_segment_chunks")


def make_workspace(op: int, q, v, decayed: bool = False):
    """Allocate (with torch, on q's device) a workspace sized for this call."""
    torch = _torch()
    B, H, T, d = q.shape
    n = workspace_bytes(op, _dtype_code(q), decayed, B, H, T, d, v.shape[-1])
    if n == 0:
        raise HLAError(5, "unsupported shape/dtype for this op")
    return torch.empty(n, dtype=torch.uint8, device=q.device)


def _call(op: int, q, k, v, gamma=None, eps: float = 1e-6, out=None, workspace=None, stream=None):
    torch = _torch()
    _check(q, k, v)
    lib = load_library()
    B, H, T, d = q.shape
    dv = v.shape[-1]
    if out is None:
        out = torch.empty((B, H, T, dv), dtype=torch.float32, device=q.device)
    if gamma is not None:
        if not gamma.is_cuda or gamma.dtype != torch.float32 or gamma.numel() != H or not gamma.is_contiguous():
            raise ValueError("gamma must be a contiguous CUDA float32 tensor of shape [H]")
    if workspace is None:
        workspace = make_workspace(op, q, v, decayed=gamma is not None)
    st = stream if stream is not None else torch.cuda.current_stream(q.device)
    sptr = ctypes.c_void_p(st.cuda_stream)
    gptr = ctypes.c_void_p(gamma.data_ptr()) if gamma is not None else ctypes.c_void_p(0)
    args = [ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()), ctypes.c_void_p(v.data_ptr()),
            ctypes.c_void_p(out.data_ptr()), B, H, T, d, dv, _dtype_code(q), gptr]
    ws = [ctypes.c_void_p(workspace.data_ptr()), ctypes.c_size_t(workspace.numel() * workspace.element_size()), sptr]
    if op == OP_HLA2:
        rc = lib.hla2_forward(*args, *ws)
    elif op == OP_HLA2_NORM:
        rc = lib.hla2_forward_normalized(*args, ctypes.c_float(eps), *ws)
    elif op == OP_AHLA:
        rc = lib.ahla_forward(*args, *ws)
    elif op == OP_HLA3:
        rc = lib.hla3_forward(*args, *ws)
    elif op == OP_HLA2_UNMASKED:
        rc = lib.hla2_forward_unmasked(*args, *ws)
    elif op == OP_AHLA_NORM:
        rc = lib.ahla_forward_normalized(*args, ctypes.c_float(eps), *ws)
    elif op == OP_HLA3_NORM:
        rc = lib.hla3_forward_normalized(*args, ctypes.c_float(eps), *ws)
    else:
        raise ValueError(op)
    if rc != HLA_OK:
        raise HLAError(rc, "HLA forward rejected the call")
    return out


def hla2(q, k, v, gamma=None, out=None, workspace=None, stream=None):
    """Second-order masked HLA forward (optional per-head decay gamma [H])."""
    return _call(OP_HLA2, q, k, v, gamma=gamma, out=out, workspace=workspace, stream=stream)


def hla2_normalized(q, k, v, eps: float = 1e-6, gamma=None, out=None, workspace=None, stream=None):
    """Ratio-normalised second-order masked HLA forward."""
    return _call(OP_HLA2_NORM, q, k, v, gamma=gamma, eps=eps, out=out, workspace=workspace, stream=stream)


def ahla(q, k, v, gamma=None, out=None, workspace=None, stream=None):
    """AHLA masked forward (optional per-head decay gamma [H])."""
    return _call(OP_AHLA, q, k, v, gamma=gamma, out=out, workspace=workspace, stream=stream)


def hla3(q, k, v, gamma=None, out=None, workspace=None, stream=None):
    """Third-order masked HLA forward (optional per-head decay gamma [H])."""
    return _call(OP_HLA3, q, k, v, gamma=gamma, out=out, workspace=workspace, stream=stream)


def hla2_unmasked(q, k, v, out=None, workspace=None, stream=None):
    """Unmasked second-order forward, o_t = q_t^T S_t C_t."""
    return _call(OP_HLA2_UNMASKED, q, k, v, out=out, workspace=workspace, stream=stream)


def hla2_backward(q, k, v, dout, workspace=None, stream=None, normalized: bool = False, eps: float = 1e-6):
    """Gradients (dq, dk, dv), fp32, of sum(O * dout) for O = hla2(q, k, v) (masked second order,
    no decay), or O = hla2_normalized(q, k, v, eps) with ``normalized``.  dout: fp32 [B, H, T, dv]
    on q's device."""
    return _backward(OP_HLA2_NORM if normalized else OP_HLA2, q, k, v, dout, workspace, stream, eps)


def ahla_backward(q, k, v, dout, workspace=None, stream=None):
    """Gradients (dq, dk, dv), fp32, of sum(O * dout) for O = ahla(q, k, v) (no decay)."""
    return _backward(OP_AHLA, q, k, v, dout, workspace, stream, 0.0)


def _backward(op, q, k, v, dout, workspace, stream, eps):
    torch = _torch()
    _check(q, k, v)
    if not dout.is_cuda or dout.dtype != torch.float32 or not dout.is_contiguous() or dout.shape != v.shape:
        raise ValueError("dout must be a contiguous CUDA float32 tensor shaped like v")
    lib = load_library()
    B, H, T, d = q.shape
    dvd = v.shape[-1]
    n = int(lib.hla_backward_workspace_bytes(op, _dtype_code(q), B, H, T, d, dvd))
    if n == 0:
        raise HLAError(5, "no backward kernel for this shape/dtype")
    if workspace is None:
        workspace = torch.empty(n, dtype=torch.uint8, device=q.device)
    dq = torch.empty((B, H, T, d), dtype=torch.float32, device=q.device)
    dk = torch.empty_like(dq)
    dv = torch.empty((B, H, T, dvd), dtype=torch.float32, device=q.device)
    st = stream if stream is not None else torch.cuda.current_stream(q.device)
    vp = ctypes.c_void_p
    head = [vp(q.data_ptr()), vp(k.data_ptr()), vp(v.data_ptr()), vp(dout.data_ptr()), vp(dq.data_ptr()),
            vp(dk.data_ptr()), vp(dv.data_ptr()), B, H, T, d, dvd, _dtype_code(q), vp(0)]
    tail = [vp(workspace.data_ptr()), ctypes.c_size_t(workspace.numel()), vp(st.cuda_stream)]
    if op == OP_HLA2_NORM:
        rc = lib.hla2_backward_normalized(*head, ctypes.c_float(eps), *tail)
    elif op == OP_AHLA:
        rc = lib.ahla_backward(*head, *tail)
    else:
        rc = lib.hla2_backward(*head, *tail)
    if rc != HLA_OK:
        raise HLAError(rc, "the backward call rejected it")
    return dq, dk, dv


def forward(op_name: str, q, k, v, gamma=None, eps: float = 1e-6, out=None, workspace=None, stream=None):
    """Dispatch by name: "hla2", "hla2n", "hla2d" (needs gamma), "ahla", "hla3", "hla2u",
    "ahlan", "hla3n" (ratio-normalised AHLA / third order), "ahlad", "hla3d" (AHLA / third order
    with decay: need gamma).  gamma, when given, selects the decayed form of any op but "hla2u"."""
    if op_name == "hla2":
        return hla2(q, k, v, out=out, workspace=workspace, stream=stream)
    if op_name == "hla2n":
        return hla2_normalized(q, k, v, eps=eps, gamma=gamma, out=out, workspace=workspace, stream=stream)
    if op_name == "hla2d":
        if gamma is None:
            raise ValueError("hla2d needs gamma")
        return hla2(q, k, v, gamma=gamma, out=out, workspace=workspace, stream=stream)
    if op_name in ("ahlad", "hla3d") and gamma is None:
        raise ValueError(f"{op_name} needs gamma")
    if op_name in ("ahla", "ahlad"):
        return ahla(q, k, v, gamma=gamma, out=out, workspace=workspace, stream=stream)
    if op_name in ("hla3", "hla3d"):
        return hla3(q, k, v, gamma=gamma, out=out, workspace=workspace, stream=stream)
    if op_name == "hla2u":
        return hla2_unmasked(q, k, v, out=out, workspace=workspace, stream=stream)
    if op_name == "ahlan":
        return _call(OP_AHLA_NORM, q, k, v, gamma=gamma, eps=eps, out=out, workspace=workspace, stream=stream)
    if op_name == "hla3n":
        return _call(OP_HLA3_NORM, q, k, v, gamma=gamma, eps=eps, out=out, workspace=workspace, stream=stream)
    raise ValueError(op_name)


OP_CODES = {"hla2": OP_HLA2, "hla2n": OP_HLA2_NORM, "hla2d": OP_HLA2, "ahla": OP_AHLA, "hla3": OP_HLA3,
            "hla2u": OP_HLA2_UNMASKED, "ahlan": OP_AHLA_NORM, "hla3n": OP_HLA3_NORM, "ahlad": OP_AHLA,
            "hla3d": OP_HLA3}


def read_device_status(workspace, stream=None) -> int:
    """Synchronise and return the device status word of the last call on ``workspace``."""
    torch = _torch()
    st = stream if stream is not None else torch.cuda.current_stream(workspace.device)
    s = ctypes.c_int(-1)
    rc = load_library().hla_read_device_status(ctypes.c_void_p(workspace.data_ptr()),
                                                ctypes.c_void_p(st.cuda_stream), ctypes.byref(s))
    if rc != HLA_OK:
        raise HLAError(rc, "hla_read_device_status")
    return s.value


def forward_profiled(op_name: str, q, k, v, events, gamma=None, eps: float = 1e-6, out=None, workspace=None,
                     stream=None):
    """Same as :func:`forward` through ``hla_forward_profiled``: ``events`` are four recorded-once
    ``torch.cuda.Event(enable_timing=True)`` objects the library records before the summary kernel,
    after it, after the scan and after the output kernel (on the call's stream)."""
    torch = _torch()
    _check(q, k, v)
    lib = load_library()
    B, H, T, d = q.shape
    dv = v.shape[-1]
    if out is None:
        out = torch.empty((B, H, T, dv), dtype=torch.float32, device=q.device)
    op = OP_CODES[op_name]
    if workspace is None:
        workspace = make_workspace(op, q, v, decayed=gamma is not None)
    st = stream if stream is not None else torch.cuda.current_stream(q.device)
    handles = (ctypes.c_void_p * 4)(*[ctypes.c_void_p(e.cuda_event) for e in events])
    rc = lib.hla_forward_profiled(
        op, ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()), ctypes.c_void_p(v.data_ptr()),
        ctypes.c_void_p(out.data_ptr()), B, H, T, d, dv, _dtype_code(q),
        ctypes.c_void_p(gamma.data_ptr()) if gamma is not None else ctypes.c_void_p(0), ctypes.c_float(eps),
        ctypes.c_void_p(workspace.data_ptr()), ctypes.c_size_t(workspace.numel()),
        ctypes.c_void_p(st.cuda_stream), ctypes.cast(handles, ctypes.c_void_p))
    if rc != HLA_OK:
        raise HLAError(rc, "hla_forward_profiled rejected the call")
    return out


# ---------------------------------------------------------------------------
# streaming state: prefill (state after T tokens) and one-token decode steps
# ---------------------------------------------------------------------------

DECAYED_OPS = ("hla2d", "ahlad", "hla3d")


def _rho_offset(op_name: str, d: int) -> int:
    """Float offset of rho in a decayed state: after the op family's matrices and vectors."""
    if op_name in ("hla2", "hla2n", "hla2d"):
        return 4 * d * d + 2 * d
    if op_name in ("ahla", "ahlan", "ahlad"):
        return 3 * d * d + 2 * d
    return 6 * d * d + 3 * d


def state_floats(op_name: str, d: int, dv: int, decayed=None) -> int:
    """Floats of one head's streaming state for ``op_name`` (see ``hla_state_floats``);
    ``decayed`` defaults to the op name's own ("hla2d", "ahlad", "hla3d"); pass True for a
    plain or ratio-normalised op used with gamma."""
    dec = op_name in DECAYED_OPS if decayed is None else bool(decayed)
    return int(load_library().hla_state_floats(OP_CODES[op_name], int(dec), d, dv))


def new_state(op_name: str, B: int, H: int, d: int, device="cuda", decayed=None):
    """The state of zero tokens: zeros, with rho = 1 for the decayed form."""
    torch = _torch()
    dec = op_name in DECAYED_OPS if decayed is None else bool(decayed)
    n = state_floats(op_name, d, d, decayed=dec)
    if n == 0:
        raise HLAError(5, "no streaming state for this op / d")
    st = torch.zeros((B, H, n), dtype=torch.float32, device=device)
    if dec:
        st[..., _rho_offset(op_name, d)] = 1.0
    return st


def state(op_name: str, q, k, v, gamma=None, out=None, workspace=None, stream=None):
    """Prefill: the streaming state [B, H, state_floats] of every head after its T tokens."""
    torch = _torch()
    _check(q, k, v)
    lib = load_library()
    B, H, T, d = q.shape
    dv = v.shape[-1]
    op = OP_CODES[op_name]
    decayed = op_name in DECAYED_OPS or (gamma is not None and op_name != "hla2u")
    if op_name in DECAYED_OPS and gamma is None:
        raise ValueError(f"{op_name} needs gamma")
    n = int(lib.hla_state_floats(op, int(decayed), d, dv))
    if out is None:
        out = torch.empty((B, H, n), dtype=torch.float32, device=q.device)
    if workspace is None:
        nb = int(lib.hla_state_workspace_bytes(op, _dtype_code(q), int(decayed), B, H, T, d, dv))
        if nb == 0:
            raise HLAError(5, "unsupported shape/dtype for this op")
        workspace = torch.empty(nb, dtype=torch.uint8, device=q.device)
    st = stream if stream is not None else torch.cuda.current_stream(q.device)
    rc = lib.hla_state(op, ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
                       ctypes.c_void_p(v.data_ptr()), ctypes.c_void_p(out.data_ptr()), B, H, T, d, dv,
                       _dtype_code(q), ctypes.c_void_p(gamma.data_ptr()) if gamma is not None else ctypes.c_void_p(0),
                       ctypes.c_void_p(workspace.data_ptr()), ctypes.c_size_t(workspace.numel()),
                       ctypes.c_void_p(st.cuda_stream))
    if rc != HLA_OK:
        raise HLAError(rc, "hla_state rejected the call")
    return out


def step(op_name: str, state_io, q, k, v, gamma=None, eps: float = 1e-6, out=None, stream=None):
    """Decode one token per head: q, k, v [B, H, d]; advances ``state_io`` in place; returns o [B, H, dv]."""
    torch = _torch()
    if op_name in DECAYED_OPS and gamma is None:
        raise ValueError(f"{op_name} needs gamma")
    for name, t in (("q", q), ("k", k), ("v", v), ("state", state_io)):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA tensor")
    if q.dim() != 3 or q.shape != k.shape or q.shape[:2] != v.shape[:2]:
        raise ValueError("q, k [B,H,d], v [B,H,dv]")
    if state_io.dtype != torch.float32:
        raise TypeError("state must be float32")
    B, H, d = q.shape
    dv = v.shape[-1]
    if out is None:
        out = torch.empty((B, H, dv), dtype=torch.float32, device=q.device)
    st = stream if stream is not None else torch.cuda.current_stream(q.device)
    rc = load_library().hla_step(
        OP_CODES[op_name], ctypes.c_void_p(state_io.data_ptr()), ctypes.c_void_p(q.data_ptr()),
        ctypes.c_void_p(k.data_ptr()), ctypes.c_void_p(v.data_ptr()), ctypes.c_void_p(out.data_ptr()),
        B, H, d, dv, _dtype_code(q), ctypes.c_void_p(gamma.data_ptr()) if gamma is not None else ctypes.c_void_p(0),
        ctypes.c_float(eps), ctypes.c_void_p(st.cuda_stream))
    if rc != HLA_OK:
        raise HLAError(rc, "hla_step rejected the call")
    return out
