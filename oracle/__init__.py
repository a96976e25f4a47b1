"""fp64 CPU oracle for the strictly causal masked HLA forward.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import this package.  The
CUDA library (``higher_order_linear_chunked_b200``) never imports it and shares
no code with it; the only module both sides use is ``hla_inputs`` (seeded
random inputs, no arithmetic of the method).

Contents
--------
* :func:`recur` - the serial token-by-token recurrences (plain C, fp64,
  ``oracle/hla_oracle.c``), one host thread per head.  This is the reference
  for every full-size parity check and the timed CPU baseline.
* :mod:`oracle.brute` - the O(T^3) masked-matrix definitions (numpy, fp64).
* :mod:`oracle.segments` - segment summaries, the semidirect-product combine
  maps and a Blelloch exclusive scan over them, on the host in fp64.
* :mod:`oracle.backward` - gradients of the second-order forward (reverse-mode
  differentiation of the masked-matrix definition, torch CPU float64).
* :func:`max_row_rel_err` - the parity metric.

All formulas come from "Resumen Técnico: Atención Lineal de Orden Superior
(HLA)" (gist.science, paper 2510.27258), sections Metodología 1-4 and
Contribuciones 1-3; each function cites its passage.

Pinning.  Every op is pinned to literal sums, brute force, closed forms and
invariants of the operator as read from the page.  Three readings have no
printed counterpart to pin against (parity unpinned against the page's own
algebra): the decay rule (the page gives no decayed formula), the third-order
nine-summary algebra (named, not printed), and the AHLA / third-order
normalisers (named, not printed; read as the operator on a ones value column).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "hla_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None

OPS = {"hla2": 0, "hla2n": 1, "hla2d": 2, "ahla": 3, "hla3": 4, "hla2u": 5, "ahlan": 6, "hla3n": 7,
       "ahlad": 3, "hla3d": 4}
# op names that require a gamma (the decayed forms); every other op except "hla2u" takes an
# optional gamma that selects its decayed form
DECAYED = ("hla2d", "ahlad", "hla3d")


def build(force: bool = False) -> str:
    """Compile ``hla_oracle.c`` into ``liboracle.so`` beside it (gcc, -O2, no fast-math)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-pthread", "-o", _LIB_PATH, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        dp = ctypes.POINTER(ctypes.c_double)
        i = ctypes.c_int
        lib.oracle_forward.argtypes = [i, i, i, i, i, i, dp, dp, dp, dp, ctypes.c_double, dp, i]
        lib.oracle_forward.restype = i
        lib.oracle_hla2_head.argtypes = [dp, dp, dp, i, i, i, i, ctypes.c_double, i, ctypes.c_double,
                                         dp, dp, dp, dp, dp, dp]
        lib.oracle_hla2_head.restype = None
        lib.oracle_ahla_head.argtypes = [dp, dp, dp, i, i, i, i, ctypes.c_double, dp, dp, dp]
        lib.oracle_ahla_head.restype = None
        lib.oracle_hla3_head.argtypes = [dp, dp, dp, i, i, i, i, ctypes.c_double, dp, dp, dp, dp]
        lib.oracle_hla3_head.restype = None
        lib.oracle_hla2u_head.argtypes = [dp, dp, dp, i, i, i, dp, dp, dp]
        lib.oracle_hla2u_head.restype = None
        _lib = lib
    return _lib


def _f64(x) -> np.ndarray:
    """Widen a torch tensor or array to a C-contiguous float64 numpy array."""
    if hasattr(x, "detach"):
        x = x.detach().to("cpu")
        import torch  # local: only when handed torch tensors
        x = x.to(torch.float64).numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a: Optional[np.ndarray]):
    if a is None:
        return ctypes.POINTER(ctypes.c_double)()
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def recur(op: str, q, k, v, gamma=None, eps: float = 1e-6, nthreads: Optional[int] = None) -> np.ndarray:
    """Serial recurrence for all heads: q, k [B,H,T,d], v [B,H,T,dv] -> o [B,H,T,dv] (fp64).

    op: "hla2" (Metodología 1 output), "hla2n" (ratio-normalised, Metodología 1
    "Normalización"), "hla2d" (decayed, Contribuciones 2; gamma [H]), "ahla"
    (Metodología 2), "hla3" (Metodología 3), "hla2u" (the unmasked configuration of
    Contribuciones 2: o_t = q_t^T S_t C_t), "ahlan" / "hla3n" (ratio-normalised: divided by
    the same operator on a ones value column, plus eps), "ahlad" / "hla3d" (AHLA / third order
    with per-head decay, gamma [H]: every state scaled by gamma before each update, the reading
    Contribuciones 2's decayed operators get for the second order).  A gamma passed with "hla2",
    "hla2n", "ahla", "hla3", "ahlan" or "hla3n" selects the decayed form of that op.
    """
    if op in DECAYED and gamma is None:
        raise ValueError(f"op {op} needs gamma")
    lib = _load()
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, T, d = q.shape
    dv = v.shape[-1]
    g = _f64(gamma) if gamma is not None else None
    o = np.zeros((B, H, T, dv), dtype=np.float64)
    n = nthreads if nthreads else (os.cpu_count() or 1)
    rc = lib.oracle_forward(OPS[op], B, H, T, d, dv, _ptr(q), _ptr(k), _ptr(v), _ptr(g),
                            float(eps), _ptr(o), int(n))
    if rc != 0:
        raise ValueError(f"oracle_forward rejected its arguments (op={op})")
    return o


# ---------------------------------------------------------------------------
# Single-head state-carrying runs (used by oracle.segments and the tests).
# ---------------------------------------------------------------------------

def hla2_run(q, k, v, state=None, gamma: Optional[float] = None, normalized: bool = False,
             eps: float = 1e-6, want_output: bool = True):
    """Run the second-order recurrence over one head's tokens from ``state``.

    q, k: [T,d]; v: [T,dv].  state = dict(S, C, G, m, h) or None (zeros).
    Returns (o or None, new_state).  Decayed when ``gamma`` is not None.
    """
    lib = _load()
    q, k, v = _f64(q), _f64(k), _f64(v)
    T, d = q.shape
    dv = v.shape[1]
    if state is None:
        st = dict(S=np.zeros((d, d)), C=np.zeros((d, dv)), G=np.zeros((d, dv)),
                  m=np.zeros(d), h=np.zeros(d))
    else:
        st = {key: np.array(val, dtype=np.float64, copy=True, order="C") for key, val in state.items()}
    o = np.zeros((T, dv)) if want_output else None
    lib.oracle_hla2_head(_ptr(q), _ptr(k), _ptr(v), T, d, dv,
                         1 if gamma is not None else 0, float(gamma if gamma is not None else 1.0),
                         1 if normalized else 0, float(eps),
                         _ptr(st["S"]), _ptr(st["C"]), _ptr(st["G"]), _ptr(st["m"]), _ptr(st["h"]),
                         _ptr(o))
    return o, st


def ahla_run(q, k, v, state=None, want_output: bool = True, gamma: Optional[float] = None):
    """AHLA recurrence over one head from ``state`` = dict(P, E) or None; decayed (P, E scaled
    by gamma before every update) when ``gamma`` is not None."""
    lib = _load()
    q, k, v = _f64(q), _f64(k), _f64(v)
    T, d = q.shape
    dv = v.shape[1]
    if state is None:
        st = dict(P=np.zeros((d, dv)), E=np.zeros((d, dv)))
    else:
        st = {key: np.array(val, dtype=np.float64, copy=True, order="C") for key, val in state.items()}
    o = np.zeros((T, dv)) if want_output else None
    lib.oracle_ahla_head(_ptr(q), _ptr(k), _ptr(v), T, d, dv, 1 if gamma is not None else 0,
                         float(gamma if gamma is not None else 1.0), _ptr(st["P"]), _ptr(st["E"]), _ptr(o))
    return o, st


def hla3_run(q, k, v, state=None, want_output: bool = True, gamma: Optional[float] = None):
    """Third-order recurrence over one head from ``state`` = dict(S, P, F) or None; decayed (S, P,
    F scaled by gamma before every update) when ``gamma`` is not None."""
    lib = _load()
    q, k, v = _f64(q), _f64(k), _f64(v)
    T, d = q.shape
    dv = v.shape[1]
    if state is None:
        st = dict(S=np.zeros((d, d)), P=np.zeros((d, dv)), F=np.zeros((d, dv)))
    else:
        st = {key: np.array(val, dtype=np.float64, copy=True, order="C") for key, val in state.items()}
    o = np.zeros((T, dv)) if want_output else None
    lib.oracle_hla3_head(_ptr(q), _ptr(k), _ptr(v), T, d, dv, 1 if gamma is not None else 0,
                         float(gamma if gamma is not None else 1.0), _ptr(st["S"]), _ptr(st["P"]),
                         _ptr(st["F"]), _ptr(o))
    return o, st


def hla2u_run(q, k, v, state=None, want_output: bool = True):
    """Unmasked second-order recurrence over one head from ``state`` = dict(S, C) or None."""
    lib = _load()
    q, k, v = _f64(q), _f64(k), _f64(v)
    T, d = q.shape
    dv = v.shape[1]
    if state is None:
        st = dict(S=np.zeros((d, d)), C=np.zeros((d, dv)))
    else:
        st = {key: np.array(val, dtype=np.float64, copy=True, order="C") for key, val in state.items()}
    o = np.zeros((T, dv)) if want_output else None
    lib.oracle_hla2u_head(_ptr(q), _ptr(k), _ptr(v), T, d, dv, _ptr(st["S"]), _ptr(st["C"]), _ptr(o))
    return o, st


def max_row_rel_err(o, ref) -> float:
    """Parity metric: max over rows (b,h,t) of ||o - ref||_2 / ||ref||_2, no floor."""
    o = _f64(o)
    ref = _f64(ref)
    num = np.linalg.norm((o - ref).reshape(-1, ref.shape[-1]), axis=1)
    den = np.linalg.norm(ref.reshape(-1, ref.shape[-1]), axis=1)
    return float(np.max(num / den)) if num.size else 0.0
