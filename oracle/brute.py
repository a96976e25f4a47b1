"""Masked-matrix definitions of the HLA forward, O(T^2 d + T^3), fp64 numpy.

TEST INFRASTRUCTURE ONLY (see the package docstring).  These are the plain
definitions the streaming algebra must reproduce exactly ("Higher-order Linear
Attention" summary, Contribuciones 1: exact masked streaming identities;
Resultados: causality, o_t depends only on j <= t).  Intended for small T.

Mask convention: L[t, j] = 1 iff j <= t (diagonal included), as the sums
sum_{j<=t} sum_{i<=j} of the second-order output require.
"""
from __future__ import annotations

import numpy as np

from . import _f64


def _tril(x):
    return np.tril(x)


def scores(q, k):
    """A = L (.) (Q K^T), per head: [..., T, T]."""
    q, k = _f64(q), _f64(k)
    return _tril(q @ np.swapaxes(k, -1, -2))


def hla2(q, k, v, normalized: bool = False, eps: float = 1e-6):
    """Second order (Metodología 1): o_t = sum_{j<=t} sum_{i<=j} (q_t.k_i)(q_j.k_i) v_j.

    In matrix form W = L (.) (A A^T) with A = L (.) Q K^T, O = W V.  The
    ratio-normalised variant divides row t by (sum_j W_tj + eps).
    """
    A = scores(q, k)
    W = _tril(A @ np.swapaxes(A, -1, -2))
    num = W @ _f64(v)
    if not normalized:
        return num
    den = W.sum(axis=-1, keepdims=True)
    return num / (den + eps)


def hla2_decay(q, k, v, gamma, normalized: bool = False, eps: float = 1e-6):
    """Decayed second order under the reading "scale every state by gamma, then update".

    Unrolling that recurrence gives, with global token indices,
        o_t = sum_{j<=t} sum_{i<=t} c(t,i,j) (q_t.k_i)(q_j.k_i) v_j,
        c(t,i,j) = gamma^(2t-i-j) - [i>j] gamma^(t-j).
    (S_t = sum gamma^(t-i) k k^T and C_t = sum gamma^(t-j) q v^T give the first
    term; G_t = sum_{j<i<=t} gamma^(t-j) k_i k_i^T q_j v_j^T the second.)
    gamma: per head, shape [H] for [B,H,T,d] inputs or a scalar for [T,d].
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    g = np.asarray(gamma, dtype=np.float64)
    lead = q.shape[:-2]
    T = q.shape[-2]
    if g.ndim == 1 and len(lead) == 2:
        g = g[None, :, None, None]          # broadcast over B, T, T
    elif g.ndim == 0:
        g = g.reshape((1,) * len(lead) + (1, 1))
    Kq = np.swapaxes(k @ np.swapaxes(q, -1, -2), -1, -2)   # Kq[..., j, i] = q_j . k_i
    QK = q @ np.swapaxes(k, -1, -2)                       # QK[..., t, i] = q_t . k_i
    out = np.zeros(q.shape[:-1] + (v.shape[-1],))
    den_all = np.zeros(q.shape[:-1])
    idx = np.arange(T, dtype=np.float64)
    for t in range(T):
        i = idx[: t + 1]
        j = idx[: t + 1]
        # weights c(t, i, j) over the (i, j) grid, i on axis -2, j on axis -1
        gi = g ** (t - i[:, None])           # gamma^(t-i)
        gj = g ** (t - j[None, :])           # gamma^(t-j)
        strict = (i[:, None] > j[None, :]).astype(np.float64)
        c = gi * gj - strict * gj            # [..., t+1, t+1]
        qk_ti = QK[..., t, : t + 1]          # (q_t . k_i)
        qk_ji = Kq[..., : t + 1, : t + 1]    # [j, i] = q_j . k_i
        # W_tj = sum_i c(t,i,j) (q_t.k_i)(q_j.k_i)
        Wt = np.einsum("...ij,...i,...ji->...j", c, qk_ti, qk_ji)
        out[..., t, :] = np.einsum("...j,...jc->...c", Wt, v[..., : t + 1, :])
        den_all[..., t] = Wt.sum(axis=-1)
    if normalized:
        out = out / (den_all[..., None] + eps)
    return out


def hla2u(q, k, v):
    """Second order without the inner mask (Contribuciones 2, unmasked configuration):
    o_t = q_t^T S_t C_t = sum_{j<=t} sum_{i<=t} (q_t.k_i)(q_j.k_i) v_j.  In matrix form
    W = L (.) (A A*^T) with A = L (.) Q K^T and A* = Q K^T (j's scores unmasked), O = W V."""
    A = scores(q, k)
    Astar = _f64(q) @ np.swapaxes(_f64(k), -1, -2)
    W = _tril(A @ np.swapaxes(Astar, -1, -2))
    return W @ _f64(v)


def ahla(q, k, v):
    """AHLA (Metodología 2): o_t = sum_{j<=t} (q_t.k_j) sum_{i<=j} (q_j.k_i) v_i, i.e. O = A (A V)."""
    A = scores(q, k)
    return A @ (A @ _f64(v))


def hla3(q, k, v):
    """Third order (Metodología 3, A A^T A): O = (M A) V, M = L (.) (A A^T), A = L (.) Q K^T."""
    A = scores(q, k)
    M = _tril(A @ np.swapaxes(A, -1, -2))
    return (M @ A) @ _f64(v)


def _decay_weights(gamma, lead, T):
    """Gamma[..., t, j] = gamma^(t - j) for j <= t, else 0; gamma per head ([H] for [B,H,T,d]
    inputs) or a scalar."""
    g = np.asarray(gamma, dtype=np.float64)
    if g.ndim == 1 and len(lead) == 2:
        g = g[None, :, None, None]
    else:
        g = g.reshape((1,) * (len(lead) + 2))
    idx = np.arange(T, dtype=np.float64)
    diff = idx[:, None] - idx[None, :]
    return np.where(diff >= 0, g ** np.maximum(diff, 0.0), 0.0)


def ahla_decay(q, k, v, gamma):
    """AHLA with per-head decay under the reading "scale every state by gamma, then update":
    P_t = gamma P + k v^T, E_t = gamma E + k (q^T P_t), o_t = q_t^T E_t, which unrolls to
        o_t = sum_{j<=t} sum_{i<=j} gamma^(t-i) (q_t.k_j)(q_j.k_i) v_i,
    i.e. O = At (At V) with At = G (.) A, G_tj = gamma^(t-j): gamma^(t-i) = gamma^(t-j) gamma^(j-i)."""
    q, k = _f64(q), _f64(k)
    At = scores(q, k) * _decay_weights(gamma, q.shape[:-2], q.shape[-2])
    return At @ (At @ _f64(v))


def hla3_decay(q, k, v, gamma):
    """Third order with per-head decay under the same reading (S, P, F scaled before each update):
        o_t = sum_{s<=t} sum_{a<=s} sum_{b<=s} gamma^(t-a) gamma^(s-b) (q_t.k_a)(q_s.k_a)(q_s.k_b) v_b,
    i.e. O = (L (.) (At A^T)) (At V) with At = G (.) A."""
    q, k = _f64(q), _f64(k)
    A = scores(q, k)
    At = A * _decay_weights(gamma, q.shape[:-2], q.shape[-2])
    M = _tril(At @ np.swapaxes(A, -1, -2))
    return M @ (At @ _f64(v))


def forward(op: str, q, k, v, gamma=None, eps: float = 1e-6):
    """Dispatch by op name, same names as :func:`oracle.recur`."""
    if op == "hla2":
        return hla2(q, k, v) if gamma is None else hla2_decay(q, k, v, gamma)
    if op == "hla2n":
        return hla2(q, k, v, normalized=True, eps=eps) if gamma is None else \
            hla2_decay(q, k, v, gamma, normalized=True, eps=eps)
    if op == "hla2d":
        return hla2_decay(q, k, v, gamma)
    if op in ("ahla", "ahlad"):
        return ahla(q, k, v) if gamma is None else ahla_decay(q, k, v, gamma)
    if op in ("hla3", "hla3d"):
        return hla3(q, k, v) if gamma is None else hla3_decay(q, k, v, gamma)
    if op == "hla2u":
        return hla2u(q, k, v)
    if op in ("ahlan", "hla3n"):
        if gamma is None:
            f = ahla if op == "ahlan" else hla3
        else:
            base = ahla_decay if op == "ahlan" else hla3_decay
            f = lambda q_, k_, v_: base(q_, k_, v_, gamma)   # noqa: E731
        ones = np.ones(_f64(q).shape[:-1] + (1,))
        return f(q, k, v) / (f(q, k, ones) + eps)
    raise ValueError(op)
