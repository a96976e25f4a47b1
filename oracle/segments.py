"""Segment summaries, semidirect-product combine maps and a Blelloch exclusive scan (fp64).

TEST INFRASTRUCTURE ONLY (see the package docstring).

"Higher-order Linear Attention" summary, Metodología 4: associative
(semidirect-product) operators concatenate token segments, accounting for the
cross terms between segments (e.g. S^K_B C^QV_A); a Blelloch exclusive scan over
the segment summaries gives forward activations identical to the serial
recurrence.  The third-order scan adds segment-level linear maps.

A *summary* of a segment is the state the serial recurrence reaches when it is
run over that segment alone from the zero state, plus the segment maps the
combine needs.  The page names the maps but prints none of them; those below
are read off the recurrences:

second order (optionally decayed, gamma = 1 for none)
    state S, C, G, m, h (the recurrence's own); maps rho = gamma^len,
    Khat = sum k k^T (undecayed).
    A then B:  S = rho_B S_A + S_B,  C = rho_B C_A + C_B,  m = rho_B m_A + m_B,
               G = rho_B G_A + G_B + rho_B Khat_B C_A,
               h = rho_B h_A + h_B + rho_B Khat_B m_A,
               Khat = Khat_A + Khat_B,  rho = rho_A rho_B.
AHLA (optionally decayed: P, E scaled by gamma before every update)
    state P, E; maps D = sum k q^T (undecayed), rho = gamma^len.
    A then B:  P = rho_B P_A + P_B,  D = D_A + D_B,  E = rho_B E_A + E_B + rho_B D_B P_A,
               rho = rho_A rho_B.
third order (optionally decayed: S, P, F scaled by gamma before every update)
    state S, P, F; maps Q2 = sum_s gamma^tau_s q_s q_s^T (tau_s = 1-based position in the
    segment), X = sum_s q_s q_s^T P_s, Z = sum_s S_s q_s q_s^T (P_s, S_s local to the segment,
    inclusive of s), rho = gamma^len.
    A then B:  S = rho_B S_A + S_B,  P = rho_B P_A + P_B,  Q2 = Q2_A + rho_A Q2_B,
               Z = Z_A + Z_B + S_A Q2_B,  X = X_A + X_B + Q2_B P_A,
               F = rho_B F_A + F_B + rho_B (S_A Q2_B P_A + S_A X_B + Z_B P_A),  rho = rho_A rho_B.
    (A token s of B sees S_s = gamma^tau_s S_A + S^B_s and P_s = gamma^tau_s P_A + P^B_s; its F term
    decays by gamma^(len_B - tau_s) to the end of B.)  With gamma = 1 every rho is 1 and Q2 the
    plain sum of q q^T.
"""
from __future__ import annotations

from typing import Callable, Dict, List, Optional

import numpy as np

from . import _f64, ahla_run, hla2_run, hla3_run

Summary = Dict[str, np.ndarray]


# --------------------------------------------------------------------------
# summaries
# --------------------------------------------------------------------------

def hla2_summary(q, k, v, gamma: Optional[float] = None) -> Summary:
    q, k, v = _f64(q), _f64(k), _f64(v)
    _, st = hla2_run(q, k, v, None, gamma=gamma, want_output=False)
    g = 1.0 if gamma is None else float(gamma)
    st["Khat"] = k.T @ k
    st["rho"] = np.array(g ** q.shape[0])
    return st


def ahla_summary(q, k, v, gamma: Optional[float] = None) -> Summary:
    q, k, v = _f64(q), _f64(k), _f64(v)
    _, st = ahla_run(q, k, v, None, want_output=False, gamma=gamma)
    st["D"] = k.T @ q
    st["rho"] = np.array((1.0 if gamma is None else float(gamma)) ** q.shape[0])
    return st


def hla3_summary(q, k, v, gamma: Optional[float] = None) -> Summary:
    q, k, v = _f64(q), _f64(k), _f64(v)
    T, d = q.shape
    dv = v.shape[1]
    g = 1.0 if gamma is None else float(gamma)
    _, st = hla3_run(q, k, v, None, want_output=False, gamma=gamma)
    S = np.zeros((d, d))
    P = np.zeros((d, dv))
    Q2 = np.zeros((d, d))
    X = np.zeros((d, dv))
    Z = np.zeros((d, d))
    for s in range(T):
        S = g * S + np.outer(k[s], k[s])
        P = g * P + np.outer(k[s], v[s])
        qq = np.outer(q[s], q[s])
        Q2 += g ** (s + 1) * qq
        X += qq @ P
        Z += S @ qq
    st["Q2"] = Q2
    st["X"] = X
    st["Z"] = Z
    st["rho"] = np.array(g ** T)
    return st


# --------------------------------------------------------------------------
# identities
# --------------------------------------------------------------------------

def hla2_identity(d: int, dv: int) -> Summary:
    return dict(S=np.zeros((d, d)), C=np.zeros((d, dv)), G=np.zeros((d, dv)), m=np.zeros(d),
                h=np.zeros(d), Khat=np.zeros((d, d)), rho=np.array(1.0))


def ahla_identity(d: int, dv: int) -> Summary:
    return dict(P=np.zeros((d, dv)), E=np.zeros((d, dv)), D=np.zeros((d, d)), rho=np.array(1.0))


def hla3_identity(d: int, dv: int) -> Summary:
    return dict(S=np.zeros((d, d)), P=np.zeros((d, dv)), F=np.zeros((d, dv)), Q2=np.zeros((d, d)),
                X=np.zeros((d, dv)), Z=np.zeros((d, d)), rho=np.array(1.0))


# --------------------------------------------------------------------------
# combine maps: combine(A, B) summarises segment A followed by segment B
# --------------------------------------------------------------------------

def hla2_combine(A: Summary, B: Summary) -> Summary:
    r = B["rho"]
    return dict(
        S=r * A["S"] + B["S"],
        C=r * A["C"] + B["C"],
        G=r * A["G"] + B["G"] + r * (B["Khat"] @ A["C"]),
        m=r * A["m"] + B["m"],
        h=r * A["h"] + B["h"] + r * (B["Khat"] @ A["m"]),
        Khat=A["Khat"] + B["Khat"],
        rho=A["rho"] * B["rho"],
    )


def ahla_combine(A: Summary, B: Summary) -> Summary:
    r = B["rho"]
    return dict(P=r * A["P"] + B["P"], E=r * A["E"] + B["E"] + r * (B["D"] @ A["P"]), D=A["D"] + B["D"],
                rho=A["rho"] * B["rho"])


def hla3_combine(A: Summary, B: Summary) -> Summary:
    r = B["rho"]
    SQ = A["S"] @ B["Q2"]
    return dict(
        S=r * A["S"] + B["S"],
        P=r * A["P"] + B["P"],
        Q2=A["Q2"] + A["rho"] * B["Q2"],
        Z=A["Z"] + B["Z"] + SQ,
        X=A["X"] + B["X"] + B["Q2"] @ A["P"],
        F=r * A["F"] + B["F"] + r * (SQ @ A["P"] + A["S"] @ B["X"] + B["Z"] @ A["P"]),
        rho=A["rho"] * B["rho"],
    )


# --------------------------------------------------------------------------
# scans
# --------------------------------------------------------------------------

def blelloch_exclusive(xs: List[Summary], combine: Callable, identity: Summary) -> List[Summary]:
    """Work-efficient exclusive scan (up-sweep, clear root, down-sweep), padded to 2^k.

    Element i of the result summarises segments 0..i-1 (identity for i = 0).
    The combine is associative but not commutative: combine(A, B) = A then B.
    """
    n = len(xs)
    if n == 0:
        return []
    size = 1
    while size < n:
        size *= 2
    a = [dict(x) for x in xs] + [dict(identity) for _ in range(size - n)]
    step = 1
    while step < size:                        # up-sweep
        for i in range(0, size, 2 * step):
            a[i + 2 * step - 1] = combine(a[i + step - 1], a[i + 2 * step - 1])
        step *= 2
    a[size - 1] = dict(identity)              # clear the root
    step = size // 2
    while step >= 1:                          # down-sweep
        for i in range(0, size, 2 * step):
            left = a[i + step - 1]
            a[i + step - 1] = a[i + 2 * step - 1]
            a[i + 2 * step - 1] = combine(a[i + 2 * step - 1], left)
        step //= 2
    return a[:n]


def fold_exclusive(xs: List[Summary], combine: Callable, identity: Summary) -> List[Summary]:
    """Left-to-right exclusive fold (the serial definition of the same prefixes)."""
    out, acc = [], dict(identity)
    for x in xs:
        out.append(acc)
        acc = combine(acc, x)
    return out


def split_points(T: int, lengths: List[int]) -> List[int]:
    """Cumulative boundaries for segment lengths that sum to T."""
    assert sum(lengths) == T
    b = [0]
    for n in lengths:
        b.append(b[-1] + n)
    return b


def hla2_scan_forward(q, k, v, lengths: List[int], gamma: Optional[float] = None,
                      normalized: bool = False, eps: float = 1e-6, scan=blelloch_exclusive):
    """Chunk-parallel forward: summaries -> exclusive scan -> each segment resumed from its prefix."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    b = split_points(q.shape[0], lengths)
    sums = [hla2_summary(q[b[i]:b[i + 1]], k[b[i]:b[i + 1]], v[b[i]:b[i + 1]], gamma)
            for i in range(len(lengths))]
    pre = scan(sums, hla2_combine, hla2_identity(q.shape[1], v.shape[1]))
    outs = []
    for i in range(len(lengths)):
        st = {key: pre[i][key] for key in ("S", "C", "G", "m", "h")}
        o, _ = hla2_run(q[b[i]:b[i + 1]], k[b[i]:b[i + 1]], v[b[i]:b[i + 1]], st, gamma=gamma,
                        normalized=normalized, eps=eps)
        outs.append(o)
    return np.concatenate(outs, axis=0)


def ahla_scan_forward(q, k, v, lengths: List[int], scan=blelloch_exclusive, gamma: Optional[float] = None):
    q, k, v = _f64(q), _f64(k), _f64(v)
    b = split_points(q.shape[0], lengths)
    sums = [ahla_summary(q[b[i]:b[i + 1]], k[b[i]:b[i + 1]], v[b[i]:b[i + 1]], gamma)
            for i in range(len(lengths))]
    pre = scan(sums, ahla_combine, ahla_identity(q.shape[1], v.shape[1]))
    outs = []
    for i in range(len(lengths)):
        st = {key: pre[i][key] for key in ("P", "E")}
        o, _ = ahla_run(q[b[i]:b[i + 1]], k[b[i]:b[i + 1]], v[b[i]:b[i + 1]], st, gamma=gamma)
        outs.append(o)
    return np.concatenate(outs, axis=0)


def hla3_scan_forward(q, k, v, lengths: List[int], scan=blelloch_exclusive, gamma: Optional[float] = None):
    q, k, v = _f64(q), _f64(k), _f64(v)
    b = split_points(q.shape[0], lengths)
    sums = [hla3_summary(q[b[i]:b[i + 1]], k[b[i]:b[i + 1]], v[b[i]:b[i + 1]], gamma)
            for i in range(len(lengths))]
    pre = scan(sums, hla3_combine, hla3_identity(q.shape[1], v.shape[1]))
    outs = []
    for i in range(len(lengths)):
        st = {key: pre[i][key] for key in ("S", "P", "F")}
        o, _ = hla3_run(q[b[i]:b[i + 1]], k[b[i]:b[i + 1]], v[b[i]:b[i + 1]], st, gamma=gamma)
        outs.append(o)
    return np.concatenate(outs, axis=0)
