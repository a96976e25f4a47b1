"""The chunk algebra of the tensor-core kernels, checked in fp64 on the CPU.

The CUDA kernels do not run the token recurrence; they run a rewritten form of it:
per-chunk matrix products, segment summaries and factored prefixes.  The GPU parity
tests check the end result; these tests check each rewrite on its own, in fp64,
against the oracle's serial recurrence and its semidirect-product combine maps, so a
derivation error (a dropped cross term, a wrong decay exponent, a transposed
operand) shows up here, away from bf16 rounding.  Every emulation below restates the
formulas written in the header comments of the kernel sources; none of them calls
into the CUDA path.

Sources: "Higher-order Linear Attention" summary (gist.science 2510.27258),
Metodología 1 (second-order state, ratio normalisation), Metodología 2 (AHLA),
Metodología 4 (chunked, scan-parallel evaluation), Contribuciones 2 (decay).
"""
import numpy as np
import pytest

import oracle
import oracle.segments as seg

EPS = 1e-6


def rel(a, b):
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300))


def rand_head(T, d, dv, seed):
    rng = np.random.default_rng(seed)
    s = 1.0 / np.sqrt(d)
    q = rng.standard_normal((T, d)) * s
    k = rng.standard_normal((T, d)) * s
    v = rng.standard_normal((T, dv))
    return q, k, v


def chunks(x, c):
    """Zero-pad the token axis to whole chunks of c and split; zero tokens add nothing."""
    T = x.shape[0]
    n = -(-T // c)
    xp = np.vstack([x, np.zeros((n * c - T, x.shape[1]))])
    return [xp[i * c:(i + 1) * c] for i in range(n)]


def recur(op, q, k, v, gamma=None):
    g = None if gamma is None else np.array([gamma])
    return oracle.recur(op, q[None, None], k[None, None], v[None, None], gamma=g, eps=EPS)[0, 0]


# ---------------------------------------------------------------------------
# second order, undecayed: the walker's per-chunk step (R-form state)
# ---------------------------------------------------------------------------

def hla2_chunk(Q, K, V1, S0, R0):
    """One chunk of the second-order walker.  V1 = [V | 1] for the normalised form.

    State carried in: S0 (key moment) and R0 = S0 C0 - G0 (with r0 as its last column
    when V1 carries the ones column).  Returns (O, S0', R0')."""
    c = Q.shape[0]
    L = np.tril(np.ones((c, c)))
    A = L * (Q @ K.T)
    P = Q @ S0
    W = L * (P @ Q.T + A @ A.T)       # W_tj = q_t^T S_j q_j
    O = Q @ R0 + W @ V1
    Z = P + A @ K                     # row j: S_j q_j
    return O, S0 + K.T @ K, R0 + Z.T @ V1


def hla2_walk(q, k, v, c, normalized, S0=None, R0=None):
    d, dv = q.shape[1], v.shape[1] + (1 if normalized else 0)
    S0 = np.zeros((d, d)) if S0 is None else S0
    R0 = np.zeros((d, dv)) if R0 is None else R0
    outs = []
    for Q, K, V in zip(chunks(q, c), chunks(k, c), chunks(v, c)):
        V1 = np.hstack([V, np.ones((V.shape[0], 1))]) if normalized else V
        O, S0, R0 = hla2_chunk(Q, K, V1, S0, R0)
        outs.append(O)
    O = np.vstack(outs)[:q.shape[0]]
    if normalized:
        O = O[:, :-1] / (O[:, -1:] + EPS)
    return O, S0, R0


def test_pair_weight_two_forms():
    """L (.) (Q S0 Q^T + A A^T) equals L (.) (Q Z^T) with Z = Q S0 + A K: the weight of the
    pair (t, j) sums (q_t . k_i)(q_j . k_i) over the carried-in keys and the keys i <= j."""
    rng = np.random.default_rng(4)
    c, d = 16, 5
    Q, K = rng.standard_normal((c, d)), rng.standard_normal((c, d))
    G = rng.standard_normal((d, d))
    S0 = G @ G.T
    L = np.tril(np.ones((c, c)))
    A = L * (Q @ K.T)
    Z = Q @ S0 + A @ K
    np.testing.assert_allclose(L * (Q @ Z.T), L * (Q @ S0 @ Q.T + A @ A.T), rtol=0, atol=1e-12)
    # the brute-force pair weight, entry by entry
    for t in range(c):
        for j in range(t + 1):
            w = Q[t] @ S0 @ Q[j] + sum((Q[t] @ K[i]) * (Q[j] @ K[i]) for i in range(j + 1))
            assert abs((Q[t] @ Z[j]) - w) < 1e-12


@pytest.mark.parametrize("normalized", [False, True])
@pytest.mark.parametrize("T,c", [(1, 8), (7, 8), (8, 8), (37, 8), (64, 16), (100, 32)])
def test_hla2_chunk_step_matches_recurrence(T, c, normalized):
    q, k, v = rand_head(T, 5, 3, seed=T * 7 + c)
    if normalized:
        k = np.abs(k)                 # keep the denominator away from zero
        q = np.abs(q)
    O, _, _ = hla2_walk(q, k, v, c, normalized)
    ref = recur("hla2n" if normalized else "hla2", q, k, v)
    assert rel(O, ref) < 1e-12


# ---------------------------------------------------------------------------
# segment prefixes: the factored forms against the exclusive fold of the combine
# ---------------------------------------------------------------------------

def r_form(s):
    """(S, C, m, R = S C - G, r = S m - h) of an oracle second-order summary."""
    return dict(S=s["S"], C=s["C"], m=s["m"], R=s["S"] @ s["C"] - s["G"], r=s["S"] @ s["m"] - s["h"])


def prefix_cross_sum(slots):
    """The two-kernel form: Y_l = R_l + S0(l) C_l, then R0(n) = sum_{l<n} Y_l."""
    out, S0, R0, r0 = [], 0.0 * slots[0]["S"], 0.0 * slots[0]["R"], 0.0 * slots[0]["r"]
    for s in slots:
        out.append(dict(S=S0, R=R0, r=r0))
        R0 = R0 + s["R"] + S0 @ s["C"]
        r0 = r0 + s["r"] + S0 @ s["m"]
        S0 = S0 + s["S"]
    return out


def prefix_fold(slots, n):
    """The in-prologue fold for the prefix of slots 0..n-1: plain sums of S, R, r plus the
    cross terms sum_{m<n-1} S_m Csuf(m+1), Csuf(m+1) = sum_{m<l<n} C_l (likewise m)."""
    S0 = sum((s["S"] for s in slots[:n]), 0.0 * slots[0]["S"])
    R0 = sum((s["R"] for s in slots[:n]), 0.0 * slots[0]["R"])
    r0 = sum((s["r"] for s in slots[:n]), 0.0 * slots[0]["r"])
    Csuf, msuf = 0.0 * slots[0]["C"], 0.0 * slots[0]["m"]
    for m in range(n - 2, -1, -1):
        Csuf = Csuf + slots[m + 1]["C"]
        msuf = msuf + slots[m + 1]["m"]
        R0 = R0 + slots[m]["S"] @ Csuf
        r0 = r0 + slots[m]["S"] @ msuf
    return dict(S=S0, R=R0, r=r0)


@pytest.mark.parametrize("lengths", [[5], [3, 9, 1], [8, 8, 8, 8, 8], [1, 2, 3, 4, 5, 6, 7]])
def test_factored_prefixes_equal_the_combine_fold(lengths):
    T, d, dv = sum(lengths), 4, 3
    q, k, v = rand_head(T, d, dv, seed=len(lengths))
    b = seg.split_points(T, lengths)
    sums = [seg.hla2_summary(q[b[i]:b[i + 1]], k[b[i]:b[i + 1]], v[b[i]:b[i + 1]]) for i in range(len(lengths))]
    ref = seg.fold_exclusive(sums, seg.hla2_combine, seg.hla2_identity(d, dv))
    slots = [r_form(s) for s in sums]
    two_kernel = prefix_cross_sum(slots)
    for n in range(len(lengths)):
        want = r_form(ref[n])
        folded = prefix_fold(slots, n)
        for key in ("S", "R", "r"):
            np.testing.assert_allclose(two_kernel[n][key], want[key], rtol=0, atol=1e-12)
            np.testing.assert_allclose(folded[key], want[key], rtol=0, atol=1e-12)


@pytest.mark.parametrize("normalized", [False, True])
@pytest.mark.parametrize("T,c,NCH,ratio", [(200, 8, 5, 1), (200, 8, 6, 3), (129, 16, 2, 2), (70, 8, 9, 1)])
def test_segment_plan_matches_recurrence(T, c, NCH, ratio, normalized):
    """Summary segments of NCH/ratio chunks walked from zero, their prefix, then output
    segments of NCH chunks walked from that prefix: the three kernel stages end to end."""
    d, dv = 4, 3
    q, k, v = rand_head(T, d, dv, seed=T + NCH)
    if normalized:
        q, k = np.abs(q), np.abs(k)
    nchunks = -(-T // c)
    NCHs = NCH // ratio
    seg_tok = NCHs * c
    n_out = -(-nchunks // NCH)
    n_sum = (n_out - 1) * ratio      # only the chunks before the last output segment
    slots = []
    for i in range(n_sum):
        sl = slice(i * seg_tok, (i + 1) * seg_tok)
        _, S, R = hla2_walk(q[sl], k[sl], v[sl], c, normalized)
        slots.append(dict(S=S, C=q[sl].T @ v[sl], m=q[sl].sum(0), R=R[:, :dv],
                          r=R[:, dv] if normalized else np.zeros(d)))
    outs = []
    for n in range(n_out):
        if n == 0:
            S0, R0, r0 = np.zeros((d, d)), np.zeros((d, dv)), np.zeros(d)
        else:
            p = prefix_fold(slots, n * ratio)
            S0, R0, r0 = p["S"], p["R"], p["r"]
        R0 = np.hstack([R0, r0[:, None]]) if normalized else R0
        sl = slice(n * NCH * c, min((n + 1) * NCH * c, T))
        O, _, _ = hla2_walk(q[sl], k[sl], v[sl], c, normalized, S0=S0, R0=R0)
        outs.append(O)
    ref = recur("hla2n" if normalized else "hla2", q, k, v)
    assert rel(np.vstack(outs), ref) < 1e-12


# ---------------------------------------------------------------------------
# AHLA: the walker's chunk step and the transposed summary slot
# ---------------------------------------------------------------------------

def ahla_walk(q, k, v, c, P0=None, E0=None):
    d, dv = q.shape[1], v.shape[1]
    P0 = np.zeros((d, dv)) if P0 is None else P0
    E0 = np.zeros((d, dv)) if E0 is None else E0
    outs = []
    for Q, K, V in zip(chunks(q, c), chunks(k, c), chunks(v, c)):
        A = np.tril(Q @ K.T)
        Y = Q @ P0 + A @ V            # row s: q_s^T P_s
        outs.append(Q @ E0 + A @ Y)
        P0 = P0 + K.T @ V
        E0 = E0 + K.T @ Y
    return np.vstack(outs)[:q.shape[0]], P0, E0


@pytest.mark.parametrize("T,c", [(1, 8), (13, 8), (64, 16), (99, 32)])
def test_ahla_chunk_step_matches_recurrence(T, c):
    q, k, v = rand_head(T, 5, 3, seed=T + 1000)
    O, _, _ = ahla_walk(q, k, v, c)
    assert rel(O, recur("ahla", q, k, v)) < 1e-12


@pytest.mark.parametrize("lengths", [[4, 4], [3, 9, 1, 6], [8, 8, 8, 8, 8, 8]])
def test_ahla_transposed_slot_uses_the_second_order_prefix(lengths):
    """(P^T, D^T, E^T) in the places of (S, C, R): the second-order factored prefix of the
    transposed slots is the transpose of the AHLA combine fold."""
    T, d, dv = sum(lengths), 5, 3
    q, k, v = rand_head(T, d, dv, seed=77 + len(lengths))
    b = seg.split_points(T, lengths)
    sums = [seg.ahla_summary(q[b[i]:b[i + 1]], k[b[i]:b[i + 1]], v[b[i]:b[i + 1]]) for i in range(len(lengths))]
    ref = seg.fold_exclusive(sums, seg.ahla_combine, seg.ahla_identity(d, dv))
    slots = [dict(S=s["P"].T, C=s["D"].T, m=np.zeros(d), R=s["E"].T, r=np.zeros(dv)) for s in sums]
    two_kernel = prefix_cross_sum(slots)
    for n in range(len(lengths)):
        folded = prefix_fold(slots, n)
        for got in (two_kernel[n], folded):
            np.testing.assert_allclose(got["S"], ref[n]["P"].T, rtol=0, atol=1e-12)
            np.testing.assert_allclose(got["R"], ref[n]["E"].T, rtol=0, atol=1e-12)


def test_ahla_segment_plan_matches_recurrence():
    T, c, NCH, d, dv = 150, 8, 4, 4, 3
    q, k, v = rand_head(T, d, dv, seed=5)
    seg_tok = NCH * c
    n_out = -(-T // seg_tok)
    slots = []
    for i in range(n_out - 1):
        sl = slice(i * seg_tok, (i + 1) * seg_tok)
        _, P, E = ahla_walk(q[sl], k[sl], v[sl], c)
        slots.append(dict(S=P.T, C=(k[sl].T @ q[sl]).T, m=np.zeros(d), R=E.T, r=np.zeros(dv)))
    outs = []
    for n in range(n_out):
        P0, E0 = np.zeros((d, dv)), np.zeros((d, dv))
        if n:
            p = prefix_fold(slots, n)
            P0, E0 = p["S"].T, p["R"].T
        sl = slice(n * seg_tok, min((n + 1) * seg_tok, T))
        outs.append(ahla_walk(q[sl], k[sl], v[sl], c, P0=P0, E0=E0)[0])
    assert rel(np.vstack(outs), recur("ahla", q, k, v)) < 1e-12


def ahla_walk_decayed(q, k, v, c, g, P0=None, E0=None):
    """The tensor-core AHLA walker with decay: At = g^(tau - j) A on the masked scores,
    Gam = diag(g^(tau+1)), Lam = diag(g^(len-1-tau)), rho = g^len per chunk:
        Y = Gam Q P0 + At V,  O = Gam Q E0 + At Y,  P0 = rho P0 + K^T Lam V,  E0 = rho E0 + K^T Lam Y.
    Chunks are the sequence's own (the last one may be short)."""
    d, dv = q.shape[1], v.shape[1]
    P0 = np.zeros((d, dv)) if P0 is None else P0
    E0 = np.zeros((d, dv)) if E0 is None else E0
    outs = []
    for t0 in range(0, q.shape[0], c):
        Q, K, V = q[t0:t0 + c], k[t0:t0 + c], v[t0:t0 + c]
        n = Q.shape[0]
        tau = np.arange(n)
        At = np.tril(Q @ K.T) * np.tril(g ** (tau[:, None] - tau[None, :]).clip(min=0))
        Gam = (g ** (tau + 1))[:, None]
        Lam = (g ** (n - 1 - tau))[:, None]
        Y = Gam * (Q @ P0) + At @ V
        outs.append(Gam * (Q @ E0) + At @ Y)
        P0 = g ** n * P0 + K.T @ (Lam * V)
        E0 = g ** n * E0 + K.T @ (Lam * Y)
    return np.vstack(outs), P0, E0


@pytest.mark.parametrize("gamma", [1.0, 0.97, 0.6])
@pytest.mark.parametrize("T,c", [(1, 8), (13, 8), (64, 16), (99, 32)])
def test_ahla_decayed_chunk_step_matches_recurrence(T, c, gamma):
    q, k, v = rand_head(T, 5, 3, seed=T + 2000)
    O, _, _ = ahla_walk_decayed(q, k, v, c, gamma)
    assert rel(O, recur("ahlad", q, k, v, gamma=gamma)) < 1e-12


@pytest.mark.parametrize("normalized", [False, True])
@pytest.mark.parametrize("gamma", [0.97, 0.6])
def test_ahla_decayed_segment_plan_matches_recurrence(gamma, normalized):
    """Decayed summary segments walked from zero (rho = g^length), the fold of their prefix with
    summary l weighted by the product of the later summaries' rho (P0, E0, and the cross term
    P^T_m D_suf^T(m+1) by the weight of m), then decayed output walks; on [V | 1] for the
    ratio-normalised form (its vectors mK, n are the ones column's P and E)."""
    T, c, NCH, d, dv = 150, 8, 3, 4, 3
    q, k, v = rand_head(T, d, dv, seed=9)
    if normalized:
        q, k = np.abs(q), np.abs(k)
    v1 = np.hstack([v, np.ones((T, 1))]) if normalized else v
    seg_tok = NCH * c
    n_out = -(-T // seg_tok)
    slots = []
    for i in range(n_out - 1):
        sl = slice(i * seg_tok, (i + 1) * seg_tok)
        _, P, E = ahla_walk_decayed(q[sl], k[sl], v1[sl], c, gamma)
        slots.append(dict(P=P, E=E, D=k[sl].T @ q[sl], rho=gamma ** seg_tok))
    outs = []
    for n in range(n_out):
        P0, E0 = np.zeros((d, v1.shape[1])), np.zeros((d, v1.shape[1]))
        w = [np.prod([s["rho"] for s in slots[l + 1:n]]) for l in range(n)]
        for l in range(n):
            P0 = P0 + w[l] * slots[l]["P"]
            E0 = E0 + w[l] * slots[l]["E"]
        for m in range(n - 1):
            Dsuf = sum(slots[l]["D"] for l in range(m + 1, n))
            E0 = E0 + w[m] * (Dsuf @ slots[m]["P"])
        sl = slice(n * seg_tok, min((n + 1) * seg_tok, T))
        outs.append(ahla_walk_decayed(q[sl], k[sl], v1[sl], c, gamma, P0=P0, E0=E0)[0])
    O = np.vstack(outs)
    if normalized:
        O = O[:, :-1] / (O[:, -1:] + EPS)
    assert rel(O, recur("ahlan" if normalized else "ahlad", q, k, v, gamma=gamma)) < 1e-12


# ---------------------------------------------------------------------------
# decayed second order: chunk summaries, prefix recurrences and the output split
# ---------------------------------------------------------------------------

def decay_forward(q, k, v, g, c, drop=None):
    """The decay kernels' algebra, chunk by chunk.  ``drop`` zeroes one named term (used
    only to show that each term is needed)."""
    T, d = q.shape
    tau = np.arange(c)
    lam = g ** (c - 1 - tau)
    rho = g ** c
    Gam = g ** (tau + 1)
    Dl = tau[:, None] - tau[None, :]
    Dg = np.where(Dl >= 0, g ** np.maximum(Dl, 0), 0.0)
    L = (Dl >= 0).astype(float)
    keep = lambda name, x: 0.0 * x if drop == name else x
    Qs, Ks, Vs = chunks(q, c), chunks(k, c), chunks(v, c)
    # k_dec_summary: every chunk from the zero state
    sums = []
    for Q, K, V in zip(Qs, Ks, Vs):
        As = Q @ K.T
        U = np.triu(As, 1)
        sums.append(dict(S=K.T @ (lam[:, None] * K), C=Q.T @ (lam[:, None] * V), Khat=K.T @ K,
                         G=K.T @ (U.T @ (lam[:, None] * V))))
    # prefix kernels, then k_dec_output
    dv = v.shape[1]
    S0, C0, G0 = np.zeros((d, d)), np.zeros((d, dv)), np.zeros((d, dv))
    outs = []
    for (Q, K, V), s in zip(zip(Qs, Ks, Vs), sums):
        As = Q @ K.T
        A = L * As
        U = np.triu(As, 1)
        At = Dg * As
        H = np.where(Dl > 0, (Dg - 1.0) * As, 0.0)
        P = Q @ S0
        W = Dg * (Gam[:, None] * (P @ Q.T) + At @ A.T + keep("HU", H @ U.T))
        O = W @ V + Gam[:, None] * ((Gam[:, None] * P + keep("HK", H @ K)) @ C0) - keep("QG0", Gam[:, None] * (Q @ G0))
        outs.append(O)
        G0 = rho * G0 + s["G"] + keep("KhatC0", rho * s["Khat"] @ C0)
        S0 = rho * S0 + s["S"]
        C0 = rho * C0 + s["C"]
    return np.vstack(outs)[:T]


@pytest.mark.parametrize("gamma", [1.0, 0.999, 0.95, 0.5])
@pytest.mark.parametrize("T,c", [(5, 8), (37, 8), (64, 16), (100, 16)])
def test_decay_chunk_algebra_matches_recurrence(T, c, gamma):
    q, k, v = rand_head(T, 4, 3, seed=T + int(gamma * 1000))
    assert rel(decay_forward(q, k, v, gamma, c), recur("hla2d", q, k, v, gamma=gamma)) < 1e-12


def test_decay_gamma_one_reduces_to_the_undecayed_walk():
    q, k, v = rand_head(61, 4, 3, seed=3)
    np.testing.assert_allclose(decay_forward(q, k, v, 1.0, 8), hla2_walk(q, k, v, 8, False)[0],
                               rtol=0, atol=1e-12)


@pytest.mark.parametrize("term", ["HU", "HK", "QG0", "KhatC0"])
def test_decay_every_term_is_needed(term):
    """Removing any one cross term breaks the match: the test above is not vacuous."""
    q, k, v = rand_head(48, 4, 3, seed=9)
    ref = recur("hla2d", q, k, v, gamma=0.9)
    assert rel(decay_forward(q, k, v, 0.9, 16, drop=term), ref) > 1e-3


def decay_walk_chunk(Q, K, V, g, S0, C0, G0, drop=None):
    """One chunk of the decayed second-order walker, state (S0, C0, G0) carried in.

    Returns O and the state after the chunk:
        S0' = rho S0 + K^T Lam K,  C0' = rho C0 + Q^T Lam V,  G0' = rho G0 + K^T Y,
        Y = U^T Lam V + rho K C0,
        O = W V + Gam (Z C0 - Q G0),  Z = Gam P + H K,  P = Q S0,
        W = Dg (.) L (.) (Gam P Q^T + At A^T + H U^T).
    ``drop`` zeroes one named term (used only to show that each term is needed)."""
    c = Q.shape[0]
    tau = np.arange(c)
    lam, rho, Gam = g ** (c - 1 - tau), g ** c, g ** (tau + 1)
    Dl = tau[:, None] - tau[None, :]
    Dg = np.where(Dl >= 0, g ** np.maximum(Dl, 0), 0.0)
    keep = lambda name, x: 0.0 * x if drop == name else x
    As = Q @ K.T
    A, U = np.tril(As), np.triu(As, 1)
    At = Dg * As
    H = np.where(Dl > 0, (Dg - 1.0) * As, 0.0)
    P = Q @ S0
    W = Dg * (Gam[:, None] * (P @ Q.T) + At @ A.T + H @ U.T)
    Z = Gam[:, None] * P + H @ K
    O = W @ V + Gam[:, None] * (Z @ C0 - Q @ G0)
    Y = U.T @ (lam[:, None] * V) + keep("rhoKC0", rho * (K @ C0))
    return O, (rho * S0 + K.T @ (lam[:, None] * K), rho * C0 + Q.T @ (lam[:, None] * V), rho * G0 + K.T @ Y)


def decay_walk_summary(q, k, v, g, c):
    """A summary walk over whole chunks from the zero state: S and the chunk contributions
    to G enter with their weight rho^(N-1-l) (applied to Lam K and to Y), C is carried chunk
    to chunk (Y needs it), Khat = K^T K is summed unweighted; rho_seg = g^(cN)."""
    d, dv = q.shape[1], v.shape[1]
    N = q.shape[0] // c
    tau = np.arange(c)
    rho = g ** c
    S, G, Kh = np.zeros((d, d)), np.zeros((d, dv)), np.zeros((d, d))
    C0 = np.zeros((d, dv))
    for l in range(N):
        Q, K, V = (x[l * c:(l + 1) * c] for x in (q, k, v))
        lam = g ** (c - 1 - tau)
        w = g ** (c * (N - l) - 1 - tau)                       # lam rho^(N-1-l)
        U = np.triu(Q @ K.T, 1)
        Y = U.T @ (lam[:, None] * V) + rho * (K @ C0)
        S = S + K.T @ (w[:, None] * K)
        G = G + K.T @ (rho ** (N - 1 - l) * Y)
        Kh = Kh + K.T @ K
        C0 = rho * C0 + Q.T @ (lam[:, None] * V)
    return dict(S=S, C=C0, G=G, Khat=Kh, rho=g ** (c * N))


def decay_fold(slots, n):
    """The output walker's prologue fold of slots 0..n-1 (exclusive prefix of slot n):
    S0 = sum w_m S_m, C0 = sum w_m C_m, G0 = sum w_m (G_m + Ksuf(m+1) C_m), with
    w_m = prod_{m<p<n} rho_p and Ksuf(m+1) = sum_{m<l<n} Khat_l (unweighted)."""
    S0, C0, G0 = (0.0 * slots[0][x] for x in ("S", "C", "G"))
    w, Ksuf = 1.0, 0.0 * slots[0]["Khat"]
    for m in range(n - 1, -1, -1):
        s = slots[m]
        S0 = S0 + w * s["S"]
        C0 = C0 + w * s["C"]
        G0 = G0 + w * (s["G"] + Ksuf @ s["C"])
        Ksuf = Ksuf + s["Khat"]
        w = w * s["rho"]
    return S0, C0, G0


@pytest.mark.parametrize("gamma", [1.0, 0.999, 0.95, 0.5])
@pytest.mark.parametrize("T,c", [(5, 8), (37, 8), (64, 16), (100, 16)])
def test_decay_walk_chunk_step_matches_recurrence(T, c, gamma):
    q, k, v = rand_head(T, 4, 3, seed=T + int(gamma * 1000))
    S0, C0, G0 = np.zeros((4, 4)), np.zeros((4, 3)), np.zeros((4, 3))
    outs = []
    for Q, K, V in zip(chunks(q, c), chunks(k, c), chunks(v, c)):
        O, (S0, C0, G0) = decay_walk_chunk(Q, K, V, gamma, S0, C0, G0)
        outs.append(O)
    assert rel(np.vstack(outs)[:T], recur("hla2d", q, k, v, gamma=gamma)) < 1e-12


def test_decay_walk_needs_the_rho_k_c0_term():
    """Without the carried C0 in Y the state walk drifts from the recurrence."""
    q, k, v = rand_head(64, 4, 3, seed=5)
    S0, C0, G0 = np.zeros((4, 4)), np.zeros((4, 3)), np.zeros((4, 3))
    outs = []
    for Q, K, V in zip(chunks(q, 16), chunks(k, 16), chunks(v, 16)):
        O, (S0, C0, G0) = decay_walk_chunk(Q, K, V, 0.9, S0, C0, G0, drop="rhoKC0")
        outs.append(O)
    assert rel(np.vstack(outs), recur("hla2d", q, k, v, gamma=0.9)) > 1e-3


@pytest.mark.parametrize("gamma", [0.999, 0.9, 0.5])
@pytest.mark.parametrize("lengths", [[2], [1, 3, 2], [2, 2, 2, 2, 2]])
def test_decay_segment_summaries_and_fold_equal_the_combine(gamma, lengths):
    """Walked segment summaries against the decayed combine of per-token summaries, and the
    prologue fold against the exclusive fold of that combine."""
    c, d, dv = 8, 4, 3
    T = c * sum(lengths)
    q, k, v = rand_head(T, d, dv, seed=sum(lengths) + int(gamma * 100))
    b = [0]
    for n in lengths:
        b.append(b[-1] + n * c)
    slots = [decay_walk_summary(q[b[i]:b[i + 1]], k[b[i]:b[i + 1]], v[b[i]:b[i + 1]], gamma, c)
             for i in range(len(lengths))]
    # reference: walk the recurrence's state over each segment and across them
    for n in range(len(lengths) + 1):
        S0, C0, G0 = decay_fold(slots, n) if n else (np.zeros((d, d)), np.zeros((d, dv)), np.zeros((d, dv)))
        S, C, G = np.zeros((d, d)), np.zeros((d, dv)), np.zeros((d, dv))
        for t in range(b[n]):
            S, C, G = gamma * S, gamma * C, gamma * G
            G = G + np.outer(k[t], k[t]) @ C
            S = S + np.outer(k[t], k[t])
            C = C + np.outer(q[t], v[t])
        for x, y in ((S0, S), (C0, C), (G0, G)):
            np.testing.assert_allclose(x, y, rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("gamma", [0.97, 0.5])
@pytest.mark.parametrize("T,c,NCH,ratio", [(200, 8, 5, 1), (200, 8, 6, 3), (129, 16, 2, 2), (70, 8, 4, 4)])
def test_decay_walk_segment_plan_matches_recurrence(T, c, NCH, ratio, gamma):
    """Summary segments of NCH/ratio chunks walked from zero, each output segment folding
    the slots before it, then walking its chunks: the decayed walker's stages end to end."""
    d, dv = 4, 3
    q, k, v = rand_head(T, d, dv, seed=T + NCH + ratio)
    nchunks = -(-T // c)
    NCHs = NCH // ratio
    n_out = -(-nchunks // NCH)
    slots = [decay_walk_summary(*(x[i * NCHs * c:(i + 1) * NCHs * c] for x in (q, k, v)), gamma, c)
             for i in range((n_out - 1) * ratio)]
    outs = []
    for n in range(n_out):
        state = decay_fold(slots, n * ratio) if n else (np.zeros((d, d)), np.zeros((d, dv)), np.zeros((d, dv)))
        lo, hi = n * NCH * c, min((n + 1) * NCH * c, T)
        for Q, K, V in zip(chunks(q[lo:hi], c), chunks(k[lo:hi], c), chunks(v[lo:hi], c)):
            O, state = decay_walk_chunk(Q, K, V, gamma, *state)
            outs.append(O)
    assert rel(np.vstack(outs)[:T], recur("hla2d", q, k, v, gamma=gamma)) < 1e-11


# ---------------------------------------------------------------------------
# ratio-normalised AHLA / third order: the combine of the normaliser vectors
# ---------------------------------------------------------------------------

def _vec_summaries(q, k, n):
    """Oracle summaries of two segments and of their concatenation, with v a ones column."""
    ones = np.ones((q.shape[0], 1))
    A = dict(q=q[:n], k=k[:n], v=ones[:n])
    B = dict(q=q[n:], k=k[n:], v=ones[n:])
    return A, B, dict(q=q, k=k, v=ones)


@pytest.mark.parametrize("n", [1, 7, 20])
def test_ahla_normaliser_vectors_combine(n):
    """mK and n are P and E with v a ones column: n_AB = n_A + n_B + D_B mK_A."""
    rng = np.random.default_rng(n)
    q, k = rng.standard_normal((31, 4)), rng.standard_normal((31, 4))
    A, B, AB = _vec_summaries(q, k, n)
    sa, sb, sab = (seg.ahla_summary(x["q"], x["k"], x["v"]) for x in (A, B, AB))
    mk_a, mk_b = sa["P"][:, 0], sb["P"][:, 0]
    n_a, n_b = sa["E"][:, 0], sb["E"][:, 0]
    np.testing.assert_allclose(mk_a + mk_b, sab["P"][:, 0], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(n_a + n_b + sb["D"] @ mk_a, sab["E"][:, 0], rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("n", [1, 9, 22])
def test_third_order_normaliser_vectors_combine(n):
    """mK, X1, F1 are P, X, F with v a ones column: X1_AB = X1_A + X1_B + Q2_B mK_A and
    F1_AB = F1_A + F1_B + S_A Q2_B mK_A + S_A X1_B + Z_B mK_A."""
    rng = np.random.default_rng(40 + n)
    q, k = rng.standard_normal((29, 3)), rng.standard_normal((29, 3))
    A, B, AB = _vec_summaries(q, k, n)
    sa, sb, sab = (seg.hla3_summary(x["q"], x["k"], x["v"]) for x in (A, B, AB))
    mk_a, x1_a, f1_a = sa["P"][:, 0], sa["X"][:, 0], sa["F"][:, 0]
    mk_b, x1_b, f1_b = sb["P"][:, 0], sb["X"][:, 0], sb["F"][:, 0]
    np.testing.assert_allclose(x1_a + x1_b + sb["Q2"] @ mk_a, sab["X"][:, 0], rtol=1e-11, atol=1e-11)
    f1 = f1_a + f1_b + sa["S"] @ sb["Q2"] @ mk_a + sa["S"] @ x1_b + sb["Z"] @ mk_a
    np.testing.assert_allclose(f1, sab["F"][:, 0], rtol=1e-11, atol=1e-11)


def test_normaliser_vectors_give_the_literal_denominator():
    """q_t . n_t (AHLA) and q_t . F1_t (third order) from the running vectors equal the masked
    operators applied to a ones column, token by token."""
    rng = np.random.default_rng(44)
    T, d = 17, 3
    q, k = np.abs(rng.standard_normal((T, d))), np.abs(rng.standard_normal((T, d)))
    ones = np.ones((T, 1))
    den_a = oracle.recur("ahla", q[None, None], k[None, None], ones[None, None])[0, 0, :, 0]
    den_3 = oracle.recur("hla3", q[None, None], k[None, None], ones[None, None])[0, 0, :, 0]
    mk, nv, S, F1 = np.zeros(d), np.zeros(d), np.zeros((d, d)), np.zeros(d)
    for t in range(T):
        mk = mk + k[t]
        nv = nv + k[t] * (q[t] @ mk)
        S = S + np.outer(k[t], k[t])
        F1 = F1 + (S @ q[t]) * (q[t] @ mk)
        assert abs(q[t] @ nv - den_a[t]) < 1e-12 * max(1.0, den_a[t])
        assert abs(q[t] @ F1 - den_3[t]) < 1e-12 * max(1.0, den_3[t])


def third_order_factored_prefix(sums, decayed=False):
    """The third-order exclusive prefix as the CUDA-core path runs it (three launches): plain
    exclusive sums S0, P0, then per chunk the corrected F_l + S0(l) Q2_l P0(l) + S0(l) X_l +
    Z_l P0(l), then its plain exclusive sum F0.  Decayed: running sums run = rho_l run + y_l
    and the cross term scaled by rho_l."""
    rho = [float(s["rho"]) if decayed else 1.0 for s in sums]
    S0 = [0.0 * sums[0]["S"]]
    P0 = [0.0 * sums[0]["P"]]
    for l, s in enumerate(sums[:-1]):
        S0.append(rho[l] * S0[-1] + s["S"])
        P0.append(rho[l] * P0[-1] + s["P"])
    Y = [s["F"] + rho[l] * (S0[l] @ s["Q2"] @ P0[l] + S0[l] @ s["X"] + s["Z"] @ P0[l])
         for l, s in enumerate(sums)]
    F0 = [0.0 * Y[0]]
    for l, y in enumerate(Y[:-1]):
        F0.append(rho[l] * F0[-1] + y)
    return [dict(S=S0[l], P=P0[l], F=F0[l]) for l in range(len(sums))]


@pytest.mark.parametrize("lengths", [[6], [3, 9, 1], [8, 8, 8, 8, 8], [1, 2, 3, 4, 5, 6, 7]])
def test_third_order_factored_prefix_equals_the_combine_fold(lengths):
    T, d, dv = sum(lengths), 4, 3
    q, k, v = rand_head(T, d, dv, seed=7 + len(lengths))
    b = seg.split_points(T, lengths)
    sums = [seg.hla3_summary(q[b[i]:b[i + 1]], k[b[i]:b[i + 1]], v[b[i]:b[i + 1]]) for i in range(len(lengths))]
    ref = seg.fold_exclusive(sums, seg.hla3_combine, seg.hla3_identity(d, dv))
    got = third_order_factored_prefix(sums)
    for n in range(len(lengths)):
        for key in ("S", "P", "F"):
            np.testing.assert_allclose(got[n][key], ref[n][key], rtol=0, atol=1e-11)


@pytest.mark.parametrize("lengths", [[6], [3, 9, 1], [8, 8, 8, 8, 8], [1, 2, 3, 4, 5, 6, 7]])
@pytest.mark.parametrize("gamma", [0.5, 0.9, 1.0])
def test_decayed_third_order_factored_prefix_equals_the_combine_fold(lengths, gamma):
    """The decayed third-order prefix in factored form (decayed running sums of S, P and of the
    rho-scaled corrected F) against the fold of the decayed combine."""
    T, d, dv = sum(lengths), 4, 3
    q, k, v = rand_head(T, d, dv, seed=11 + len(lengths))
    b = seg.split_points(T, lengths)
    sums = [seg.hla3_summary(q[b[i]:b[i + 1]], k[b[i]:b[i + 1]], v[b[i]:b[i + 1]], gamma=gamma)
            for i in range(len(lengths))]
    ref = seg.fold_exclusive(sums, seg.hla3_combine, seg.hla3_identity(d, dv))
    got = third_order_factored_prefix(sums, decayed=True)
    for n in range(len(lengths)):
        for key in ("S", "P", "F"):
            np.testing.assert_allclose(got[n][key], ref[n][key], rtol=0, atol=1e-11)
    # a planted mistake: the cross term without its rho differs once there is decay
    if gamma < 1.0 and len(lengths) > 2:
        wrong = third_order_factored_prefix([dict(s, rho=np.array(1.0)) if i else s for i, s in enumerate(sums)],
                                            decayed=True)
        assert max(np.abs(wrong[n]["F"] - ref[n]["F"]).max() for n in range(len(lengths))) > 1e-6
