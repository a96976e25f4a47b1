"""Groundwork for the backward pass (CPU, fp64): the gradient reference and the chunked
reverse walk a kernel would run.

"Higher-order Linear Attention" summary (gist.science 2510.27258), Metodología 4 and
Contribuciones 2 claim exact scan-based training but print no gradient.  The reference,
``oracle.backward.hla2_grads``, is reverse-mode differentiation of the masked-matrix definition.
It is pinned here by central finite differences of the independent numpy definition and by the
single-token closed form.  The chunked reverse walk is then checked against it: the forward
walk over chunks carries (S0, R0); the backward walk runs over the chunks in reverse order,
carrying their adjoints (dS0, dR0), and forms the chunk's dQ, dK, dV with the same masked
chunk-local products as the forward.
"""
import numpy as np
import pytest

import oracle.brute as brute
from oracle.backward import ahla_grads, hla2_grads, hla2n_grads, hla3_grads


def rand(T, d, dv, seed):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((T, d)) / np.sqrt(d), rng.standard_normal((T, d)) / np.sqrt(d),
            rng.standard_normal((T, dv)), rng.standard_normal((T, dv)))


def test_reference_matches_finite_differences():
    q, k, v, do = rand(6, 3, 2, 1)
    gq, gk, gv = hla2_grads(q, k, v, do)
    f = lambda q_, k_, v_: float(np.sum(brute.hla2(q_, k_, v_) * do))   # noqa: E731
    h = 1e-6
    for x, g, which in ((q, gq, 0), (k, gk, 1), (v, gv, 2)):
        num = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args_p = [q, k, v]
            args_m = [q, k, v]
            args_p[which], args_m[which] = xp, xm
            num[idx] = (f(*args_p) - f(*args_m)) / (2 * h)
        np.testing.assert_allclose(g, num, rtol=1e-6, atol=1e-8)


def test_normalised_reference_matches_finite_differences():
    rng = np.random.default_rng(3)
    T, d, dv = 5, 3, 2
    q, k = np.abs(rng.standard_normal((T, d))), np.abs(rng.standard_normal((T, d)))
    v, do = rng.standard_normal((T, dv)), rng.standard_normal((T, dv))
    gq, gk, gv = hla2n_grads(q, k, v, do, 1e-6)
    f = lambda q_, k_, v_: float(np.sum(brute.hla2(q_, k_, v_, normalized=True, eps=1e-6) * do))  # noqa: E731
    h = 1e-6
    for x, g, which in ((q, gq, 0), (k, gk, 1), (v, gv, 2)):
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args_p, args_m = [q, k, v], [q, k, v]
            args_p[which], args_m[which] = xp, xm
            num = (f(*args_p) - f(*args_m)) / (2 * h)
            assert abs(g[idx] - num) <= 1e-6 * max(1.0, abs(num))


def test_reference_single_token_closed_form():
    q, k, v, do = rand(1, 4, 3, 2)
    gq, gk, gv = hla2_grads(q, k, v, do)
    s, w = float(q[0] @ k[0]), float(v[0] @ do[0])
    np.testing.assert_allclose(gq[0], 2 * s * w * k[0], rtol=1e-12)
    np.testing.assert_allclose(gk[0], 2 * s * w * q[0], rtol=1e-12)
    np.testing.assert_allclose(gv[0], s * s * do[0], rtol=1e-12)


def chunks(x, c):
    T = x.shape[0]
    n = -(-T // c)
    return [np.vstack([x, np.zeros((n * c - T, x.shape[1]))])[i * c:(i + 1) * c] for i in range(n)]


def chunked_backward(q, k, v, do, c, drop=None):
    """Reverse walk over chunks.  Forward per chunk (S0, R0 carried in):
        A = L (.) Q K^T,  P = Q S0,  W = L (.) (P Q^T + A A^T),  O = Q R0 + W V,
        Z = P + A K,  S0' = S0 + K^T K,  R0' = R0 + Z^T V.
    Backward per chunk, given dO and the adjoints (dS0', dR0') of the states it hands on:
        dV = W^T dO + Z dR0';  dZ = V dR0'^T;  dW = L (.) dO V^T;
        dP = dZ + dW Q;  dA = L (.) (dZ K^T + (dW + dW^T) A);
        dQ = dO R0^T + dW^T P + dP S0^T + dA K;  dK = K (dS0' + dS0'^T) + A^T dZ + dA^T Q;
        dS0 = dS0' + Q^T dP;  dR0 = dR0' + Q^T dO.
    ``drop`` ("dS" or "dR") withholds one carried adjoint, only to show that it is needed."""
    d, dv = q.shape[1], v.shape[1]
    Qs, Ks, Vs, Gs = chunks(q, c), chunks(k, c), chunks(v, c), chunks(do, c)
    L = np.tril(np.ones((c, c)))
    S0, R0 = np.zeros((d, d)), np.zeros((d, dv))
    saved = []
    for Q, K, V in zip(Qs, Ks, Vs):                     # forward walk: keep the carried states
        saved.append((S0, R0))
        A = L * (Q @ K.T)
        Z = Q @ S0 + A @ K
        S0, R0 = S0 + K.T @ K, R0 + Z.T @ V
    dS, dR = np.zeros((d, d)), np.zeros((d, dv))
    gq, gk, gv = [], [], []
    for (Q, K, V, dO), (S0, R0) in zip(reversed(list(zip(Qs, Ks, Vs, Gs))), reversed(saved)):
        A = L * (Q @ K.T)
        P = Q @ S0
        W = L * (P @ Q.T + A @ A.T)
        Z = P + A @ K
        dV = W.T @ dO + Z @ dR
        dZ = V @ dR.T
        dW = L * (dO @ V.T)
        dP = dZ + dW @ Q
        dA = L * (dZ @ K.T + (dW + dW.T) @ A)
        dQ = dO @ R0.T + dW.T @ P + dP @ S0.T + dA @ K
        dK = K @ (dS + dS.T) + A.T @ dZ + dA.T @ Q
        dS, dR = dS + Q.T @ dP, dR + Q.T @ dO
        if drop == "dS":
            dS = np.zeros_like(dS)
        if drop == "dR":
            dR = np.zeros_like(dR)
        gq.append(dQ); gk.append(dK); gv.append(dV)
    T = q.shape[0]
    return (np.vstack(gq[::-1])[:T], np.vstack(gk[::-1])[:T], np.vstack(gv[::-1])[:T])


@pytest.mark.parametrize("T,c", [(1, 4), (7, 4), (16, 4), (37, 8), (64, 16), (100, 32)])
def test_chunked_reverse_walk_matches_the_reference(T, c):
    q, k, v, do = rand(T, 5, 3, T + c)
    want = hla2_grads(q, k, v, do)
    got = chunked_backward(q, k, v, do, c)
    for a, b in zip(got, want):
        np.testing.assert_allclose(a, b, rtol=1e-10, atol=1e-10)


def z_form_backward(q, k, v, do, c):
    """The tensor-core gradient stage's algebra, chunk-parallel: carried (S0, R0) by the forward's
    exclusive prefixes; the adjoints leaving each chunk by exclusive suffix sums of its terms
        Y = Q^T dO,  U = Q^T (dW Q),  C = Q^T V:   dR'(c) = sum_{m>c} Y_m,
        dS'(c) = sum_{m>c} (U_m + C_m dR'(m)^T);
    then per chunk, in the Z form (Z = Q S0 + A K, W = L (.) Q Z^T):
        dW = L (.) dO V^T,  dZ = dW^T Q + V dR'^T,  dA = L (.) dZ K^T,
        dQ = dO R0^T + dZ S0 + dW Z + dA K,  dK = K (dS' + dS'^T) + A^T dZ + dA^T Q,
        dV = W^T dO + Z dR'."""
    d, dv = q.shape[1], v.shape[1]
    Qs, Ks, Vs, Gs = chunks(q, c), chunks(k, c), chunks(v, c), chunks(do, c)
    n = len(Qs)
    L = np.tril(np.ones((c, c)))
    S0s, R0s = [], []
    S0, R0 = np.zeros((d, d)), np.zeros((d, dv))
    for Q, K, V in zip(Qs, Ks, Vs):
        S0s.append(S0); R0s.append(R0)
        Z = Q @ S0 + (L * (Q @ K.T)) @ K
        S0, R0 = S0 + K.T @ K, R0 + Z.T @ V
    Y = [Q.T @ dO for Q, dO in zip(Qs, Gs)]
    U = [Q.T @ ((L * (dO @ V.T)) @ Q) for Q, V, dO in zip(Qs, Vs, Gs)]
    Cm = [Q.T @ V for Q, V in zip(Qs, Vs)]
    dR = [sum((Y[m] for m in range(i + 1, n)), np.zeros((d, dv))) for i in range(n)]
    dS = [sum((U[m] + Cm[m] @ dR[m].T for m in range(i + 1, n)), np.zeros((d, d))) for i in range(n)]
    gq, gk, gv = [], [], []
    for i, (Q, K, V, dO) in enumerate(zip(Qs, Ks, Vs, Gs)):
        A = L * (Q @ K.T)
        Z = Q @ S0s[i] + A @ K
        W = L * (Q @ Z.T)
        dW = L * (dO @ V.T)
        dZ = dW.T @ Q + V @ dR[i].T
        dA = L * (dZ @ K.T)
        gq.append(dO @ R0s[i].T + dZ @ S0s[i] + dW @ Z + dA @ K)
        gk.append(K @ (dS[i] + dS[i].T) + A.T @ dZ + dA.T @ Q)
        gv.append(W.T @ dO + Z @ dR[i])
    T = q.shape[0]
    return (np.vstack(gq)[:T], np.vstack(gk)[:T], np.vstack(gv)[:T])


@pytest.mark.parametrize("T,c", [(1, 4), (7, 4), (16, 4), (37, 8), (64, 16), (100, 32), (300, 128)])
def test_z_form_chunk_parallel_gradients_match_the_reference(T, c):
    q, k, v, do = rand(T, 5, 3, T + 3 * c)
    want = hla2_grads(q, k, v, do)
    got = z_form_backward(q, k, v, do, c)
    for a, b in zip(got, want):
        np.testing.assert_allclose(a, b, rtol=1e-10, atol=1e-10)


@pytest.mark.parametrize("drop", ["dS", "dR"])
def test_reverse_walk_needs_both_carried_adjoints(drop):
    """Withholding either carried adjoint breaks the gradients once there are several chunks
    (and changes nothing with one chunk): the match above covers the cross-chunk terms."""
    q, k, v, do = rand(40, 4, 3, 5)
    want = hla2_grads(q, k, v, do)
    one = chunked_backward(q, k, v, do, 40, drop=drop)
    for a, b in zip(one, want):
        np.testing.assert_allclose(a, b, rtol=1e-10, atol=1e-10)
    many = chunked_backward(q, k, v, do, 8, drop=drop)
    assert max(np.abs(a - b).max() / np.abs(b).max() for a, b in zip(many, want)) > 1e-3


@pytest.mark.parametrize("T,c", [(1, 4), (23, 8), (64, 16)])
def test_normalised_backward_is_the_walk_on_ones_augmented_values(T, c):
    """The ratio-normalised output is num / (den + eps) with den the operator on a ones column,
    so its backward is the same reverse walk on [V | 1] with the output gradient
    [dO / (den + eps) | -sum_c dO num / (den + eps)^2], the last dV column discarded."""
    rng = np.random.default_rng(T)
    q, k = np.abs(rng.standard_normal((T, 4))) / 2, np.abs(rng.standard_normal((T, 4))) / 2
    v, do = rng.standard_normal((T, 3)), rng.standard_normal((T, 3))
    eps = 1e-6
    v1 = np.hstack([v, np.ones((T, 1))])
    out = brute.hla2(q, k, v1)
    num, den = out[:, :3], out[:, 3:]
    g = np.hstack([do / (den + eps), -(do * num).sum(axis=1, keepdims=True) / (den + eps) ** 2])
    gq, gk, gv = chunked_backward(q, k, v1, g, c)
    want = hla2n_grads(q, k, v, do, eps)
    np.testing.assert_allclose(gq, want[0], rtol=1e-9, atol=1e-10)
    np.testing.assert_allclose(gk, want[1], rtol=1e-9, atol=1e-10)
    np.testing.assert_allclose(gv[:, :3], want[2], rtol=1e-9, atol=1e-10)


# ---------------------------------------------------------------------------
# AHLA (Metodología 2): O = A (A V)
# ---------------------------------------------------------------------------

def test_ahla_reference_matches_finite_differences():
    q, k, v, do = rand(6, 3, 2, 11)
    gq, gk, gv = ahla_grads(q, k, v, do)
    f = lambda q_, k_, v_: float(np.sum(brute.ahla(q_, k_, v_) * do))   # noqa: E731
    h = 1e-6
    for x, g, which in ((q, gq, 0), (k, gk, 1), (v, gv, 2)):
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args_p, args_m = [q, k, v], [q, k, v]
            args_p[which], args_m[which] = xp, xm
            num = (f(*args_p) - f(*args_m)) / (2 * h)
            assert abs(g[idx] - num) <= 1e-6 * max(1.0, abs(num))


def ahla_chunked_backward(q, k, v, do, c):
    """Reverse walk for AHLA.  Forward per chunk (P0, E0 carried in):
        A = L (.) Q K^T,  Y = Q P0 + A V,  O = Q E0 + A Y,  P0' = P0 + K^T V,  E0' = E0 + K^T Y.
    Backward per chunk, given dO and the adjoints (dP0', dE0') of the states it hands on:
        dY = A^T dO + K dE0';  dA = L (.) (dO Y^T + dY V^T);
        dQ = dO E0^T + dY P0^T + dA K;  dK = Y dE0'^T + V dP0'^T + dA^T Q;  dV = K dP0' + A^T dY;
        dE0 = dE0' + Q^T dO;  dP0 = dP0' + Q^T dY."""
    d, dv = q.shape[1], v.shape[1]
    Qs, Ks, Vs, Gs = chunks(q, c), chunks(k, c), chunks(v, c), chunks(do, c)
    L = np.tril(np.ones((c, c)))
    P0, E0 = np.zeros((d, dv)), np.zeros((d, dv))
    saved = []
    for Q, K, V in zip(Qs, Ks, Vs):
        saved.append((P0, E0))
        A = L * (Q @ K.T)
        Y = Q @ P0 + A @ V
        P0, E0 = P0 + K.T @ V, E0 + K.T @ Y
    dP, dE = np.zeros((d, dv)), np.zeros((d, dv))
    gq, gk, gv = [], [], []
    for (Q, K, V, dO), (P0, E0) in zip(reversed(list(zip(Qs, Ks, Vs, Gs))), reversed(saved)):
        A = L * (Q @ K.T)
        Y = Q @ P0 + A @ V
        dY = A.T @ dO + K @ dE
        dA = L * (dO @ Y.T + dY @ V.T)
        gq.append(dO @ E0.T + dY @ P0.T + dA @ K)
        gk.append(Y @ dE.T + V @ dP.T + dA.T @ Q)
        gv.append(K @ dP + A.T @ dY)
        dE, dP = dE + Q.T @ dO, dP + Q.T @ dY
    T = q.shape[0]
    return tuple(np.vstack(g[::-1])[:T] for g in (gq, gk, gv))


def ahla_chunk_parallel_backward(q, k, v, do, c):
    """The AHLA GPU backward's algebra, chunk-parallel: carried (P0, E0) from the forward's
    prefixes; adjoints leaving each chunk as suffix sums of its terms
        Y = Q^T dO,  U = Q^T (A^T dO),  M = Q^T K:   dE'(c) = sum_{m>c} Y_m,
        dP'(c) = sum_{m>c} (U_m + M_m dE'(m));
    then per chunk dY = A^T dO + K dE', dA = L (.) (dO Y^T + dY V^T),
        dQ = dO E0^T + dY P0^T + dA K,  dK = Y dE'^T + V dP'^T + dA^T Q,  dV = K dP' + A^T dY."""
    d, dv = q.shape[1], v.shape[1]
    Qs, Ks, Vs, Gs = chunks(q, c), chunks(k, c), chunks(v, c), chunks(do, c)
    n = len(Qs)
    L = np.tril(np.ones((c, c)))
    P0s, E0s = [], []
    P0, E0 = np.zeros((d, dv)), np.zeros((d, dv))
    for Q, K, V in zip(Qs, Ks, Vs):
        P0s.append(P0); E0s.append(E0)
        A = L * (Q @ K.T)
        Y = Q @ P0 + A @ V
        P0, E0 = P0 + K.T @ V, E0 + K.T @ Y
    Yt = [Q.T @ dO for Q, dO in zip(Qs, Gs)]
    U = [Q.T @ ((L * (Q @ K.T)).T @ dO) for Q, K, dO in zip(Qs, Ks, Gs)]
    M = [Q.T @ K for Q, K in zip(Qs, Ks)]
    dE = [sum((Yt[m] for m in range(i + 1, n)), np.zeros((d, dv))) for i in range(n)]
    dP = [sum((U[m] + M[m] @ dE[m] for m in range(i + 1, n)), np.zeros((d, dv))) for i in range(n)]
    gq, gk, gv = [], [], []
    for i, (Q, K, V, dO) in enumerate(zip(Qs, Ks, Vs, Gs)):
        A = L * (Q @ K.T)
        Y = Q @ P0s[i] + A @ V
        dY = A.T @ dO + K @ dE[i]
        dA = L * (dO @ Y.T + dY @ V.T)
        gq.append(dO @ E0s[i].T + dY @ P0s[i].T + dA @ K)
        gk.append(Y @ dE[i].T + V @ dP[i].T + dA.T @ Q)
        gv.append(K @ dP[i] + A.T @ dY)
    T = q.shape[0]
    return tuple(np.vstack(g)[:T] for g in (gq, gk, gv))


@pytest.mark.parametrize("T,c", [(1, 4), (9, 4), (37, 8), (64, 16), (100, 32)])
def test_ahla_chunk_parallel_gradients_match_the_reference(T, c):
    q, k, v, do = rand(T, 5, 3, T + 5 * c)
    want = ahla_grads(q, k, v, do)
    got = ahla_chunk_parallel_backward(q, k, v, do, c)
    for a, b in zip(got, want):
        np.testing.assert_allclose(a, b, rtol=1e-10, atol=1e-10)


@pytest.mark.parametrize("T,c", [(1, 4), (9, 4), (37, 8), (64, 16), (100, 32)])
def test_ahla_chunked_reverse_walk_matches_the_reference(T, c):
    q, k, v, do = rand(T, 5, 3, T + 2 * c)
    want = ahla_grads(q, k, v, do)
    got = ahla_chunked_backward(q, k, v, do, c)
    for a, b in zip(got, want):
        np.testing.assert_allclose(a, b, rtol=1e-10, atol=1e-10)


# ---------------------------------------------------------------------------
# third order (Metodología 3): O = (M A) V, M = L (.) (A A^T)
# ---------------------------------------------------------------------------

def test_hla3_reference_matches_finite_differences():
    q, k, v, do = rand(6, 3, 2, 12)
    gq, gk, gv = hla3_grads(q, k, v, do)
    f = lambda q_, k_, v_: float(np.sum(brute.hla3(q_, k_, v_) * do))   # noqa: E731
    h = 1e-6
    for x, g, which in ((q, gq, 0), (k, gk, 1), (v, gv, 2)):
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args_p, args_m = [q, k, v], [q, k, v]
            args_p[which], args_m[which] = xp, xm
            num = (f(*args_p) - f(*args_m)) / (2 * h)
            assert abs(g[idx] - num) <= 1e-6 * max(1.0, abs(num))


def hla3_chunked_backward(q, k, v, do, c):
    """Reverse walk for the third order.  Forward per chunk (S0, P0, F0 carried in):
        A = L (.) Q K^T,  P = Q S0,  W = L (.) (P Q^T + A A^T),  Y = Q P0 + A V,  Z = P + A K,
        O = Q F0 + W Y,   S0' = S0 + K^T K,  P0' = P0 + K^T V,  F0' = F0 + Z^T Y.
    Backward per chunk, given dO and the adjoints (dS0', dP0', dF0'):
        dY = W^T dO + Z dF0';  dW = L (.) dO Y^T;  dZ = Y dF0'^T;  dP = dZ + dW Q;
        dA = L (.) (dZ K^T + dY V^T + (dW + dW^T) A);
        dQ = dO F0^T + dW^T P + dY P0^T + dP S0^T + dA K;
        dK = K (dS0' + dS0'^T) + V dP0'^T + A^T dZ + dA^T Q;  dV = K dP0' + A^T dY;
        dS0 = dS0' + Q^T dP;  dP0 = dP0' + Q^T dY;  dF0 = dF0' + Q^T dO."""
    d, dv = q.shape[1], v.shape[1]
    Qs, Ks, Vs, Gs = chunks(q, c), chunks(k, c), chunks(v, c), chunks(do, c)
    L = np.tril(np.ones((c, c)))
    S0, P0, F0 = np.zeros((d, d)), np.zeros((d, dv)), np.zeros((d, dv))
    saved = []
    for Q, K, V in zip(Qs, Ks, Vs):
        saved.append((S0, P0, F0))
        A = L * (Q @ K.T)
        Y = Q @ P0 + A @ V
        Z = Q @ S0 + A @ K
        S0, P0, F0 = S0 + K.T @ K, P0 + K.T @ V, F0 + Z.T @ Y
    dS, dP0a, dF = np.zeros((d, d)), np.zeros((d, dv)), np.zeros((d, dv))
    gq, gk, gv = [], [], []
    for (Q, K, V, dO), (S0, P0, F0) in zip(reversed(list(zip(Qs, Ks, Vs, Gs))), reversed(saved)):
        A = L * (Q @ K.T)
        P = Q @ S0
        W = L * (P @ Q.T + A @ A.T)
        Y = Q @ P0 + A @ V
        Z = P + A @ K
        dY = W.T @ dO + Z @ dF
        dW = L * (dO @ Y.T)
        dZ = Y @ dF.T
        dP = dZ + dW @ Q
        dA = L * (dZ @ K.T + dY @ V.T + (dW + dW.T) @ A)
        gq.append(dO @ F0.T + dW.T @ P + dY @ P0.T + dP @ S0.T + dA @ K)
        gk.append(K @ (dS + dS.T) + V @ dP0a.T + A.T @ dZ + dA.T @ Q)
        gv.append(K @ dP0a + A.T @ dY)
        dS, dP0a, dF = dS + Q.T @ dP, dP0a + Q.T @ dY, dF + Q.T @ dO
    T = q.shape[0]
    return tuple(np.vstack(g[::-1])[:T] for g in (gq, gk, gv))


@pytest.mark.parametrize("T,c", [(1, 4), (9, 4), (37, 8), (64, 16), (100, 32)])
def test_hla3_chunked_reverse_walk_matches_the_reference(T, c):
    q, k, v, do = rand(T, 4, 3, T + 3 * c)
    want = hla3_grads(q, k, v, do)
    got = hla3_chunked_backward(q, k, v, do, c)
    for a, b in zip(got, want):
        np.testing.assert_allclose(a, b, rtol=1e-9, atol=1e-10)
