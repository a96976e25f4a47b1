"""Pins of the fp64 oracle to things other than itself (CPU only).

* hand-worked values (tests/golden/hand_examples.json, derivations in the .md);
* the literal double sums of the definitions, as pure-Python loops, on tiny inputs;
* closed forms (T = 1; d = 1 with all-ones inputs);
* invariants: homogeneity, causality, constant-v normalisation, gamma = 1;
* the decayed closed form derived from the stated reading;
* exactness of the segment scan (Blelloch and left fold) against the serial
  recurrence, combine associativity and identity;
* planted mistakes (in the oracle, on the CPU) that these pins must catch.

Sources: "Higher-order Linear Attention" summary (gist.science 2510.27258),
Metodología 1-4, Contribuciones 1-3, Resultados (exactness, causality).
"""
import json
import os

import numpy as np
import pytest

import oracle
import oracle.brute as brute
import oracle.segments as seg

GOLD = os.path.join(os.path.dirname(__file__), "golden", "hand_examples.json")
EPS = 1e-6


def rel(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300))


def one_head(x):
    x = np.asarray(x, dtype=np.float64)
    return x[None, None]


# ---------------------------------------------------------------------------
# hand-worked values
# ---------------------------------------------------------------------------

with open(GOLD) as f:
    GOLDEN = json.load(f)["cases"]


@pytest.mark.parametrize("case", GOLDEN, ids=[c["name"] for c in GOLDEN])
def test_golden_hand_examples(case):
    q, k, v = (one_head(case[n]) for n in ("q", "k", "v"))
    for op in ("hla2", "ahla", "hla3"):
        exp = np.asarray(case[op], dtype=np.float64)
        np.testing.assert_allclose(oracle.recur(op, q, k, v)[0, 0], exp, rtol=0, atol=1e-12)
        np.testing.assert_allclose(brute.forward(op, q, k, v)[0, 0], exp, rtol=0, atol=1e-12)
    num = np.asarray(case["hla2n_num"], dtype=np.float64)
    den = np.asarray(case["hla2n_den"], dtype=np.float64)[:, None]
    exp = num / (den + EPS)
    np.testing.assert_allclose(oracle.recur("hla2n", q, k, v, eps=EPS)[0, 0], exp, rtol=1e-14, atol=0)
    np.testing.assert_allclose(brute.hla2(q, k, v, True, EPS)[0, 0], exp, rtol=1e-14, atol=0)
    if "hla2d" in case:
        g = np.array([case["hla2d_gamma"]])
        exp = np.asarray(case["hla2d"], dtype=np.float64)
        np.testing.assert_allclose(oracle.recur("hla2d", q, k, v, gamma=g)[0, 0], exp, rtol=0, atol=1e-12)
        np.testing.assert_allclose(brute.hla2_decay(q, k, v, g)[0, 0], exp, rtol=0, atol=1e-12)
    for op in ("ahlad", "hla3d"):
        if op in case:
            g = np.array([case["hla2d_gamma"]])
            exp = np.asarray(case[op], dtype=np.float64)
            np.testing.assert_allclose(oracle.recur(op, q, k, v, gamma=g)[0, 0], exp, rtol=0, atol=1e-12)
            np.testing.assert_allclose(brute.forward(op, q, k, v, gamma=g)[0, 0], exp, rtol=0, atol=1e-12)


# ---------------------------------------------------------------------------
# literal sums of the definitions (pure Python, tiny)
# ---------------------------------------------------------------------------

def _dot(a, b):
    return sum(x * y for x, y in zip(a, b))


def literal_hla2(q, k, v, normalized=False, eps=EPS):
    T, dv = len(q), len(v[0])
    out = []
    for t in range(T):
        num = [0.0] * dv
        den = 0.0
        for j in range(t + 1):
            w = 0.0
            for i in range(j + 1):
                w += _dot(q[t], k[i]) * _dot(q[j], k[i])
            den += w
            for c in range(dv):
                num[c] += w * v[j][c]
        out.append([x / (den + eps) for x in num] if normalized else num)
    return out


def literal_ahla(q, k, v):
    T, dv = len(q), len(v[0])
    out = []
    for t in range(T):
        o = [0.0] * dv
        for j in range(t + 1):
            inner = [0.0] * dv
            for i in range(j + 1):
                s = _dot(q[j], k[i])
                for c in range(dv):
                    inner[c] += s * v[i][c]
            a = _dot(q[t], k[j])
            for c in range(dv):
                o[c] += a * inner[c]
        out.append(o)
    return out


def literal_hla3(q, k, v):
    """o_t = sum_s M_ts sum_u A_su v_u with A_su = q_s.k_u (u<=s), M_ts = sum_{i<=s} A_ti A_si (s<=t)."""
    T, dv = len(q), len(v[0])
    out = []
    for t in range(T):
        o = [0.0] * dv
        for s in range(t + 1):
            m = sum(_dot(q[t], k[i]) * _dot(q[s], k[i]) for i in range(s + 1))
            for u in range(s + 1):
                a = _dot(q[s], k[u])
                for c in range(dv):
                    o[c] += m * a * v[u][c]
        out.append(o)
    return out


def literal_hla2_decay(q, k, v, g):
    """The recurrence as stated, with scalar Python loops: scale every state, then update."""
    T, d, dv = len(q), len(q[0]), len(v[0])
    S = [[0.0] * d for _ in range(d)]
    C = [[0.0] * dv for _ in range(d)]
    G = [[0.0] * dv for _ in range(d)]
    out = []
    for t in range(T):
        for a in range(d):
            for b in range(d):
                S[a][b] *= g
            for c in range(dv):
                C[a][c] *= g
                G[a][c] *= g
        kc = [sum(k[t][a] * C[a][c] for a in range(d)) for c in range(dv)]
        for a in range(d):
            for c in range(dv):
                G[a][c] += k[t][a] * kc[c]
        for a in range(d):
            for b in range(d):
                S[a][b] += k[t][a] * k[t][b]
            for c in range(dv):
                C[a][c] += q[t][a] * v[t][c]
        SC = [[sum(S[a][b] * C[b][c] for b in range(d)) for c in range(dv)] for a in range(d)]
        out.append([sum(q[t][a] * (SC[a][c] - G[a][c]) for a in range(d)) for c in range(dv)])
    return out


@pytest.mark.parametrize("seed", [0, 1])
def test_literal_sums(seed):
    rng = np.random.default_rng(seed)
    T, d, dv = 7, 3, 2
    q, k, v = rng.standard_normal((T, d)), rng.standard_normal((T, d)), rng.standard_normal((T, dv))
    ql, kl, vl = q.tolist(), k.tolist(), v.tolist()
    Q, K, V = one_head(q), one_head(k), one_head(v)
    assert rel(oracle.recur("hla2", Q, K, V)[0, 0], literal_hla2(ql, kl, vl)) < 1e-12
    assert rel(oracle.recur("hla2n", Q, K, V, eps=EPS)[0, 0], literal_hla2(ql, kl, vl, True)) < 1e-12
    assert rel(oracle.recur("ahla", Q, K, V)[0, 0], literal_ahla(ql, kl, vl)) < 1e-12
    assert rel(oracle.recur("hla3", Q, K, V)[0, 0], literal_hla3(ql, kl, vl)) < 1e-12
    g = 0.83
    assert rel(oracle.recur("hla2d", Q, K, V, gamma=np.array([g]))[0, 0],
               literal_hla2_decay(ql, kl, vl, g)) < 1e-12


# ---------------------------------------------------------------------------
# recurrence vs masked-matrix definition (exactness claim)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("op", ["hla2", "hla2n", "hla2d", "ahla", "hla3", "hla2u", "ahlan", "hla3n", "ahlad",
                                "hla3d", "hla2n+g", "ahlan+g", "hla3n+g"])
@pytest.mark.parametrize("shape", [(1, 1, 1, 1, 1), (1, 2, 17, 3, 2), (2, 2, 64, 4, 4), (1, 1, 40, 1, 3)])
def test_recur_equals_brute(op, shape):
    """The serial recurrence equals the masked-matrix definition for every op; "op+g" is the
    ratio-normalised op with per-head decay (the gamma argument selects the decayed form)."""
    B, H, T, d, dv = shape
    rng = np.random.default_rng(T * 31 + d)
    q = rng.standard_normal((B, H, T, d)) / np.sqrt(d)
    k = rng.standard_normal((B, H, T, d)) / np.sqrt(d)
    v = rng.standard_normal((B, H, T, dv))
    name = op.split("+")[0]
    if name in ("hla2n", "ahlan", "hla3n"):
        q, k = np.abs(q), np.abs(k)
    g = rng.uniform(0.9, 0.999, size=H) if (op.endswith("+g") or name in oracle.DECAYED) else None
    op = name
    r = oracle.recur(op, q, k, v, gamma=g, eps=EPS)
    b = brute.forward(op, q, k, v, gamma=g, eps=EPS)
    assert oracle.max_row_rel_err(r, b) < 1e-11


# ---------------------------------------------------------------------------
# closed forms
# ---------------------------------------------------------------------------

def test_closed_form_single_token():
    rng = np.random.default_rng(5)
    q, k, v = rng.standard_normal((1, 1, 1, 4)), rng.standard_normal((1, 1, 1, 4)), rng.standard_normal((1, 1, 1, 3))
    s = float(q[0, 0, 0] @ k[0, 0, 0])
    np.testing.assert_allclose(oracle.recur("hla2", q, k, v)[0, 0, 0], s * s * v[0, 0, 0], rtol=1e-14)
    np.testing.assert_allclose(oracle.recur("ahla", q, k, v)[0, 0, 0], s * s * v[0, 0, 0], rtol=1e-14)
    np.testing.assert_allclose(oracle.recur("hla3", q, k, v)[0, 0, 0], s ** 3 * v[0, 0, 0], rtol=1e-14)
    np.testing.assert_allclose(oracle.recur("hla2n", q, k, v, eps=EPS)[0, 0, 0],
                               s * s * v[0, 0, 0] / (s * s + EPS), rtol=1e-14)
    np.testing.assert_allclose(oracle.recur("hla2d", q, k, v, gamma=np.array([0.5]))[0, 0, 0],
                               s * s * v[0, 0, 0], rtol=1e-14)


def test_closed_form_all_ones():
    T = 50
    one = np.ones((1, 1, T, 1))
    t = np.arange(T, dtype=np.float64)
    np.testing.assert_allclose(oracle.recur("hla2", one, one, one)[0, 0, :, 0], (t + 1) * (t + 2) / 2, rtol=1e-14)
    np.testing.assert_allclose(oracle.recur("ahla", one, one, one)[0, 0, :, 0], (t + 1) * (t + 2) / 2, rtol=1e-14)
    np.testing.assert_allclose(oracle.recur("hla3", one, one, one)[0, 0, :, 0],
                               (t + 1) * (t + 2) * (2 * t + 3) / 6, rtol=1e-14)
    den = (t + 1) * (t + 2) / 2
    np.testing.assert_allclose(oracle.recur("hla2n", one, one, one, eps=EPS)[0, 0, :, 0], den / (den + EPS),
                               rtol=1e-14)


def test_decay_all_ones_geometric():
    """d = 1, all ones: o_t = sum_{i,j<=t} c(t,i,j); summed in closed form with geometric series."""
    T, g = 30, 0.9
    one = np.ones((1, 1, T, 1))
    got = oracle.recur("hla2d", one, one, one, gamma=np.array([g]))[0, 0, :, 0]
    for t in range(T):
        n = t + 1
        s1 = (1 - g ** n) / (1 - g)                 # sum_{i<=t} g^(t-i)
        full = s1 * s1                              # sum_{i,j} g^(2t-i-j)
        # sum_{j<i<=t} g^(t-j) = sum_j g^(t-j) * (t - j)  (number of i above j)
        strict = sum(g ** (t - j) * (t - j) for j in range(n))
        assert abs(got[t] - (full - strict)) < 1e-12 * max(1.0, abs(full))


# ---------------------------------------------------------------------------
# invariants
# ---------------------------------------------------------------------------

def _rand(T=24, d=3, dv=2, seed=11, positive=False):
    rng = np.random.default_rng(seed)
    q, k, v = (rng.standard_normal((1, 2, T, d)), rng.standard_normal((1, 2, T, d)),
               rng.standard_normal((1, 2, T, dv)))
    if positive:
        q, k = np.abs(q), np.abs(k)
    return q, k, v


def test_homogeneity():
    q, k, v = _rand()
    a, b, c = 1.5, 0.5, -2.0
    for op, (pa, pb) in (("hla2", (2, 2)), ("ahla", (2, 2)), ("hla3", (3, 3))):
        base = oracle.recur(op, q, k, v)
        scaled = oracle.recur(op, a * q, b * k, c * v)
        np.testing.assert_allclose(scaled, (a ** pa) * (b ** pb) * c * base, rtol=1e-11, atol=1e-12)
    g = np.array([0.9, 0.8])
    base = oracle.recur("hla2d", q, k, v, gamma=g)
    np.testing.assert_allclose(oracle.recur("hla2d", a * q, b * k, c * v, gamma=g),
                               a * a * b * b * c * base, rtol=1e-11, atol=1e-12)
    # ratio-normalised, eps = 0: invariant to q, k scale, linear in v
    base = oracle.recur("hla2n", q, k, v, eps=0.0)
    np.testing.assert_allclose(oracle.recur("hla2n", a * q, b * k, c * v, eps=0.0), c * base, rtol=1e-9)


@pytest.mark.parametrize("op", ["hla2", "hla2n", "hla2d", "ahla", "hla3"])
def test_causality(op):
    q, k, v = _rand(positive=(op == "hla2n"))
    g = np.array([0.95, 0.9])
    base = oracle.recur(op, q, k, v, gamma=g, eps=EPS)
    s = 13
    q2, k2, v2 = q.copy(), k.copy(), v.copy()
    q2[..., s:, :] += 3.0
    k2[..., s:, :] -= 1.0
    v2[..., s:, :] *= -7.0
    pert = oracle.recur(op, q2, k2, v2, gamma=g, eps=EPS)
    assert np.array_equal(base[..., :s, :], pert[..., :s, :])
    assert not np.allclose(base[..., s:, :], pert[..., s:, :])


def test_normalized_constant_v():
    q, k, _ = _rand(positive=True)
    v = np.full((1, 2, q.shape[2], 2), 3.25)
    o = oracle.recur("hla2n", q, k, v, eps=EPS)
    W = brute.hla2(q, k, np.ones_like(v[..., :1]))   # W 1 = the denominators
    np.testing.assert_allclose(o, 3.25 * W / (W + EPS) * np.ones_like(v), rtol=1e-12)


def test_decay_gamma_one_is_undecayed_bitwise():
    q, k, v = _rand()
    a = oracle.recur("hla2d", q, k, v, gamma=np.array([1.0, 1.0]))
    b = oracle.recur("hla2", q, k, v)
    assert np.array_equal(a, b)


# ---------------------------------------------------------------------------
# segment scan (Metodología 4): exactness, associativity, identity
# ---------------------------------------------------------------------------

SEGMENTATIONS = [[40], [1] * 40, [7, 1, 12, 20], [16, 16, 8], [3, 5, 9, 2, 1, 6, 14]]


@pytest.mark.parametrize("lengths", SEGMENTATIONS)
@pytest.mark.parametrize("scan", [seg.blelloch_exclusive, seg.fold_exclusive])
def test_scan_matches_recurrence(lengths, scan):
    q, k, v = _rand(T=40, d=3, dv=2, seed=3)
    qp, kp = np.abs(q), np.abs(k)
    h = 0
    ref = oracle.recur("hla2", q, k, v)[0, h]
    assert rel(seg.hla2_scan_forward(q[0, h], k[0, h], v[0, h], lengths, scan=scan), ref) < 1e-11
    ref = oracle.recur("hla2n", qp, kp, v, eps=EPS)[0, h]
    assert rel(seg.hla2_scan_forward(qp[0, h], kp[0, h], v[0, h], lengths, normalized=True, eps=EPS,
                                     scan=scan), ref) < 1e-11
    ref = oracle.recur("hla2d", q, k, v, gamma=np.array([0.93, 0.9]))[0, h]
    assert rel(seg.hla2_scan_forward(q[0, h], k[0, h], v[0, h], lengths, gamma=0.93, scan=scan), ref) < 1e-11
    ref = oracle.recur("ahla", q, k, v)[0, h]
    assert rel(seg.ahla_scan_forward(q[0, h], k[0, h], v[0, h], lengths, scan=scan), ref) < 1e-11
    ref = oracle.recur("hla3", q, k, v)[0, h]
    assert rel(seg.hla3_scan_forward(q[0, h], k[0, h], v[0, h], lengths, scan=scan), ref) < 1e-10


def _close_summary(a, b):
    for key in a:
        np.testing.assert_allclose(a[key], b[key], rtol=1e-11, atol=1e-11)


@pytest.mark.parametrize("kind", ["hla2", "hla2d", "ahla", "hla3"])
def test_combine_is_concatenation_and_associative(kind):
    q, k, v = (x[0, 0] for x in _rand(T=30, d=3, dv=2, seed=8))
    b = [0, 9, 17, 30]
    if kind in ("hla2", "hla2d"):
        g = 0.9 if kind == "hla2d" else None
        summ = lambda s, e: seg.hla2_summary(q[s:e], k[s:e], v[s:e], g)
        comb, ident = seg.hla2_combine, seg.hla2_identity(3, 2)
    elif kind == "ahla":
        summ = lambda s, e: seg.ahla_summary(q[s:e], k[s:e], v[s:e])
        comb, ident = seg.ahla_combine, seg.ahla_identity(3, 2)
    else:
        summ = lambda s, e: seg.hla3_summary(q[s:e], k[s:e], v[s:e])
        comb, ident = seg.hla3_combine, seg.hla3_identity(3, 2)
    A, B, C = summ(b[0], b[1]), summ(b[1], b[2]), summ(b[2], b[3])
    _close_summary(comb(A, B), summ(b[0], b[2]))                 # concatenation
    _close_summary(comb(comb(A, B), C), comb(A, comb(B, C)))     # associativity
    _close_summary(comb(ident, A), A)                            # identity, both sides
    _close_summary(comb(A, ident), A)


# ---------------------------------------------------------------------------
# planted mistakes: the pins above must notice each of these
# ---------------------------------------------------------------------------

def test_planted_mistakes_are_caught():
    case = GOLDEN[1]
    q, k, v = (one_head(case[n]) for n in ("q", "k", "v"))
    exp = np.asarray(case["hla2"])
    # (1) transposed score matrix
    A_t = np.tril(k[0, 0] @ q[0, 0].T)
    wrong = np.tril(A_t @ A_t.T) @ v[0, 0]
    assert not np.allclose(wrong, exp)
    # (2) strict mask (diagonal dropped)
    A_s = np.tril(q[0, 0] @ k[0, 0].T, -1)
    wrong = np.tril(A_s @ A_s.T) @ v[0, 0]
    assert not np.allclose(wrong, exp)
    # (3) combine without its cross term
    qq, kk, vv = (x[0, 0] for x in _rand(T=20, d=3, dv=2, seed=2))
    ref = oracle.recur("hla2", qq[None, None], kk[None, None], vv[None, None])[0, 0]

    def bad(A, B):
        out = seg.hla2_combine(A, B)
        out["G"] = out["G"] - B["rho"] * (B["Khat"] @ A["C"])
        return out

    sums = [seg.hla2_summary(qq[s:s + 5], kk[s:s + 5], vv[s:s + 5]) for s in range(0, 20, 5)]
    pre = seg.blelloch_exclusive(sums, bad, seg.hla2_identity(3, 2))
    o, _ = oracle.hla2_run(qq[15:], kk[15:], vv[15:], {x: pre[3][x] for x in ("S", "C", "G", "m", "h")})
    assert rel(o, ref[15:]) > 1e-3
    # (4) the other decay reading: G decays, but its cross term uses the
    # undecayed C_{t-1} (G_t = g G_{t-1} + k k^T C_{t-1})
    g = 0.8
    T = 6
    rng = np.random.default_rng(4)
    q4, k4, v4 = rng.standard_normal((T, 2)), rng.standard_normal((T, 2)), rng.standard_normal((T, 2))
    ok = oracle.recur("hla2d", q4[None, None], k4[None, None], v4[None, None], gamma=np.array([g]))[0, 0]
    closed = brute.hla2_decay(q4, k4, v4, g)
    assert rel(ok, closed) < 1e-12
    S = np.zeros((2, 2)); C = np.zeros((2, 2)); G = np.zeros((2, 2)); out = []
    for t in range(T):
        G = g * G + np.outer(k4[t], k4[t]) @ C
        S = g * S + np.outer(k4[t], k4[t])
        C = g * C + np.outer(q4[t], v4[t])
        out.append(q4[t] @ (S @ C - G))
    assert rel(np.array(out), closed) > 1e-3


def test_metric():
    ref = np.array([[[[3.0, 4.0], [1.0, 0.0]]]])
    o = np.array([[[[3.0, 4.5], [1.0, 0.0]]]])
    assert abs(oracle.max_row_rel_err(o, ref) - 0.1) < 1e-15


# ---------------------------------------------------------------------------
# the unmasked configuration (Contribuciones 2): o_t = q_t^T S_t C_t
# ---------------------------------------------------------------------------

def test_unmasked_literal_double_sum():
    rng = np.random.default_rng(21)
    T, d, dv = 9, 3, 2
    q, k, v = rng.standard_normal((T, d)), rng.standard_normal((T, d)), rng.standard_normal((T, dv))
    want = np.zeros((T, dv))
    for t in range(T):
        for i in range(t + 1):
            for j in range(t + 1):
                want[t] += _dot(q[t], k[i]) * _dot(q[j], k[i]) * v[j]
    got = oracle.recur("hla2u", one_head(q), one_head(k), one_head(v))[0, 0]
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(brute.hla2u(q, k, v), want, rtol=1e-12, atol=1e-12)


def test_unmasked_minus_masked_is_the_cross_summary():
    """Metodología 1: G_t corrects the future terms of the naive product, so the unmasked
    output minus the masked one is q_t^T G_t, with G from the masked recurrence's own state."""
    rng = np.random.default_rng(22)
    T, d, dv = 30, 4, 3
    q, k, v = rng.standard_normal((T, d)), rng.standard_normal((T, d)), rng.standard_normal((T, dv))
    ou = oracle.recur("hla2u", one_head(q), one_head(k), one_head(v))[0, 0]
    om = oracle.recur("hla2", one_head(q), one_head(k), one_head(v))[0, 0]
    st = None
    for t in range(T):
        _, st = oracle.hla2_run(q[t:t + 1], k[t:t + 1], v[t:t + 1], st, want_output=False)
        np.testing.assert_allclose(ou[t] - om[t], q[t] @ st["G"], rtol=1e-10, atol=1e-12)


def test_unmasked_single_token_and_planted_mask():
    rng = np.random.default_rng(23)
    q, k, v = rng.standard_normal((1, 5)), rng.standard_normal((1, 5)), rng.standard_normal((1, 2))
    o = oracle.recur("hla2u", one_head(q), one_head(k), one_head(v))[0, 0]
    np.testing.assert_allclose(o[0], (q[0] @ k[0]) ** 2 * v[0], rtol=1e-13)
    # a planted mistake: masking the j side too gives the masked operator, which the pins reject
    T = 12
    q, k, v = rng.standard_normal((T, 3)), rng.standard_normal((T, 3)), rng.standard_normal((T, 2))
    assert oracle.max_row_rel_err(brute.hla2(q, k, v), oracle.recur("hla2u", one_head(q), one_head(k),
                                                                    one_head(v))[0, 0]) > 1e-3


# ---------------------------------------------------------------------------
# ratio-normalised AHLA and third order: the same operator on a ones value column
# ---------------------------------------------------------------------------

def test_normalised_ahla_literal_and_named_summaries():
    """Metodología 2 names the AHLA summaries (P^KV, m^K, E, n).  With m^K = sum k and
    n_t = sum_{j<=t} k_j (q_j . m^K_j), the denominator is q_t . n_t: the literal masked sum
    of the operator with every v replaced by 1."""
    rng = np.random.default_rng(31)
    T, d, dv = 11, 3, 2
    q, k = np.abs(rng.standard_normal((T, d))), np.abs(rng.standard_normal((T, d)))
    v = rng.standard_normal((T, dv))
    num = np.zeros((T, dv))
    den = np.zeros(T)
    mK = np.zeros(d)
    n = np.zeros(d)
    for t in range(T):
        for j in range(t + 1):
            for i in range(j + 1):
                w = _dot(q[t], k[j]) * _dot(q[j], k[i])
                num[t] += w * v[i]
                den[t] += w
        mK += k[t]
        n += k[t] * _dot(q[t], mK)
        assert abs(_dot(q[t], n) - den[t]) < 1e-12 * max(1.0, den[t])
    got = oracle.recur("ahlan", one_head(q), one_head(k), one_head(v), eps=EPS)[0, 0]
    np.testing.assert_allclose(got, num / (den[:, None] + EPS), rtol=1e-12)


def test_normalised_third_order_literal():
    rng = np.random.default_rng(32)
    T, d, dv = 8, 3, 2
    q, k = np.abs(rng.standard_normal((T, d))), np.abs(rng.standard_normal((T, d)))
    v = rng.standard_normal((T, dv))
    A = np.tril(q @ k.T)
    M = np.tril(A @ A.T)
    W = M @ A                                 # o = W v: the masked A A^T A weights
    num = W @ v
    den = W.sum(axis=1)
    got = oracle.recur("hla3n", one_head(q), one_head(k), one_head(v), eps=EPS)[0, 0]
    np.testing.assert_allclose(got, num / (den[:, None] + EPS), rtol=1e-12)


@pytest.mark.parametrize("op", ["ahlan", "hla3n"])
def test_normalised_constant_v_and_homogeneity(op):
    rng = np.random.default_rng(33)
    T, d = 20, 4
    q, k = np.abs(rng.standard_normal((T, d))), np.abs(rng.standard_normal((T, d)))
    v = np.full((T, 3), 2.5)
    o = oracle.recur(op, one_head(q), one_head(k), one_head(v), eps=1e-12)[0, 0]
    np.testing.assert_allclose(o, 2.5, rtol=1e-9)
    v = rng.standard_normal((T, 3))
    o1 = oracle.recur(op, one_head(q), one_head(k), one_head(v), eps=0.0)[0, 0]
    o2 = oracle.recur(op, one_head(3.0 * q), one_head(k), one_head(v), eps=0.0)[0, 0]
    np.testing.assert_allclose(o1, o2, rtol=1e-10)     # degree 0 in q (ratio of equal degrees)


# ---------------------------------------------------------------------------
# decayed AHLA and third order (Contribuciones 2 with Metodología 2 and 3; reading: every state
# of the recurrence scaled by gamma before each token's update)
# ---------------------------------------------------------------------------

def literal_ahla_decay(q, k, v, g):
    """o_t = sum_{j<=t} sum_{i<=j} g^(t-i) (q_t.k_j)(q_j.k_i) v_i, as plain loops."""
    T, dv = len(q), len(v[0])
    out = []
    for t in range(T):
        o = [0.0] * dv
        for j in range(t + 1):
            for i in range(j + 1):
                w = g ** (t - i) * _dot(q[t], k[j]) * _dot(q[j], k[i])
                for c in range(dv):
                    o[c] += w * v[i][c]
        out.append(o)
    return np.asarray(out)


def literal_hla3_decay(q, k, v, g):
    """o_t = sum_{s<=t} sum_{a<=s} sum_{b<=s} g^(t-a) g^(s-b) (q_t.k_a)(q_s.k_a)(q_s.k_b) v_b."""
    T, dv = len(q), len(v[0])
    out = []
    for t in range(T):
        o = [0.0] * dv
        for s in range(t + 1):
            for a in range(s + 1):
                for b in range(s + 1):
                    w = g ** (t - a) * g ** (s - b) * _dot(q[t], k[a]) * _dot(q[s], k[a]) * _dot(q[s], k[b])
                    for c in range(dv):
                        o[c] += w * v[b][c]
        out.append(o)
    return np.asarray(out)


@pytest.mark.parametrize("g", [0.5, 0.9, 1.0])
def test_decayed_ahla_hla3_literal_sums(g):
    rng = np.random.default_rng(int(g * 100))
    T, d, dv = 9, 3, 2
    q, k, v = rng.standard_normal((T, d)), rng.standard_normal((T, d)), rng.standard_normal((T, dv))
    gam = np.array([g])
    np.testing.assert_allclose(oracle.recur("ahlad", one_head(q), one_head(k), one_head(v), gamma=gam)[0, 0],
                               literal_ahla_decay(q.tolist(), k.tolist(), v.tolist(), g), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(oracle.recur("hla3d", one_head(q), one_head(k), one_head(v), gamma=gam)[0, 0],
                               literal_hla3_decay(q.tolist(), k.tolist(), v.tolist(), g), rtol=1e-12, atol=1e-12)


def test_decayed_ahla_hla3_all_ones_closed_forms():
    """d = 1, all ones: AHLA o_t = sum_{m=0}^{t} (m+1) g^m (the pairs i <= j <= t with t - i = m
    number m + 1); third order o_t = sum_{s<=t} g^(t-s) ((1 - g^(s+1)) / (1 - g))^2."""
    T, g = 40, 0.8
    one = np.ones((1, 1, T, 1))
    a = oracle.recur("ahlad", one, one, one, gamma=np.array([g]))[0, 0, :, 0]
    h = oracle.recur("hla3d", one, one, one, gamma=np.array([g]))[0, 0, :, 0]
    for t in range(T):
        assert abs(a[t] - sum((m + 1) * g ** m for m in range(t + 1))) < 1e-12 * max(1.0, a[t])
        ref = sum(g ** (t - s) * ((1 - g ** (s + 1)) / (1 - g)) ** 2 for s in range(t + 1))
        assert abs(h[t] - ref) < 1e-12 * max(1.0, ref)


def test_decayed_ahla_hla3_gamma_one_is_undecayed_bitwise():
    q, k, v = _rand()
    qp, kp = np.abs(q), np.abs(k)
    ones = np.array([1.0, 1.0])
    for op, base in (("ahlad", "ahla"), ("hla3d", "hla3")):
        assert np.array_equal(oracle.recur(op, q, k, v, gamma=ones), oracle.recur(base, q, k, v))
    for op in ("ahlan", "hla3n"):
        assert np.array_equal(oracle.recur(op, qp, kp, v, gamma=ones, eps=EPS), oracle.recur(op, qp, kp, v, eps=EPS))


def test_decayed_ahla_hla3_homogeneity_and_causality():
    q, k, v = _rand()
    g = np.array([0.9, 0.7])
    a, b, c = 1.5, 0.5, -2.0
    for op, p in (("ahlad", 2), ("hla3d", 3)):
        base = oracle.recur(op, q, k, v, gamma=g)
        np.testing.assert_allclose(oracle.recur(op, a * q, b * k, c * v, gamma=g), a ** p * b ** p * c * base,
                                   rtol=1e-11, atol=1e-12)
        s = 11
        q2, k2, v2 = q.copy(), k.copy(), v.copy()
        q2[..., s:, :] += 2.0
        v2[..., s:, :] *= -3.0
        pert = oracle.recur(op, q2, k2, v2, gamma=g)
        assert np.array_equal(base[..., :s, :], pert[..., :s, :])
        assert not np.allclose(base[..., s:, :], pert[..., s:, :])


@pytest.mark.parametrize("lengths", SEGMENTATIONS)
@pytest.mark.parametrize("scan", [seg.blelloch_exclusive, seg.fold_exclusive])
def test_decayed_ahla_hla3_scan_matches_recurrence(lengths, scan):
    q, k, v = _rand(T=40, d=3, dv=2, seed=5)
    g = np.array([0.93, 0.8])
    for op, fwd in (("ahlad", seg.ahla_scan_forward), ("hla3d", seg.hla3_scan_forward)):
        ref = oracle.recur(op, q, k, v, gamma=g)[0, 1]
        assert rel(fwd(q[0, 1], k[0, 1], v[0, 1], lengths, scan=scan, gamma=0.8), ref) < 1e-10


@pytest.mark.parametrize("kind", ["ahla", "hla3"])
def test_decayed_combine_is_concatenation_and_associative(kind):
    q, k, v = (x[0, 0] for x in _rand(T=30, d=3, dv=2, seed=9))
    b = [0, 9, 17, 30]
    g = 0.85
    if kind == "ahla":
        summ = lambda s, e: seg.ahla_summary(q[s:e], k[s:e], v[s:e], g)   # noqa: E731
        comb, ident = seg.ahla_combine, seg.ahla_identity(3, 2)
    else:
        summ = lambda s, e: seg.hla3_summary(q[s:e], k[s:e], v[s:e], g)   # noqa: E731
        comb, ident = seg.hla3_combine, seg.hla3_identity(3, 2)
    A, B, C = summ(b[0], b[1]), summ(b[1], b[2]), summ(b[2], b[3])
    _close_summary(comb(A, B), summ(b[0], b[2]))
    _close_summary(comb(comb(A, B), C), comb(A, comb(B, C)))
    _close_summary(comb(ident, A), A)
    _close_summary(comb(A, ident), A)


def test_decayed_ahla_hla3_planted_mistakes_are_caught():
    """Mistakes a decayed implementation could make, planted in copies of the oracle's maps: the
    pins above must tell each apart from the real thing."""
    q, k, v = (x[0, 0] for x in _rand(T=24, d=3, dv=2, seed=4))
    g = 0.8
    # (1) AHLA with only P decayed (E accumulated undecayed) disagrees with the literal sum
    P = np.zeros((3, 2))
    E = np.zeros((3, 2))
    wrong = []
    for t in range(24):
        P = g * P + np.outer(k[t], v[t])
        E = E + np.outer(k[t], q[t] @ P)
        wrong.append(q[t] @ E)
    lit = literal_ahla_decay(q.tolist(), k.tolist(), v.tolist(), g)
    assert rel(np.asarray(wrong), lit) > 1e-3
    # (2) the third-order combine with an undecayed Q2 map breaks concatenation
    summ = lambda s, e: seg.hla3_summary(q[s:e], k[s:e], v[s:e], g)   # noqa: E731
    A, B = summ(0, 10), summ(10, 24)
    B_plain = dict(B)
    B_plain["Q2"] = q[10:24].T @ q[10:24]
    bad = seg.hla3_combine(A, B_plain)
    assert rel(bad["F"], summ(0, 24)["F"]) > 1e-3
    # (3) the AHLA combine without rho on the cross term breaks concatenation
    sA, sB = seg.ahla_summary(q[:10], k[:10], v[:10], g), seg.ahla_summary(q[10:], k[10:], v[10:], g)
    E_bad = sB["rho"] * sA["E"] + sB["E"] + sB["D"] @ sA["P"]
    assert rel(E_bad, seg.ahla_summary(q, k, v, g)["E"]) > 1e-3
