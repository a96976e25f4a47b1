"""GPU backward pass of the masked second-order output against the fp64 gradient reference.

"Higher-order Linear Attention" summary (gist.science 2510.27258), Metodología 4 and
Contribuciones 2: exact scan-based training.  The reference is ``oracle.backward.hla2_grads``
(reverse-mode differentiation of the masked-matrix definition, pinned by finite differences in
``tests/test_backward_algebra.py``).  The library's hla2_backward runs the chunk-parallel reverse
walk on the GPU: fp32 on the CUDA cores, except the last stage (the gradients of every chunk) for
bf16 inputs at d = 64, which runs on the tensor cores with bf16 operands.  Metric and gates as for
the forward: max row-wise relative L2 error, 1e-4 for fp32 inputs, 2e-2 for bf16 inputs.
"""
import numpy as np
import pytest

import hla_inputs
import oracle
from oracle.backward import hla2_grads

torch = pytest.importorskip("torch")
import higher_order_linear_chunked_b200 as hla  # noqa: E402

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-4, "bf16": 2e-2}


def _case(dtype, B, H, T, d, seed):
    w = hla_inputs.Workload(f"bwd_{T}", "hla2", dtype, B, H, T, d, d, "scaled", "scaled", seed=seed)
    q, k, v, _ = hla_inputs.make_inputs(w)
    g = torch.Generator("cpu").manual_seed(seed + 1000)
    do = torch.randn((B, H, T, d), generator=g, dtype=torch.float32)
    return q, k, v, do


def _check(dtype, q, k, v, do):
    dev = torch.device("cuda:0")
    got = hla.hla2_backward(q.to(dev), k.to(dev), v.to(dev), do.to(dev))
    torch.cuda.synchronize()
    B, H = q.shape[:2]
    for bh in range(B * H):
        b, h = divmod(bh, H)
        want = hla2_grads(q[b, h], k[b, h], v[b, h], do[b, h])
        for name, gt, wt in zip(("dq", "dk", "dv"), got, want):
            err = oracle.max_row_rel_err(gt[b, h].cpu(), wt)
            assert err <= TOL[dtype], (name, bh, err)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("d", [32, 64])
@pytest.mark.parametrize("T", [1, 63, 64, 65, 200, 333])
def test_backward_parity(dtype, d, T):
    q, k, v, do = _case(dtype, 1, 2, T, d, seed=T + d)
    _check(dtype, q, k, v, do)


def test_backward_many_heads_and_chunks():
    q, k, v, do = _case("bf16", 2, 3, 1000, 64, seed=7)
    _check("bf16", q, k, v, do)


def test_backward_matches_autograd_of_the_gpu_forward_at_the_headline_shape():
    """At B=4, H=16, T=4096, d=64 the fp64 reference is too large to run per head in the test, so
    the gradient is checked by a property that holds at any size: for a random direction (dQ, dK,
    dV)-weighted sum, <grad, delta> equals the directional derivative of <O, dO> computed from the
    oracle's forward by central differences on two heads.

    Gate: for delta with independent standard normal entries, <grad, delta> and <err, delta> are
    centred with standard deviations ||grad|| and ||err||, so the error is measured in units of
    ||grad|| (the gradient of the heads checked): |ana - num| <= 2e-2 ||grad||, the bf16 parity
    gate.  bf16 inputs at d = 64 take the tensor-core gradient kernel, whose bf16 operands leave
    about 2e-3 of ||grad|| (checked chunk by chunk against the fp64 reference in
    test_backward_full_length_head); |num| itself has no fixed relation to ||grad||."""
    B, H, T, d = 4, 16, 4096, 64
    q, k, v, do = _case("bf16", B, H, T, d, seed=11)
    dev = torch.device("cuda:0")
    dq, dk, dv = (x.cpu().double().numpy() for x in hla.hla2_backward(q.to(dev), k.to(dev), v.to(dev), do.to(dev)))
    assert np.isfinite(dq).all() and np.isfinite(dk).all() and np.isfinite(dv).all()
    rng = np.random.default_rng(0)
    for bh in (0, B * H - 1):
        b, h = divmod(bh, H)
        qh, kh, vh, doh = (x[b, h].double().numpy() for x in (q, k, v, do))
        dirs = [rng.standard_normal(x.shape) for x in (qh, kh, vh)]
        eps = 1e-4

        def f(s):
            o = oracle.recur("hla2", (qh + s * dirs[0])[None, None], (kh + s * dirs[1])[None, None],
                             (vh + s * dirs[2])[None, None])[0, 0]
            return float(np.sum(o * doh))
        num = (f(eps) - f(-eps)) / (2 * eps)
        ana = float(np.sum(dq[b, h] * dirs[0]) + np.sum(dk[b, h] * dirs[1]) + np.sum(dv[b, h] * dirs[2]))
        gnorm = float(np.sqrt(np.sum(dq[b, h] ** 2) + np.sum(dk[b, h] ** 2) + np.sum(dv[b, h] ** 2)))
        assert abs(ana - num) <= TOL["bf16"] * gnorm, (bh, ana, num, gnorm)


def test_backward_full_length_head():
    """One head at the headline's length (T = 4096, 32 tensor-core chunks, the carried state and
    adjoints at their largest) against the fp64 reference gradient, row by row."""
    q, k, v, do = _case("bf16", 1, 1, 4096, 64, seed=11)
    _check("bf16", q, k, v, do)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("d", [32, 64])
@pytest.mark.parametrize("T", [2, 65, 200])
def test_normalised_backward_parity(dtype, d, T):
    """The ratio-normalised output's gradient (hla2_backward_normalized) against
    ``oracle.backward.hla2n_grads`` (reverse-mode through num / (den + eps), pinned by finite
    differences), on the normalised workload's input distribution (positive q and k).  A single
    token is the degenerate case, tested below: there o = v s^2 / (s^2 + eps) with s = q.k does
    not depend on q or k up to eps."""
    from oracle.backward import hla2n_grads
    w = hla_inputs.Workload(f"bwdn_{T}", "hla2n", dtype, 1, 2, T, d, d, "softplus", "unit", seed=T + 3 * d)
    q, k, v, _ = hla_inputs.make_inputs(w)
    do = torch.randn((1, 2, T, d), generator=torch.Generator("cpu").manual_seed(T), dtype=torch.float32)
    dev = torch.device("cuda:0")
    got = hla.hla2_backward(q.to(dev), k.to(dev), v.to(dev), do.to(dev), normalized=True, eps=w.eps)
    torch.cuda.synchronize()
    for h in range(2):
        want = hla2n_grads(q[0, h], k[0, h], v[0, h], do[0, h], w.eps)
        for name, gt, wt in zip(("dq", "dk", "dv"), got, want):
            err = oracle.max_row_rel_err(gt[0, h].cpu(), wt)
            assert err <= TOL[dtype], (name, h, err)


def test_normalised_backward_single_token():
    """T = 1: dv = s^2 / (s^2 + eps) dO exactly; dq and dk are of order eps, the difference of the
    numerator's and the denominator's terms, each of size 2 |v.dO| |k| / |s|.  The GPU result must
    be small against those terms (fp32 cancellation leaves a few units of 1e-7 of them)."""
    w = hla_inputs.Workload("bwdn_1", "hla2n", "f32", 1, 2, 1, 32, 32, "softplus", "unit", seed=5)
    q, k, v, _ = hla_inputs.make_inputs(w)
    do = torch.randn((1, 2, 1, 32), generator=torch.Generator("cpu").manual_seed(1), dtype=torch.float32)
    dev = torch.device("cuda:0")
    dq, dk, dv = (x.cpu().double() for x in hla.hla2_backward(q.to(dev), k.to(dev), v.to(dev), do.to(dev),
                                                              normalized=True, eps=w.eps))
    for h in range(2):
        qh, kh, vh, dh = (x[0, h, 0].double() for x in (q, k, v, do))
        s = float(qh @ kh)
        np.testing.assert_allclose(dv[0, h, 0].numpy(), (s * s / (s * s + w.eps) * dh).numpy(), rtol=1e-6)
        scale = 2 * abs(float(vh @ dh)) / abs(s)
        assert float(dq[0, h, 0].norm()) <= 1e-5 * scale * float(kh.norm())
        assert float(dk[0, h, 0].norm()) <= 1e-5 * scale * float(qh.norm())


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("d", [32, 64])
@pytest.mark.parametrize("T", [1, 63, 64, 65, 200, 333])
def test_ahla_backward_parity(dtype, d, T):
    """AHLA's gradient (ahla_backward, fp32 on the CUDA cores) against ``oracle.backward.ahla_grads``
    (reverse-mode through O = A (A V), pinned by finite differences)."""
    from oracle.backward import ahla_grads
    q, k, v, do = _case(dtype, 1, 2, T, d, seed=T + 2 * d)
    dev = torch.device("cuda:0")
    got = hla.ahla_backward(q.to(dev), k.to(dev), v.to(dev), do.to(dev))
    torch.cuda.synchronize()
    for h in range(2):
        want = ahla_grads(q[0, h], k[0, h], v[0, h], do[0, h])
        for name, gt, wt in zip(("dq", "dk", "dv"), got, want):
            err = oracle.max_row_rel_err(gt[0, h].cpu(), wt)
            assert err <= TOL[dtype], (name, h, err)


def test_ahla_backward_many_heads_and_chunks():
    from oracle.backward import ahla_grads
    q, k, v, do = _case("bf16", 2, 3, 1000, 64, seed=8)
    dev = torch.device("cuda:0")
    got = hla.ahla_backward(q.to(dev), k.to(dev), v.to(dev), do.to(dev))
    torch.cuda.synchronize()
    for bh in range(6):
        b, h = divmod(bh, 3)
        want = ahla_grads(q[b, h], k[b, h], v[b, h], do[b, h])
        for name, gt, wt in zip(("dq", "dk", "dv"), got, want):
            assert oracle.max_row_rel_err(gt[b, h].cpu(), wt) <= TOL["bf16"], (name, bh)
