"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Inputs come from the seeded generators of ``hla_inputs``; the oracle consumes
exactly the values the kernels receive (bf16 workloads are rounded once, then
widened).  Bar: max row-wise relative L2 error <= 1e-4 for fp32 inputs and
<= 2e-2 for bf16 inputs (the problem's stated tolerances).
"""
import math

import numpy as np
import pytest

import hla_inputs
import oracle
import oracle.brute as brute

torch = pytest.importorskip("torch")
import higher_order_linear_chunked_b200 as hla  # noqa: E402

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-4, "bf16": 2e-2}
OPS = ["hla2", "hla2n", "hla2d", "ahla", "hla3"]


def recipe(op, dtype, B, H, T, d, seed=0):
    """Workload of an op name; "ahlan_g" is the ratio-normalised AHLA with per-head decay."""
    decayed = op in ("hla2d", "ahlad", "ahlan_g")
    op = "ahlan" if op == "ahlan_g" else op
    qk = "softplus" if op in ("hla2n", "ahlan") else "scaled"
    v = "unit" if op in ("hla2n", "ahlan") else "scaled"
    g = ((0.95, 0.999) if op == "hla2d" else (0.9, 0.999)) if decayed else None
    return hla_inputs.Workload(f"{op}_{dtype}_{B}x{H}x{T}x{d}", op, dtype, B, H, T, d, d, qk, v,
                               gamma_range=g, seed=seed)


def gpu_forward(op, q, k, v, gamma, eps=1e-6):
    dev = torch.device("cuda:0")
    qd, kd, vd = (x.to(dev) for x in (q, k, v))
    gd = gamma.to(dev) if gamma is not None else None
    o = hla.forward(op, qd, kd, vd, gamma=gd, eps=eps)
    torch.cuda.synchronize()
    return o


def reference(op, q, k, v, gamma, eps=1e-6):
    if q.shape[2] <= 256:
        return brute.forward(op, q, k, v, gamma=gamma, eps=eps)
    return oracle.recur(op, q, k, v, gamma=gamma, eps=eps)


# ---------------------------------------------------------------------------
# tensor-core layout self-check (one tcgen05 MMA), against fp64 on the host
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("case", [0, 1, 2, 3, 4, 5, 6, 7, 12, 13, 14, 15, 16, 17])
@pytest.mark.parametrize("N,K", [(64, 64), (128, 64), (64, 128), (128, 128), (192, 64), (256, 64), (256, 128)])
def test_umma_layouts(case, N, K):
    g = torch.Generator().manual_seed(case * 7 + N + K)
    M = 64 if case & 4 else 128
    A = torch.randn(M, K, generator=g).to(torch.bfloat16)
    B = torch.randn(K, N, generator=g).to(torch.bfloat16)
    a = A if not (case & 2) else A.t().contiguous()        # [M][K] or [K][M]
    b = B.t().contiguous() if not (case & 1) else B        # [N][K] or [K][N]
    ad, bd = a.cuda(), b.cuda()
    d = torch.full((M, N), float("nan"), device="cuda")
    import ctypes
    lib = hla.load_library()
    rc = lib.hla_selftest_umma(case, ctypes.c_void_p(ad.data_ptr()), ctypes.c_void_p(bd.data_ptr()),
                               ctypes.c_void_p(d.data_ptr()), N, K,
                               ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0
    torch.cuda.synchronize()
    ref = A.double() @ B.double()
    err = (d.cpu().double() - ref).abs().max().item()
    assert err <= 1e-4 * max(1.0, ref.abs().max().item()), err


# ---------------------------------------------------------------------------
# small shapes: every op x dtype x d, ragged tails, several chunks
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("op", OPS)
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("d", [32, 64])
@pytest.mark.parametrize("T", [1, 63, 64, 65, 200, 333])
def test_small_parity(op, dtype, d, T):
    w = recipe(op, dtype, 1, 2, T, d, seed=T)
    q, k, v, g = hla_inputs.make_inputs(w)
    o = gpu_forward(op, q, k, v, g)
    ref = reference(op, q, k, v, g)
    err = oracle.max_row_rel_err(o.cpu(), ref)
    assert err <= TOL[dtype], err


@pytest.mark.parametrize("op", OPS)
def test_many_heads_short_sequences(op):
    w = recipe(op, "bf16", 3, 5, 97, 64, seed=3)
    q, k, v, g = hla_inputs.make_inputs(w)
    o = gpu_forward(op, q, k, v, g)
    assert oracle.max_row_rel_err(o.cpu(), reference(op, q, k, v, g)) <= TOL["bf16"]


@pytest.mark.parametrize("op", ["hla2", "hla2n", "hla2d", "ahla"])
@pytest.mark.parametrize("T", [127, 128, 129, 1000, 1024, 2049])
def test_bf16_d64_parity_across_segments(op, T):
    """bf16 d = 64 (the tensor-core shapes) over many chunks and a ragged tail."""
    w = recipe(op, "bf16", 1, 3, T, 64, seed=T + 1)
    q, k, v, g = hla_inputs.make_inputs(w)
    o = gpu_forward(op, q, k, v, g)
    err = oracle.max_row_rel_err(o.cpu(), oracle.recur(op, q, k, v, gamma=g))
    assert err <= TOL["bf16"], err


@pytest.mark.parametrize("op", ["hla2", "hla2n", "hla2d", "ahla", "ahlan", "ahlad", "ahlan_g"])
@pytest.mark.parametrize("nch", [1, 2, 4, 8, 16])
@pytest.mark.parametrize("T", [129, 1000, 2049])
def test_segment_length_invariance(op, nch, T):
    """Tensor-core walk over 1..16 chunks per segment: same result (to rounding) as the oracle.
    (The decayed AHLA walk folds its prefix in the output walker; a plan with more summary slots
    than that fold takes runs on the CUDA cores, which the oracle checks the same way.)"""
    w = recipe(op, "bf16", 2, 2, T, 64, seed=nch + T)
    q, k, v, g = hla_inputs.make_inputs(w)
    hla.set_segment_chunks(nch)
    try:
        o = gpu_forward(w.op, q, k, v, g, eps=w.eps)
    finally:
        hla.set_segment_chunks(0)
    err = oracle.max_row_rel_err(o.cpu(), oracle.recur(w.op, q, k, v, gamma=g, eps=w.eps))
    assert err <= TOL["bf16"], err


@pytest.mark.parametrize("op", ["ahlad", "ahlan_g"])
@pytest.mark.parametrize("gam", [0.3, 0.9, 0.999, 1.0])
def test_decayed_ahla_tensor_cores_gamma_range(op, gam):
    """Decayed AHLA on the tensor-core walker from strong to no decay: many output segments per
    head (the decayed fold), a ragged tail, one gamma per head pair."""
    w = recipe(op, "bf16", 1, 2, 1500, 64, seed=int(gam * 100) + 5)
    q, k, v, _ = hla_inputs.make_inputs(w)
    g = torch.full((2,), gam)
    lib_uses = hla.uses_tensor_cores(hla.OP_AHLA_NORM if w.op == "ahlan" else hla.OP_AHLA, hla.HLA_BF16, True,
                                     1, 2, 1500, 64, 64)
    assert lib_uses
    o = gpu_forward(w.op, q, k, v, g, eps=w.eps)
    err = oracle.max_row_rel_err(o.cpu(), oracle.recur(w.op, q, k, v, gamma=g, eps=w.eps))
    assert err <= TOL["bf16"], err


@pytest.mark.parametrize("op", ["hla2n", "ahla"])
@pytest.mark.parametrize("nch,T", [(1, 4097), (1, 8193), (2, 8193)])
def test_many_segments_per_head(op, nch, T):
    """More than 32 segments per head (the scan leaves shared memory) and exactly 32 / 64."""
    w = recipe(op, "bf16", 1, 2, T, 64, seed=nch * 7 + T)
    q, k, v, g = hla_inputs.make_inputs(w)
    hla.set_segment_chunks(nch)
    try:
        o = gpu_forward(op, q, k, v, g)
    finally:
        hla.set_segment_chunks(0)
    err = oracle.max_row_rel_err(o.cpu(), oracle.recur(op, q, k, v, gamma=g))
    assert err <= TOL["bf16"], err


def test_tensor_core_path_is_used_for_bf16_d64():
    assert hla.uses_tensor_cores(hla.OP_HLA2_NORM, hla.HLA_BF16, False, 4, 16, 4096, 64, 64)
    assert hla.uses_tensor_cores(hla.OP_HLA2, hla.HLA_BF16, False, 1, 1, 100, 64, 64)
    assert not hla.uses_tensor_cores(hla.OP_HLA2, hla.HLA_F32, False, 1, 1, 100, 64, 64)
    assert hla.uses_tensor_cores(hla.OP_HLA2, hla.HLA_BF16, True, 2, 16, 16384, 64, 64)       # decayed
    assert not hla.uses_tensor_cores(hla.OP_HLA2_NORM, hla.HLA_BF16, True, 1, 1, 100, 64, 64)  # normalised + decay
    assert hla.uses_tensor_cores(hla.OP_AHLA, hla.HLA_BF16, False, 4, 16, 8192, 64, 64)
    assert not hla.uses_tensor_cores(hla.OP_AHLA, hla.HLA_BF16, False, 1, 1, 100, 32, 32)
    assert not hla.uses_tensor_cores(hla.OP_HLA3, hla.HLA_BF16, False, 1, 1, 100, 64, 64)


# ---------------------------------------------------------------------------
# properties
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("op", OPS)
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_deterministic_and_causal(op, dtype):
    w = recipe(op, dtype, 1, 2, 300, 64, seed=11)
    q, k, v, g = hla_inputs.make_inputs(w)
    a = gpu_forward(op, q, k, v, g)
    b = gpu_forward(op, q, k, v, g)
    assert torch.equal(a, b)                                  # run-to-run bitwise
    s = 150
    q2, k2, v2 = q.clone(), k.clone(), v.clone()
    q2[:, :, s:] = q2[:, :, s:] * 2
    k2[:, :, s:] = -k2[:, :, s:]
    v2[:, :, s:] = v2[:, :, s:] + 1
    c = gpu_forward(op, q2, k2, v2, g)
    assert torch.equal(a[:, :, :s], c[:, :, :s])              # rows before s untouched
    assert not torch.equal(a[:, :, s:], c[:, :, s:])


@pytest.mark.parametrize("op", OPS)
def test_no_write_outside_output(op):
    w = recipe(op, "bf16", 1, 2, 190, 64, seed=5)
    q, k, v, g = hla_inputs.make_inputs(w)
    dev = torch.device("cuda:0")
    n = q.shape[0] * q.shape[1] * q.shape[2] * 64
    guard = 4096
    buf = torch.full((n + 2 * guard,), float("nan"), device=dev)
    out = buf[guard:guard + n].view(1, 2, 190, 64)
    ws = hla.make_workspace(hla.OP_CODES[op], q.to(dev), v.to(dev), decayed=g is not None)
    hla.forward(op, q.to(dev), k.to(dev), v.to(dev), gamma=g.to(dev) if g is not None else None,
                out=out, workspace=ws)
    torch.cuda.synchronize()
    assert torch.isnan(buf[:guard]).all() and torch.isnan(buf[guard + n:]).all()
    assert torch.isfinite(out).all()
    assert hla.read_device_status(ws) == 0


@pytest.mark.parametrize("op", ["hla2", "hla3"])
@pytest.mark.parametrize("T", [1, 190, 4097])
def test_no_write_outside_output_fp32_tensor_cores(op, T):
    """The fp32, d = 32 tensor-core kernels store O rows with plain stores: NaN guard bands on
    both sides of the output stay untouched, and every output value is finite."""
    w = recipe(op, "f32", 1, 2, T, 32, seed=T)
    q, k, v, g = hla_inputs.make_inputs(w)
    dev = torch.device("cuda:0")
    n = 2 * T * 32
    guard = 4096
    buf = torch.full((n + 2 * guard,), float("nan"), device=dev)
    out = buf[guard:guard + n].view(1, 2, T, 32)
    ws = hla.make_workspace(hla.OP_CODES[op], q.to(dev), v.to(dev), decayed=False)
    hla.forward(op, q.to(dev), k.to(dev), v.to(dev), gamma=None, out=out, workspace=ws)
    torch.cuda.synchronize()
    assert torch.isnan(buf[:guard]).all() and torch.isnan(buf[guard + n:]).all()
    assert torch.isfinite(out).all()
    assert hla.read_device_status(ws) == 0


def test_normalized_constant_v_gives_den_ratio():
    w = recipe("hla2n", "bf16", 1, 2, 300, 64, seed=9)
    q, k, _, _ = hla_inputs.make_inputs(w)
    v = torch.full((1, 2, 300, 64), 2.5, dtype=torch.bfloat16)
    o = gpu_forward("hla2n", q, k, v, None).cpu().double()
    # den >> eps for positive q, k: the output is 2.5 up to rounding
    assert (o - 2.5).abs().max().item() < 2.5 * 2e-2


def test_decay_gamma_one_matches_undecayed():
    """gamma = 1 reduces the decayed op (CUDA cores, fp32 FFMA) to the undecayed one (at fp32 and
    d = 32 the tensor-core kernels with split products, about 2e-5 from the oracle): both match
    the oracle at the fp32 gate, and each other within two of it."""
    w = recipe("hla2", "f32", 1, 2, 200, 32, seed=4)
    q, k, v, _ = hla_inputs.make_inputs(w)
    a = gpu_forward("hla2d", q, k, v, torch.ones(2))
    b = gpu_forward("hla2", q, k, v, None)
    ref = oracle.recur("hla2", q, k, v)
    assert oracle.max_row_rel_err(a.cpu(), ref) <= TOL["f32"]
    assert oracle.max_row_rel_err(b.cpu(), ref) <= TOL["f32"]
    assert oracle.max_row_rel_err(a.cpu(), b.cpu()) <= 2 * TOL["f32"]


@pytest.mark.parametrize("T", [300, 2049])
def test_decay_gamma_one_matches_undecayed_tensor_cores(T):
    """bf16 d = 64: the decayed tensor-core path at gamma = 1 against the undecayed one (both
    differ from the oracle only by bf16 operand rounding)."""
    w = recipe("hla2", "bf16", 1, 2, T, 64, seed=T)
    q, k, v, _ = hla_inputs.make_inputs(w)
    a = gpu_forward("hla2d", q, k, v, torch.ones(2))
    b = gpu_forward("hla2", q, k, v, None)
    ref = oracle.recur("hla2", q, k, v)
    assert oracle.max_row_rel_err(a.cpu(), ref) <= TOL["bf16"]
    assert oracle.max_row_rel_err(a.cpu(), b.cpu()) <= TOL["bf16"]


@pytest.mark.parametrize("gam", [0.3, 0.5, 0.95, 0.999, 1.0])
@pytest.mark.parametrize("nch,T", [(1, 2049), (2, 4097), (4, 1500), (16, 5000)])
def test_decayed_walk_segment_plans(gam, nch, T):
    """The decayed second-order walk from strong to no decay over forced segment plans: up to
    32 summary slots folded by one output CTA, ragged tails, one gamma per head pair."""
    w = recipe("hla2d", "bf16", 1, 2, T, 64, seed=nch * 31 + int(gam * 100))
    q, k, v, _ = hla_inputs.make_inputs(w)
    g = torch.full((2,), gam)
    hla.set_segment_chunks(nch)
    try:
        o = gpu_forward("hla2d", q, k, v, g)
    finally:
        hla.set_segment_chunks(0)
    err = oracle.max_row_rel_err(o.cpu(), oracle.recur("hla2d", q, k, v, gamma=g))
    assert err <= TOL["bf16"], err


@pytest.mark.parametrize("T", [1, 63, 64, 65, 127, 128, 129, 255, 257, 1000, 4097])
def test_third_order_tensor_core_output(T):
    """The plain third order with fp32 inputs at d = 32: tensor-core summaries and output over
    128-token chunks, the factored prefix on the CUDA cores between them; ragged tails, fp32
    tolerance."""
    assert hla.uses_tensor_cores(hla.OP_HLA3, hla.HLA_F32, False, 1, 3, T, 32, 32) == 2
    w = recipe("hla3", "f32", 1, 3, T, 32, seed=T + 17)
    q, k, v, g = hla_inputs.make_inputs(w)
    o = gpu_forward("hla3", q, k, v, g)
    err = oracle.max_row_rel_err(o.cpu(), oracle.recur("hla3", q, k, v))
    assert err <= TOL["f32"], err


@pytest.mark.parametrize("T", [1, 100, 128, 129, 256, 1000, 4097, 8192, 8193])
def test_second_order_fp32_tensor_cores(T):
    """The plain second order with fp32 inputs at d = 32: tensor-core summaries and output with
    the prefix folded into every output CTA, up to 64 chunks per head; one chunk more takes the
    CUDA-core path.  fp32 tolerance either way."""
    on_tc = hla.uses_tensor_cores(hla.OP_HLA2, hla.HLA_F32, False, 1, 2, T, 32, 32)
    assert on_tc == (2 if T <= 8192 else 0)
    w = recipe("hla2", "f32", 1, 2, T, 32, seed=T + 29)
    q, k, v, g = hla_inputs.make_inputs(w)
    o = gpu_forward("hla2", q, k, v, g)
    err = oracle.max_row_rel_err(o.cpu(), oracle.recur("hla2", q, k, v))
    assert err <= TOL["f32"], err


def test_third_order_tensor_cores_many_items_per_cta():
    """21 heads x 33 chunks (the last one 1 token long) = 693 chunk x head items: every persistent
    CTA of the summary and output kernels walks four or five of them, so the next item's loads,
    the carried barrier phase and the reused TMEM and shared tiles all come into play, across
    head boundaries and ragged tails."""
    w = recipe("hla3", "f32", 3, 7, 4097, 32, seed=41)
    q, k, v, g = hla_inputs.make_inputs(w)
    o = gpu_forward("hla3", q, k, v, g)
    err = oracle.max_row_rel_err(o.cpu(), oracle.recur("hla3", q, k, v))
    assert err <= TOL["f32"], err


@pytest.mark.parametrize("op,dtype,d", [("hla2n", "bf16", 64), ("ahla", "bf16", 64), ("hla2d", "bf16", 64),
                                         ("hla3", "f32", 32)])
def test_long_single_head(op, dtype, d):
    """One head of 262,181 tokens (2,049 chunks of 128, the last one 37 tokens long): the
    longest plans, with hundreds of summary slots per head and the many-slot prefix paths,
    against the fp64 recurrence over the whole sequence."""
    w = recipe(op, dtype, 1, 1, 262144 + 37, d, seed=5)
    q, k, v, g = hla_inputs.make_inputs(w)
    o = gpu_forward(w.op, q, k, v, g, eps=w.eps)
    err = oracle.max_row_rel_err(o.cpu(), oracle.recur(w.op, q, k, v, gamma=g, eps=w.eps))
    assert err <= TOL[dtype], err


def test_third_order_tensor_core_output_large_values():
    """Inputs 8x larger than the workload's (a wider dynamic range for the bf16 splits)."""
    w = recipe("hla3", "f32", 1, 2, 2000, 32, seed=3)
    q, k, v, g = hla_inputs.make_inputs(w)
    q, k, v = q * 8, k * 8, v * 8
    o = gpu_forward("hla3", q, k, v, g)
    err = oracle.max_row_rel_err(o.cpu(), oracle.recur("hla3", q, k, v))
    assert err <= TOL["f32"], err


@pytest.mark.parametrize("gam", [0.5, 0.95, 0.999])
def test_decay_strong_and_weak_tensor_cores(gam):
    """bf16 d = 64 decayed path for one gamma per run, strong to weak decay, ragged tail."""
    w = recipe("hla2d", "bf16", 1, 2, 777, 64, seed=int(gam * 1000))
    q, k, v, _ = hla_inputs.make_inputs(w)
    g = torch.full((2,), gam)
    o = gpu_forward("hla2d", q, k, v, g)
    err = oracle.max_row_rel_err(o.cpu(), oracle.recur("hla2d", q, k, v, gamma=g))
    assert err <= TOL["bf16"], err


# ---------------------------------------------------------------------------
# the full-size workloads: whole GPU forward against the oracle on every head and token
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("name", list(hla_inputs.WORKLOADS))
def test_full_size_workloads(name):
    w = hla_inputs.workload(name)
    q, k, v, g = hla_inputs.make_inputs(w)
    o = gpu_forward(w.op, q, k, v, g, eps=w.eps).cpu()
    assert torch.isfinite(o).all()
    ref = oracle.recur(w.op, q, k, v, gamma=g, eps=w.eps)         # every head (host threads)
    BH = w.B * w.H
    per_head = [oracle.max_row_rel_err(o.reshape(BH, w.T, w.dv)[bh], ref.reshape(BH, w.T, w.dv)[bh])
                for bh in range(BH)]
    worst = max(range(BH), key=lambda bh: per_head[bh])
    assert per_head[worst] <= TOL[w.dtype], (name, worst, per_head[worst])


# ---------------------------------------------------------------------------
# the unmasked configuration (CUDA-core kernels): o_t = q_t^T S_t C_t
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("d", [32, 64])
@pytest.mark.parametrize("T", [1, 63, 64, 65, 200, 333, 1000])
def test_unmasked_parity(dtype, d, T):
    w = recipe("hla2u", dtype, 1, 2, T, d, seed=T + 5)
    q, k, v, _ = hla_inputs.make_inputs(w)
    o = gpu_forward("hla2u", q, k, v, None)
    assert oracle.max_row_rel_err(o.cpu(), reference("hla2u", q, k, v, None)) <= TOL[dtype]


def test_unmasked_many_heads():
    w = recipe("hla2u", "bf16", 3, 5, 97, 64, seed=4)
    q, k, v, _ = hla_inputs.make_inputs(w)
    o = gpu_forward("hla2u", q, k, v, None)
    assert oracle.max_row_rel_err(o.cpu(), reference("hla2u", q, k, v, None)) <= TOL["bf16"]


# ---------------------------------------------------------------------------
# ratio-normalised AHLA and third order (CUDA-core kernels)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("op", ["ahlan", "hla3n"])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("d", [32, 64])
@pytest.mark.parametrize("T", [1, 63, 65, 200, 1000])
def test_normalised_ahla_hla3_parity(op, dtype, d, T):
    w = hla_inputs.Workload(f"{op}_{dtype}_1x2x{T}x{d}", op, dtype, 1, 2, T, d, d, "softplus", "unit", seed=T + 9)
    q, k, v, _ = hla_inputs.make_inputs(w)
    o = gpu_forward(op, q, k, v, None, eps=w.eps)
    ref = reference(op, q, k, v, None, eps=w.eps)
    assert oracle.max_row_rel_err(o.cpu(), ref) <= TOL[dtype]


# ---------------------------------------------------------------------------
# decayed AHLA and third order, plain and ratio-normalised (CUDA-core kernels)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("op", ["ahlad", "hla3d", "ahlan", "hla3n"])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("d", [32, 64])
@pytest.mark.parametrize("T", [1, 63, 65, 200, 1000])
def test_decayed_ahla_hla3_parity(op, dtype, d, T):
    norm = op.endswith("n")
    w = hla_inputs.Workload(f"{op}_{dtype}_1x2x{T}x{d}", op, dtype, 1, 2, T, d, d,
                            "softplus" if norm else "scaled", "unit" if norm else "scaled", seed=T + 17,
                            gamma_range=(0.9, 0.999))
    q, k, v, g = hla_inputs.make_inputs(w)
    o = gpu_forward(op, q, k, v, g, eps=w.eps)
    ref = reference(op, q, k, v, g, eps=w.eps)
    assert oracle.max_row_rel_err(o.cpu(), ref) <= TOL[dtype]


@pytest.mark.parametrize("op", ["ahlad", "hla3d"])
@pytest.mark.parametrize("gam", [0.5, 0.95, 0.999])
def test_decayed_ahla_hla3_strong_and_weak(op, gam):
    """One gamma per run, from strong to weak decay, several chunks and a ragged tail."""
    d = 64 if op == "ahlad" else 32
    dtype = "bf16" if op == "ahlad" else "f32"
    w = hla_inputs.Workload(f"{op}_{gam}", op, dtype, 1, 2, 777, d, d, "scaled", "scaled", seed=int(gam * 1000))
    q, k, v, _ = hla_inputs.make_inputs(w)
    g = torch.full((2,), gam)
    o = gpu_forward(op, q, k, v, g)
    assert oracle.max_row_rel_err(o.cpu(), oracle.recur(op, q, k, v, gamma=g)) <= TOL[dtype]


@pytest.mark.parametrize("op", ["ahla", "hla3"])
def test_decayed_gamma_one_matches_undecayed(op):
    d, dtype = (64, "bf16") if op == "ahla" else (32, "f32")
    w = hla_inputs.Workload(f"{op}_g1", op, dtype, 1, 2, 300, d, d, "scaled", "scaled", seed=3)
    q, k, v, _ = hla_inputs.make_inputs(w)
    a = gpu_forward(op + "d", q, k, v, torch.ones(2))
    b = gpu_forward(op, q, k, v, None)
    assert oracle.max_row_rel_err(a.cpu(), b.cpu()) <= TOL[dtype]
