"""The allocation-free entry point, hla2_forward_normalized_noalloc, through the C ABI.

Callers that may not allocate device memory while they run (a plugin inside
another framework that owns all device memory, a serving loop that allocates
only at start-up because cudaMalloc/cudaFree can stall the device) use this
entry point: its scratch is a fixed array built into the library.

The no-alloc call runs the same kernels as the regular entry point on the same
inputs, only with another scratch address, so the two outputs must be equal bit
for bit; the oracle checks one of them independently.  Each case calls the
entry point twice in a row, a longer sequence then a shorter one, so that a
slot left over from the first call in the shared array would show up in the
second.  The cases cover the tensor-core path (bf16, d = 64), the decayed form
(per-head gamma: CUDA-core kernels with their own workspace layout) and the
fp32 d = 32 CUDA-core path.  The device's free memory must not change across a
warmed-up call, the status word of the built-in array must read HLA_OK, and a
request larger than the array is refused.

The file name sorts last so that a run that stops at its first failure has
already run every other test.
"""
import ctypes

import numpy as np
import pytest

import hla_inputs
import oracle

torch = pytest.importorskip("torch")
import higher_order_linear_chunked_b200 as hla  # noqa: E402

pytestmark = pytest.mark.gpu

TOL = {"bf16": 2e-2, "f32": 1e-4}   # the parity tolerances of every other test
SCRATCH = 64 << 20

CASES = [
    # (name, dtype, d, decayed, (T of the first call, T of the second call), B, H)
    ("tensor_cores_bf16_d64", "bf16", 64, False, (4096, 1000), 4, 16),
    ("decayed_bf16_d64", "bf16", 64, True, (2048, 333), 2, 8),
    ("cuda_cores_f32_d32", "f32", 32, False, (1024, 65), 2, 4),
]


def _inputs(seed, dtype, B, H, T, d, decayed):
    w = hla_inputs.Workload(f"noalloc_{seed}", "hla2n", dtype, B, H, T, d, d, "softplus", "unit", seed=seed,
                            gamma_range=(0.95, 0.999) if decayed else None)
    q, k, v, g = hla_inputs.make_inputs(w)
    return q, k, v, g


def _noalloc(lib, q, k, v, g, out, eps=1e-6):
    B, H, T, d = q.shape
    vp = ctypes.c_void_p
    code = hla.HLA_BF16 if q.dtype == torch.bfloat16 else hla.HLA_F32
    return lib.hla2_forward_normalized_noalloc(
        vp(q.data_ptr()), vp(k.data_ptr()), vp(v.data_ptr()), vp(out.data_ptr()), B, H, T, d, v.shape[-1],
        code, vp(g.data_ptr() if g is not None else 0), ctypes.c_float(eps),
        vp(torch.cuda.current_stream().cuda_stream))


def _oracle(q, k, v, g):
    """fp64 ratio-normalised second order; decayed per head when g is given."""
    if g is None:
        return oracle.recur("hla2n", q, k, v, eps=1e-6)
    B, H = q.shape[:2]
    ref = np.zeros(tuple(v.shape), dtype=np.float64)
    for b in range(B):
        for h in range(H):
            ref[b, h] = oracle.hla2_run(q[b, h], k[b, h], v[b, h], gamma=float(g[h]), normalized=True,
                                        eps=1e-6)[0]
    return ref


def _noalloc_status(lib):
    s = ctypes.c_int(-1)
    rc = lib.hla_noalloc_read_device_status(ctypes.c_void_p(torch.cuda.current_stream().cuda_stream),
                                             ctypes.byref(s))
    assert rc == 0, hla.STATUS_NAMES.get(rc, rc)
    return s.value


@pytest.mark.parametrize("name,dtype,d,decayed,Ts,B,H", CASES, ids=[c[0] for c in CASES])
def test_noalloc_equals_workspace_entry_point(name, dtype, d, decayed, Ts, B, H):
    torch.cuda.init()
    lib = hla.load_library()
    dev = torch.device("cuda:0")
    for i, T in enumerate(Ts):                 # two calls in a row: a long sequence, then a short one
        q, k, v, g = _inputs(31 + i, dtype, B, H, T, d, decayed)
        qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
        gd = g.to(dev) if g is not None else None
        ref = hla.hla2_normalized(qd, kd, vd, eps=1e-6, gamma=gd)     # regular entry, caller workspace
        out = torch.full_like(ref, float("nan"))
        torch.cuda.synchronize()
        rc = _noalloc(lib, qd, kd, vd, gd, out)
        assert rc == 0, hla.STATUS_NAMES.get(rc, rc)
        torch.cuda.synchronize()
        assert _noalloc_status(lib) == 0
        assert torch.equal(out, ref), (name, T, (out - ref).abs().max().item())
        if i == 0:                             # one call checked against the fp64 oracle as well
            assert oracle.max_row_rel_err(out.cpu(), _oracle(q, k, v, g)) <= TOL[dtype], name


def test_noalloc_allocates_nothing():
    lib = hla.load_library()
    dev = torch.device("cuda:0")
    q, k, v, _ = _inputs(41, "bf16", 4, 16, 2048, 64, False)
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    out = torch.empty((4, 16, 2048, 64), dtype=torch.float32, device=dev)
    assert _noalloc(lib, qd, kd, vd, None, out) == 0     # warm: first-call set-up done
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info(dev)
    for _ in range(3):
        assert _noalloc(lib, qd, kd, vd, None, out) == 0
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info(dev)
    assert free1 == free0, (free0, free1)
    assert _noalloc_status(lib) == 0


def test_noalloc_refuses_requests_larger_than_its_array():
    lib = hla.load_library()
    dev = torch.device("cuda:0")
    q, k, v, _ = _inputs(43, "bf16", 4, 16, 128, 64, False)
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    out = torch.empty((4, 16, 128, 64), dtype=torch.float32, device=dev)
    # a sequence length whose workspace exceeds the built-in array: refused before any launch
    big_T = 1 << 17
    need = hla.workspace_bytes(hla.OP_HLA2_NORM, hla.HLA_BF16, False, 4, 16, big_T, 64, 64)
    assert need > SCRATCH
    vp = ctypes.c_void_p
    rc = lib.hla2_forward_normalized_noalloc(vp(qd.data_ptr()), vp(kd.data_ptr()), vp(vd.data_ptr()),
                                              vp(out.data_ptr()), 4, 16, big_T, 64, 64, hla.HLA_BF16, vp(0),
                                              ctypes.c_float(1e-6), vp(0))
    assert hla.STATUS_NAMES[rc] == "HLA_ERR_WORKSPACE"
