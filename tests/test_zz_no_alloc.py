"""The allocation-free entry point, hla2_forward_normalized_noalloc, through the C ABI.

Callers that may not allocate device memory while they run (a plugin inside
another framework that owns all device memory, a serving loop that allocates
only at start-up because cudaMalloc/cudaFree can stall the device) use this
entry point: its scratch is a fixed array built into the library.  This test
checks that it gives the same output as the regular entry point, which takes a
caller-allocated workspace, on two calls in a row, and that a request larger
than the built-in array is refused.

The file name sorts last so that a run that stops at its first failure has
already run every other test.
"""
import ctypes

import pytest

import hla_inputs
import oracle

torch = pytest.importorskip("torch")
import higher_order_linear_chunked_b200 as hla  # noqa: E402

pytestmark = pytest.mark.gpu

TOL = 2e-2   # bf16-input tolerance used by every parity test
SCRATCH = 64 << 20


def _inputs(seed, T=4096, op="hla2n"):
    w = hla_inputs.Workload(f"noalloc_{seed}", op, "bf16", 4, 16, T, 64, 64, "softplus", "unit", seed=seed)
    q, k, v, _ = hla_inputs.make_inputs(w)
    dev = torch.device("cuda:0")
    return q.to(dev), k.to(dev), v.to(dev)


def _noalloc(lib, q, k, v, out, eps=1e-6):
    B, H, T, d = q.shape
    vp = ctypes.c_void_p
    return lib.hla2_forward_normalized_noalloc(
        vp(q.data_ptr()), vp(k.data_ptr()), vp(v.data_ptr()), vp(out.data_ptr()), B, H, T, d, v.shape[-1],
        hla.HLA_BF16, vp(0), ctypes.c_float(eps), vp(torch.cuda.current_stream().cuda_stream))


def test_noalloc_matches_workspace_entry_point_twice():
    torch.cuda.init()
    lib = hla.load_library()
    for seed in (21, 22):                      # two calls in a row, different inputs
        q, k, v = _inputs(seed)
        ref = hla.hla2_normalized(q, k, v, eps=1e-6)        # regular entry, caller workspace
        out = torch.full_like(ref, float("nan"))
        rc = _noalloc(lib, q, k, v, out)
        assert rc == 0, hla.STATUS_NAMES.get(rc, rc)
        torch.cuda.synchronize()
        assert torch.isfinite(out).all()
        assert oracle.max_row_rel_err(out.cpu(), ref.cpu()) <= TOL


def test_noalloc_refuses_requests_larger_than_its_array():
    lib = hla.load_library()
    q, k, v = _inputs(23, T=128)
    out = torch.empty((4, 16, 128, 64), dtype=torch.float32, device=q.device)
    # a sequence length whose workspace exceeds the built-in array: refused before any launch
    big_T = 1 << 17
    need = hla.workspace_bytes(hla.OP_HLA2_NORM, hla.HLA_BF16, False, 4, 16, big_T, 64, 64)
    assert need > SCRATCH
    vp = ctypes.c_void_p
    rc = lib.hla2_forward_normalized_noalloc(vp(q.data_ptr()), vp(k.data_ptr()), vp(v.data_ptr()),
                                              vp(out.data_ptr()), 4, 16, big_T, 64, 64, hla.HLA_BF16, vp(0),
                                              ctypes.c_float(1e-6), vp(0))
    assert hla.STATUS_NAMES[rc] == "HLA_ERR_WORKSPACE"
