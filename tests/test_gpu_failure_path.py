"""The bounded-wait failure path on the GPU, made to run out on purpose.

Every mbarrier wait in the tensor-core kernels gives up after a wall-clock limit, records
HLA_ERR_TIMEOUT in the workspace status word, frees its tensor memory and returns.  This
test drives that path with hla_selftest_wait_timeout (a kernel waits on a barrier nothing
arrives on, with a 2 ms limit), reads the status back, and then checks that the context
still runs a forward correctly.  Nothing faults, traps or hangs.
"""
import ctypes

import pytest

import hla_inputs
import oracle

torch = pytest.importorskip("torch")
import higher_order_linear_chunked_b200 as hla  # noqa: E402

pytestmark = pytest.mark.gpu


def _status(lib, ws):
    out = ctypes.c_int(-1)
    rc = lib.hla_read_device_status(ctypes.c_void_p(ws.data_ptr()),
                                    ctypes.c_void_p(torch.cuda.current_stream().cuda_stream), ctypes.byref(out))
    assert rc == 0
    return out.value


def test_wait_runs_out_reports_timeout_and_context_survives():
    lib = hla.load_library()
    ws = torch.zeros(64, dtype=torch.int32, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = lib.hla_selftest_wait_timeout(ctypes.c_void_p(ws.data_ptr()), ws.numel() * 4, 2000, stream)
    assert rc == 0
    assert hla.STATUS_NAMES[_status(lib, ws)] == "HLA_ERR_TIMEOUT"
    # the same context still computes a forward, whose own status word stays clear
    w = hla_inputs.Workload("after_timeout", "hla2n", "bf16", 1, 2, 300, 64, 64, "softplus", "unit", seed=5)
    q, k, v, _ = hla_inputs.make_inputs(w)
    dev = torch.device("cuda:0")
    B, H, T, d = q.shape
    wsb = hla.workspace_bytes(hla.OP_HLA2_NORM, hla.HLA_BF16, False, B, H, T, d, d)
    fws = torch.empty(wsb, dtype=torch.uint8, device=dev)
    o = hla.hla2_normalized(q.to(dev), k.to(dev), v.to(dev), eps=1e-6, workspace=fws)
    torch.cuda.synchronize()
    assert _status(lib, fws) == 0
    assert oracle.max_row_rel_err(o.cpu(), oracle.recur("hla2n", q, k, v, eps=1e-6)) <= 2e-2
    # and a second timeout run reports again (the status word is cleared per call)
    rc = lib.hla_selftest_wait_timeout(ctypes.c_void_p(ws.data_ptr()), ws.numel() * 4, 1000, stream)
    assert rc == 0
    assert hla.STATUS_NAMES[_status(lib, ws)] == "HLA_ERR_TIMEOUT"
