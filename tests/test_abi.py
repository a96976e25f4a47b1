"""Host-side checks of the C ABI (no GPU needed, no compute calls).

The library must load on a machine without a GPU, export every function
include/hla.h declares, size workspaces, and reject bad arguments with the
documented status codes before touching the device.
"""
import ctypes
import os
import re

import pytest

import higher_order_linear_chunked_b200 as hla

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "hla.h")


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(hla.LIB_PATH):
        from higher_order_linear_chunked_b200 import build
        build.build()
    return hla.load_library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b((?:a?hla)\w*)\s*\(", text)))


def test_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert set(names) == set(hla.EXPORTS), names
    for name in names:
        assert hasattr(lib, name), name


def test_abi_version_and_status_strings(lib):
    assert lib.hla_abi_version() == 2
    for code in range(9):
        s = lib.hla_status_str(code).decode()
        assert s.startswith(hla.STATUS_NAMES[code])
    assert lib.hla_status_str(99).decode() == "unknown hla_status_t"


def test_workspace_sizes(lib):
    ws = lambda *a: lib.hla_workspace_bytes(*a)
    # supported requests have a positive size, growing with the sequence
    for op in range(4):
        for dtype in (hla.HLA_F32, hla.HLA_BF16):
            for d in (32, 64):
                a = ws(op, dtype, 0, 1, 2, 256, d, d)
                b = ws(op, dtype, 0, 1, 2, 4096, d, d)
                assert 0 < a <= b
    assert ws(hla.OP_HLA2, hla.HLA_BF16, 1, 2, 16, 16384, 64, 64) > 0       # decayed
    # invalid or unsupported requests size to 0
    assert ws(hla.OP_HLA2, hla.HLA_F32, 0, 1, 1, 10, 48, 48) == 0          # d not in {32, 64}
    assert ws(hla.OP_HLA2, hla.HLA_F32, 0, 1, 1, 10, 64, 32) == 0          # d != dv
    assert ws(hla.OP_HLA2, hla.HLA_F32, 0, 0, 1, 10, 64, 64) == 0          # B = 0
    assert ws(hla.OP_HLA2, 7, 0, 1, 1, 10, 64, 64) == 0                    # bad dtype
    assert ws(hla.OP_AHLA, hla.HLA_F32, 1, 1, 1, 10, 64, 64) > 0           # decayed AHLA
    assert ws(hla.OP_HLA3, hla.HLA_F32, 1, 1, 1, 10, 32, 32) > 0           # decayed third order
    assert ws(hla.OP_HLA2_UNMASKED, hla.HLA_F32, 1, 1, 1, 10, 64, 64) == 0  # no decayed unmasked op
    assert ws(9, hla.HLA_F32, 0, 1, 1, 10, 64, 64) == 0                    # bad op


def test_tensor_core_routing_launches_and_workspace(lib):
    """Host-side routing: which requests take the tcgen05 kernels, how many launches a
    forward enqueues, and the workspace each path sizes (no GPU needed)."""
    use = lambda op, dt, dec, T=4096, d=64: lib.hla_uses_tensor_cores(op, dt, dec, 4, 16, T, d, d)
    launches = lambda op, dt, dec, T=4096, d=64: lib.hla_kernel_launches(op, dt, dec, 4, 16, T, d, d)
    bf16, f32 = hla.HLA_BF16, hla.HLA_F32
    # bf16, d = 64: second order (plain, normalised, decayed) and AHLA (plain, normalised) run on
    # the tensor cores
    for op, dec in ((hla.OP_HLA2, 0), (hla.OP_HLA2_NORM, 0), (hla.OP_HLA2, 1), (hla.OP_AHLA, 0),
                    (hla.OP_AHLA_NORM, 0), (hla.OP_AHLA, 1), (hla.OP_AHLA_NORM, 1)):
        assert use(op, bf16, dec) == 1, (op, dec)
    # the rest on CUDA cores: fp32 inputs, d = 32, third order, normalised with decay
    assert use(hla.OP_HLA2, f32, 0) == 0
    assert use(hla.OP_HLA2, bf16, 0, d=32) == 0
    assert use(hla.OP_HLA3, bf16, 0) == 0
    # the plain third order with fp32 inputs at d = 32: the output kernel on the tensor cores (2),
    # not the normalised or decayed forms, nor d = 64 or bf16 inputs
    assert use(hla.OP_HLA3, f32, 0, d=32) == 2
    assert use(hla.OP_HLA3, f32, 1, d=32) == 0 and use(hla.OP_HLA3_NORM, f32, 0, d=32) == 0
    assert use(hla.OP_HLA3, f32, 0) == 0 and use(hla.OP_HLA3, bf16, 0, d=32) == 0
    # the plain second order with fp32 inputs at d = 32: summaries and output on the tensor cores
    # while the output CTAs can fold the summaries (up to 64 chunks of 128 tokens per head)
    assert use(hla.OP_HLA2, f32, 0, d=32) == 2 and launches(hla.OP_HLA2, f32, 0, d=32) == 2
    assert use(hla.OP_HLA2, f32, 0, T=8192, d=32) == 2 and use(hla.OP_HLA2, f32, 0, T=8193, d=32) == 0
    assert launches(hla.OP_HLA2, f32, 0, T=8193, d=32) == 3
    assert use(hla.OP_HLA2_NORM, f32, 0, d=32) == 0 and use(hla.OP_HLA2, f32, 1, d=32) == 0
    assert use(hla.OP_HLA2_NORM, bf16, 1) == 0
    # launches per forward: summary walker, the prefix (with up to nine summary slots per head
    # folded into the output walker; else three kernels), output walker; the decayed second
    # order folds its prefix in the output walker at every plan
    assert launches(hla.OP_HLA2_NORM, bf16, 0) == 2   # the output walker folds the prefix
    assert launches(hla.OP_AHLA, bf16, 0) == 2
    assert launches(hla.OP_AHLA_NORM, bf16, 0) == 2
    assert launches(hla.OP_AHLA, bf16, 1) == 2                                          # decayed AHLA
    # the decayed AHLA walk folds its prefix in the output walker: a plan with more summary slots
    # than that (one long head) runs on the CUDA cores
    assert lib.hla_uses_tensor_cores(hla.OP_AHLA, bf16, 1, 1, 1, 65536, 64, 64) == 0
    assert lib.hla_uses_tensor_cores(hla.OP_AHLA, bf16, 0, 1, 1, 65536, 64, 64) == 1
    # the normalised AHLA walker runs one CTA per SM (512 TMEM columns): its segment plan, and
    # so its workspace, differs from the plain walker's (two per SM) at the same shape
    ws_tc = lambda op, B, H, T: lib.hla_workspace_bytes(op, bf16, 0, B, H, T, 64, 64)
    assert ws_tc(hla.OP_AHLA_NORM, 4, 16, 8192) > 0 and ws_tc(hla.OP_AHLA, 4, 16, 8192) > 0
    assert lib.hla_kernel_launches(hla.OP_AHLA_NORM, bf16, 0, 1, 1, 65536, 64, 64) == 5   # many slots
    assert lib.hla_kernel_launches(hla.OP_HLA2_NORM, bf16, 0, 1, 1, 65536, 64, 64) == 5   # many slots
    assert launches(hla.OP_HLA2, bf16, 1) == 2
    assert lib.hla_kernel_launches(hla.OP_HLA2, bf16, 1, 1, 2, 200, 64, 64) == 1   # one segment per head
    # CUDA-core path: chunk kernel, one scan launch (a per-head fold) and the output kernel;
    # the third order, decayed or not, takes the factored prefix (three launches)
    assert launches(hla.OP_HLA2, f32, 0) == 3
    assert launches(hla.OP_AHLA_NORM, f32, 0) == 3
    assert launches(hla.OP_HLA2_UNMASKED, bf16, 0) == 3
    assert launches(hla.OP_HLA3, f32, 0, d=32) == 2 + 3      # the factored third-order prefix
    assert launches(hla.OP_HLA3, f32, 0) == 2 + 3
    assert launches(hla.OP_HLA3, f32, 1, d=32) == 2 + 3      # decayed: the same three prefix launches
    # decayed workspace: 256 B status block + segment summaries only, each slot S, C, G, Khat
    # (4 x 64 x 64 fp32) and rho, a whole number of slots per head and fewer than one per four
    # 128-token chunks at this shape
    T, slot = 16384, (4 * 64 * 64 + 32) * 4
    for t in (T, T + 1):
        body = lib.hla_workspace_bytes(hla.OP_HLA2, bf16, 1, 2, 16, t, 64, 64) - 256
        assert body > 0 and body % (32 * slot) == 0 and body // (32 * slot) <= T // 128 // 4


def _call(lib, name, q=16, k=16, v=16, o=16, B=1, H=1, T=8, d=32, dv=32, dtype=0, gamma=0, ws=16,
          wsb=1 << 30, eps=None):
    vp = ctypes.c_void_p
    args = [vp(q), vp(k), vp(v), vp(o), B, H, T, d, dv, dtype, vp(gamma)]
    tail = [vp(ws), ctypes.c_size_t(wsb), vp(0)]
    fn = getattr(lib, name)
    if name == "hla2_forward_normalized":
        return fn(*args, ctypes.c_float(1e-6 if eps is None else eps), *tail)
    return fn(*args, *tail)


@pytest.mark.parametrize("name", ["hla2_forward", "hla2_forward_normalized", "ahla_forward", "hla3_forward"])
def test_argument_errors_are_reported_before_any_launch(lib, name):
    assert _call(lib, name, q=0) == 1                      # HLA_ERR_NULL
    assert _call(lib, name, o=0) == 1
    assert _call(lib, name, B=0) == 2                      # HLA_ERR_SHAPE
    assert _call(lib, name, T=0) == 2
    assert _call(lib, name, B=1 << 16, H=1 << 10, T=1 << 10) == 2
    assert _call(lib, name, B=256, H=256, T=1) == 2        # B*H above 65535 heads
    assert _call(lib, name, B=3, H=21845, T=1, ws=0) == 6  # 65535 heads: the shape passes
    assert _call(lib, name, dtype=5) == 4                  # HLA_ERR_DTYPE
    assert _call(lib, name, d=32, dv=64) == 5              # HLA_ERR_UNSUPPORTED
    assert _call(lib, name, d=48, dv=48) == 5
    assert _call(lib, name, q=24) == 3                     # HLA_ERR_ALIGN
    assert _call(lib, name, ws=0) == 6                     # HLA_ERR_WORKSPACE
    assert _call(lib, name, wsb=64) == 6
    assert _call(lib, name, ws=32 + 8) == 3
    assert _call(lib, name, gamma=66) == 3                 # misaligned gamma


def test_segment_chunks_knob(lib):
    base = lib.hla_workspace_bytes(hla.OP_HLA2, hla.HLA_BF16, 0, 1, 2, 4096, 64, 64)
    for n in (1, 2, 4, 8, 16):
        assert lib.hla_set_segment_chunks(n) == 0
        assert lib.hla_workspace_bytes(hla.OP_HLA2, hla.HLA_BF16, 0, 1, 2, 4096, 64, 64) > 0
    for bad in (-1, 3, 5, 32):
        assert lib.hla_set_segment_chunks(bad) == 2
    assert lib.hla_set_segment_chunks(0) == 0
    assert lib.hla_workspace_bytes(hla.OP_HLA2, hla.HLA_BF16, 0, 1, 2, 4096, 64, 64) == base


def test_selftest_argument_errors(lib):
    vp = ctypes.c_void_p
    assert lib.hla_selftest_umma(0, vp(0), vp(16), vp(16), 64, 64, vp(0)) == 1
    assert lib.hla_selftest_umma(32, vp(16), vp(16), vp(16), 64, 64, vp(0)) == 5
    assert lib.hla_selftest_umma(18, vp(16), vp(16), vp(16), 64, 64, vp(0)) == 5   # TMEM A, MN-major
    assert lib.hla_selftest_umma(20, vp(16), vp(16), vp(16), 64, 64, vp(0)) == 5   # TMEM A, M = 64
    assert lib.hla_selftest_umma(8, vp(16), vp(16), vp(16), 64, 64, vp(0)) == 5
    assert lib.hla_selftest_umma(0, vp(16), vp(16), vp(16), 96, 64, vp(0)) == 2
    assert lib.hla_selftest_umma(0, vp(16), vp(16), vp(16), 320, 64, vp(0)) == 2
    assert lib.hla_read_device_status(vp(0), vp(0), None) == 1
    wt = lib.hla_selftest_wait_timeout
    assert wt(vp(0), 256, 1000, vp(0)) == 1                     # NULL workspace
    assert wt(vp(8), 256, 1000, vp(0)) == 3                     # not 16-byte aligned
    assert wt(vp(16), 64, 1000, vp(0)) == 6                     # smaller than the status block
    assert wt(vp(16), 256, 0, vp(0)) == 2                       # timeout out of range
    assert wt(vp(16), 256, 2000000, vp(0)) == 2


def test_streaming_state_sizes_and_argument_errors(lib):
    """State sizes follow the summary layout; bad calls are refused before any launch."""
    vp, f = ctypes.c_void_p, ctypes.c_float
    d = 64
    pad = lambda n: (n + 31) // 32 * 32                       # noqa: E731
    assert lib.hla_state_floats(0, 0, d, d) == pad(3 * d * d + 2 * d + 4)     # S, C, R ; m, r
    assert lib.hla_state_floats(1, 1, d, d) == pad(4 * d * d + 2 * d + 4)     # decayed: + Khat, rho
    assert lib.hla_state_floats(2, 0, d, d) == pad(3 * d * d + 2 * d + 4)     # P, E, D ; mK, n
    assert lib.hla_state_floats(3, 0, 32, 32) == pad(6 * 32 * 32 + 3 * 32 + 4)   # S Q2 P F X Z ; mK X1 F1
    assert lib.hla_state_floats(5, 0, d, d) == lib.hla_state_floats(2, 0, d, d)   # normalised: same state
    assert lib.hla_state_floats(6, 0, 32, 32) == lib.hla_state_floats(3, 0, 32, 32)
    assert lib.hla_state_floats(2, 1, d, d) == lib.hla_state_floats(2, 0, d, d)   # decayed AHLA: + rho
    assert lib.hla_state_floats(3, 1, 32, 32) == lib.hla_state_floats(3, 0, 32, 32)
    assert lib.hla_state_floats(4, 1, d, d) == 0                              # no decayed unmasked op
    assert lib.hla_state_floats(0, 0, 48, 48) == 0
    assert lib.hla_state_floats(0, 0, 64, 32) == 0
    # workspace: status block + the CUDA-core chunk summaries (64-token chunks, padded to 2^k)
    n = lib.hla_state_workspace_bytes(0, 0, 0, 4, 16, 4096, d, d)
    assert n == 256 + 4 * 64 * 64 * lib.hla_state_floats(0, 0, d, d)
    assert lib.hla_state_workspace_bytes(2, 1, 1, 4, 16, 4096, d, d) > 0       # decayed AHLA (CUDA cores)
    assert lib.hla_state_workspace_bytes(4, 1, 1, 4, 16, 4096, d, d) == 0
    assert lib.hla_state_kernel_launches(0, 0, 0, 4, 16, 4096, d, d) == 2 + 6     # 64 chunks: 6 levels
    # bf16, d = 64, undecayed second order: the tensor-core summary walker over 16-chunk segments
    # (two per head at T = 4096), then one combine per head
    n = lib.hla_state_workspace_bytes(0, 1, 0, 4, 16, 4096, d, d)
    assert n == 256 + 64 * 2 * 4 * lib.hla_state_floats(0, 0, d, d)
    assert lib.hla_state_kernel_launches(0, 1, 0, 4, 16, 4096, d, d) == 2
    assert lib.hla_state_kernel_launches(1, 1, 0, 4, 16, 4096, d, d) == 2
    assert lib.hla_state_kernel_launches(0, 1, 1, 4, 16, 4096, d, d) == 2 + 6     # decayed: CUDA cores
    assert lib.hla_state_kernel_launches(0, 0, 0, 1, 1, 64, 32, 32) == 2
    st = lib.hla_state
    a = [vp(16), vp(16), vp(16), vp(16)]
    assert st(0, vp(0), *a[1:], 1, 1, 64, d, d, 0, vp(0), vp(16), 1 << 20, vp(0)) == 1      # NULL q
    assert st(7, *a, 1, 1, 64, d, d, 0, vp(0), vp(16), 1 << 20, vp(0)) == 5                # bad op
    assert st(0, *a, 0, 1, 64, d, d, 0, vp(0), vp(16), 1 << 20, vp(0)) == 2                # B = 0
    assert st(0, *a, 1, 1, 64, d, d, 7, vp(0), vp(16), 1 << 20, vp(0)) == 4                # dtype
    assert st(4, *a, 1, 1, 64, d, d, 0, vp(16), vp(16), 1 << 20, vp(0)) == 5               # gamma + unmasked
    assert st(0, vp(8), *a[1:], 1, 1, 64, d, d, 0, vp(0), vp(16), 1 << 20, vp(0)) == 3     # alignment
    assert st(0, *a, 1, 1, 64, d, d, 0, vp(0), vp(0), 1 << 20, vp(0)) == 6                 # no workspace
    assert st(0, *a, 1, 1, 64, d, d, 0, vp(0), vp(16), 64, vp(0)) == 6                     # too small
    sp = lib.hla_step
    b = [vp(16)] * 5
    assert sp(0, vp(0), *b[1:], 1, 1, d, d, 0, vp(0), f(1e-6), vp(0)) == 1                 # NULL state
    assert sp(0, *b, 1, 1, 48, 48, 0, vp(0), f(1e-6), vp(0)) == 5                          # d = 48
    assert sp(0, *b, 1, 0, d, d, 0, vp(0), f(1e-6), vp(0)) == 2                            # H = 0
    assert sp(4, *b, 1, 1, 32, 32, 0, vp(16), f(1e-6), vp(0)) == 5                         # gamma + unmasked
    assert sp(0, vp(24), *b[1:], 1, 1, d, d, 0, vp(0), f(1e-6), vp(0)) == 3                # alignment


def test_normalised_ahla_hla3_routing_and_errors(lib):
    """Ratio-normalised AHLA / third order: the tensor-core walker for bf16 AHLA at d = 64 (a
    ones column beside V), CUDA-core kernels otherwise (the third order, fp32, d = 32, decay)
    with the plain op's workspace."""
    vp, f = ctypes.c_void_p, ctypes.c_float
    assert lib.hla_uses_tensor_cores(hla.OP_AHLA_NORM, hla.HLA_BF16, 0, 4, 16, 4096, 64, 64) == 1
    assert lib.hla_uses_tensor_cores(hla.OP_HLA3_NORM, hla.HLA_BF16, 0, 4, 16, 4096, 64, 64) == 0
    assert lib.hla_uses_tensor_cores(hla.OP_AHLA_NORM, hla.HLA_BF16, 1, 4, 16, 4096, 64, 64) == 1   # + decay
    assert lib.hla_uses_tensor_cores(hla.OP_HLA3_NORM, hla.HLA_BF16, 1, 4, 16, 4096, 64, 64) == 0
    for op, plain in ((hla.OP_AHLA_NORM, hla.OP_AHLA), (hla.OP_HLA3_NORM, hla.OP_HLA3)):
        assert lib.hla_workspace_bytes(op, hla.HLA_BF16, 1, 4, 16, 4096, 64, 64) > 0            # decayed form
        assert lib.hla_workspace_bytes(op, hla.HLA_F32, 0, 2, 8, 4096, 32, 32) == \
            lib.hla_workspace_bytes(plain, hla.HLA_F32, 0, 2, 8, 4096, 32, 32)
    assert lib.hla_uses_tensor_cores(hla.OP_AHLA, hla.HLA_BF16, 0, 4, 16, 4096, 64, 64) == 1
    a = [vp(16)] * 4
    for fn in (lib.ahla_forward_normalized, lib.hla3_forward_normalized):
        assert fn(*a, 1, 1, 64, 64, 64, 0, vp(16), f(1e-6), vp(16), 64, vp(0)) == 6          # gamma: decayed,
        assert fn(*a, 1, 1, 64, 64, 64, 0, vp(18), f(1e-6), vp(16), 1 << 20, vp(0)) == 3     # sized, aligned
        assert fn(vp(0), *a[1:], 1, 1, 64, 64, 64, 0, vp(0), f(1e-6), vp(16), 1 << 20, vp(0)) == 1
        assert fn(*a, 1, 1, 64, 64, 64, 0, vp(0), f(1e-6), vp(16), 64, vp(0)) == 6           # workspace


def test_unmasked_op_sizes_and_errors(lib):
    """The unmasked second-order op: CUDA-core kernels only, no decayed form, state (S, C)."""
    vp = ctypes.c_void_p
    op = hla.OP_HLA2_UNMASKED
    assert lib.hla_workspace_bytes(op, hla.HLA_BF16, 0, 4, 16, 4096, 64, 64) > 0
    assert lib.hla_workspace_bytes(op, hla.HLA_BF16, 1, 4, 16, 4096, 64, 64) == 0          # no decay
    assert lib.hla_uses_tensor_cores(op, hla.HLA_BF16, 0, 4, 16, 4096, 64, 64) == 0
    assert lib.hla_state_floats(op, 0, 64, 64) == (2 * 64 * 64 + 4 + 31) // 32 * 32
    f = lib.hla2_forward_unmasked
    a = [vp(16)] * 4
    assert f(*a, 1, 1, 64, 64, 64, 0, vp(16), vp(16), 1 << 20, vp(0)) == 5                  # gamma given
    assert f(vp(0), *a[1:], 1, 1, 64, 64, 64, 0, vp(0), vp(16), 1 << 20, vp(0)) == 1        # NULL q
    assert f(*a, 1, 1, 64, 48, 48, 0, vp(0), vp(16), 1 << 20, vp(0)) == 5                  # d = 48
    assert f(*a, 1, 1, 64, 64, 64, 0, vp(0), vp(16), 64, vp(0)) == 6                       # workspace


def test_header_is_plain_c(tmp_path):
    """include/hla.h is a C ABI: it compiles as strict C99 (and as C++) with no CUDA header."""
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("no gcc")
    src = tmp_path / "use_hla.c"
    src.write_text('#include "hla.h"\nint main(void) { return hla_abi_version() > 0 ? 0 : 1; }\n')
    inc = os.path.join(ROOT, "include")
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-fsyntax-only", "-I", inc,
                    str(src)], check=True)
    subprocess.run(["g++", "-std=c++17", "-Wall", "-Wextra", "-Werror", "-fsyntax-only", "-x", "c++", "-I", inc,
                    str(src)], check=True)


def test_product_path_never_touches_the_oracle():
    """The package (binding + CUDA sources) must not import, call or link oracle/."""
    pkg = os.path.join(ROOT, "higher_order_linear_chunked_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                text = open(os.path.join(dirpath, f), encoding="utf-8").read()
                assert not re.search(r"\boracle\b", text), os.path.join(dirpath, f)


def test_python_binding_rejects_cpu_tensors():
    torch = pytest.importorskip("torch")
    q = torch.zeros(1, 1, 4, 32)
    with pytest.raises(ValueError, match="CUDA tensor"):
        hla.hla2(q, q, q)
