"""Host-side checks of the C ABI (no GPU needed).

The library must load on a machine without a GPU, export every entry point
``include/fa2.h`` declares, and reject bad arguments with the documented status
codes before touching the device.
"""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fa2.h")


@pytest.fixture(scope="module")
def lib():
    from exact_tiled_attention_30_b200 import build

    build.build()
    import exact_tiled_attention_30_b200 as m

    return m.load_library()


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"FA2_API[^;(]*?\b(fa2_\w+)\s*\(", text)))


def test_header_declares_the_abi():
    assert {"fa2_forward", "fa2_backward", "fa2_backward_workspace_size", "fa2_status_string",
            "fa2_get_device_status", "fa2_clear_device_status", "fa2_backward_preprocess",
            "fa2_backward_main", "fa2_backward_dq_convert"} <= set(declared_symbols())


def test_library_exports_every_declared_symbol(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name


def test_library_exports_nothing_else(lib):
    out = os.popen(f"nm -D --defined-only {lib._name}").read()
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    ours = {s for s in exported if s.startswith("fa2")}
    assert ours == set(declared_symbols())


def test_status_strings(lib):
    import exact_tiled_attention_30_b200 as m

    for code, name in m.STATUS.items():
        assert m.fa2_status_string(code) == name
    assert m.fa2_status_string(99) == "FA2_ERR_UNKNOWN"


A = 0x10000  # aligned fake device address (never dereferenced: checks fail first)


def fwd(lib, q=A, k=A, v=A, o=A, lse=A, B=1, H=1, N=128, d=64, causal=0, scale=0.125):
    return lib.fa2_forward(q, k, v, o, lse, B, H, N, d, causal, ctypes.c_float(scale), None)


def test_forward_rejects_bad_arguments(lib):
    assert fwd(lib, q=None) == 1
    assert fwd(lib, lse=None) == 1
    assert fwd(lib, N=0) == 1
    assert fwd(lib, B=0) == 1
    assert fwd(lib, H=-1) == 1
    assert fwd(lib, scale=float("nan")) == 1
    assert fwd(lib, scale=float("inf")) == 1
    assert fwd(lib, scale=-0.5) == 1
    assert fwd(lib, d=96) == 2
    assert fwd(lib, d=256) == 2
    assert fwd(lib, B=256, H=256) == 2
    assert fwd(lib, q=A + 8) == 3
    assert fwd(lib, o=A + 2) == 3
    assert fwd(lib, lse=A + 4) == 3


def test_workspace_size(lib):
    import exact_tiled_attention_30_b200 as m

    assert m.fa2_backward_workspace_size(1, 1, 128, 64) == 128 * 64 * 4 + 2 * 128 * 4 + 16
    assert m.fa2_backward_workspace_size(2, 3, 129, 128) == 6 * 256 * 128 * 4 + 2 * 6 * 256 * 4 + 16
    assert m.fa2_backward_workspace_size(1, 1, 0, 64) == 0
    assert m.fa2_backward_workspace_size(1, 1, 10, 32) == 0


def bwd(lib, ptrs=None, B=1, H=1, N=128, d=64, scale=0.125, ws_bytes=None):
    p = [A] * 10 if ptrs is None else ptrs
    if ws_bytes is None:
        ws_bytes = lib.fa2_backward_workspace_size(B, H, N, d)
    return lib.fa2_backward(*p[:9], B, H, N, d, 0, ctypes.c_float(scale), p[9], ws_bytes, None)


def test_backward_rejects_bad_arguments(lib):
    for i in range(10):
        p = [A] * 10
        p[i] = None
        assert bwd(lib, p) == 1, i
    assert bwd(lib, ws_bytes=100) == 1
    assert bwd(lib, N=0) == 1
    assert bwd(lib, d=32) == 2
    assert bwd(lib, scale=float("nan")) == 1
    for i in range(10):
        p = [A] * 10
        p[i] = A + 4
        assert bwd(lib, p) == 3, i


def test_backward_stages_reject_bad_arguments(lib):
    ws = lib.fa2_backward_workspace_size(1, 1, 128, 64)
    f = ctypes.c_float
    assert lib.fa2_backward_preprocess(None, A, A, 1, 1, 128, 64, A, ws, None) == 1
    assert lib.fa2_backward_preprocess(A, A, A, 1, 1, 128, 64, None, ws, None) == 1
    assert lib.fa2_backward_preprocess(A, A, A, 1, 1, 128, 64, A, ws - 1, None) == 1
    assert lib.fa2_backward_preprocess(A, A, A, 1, 1, 128, 48, A, ws, None) == 2
    assert lib.fa2_backward_preprocess(A, A + 4, A, 1, 1, 128, 64, A, ws, None) == 3
    assert lib.fa2_backward_main(A, A, A, A, A, None, 1, 1, 128, 64, 0, f(0.1), A, ws, None) == 1
    assert lib.fa2_backward_main(A, A, A, A, A, A, 1, 1, 128, 64, 0, f(-1.0), A, ws, None) == 1
    assert lib.fa2_backward_main(A, A, A, A, A, A, 1, 1, 128, 64, 0, f(0.1), A + 8, ws, None) == 3
    assert lib.fa2_backward_main(A, A, A, A + 2, A, A, 1, 1, 128, 64, 0, f(0.1), A, ws, None) == 3
    assert lib.fa2_backward_dq_convert(None, 1, 1, 128, 64, f(0.1), A, ws, None) == 1
    assert lib.fa2_backward_dq_convert(A, 1, 1, 128, 64, f(0.1), A, 16, None) == 1
    assert lib.fa2_backward_dq_convert(A + 2, 1, 1, 128, 64, f(0.1), A, ws, None) == 3


def test_backward_ex_rejects_bad_strategy(lib):
    ws = lib.fa2_backward_workspace_size(1, 1, 128, 64)
    args = [A] * 9 + [1, 1, 128, 64, 0, ctypes.c_float(0.125), A, ws]
    assert lib.fa2_backward_ex(*args, 3, None) == 1
    assert lib.fa2_backward_ex(*args, -1, None) == 1
    assert lib.fa2_backward_dq_strategy(1, 1, 128, 64, 0) in (1, 2)
    assert lib.fa2_backward_dq(None, A, A, A, A, 1, 1, 128, 64, 0, ctypes.c_float(0.1), A, ws, None) == 1
    assert lib.fa2_backward_main_dkdv(A, A, A, A, A, A, 1, 1, 128, 64, 0, ctypes.c_float(0.1), A, 8, None) == 1


def test_host_path_workspace_size(lib):
    """Three chunk slots of: 8 bf16 tensors + fp32 LSE + the chunk's backward workspace,
    each rounded up to 256 bytes; heads_per_chunk 0 means ceil(B*H / 8)."""
    def r256(x):
        return (x + 255) // 256 * 256

    def expect(B, H, N, d, hpc):
        c = hpc if hpc > 0 else (B * H + 7) // 8
        c = max(1, min(c, B * H))
        slot = (8 * r256(c * N * d * 2) + r256(c * N * 4)
                + r256(lib.fa2_backward_workspace_size(1, c, N, d)))
        return 3 * slot

    for args in [(2, 3, 129, 64, 2), (2, 3, 129, 64, 0), (8, 16, 2048, 128, 0), (1, 5, 1, 128, 9),
                 (1, 1, 300, 64, 1)]:
        assert lib.fa2_forward_backward_host_workspace_size(*args) == expect(*args), args
    assert lib.fa2_forward_backward_host_workspace_size(1, 1, 128, 64, -1) == 0
    assert lib.fa2_forward_backward_host_workspace_size(1, 1, 128, 32, 0) == 0


def host(lib, ptrs=None, B=1, H=2, N=128, d=64, scale=0.125, hpc=0, ws_bytes=None):
    p = [A] * 10 if ptrs is None else ptrs
    if ws_bytes is None:
        ws_bytes = lib.fa2_forward_backward_host_workspace_size(B, H, N, d, max(hpc, 0))
    return lib.fa2_forward_backward_host(*p[:9], B, H, N, d, 1, ctypes.c_float(scale), hpc, p[9],
                                         ws_bytes, None)


def test_host_path_rejects_bad_arguments(lib):
    for i in range(10):
        p = [A] * 10
        p[i] = None
        assert host(lib, p) == 1, i
    assert host(lib, hpc=-1) == 1
    assert host(lib, ws_bytes=1000) == 1
    assert host(lib, N=0) == 1
    assert host(lib, scale=float("nan")) == 1
    assert host(lib, d=80) == 2
    p = [A] * 10
    p[9] = A + 16  # the device workspace must be 256-byte aligned
    assert host(lib, p) == 3


def test_qk_entry_points_reject_bad_arguments(lib):
    f = ctypes.c_float

    def fwd_qk(Nq=100, Nk=300, causal=1, d=64, p=None):
        p = [A] * 5 if p is None else p
        return lib.fa2_forward_qk(*p, 1, 2, Nq, Nk, d, causal, f(0.125), None)

    assert fwd_qk(Nq=300, Nk=100, causal=1) == 2  # causal needs Nq <= Nk
    assert fwd_qk(Nq=0) == 1 and fwd_qk(Nk=0) == 1
    assert fwd_qk(d=80) == 2
    assert fwd_qk(p=[A, None, A, A, A]) == 1
    assert fwd_qk(p=[A, A + 8, A, A, A]) == 3
    ws = lib.fa2_backward_workspace_size(1, 2, 100, 64)

    def bwd_qk(Nq=100, Nk=300, causal=1, wsb=ws, p=None):
        p = [A] * 10 if p is None else p
        return lib.fa2_backward_qk(*p[:9], 1, 2, Nq, Nk, 64, causal, f(0.125), p[9], wsb, None)

    assert bwd_qk(Nq=300, Nk=100, causal=1) == 2
    assert bwd_qk(wsb=ws - 1) == 1
    for i in range(10):
        p = [A] * 10
        p[i] = None
        assert bwd_qk(p=p) == 1, i
    p = [A] * 10
    p[7] = A + 4
    assert bwd_qk(p=p) == 3
