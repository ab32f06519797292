"""Bounded waits end with an error status, and the context stays usable.

Every mbarrier wait in the kernels is bounded: when one runs out, the thread
records a site code in the library's device status word, raises the CTA's
abort flag, every role leaves its loop, the MMA warp waits for its own tensor
core operations, the TMA warp for its copies in flight, TMEM is freed and the
kernel returns. fa2_get_device_status then reports FA2_ERR_TIMEOUT and the site.

To make a wait run out without any fault, these tests load the test-hooks build
of the library (never the shipped one): its waits give up after 20 ms instead
of 2 s, and fa2_debug_set_stall(n) makes the forward producer skip the load of
each CTA's n-th key tile (it neither issues the copy nor expects its bytes), so
the MMA warp's wait on that stage is one that nothing completes. After the
stalled call the status is cleared and the same library, in the same context,
must run a normal forward that matches the oracle.
"""
import ctypes
import math

import numpy as np
import pytest

from tests import gpu_helpers as gh

FA2_ERR_TIMEOUT = 5


def _test_hooks_lib():
    from exact_tiled_attention_30_b200 import build

    lib = ctypes.CDLL(build.build_test_hooks())
    vp, i = ctypes.c_void_p, ctypes.c_int
    lib.fa2_forward.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, ctypes.c_float, vp]
    lib.fa2_forward.restype = i
    lib.fa2_get_device_status.argtypes = [vp, ctypes.POINTER(i)]
    lib.fa2_get_device_status.restype = i
    lib.fa2_clear_device_status.argtypes = []
    lib.fa2_clear_device_status.restype = i
    lib.fa2_debug_set_stall.argtypes = [i]
    lib.fa2_debug_set_stall.restype = i
    return lib


def test_shipped_library_has_no_test_hooks():
    import exact_tiled_attention_30_b200 as fa2

    lib = fa2.load_library()
    assert not hasattr(lib, "fa2_debug_set_stall")
    assert not hasattr(lib, "fa2_debug_forward_tag_skew")
    assert fa2.fa2_status_string(6) == "FA2_ERR_CONFLICT"


@pytest.mark.gpu
@pytest.mark.parametrize("d,causal", [(64, False), (128, True), (128, False)])
def test_stalled_wait_times_out_then_context_recovers(oracle_mod, d, causal):
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    lib = _test_hooks_lib()
    B, H, N = 1, 2, 384
    scale = 1.0 / math.sqrt(d)
    t = gh.inputs(0, B, H, N, d)
    q, k, v = (gh.to_device(t[n]) for n in ("q", "k", "v"))
    stream = torch.cuda.current_stream()
    sp = ctypes.c_void_p(stream.cuda_stream)
    info = ctypes.c_int(0)

    def forward(o, lse):
        return lib.fa2_forward(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                               lse.data_ptr(), B, H, N, d, int(causal), ctypes.c_float(scale), sp)

    assert lib.fa2_clear_device_status() == 0
    o, lse = torch.empty_like(q), torch.empty(B, H, N, device="cuda", dtype=torch.float32)
    assert lib.fa2_debug_set_stall(2) == 0  # each CTA's second key tile
    try:
        assert forward(o, lse) == 0  # the launch itself succeeds
        st = lib.fa2_get_device_status(sp, ctypes.byref(info))
    finally:
        assert lib.fa2_debug_set_stall(0) == 0
    assert st == FA2_ERR_TIMEOUT, f"status {st}, site {info.value:#x}"
    # forward sites: 0x1xx producer, 0x2xx MMA issuer, 0x3xx softmax warps
    assert 0x100 <= info.value < 0x400, f"site {info.value:#x}"

    # same library, same context: clear the word and run a normal forward
    assert lib.fa2_clear_device_status() == 0
    o2, lse2 = torch.empty_like(q), torch.empty_like(lse)
    assert forward(o2, lse2) == 0
    st = lib.fa2_get_device_status(sp, ctypes.byref(info))
    assert st == 0, f"status {st} after clearing, site {info.value:#x}"
    ro, rl = oracle_mod.attention_forward(t["q"], t["k"], t["v"], causal, scale)
    where = f"after a timed-out call, B={B} H={H} N={N} d={d} causal={causal}"
    gh.check_o(gh.to_host_f64(o2), ro, where)
    gh.check_lse(lse2.cpu().numpy().astype(np.float64), rl, where)


FA2_ERR_CONFLICT = 6


@pytest.mark.gpu
def test_foreign_counter_tag_is_reported_as_conflict(oracle_mod):
    """A forward whose work counter holds another launch's tag (what happens when
    more than 256 forwards on different streams are in flight at once and the
    counter ring wraps onto a running launch) stops taking work and reports
    FA2_ERR_CONFLICT instead of sharing items silently. The test-hooks build
    makes every launch see a foreign tag (fa2_debug_forward_tag_skew); with the
    skew removed and the status cleared, the same context computes correctly."""
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    lib = _test_hooks_lib()
    lib.fa2_debug_forward_tag_skew.argtypes = [ctypes.c_int]
    lib.fa2_debug_forward_tag_skew.restype = ctypes.c_int
    B, H, N, d, causal = 2, 2, 640, 128, True
    scale = 1.0 / math.sqrt(d)
    t = gh.inputs(33, B, H, N, d)
    q, k, v = (gh.to_device(t[n]) for n in ("q", "k", "v"))
    sp = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    info = ctypes.c_int(0)

    def forward(o, lse):
        return lib.fa2_forward(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                               lse.data_ptr(), B, H, N, d, int(causal), ctypes.c_float(scale), sp)

    assert lib.fa2_clear_device_status() == 0
    o, lse = torch.empty_like(q), torch.empty(B, H, N, device="cuda", dtype=torch.float32)
    assert lib.fa2_debug_forward_tag_skew(1) == 0
    try:
        assert forward(o, lse) == 0
        st = lib.fa2_get_device_status(sp, ctypes.byref(info))
    finally:
        lib.fa2_debug_forward_tag_skew(0)
    assert st == FA2_ERR_CONFLICT, f"status {st}, site {info.value:#x}"
    assert info.value == 0x10A

    assert lib.fa2_clear_device_status() == 0
    o2, lse2 = torch.empty_like(q), torch.empty_like(lse)
    assert forward(o2, lse2) == 0
    st = lib.fa2_get_device_status(sp, ctypes.byref(info))
    assert st == 0, f"status {st} after clearing, site {info.value:#x}"
    ro, rl = oracle_mod.attention_forward(t["q"], t["k"], t["v"], causal, scale)
    where = f"after a conflict, B={B} H={H} N={N} d={d} causal={causal}"
    gh.check_o(gh.to_host_f64(o2), ro, where)
    gh.check_lse(lse2.cpu().numpy().astype(np.float64), rl, where)
