"""fa2_backward_noalloc, the backward entry point that allocates nothing.

It exists for callers that cannot allocate device memory when they run the
backward pass (memory reserved up front, hosts that forbid allocation on the
hot path, C callers without an allocator). These tests call it through the C
ABI and compare it with fa2_backward (caller-provided workspace) and with the
fp64 oracle on two calls in a row, so that a second call sees the first call's
leftovers in the shared scratch array. This file is collected last on purpose.
"""
import ctypes
import math

import pytest

from tests import gpu_helpers as gh

A = 0x10000  # aligned fake device address, for checks that fail before any launch


def _lib():
    import exact_tiled_attention_30_b200 as m

    lib = m.load_library()
    fn = lib.fa2_backward_noalloc
    vp, i = ctypes.c_void_p, ctypes.c_int
    fn.argtypes = [vp] * 9 + [i, i, i, i, i, ctypes.c_float, vp]
    fn.restype = i
    return lib


def test_noalloc_rejects_sizes_beyond_the_scratch():
    lib = _lib()
    limit = 64 << 20
    # B*H*N*d fp32 accumulator alone above 64 MiB
    assert lib.fa2_backward_workspace_size(1, 64, 4096, 64) > limit
    assert lib.fa2_backward_noalloc(*([A] * 9), 1, 64, 4096, 64, 0, ctypes.c_float(0.125),
                                    None) == 2
    assert lib.fa2_backward_noalloc(*([A] * 8), None, 1, 1, 128, 64, 0, ctypes.c_float(0.125),
                                    None) == 1


@pytest.mark.gpu
@pytest.mark.parametrize("B,H,N,d,causal", [(2, 3, 384, 128, True), (1, 4, 1000, 64, False)])
def test_noalloc_matches_workspace_backward(oracle_mod, B, H, N, d, causal):
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import exact_tiled_attention_30_b200 as fa2

    lib = _lib()
    scale = 1.0 / math.sqrt(d)
    t = gh.inputs(21, B, H, N, d, with_do=True)
    q, k, v, do = (gh.to_device(t[n]) for n in ("q", "k", "v", "do"))
    o, lse = fa2.attention_forward(q, k, v, causal=causal, scale=scale)
    ref = fa2.attention_backward(q, k, v, o, lse, do, causal=causal, scale=scale)
    oracle_ref = oracle_mod.attention_backward(t["q"], t["k"], t["v"], t["do"], causal, scale)
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        st = lib.fa2_backward_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                      lse.data_ptr(), do.data_ptr(), dq.data_ptr(),
                                      dk.data_ptr(), dv.data_ptr(), B, H, N, d, int(causal),
                                      ctypes.c_float(scale), stream)
        assert st == 0, fa2.fa2_status_string(st)
        torch.cuda.synchronize()
        for got, want, name in zip((dq, dk, dv), ref, ("dq", "dk", "dv")):
            err = gh.rel_fro(gh.to_host_f64(got), gh.to_host_f64(want))
            assert err <= gh.GRAD_RTOL, f"call {call}: {name} differs by {err:.3e}"
            # and against the fp64 oracle, with the tolerance of the parity tests
            gh.check_grad(name, gh.to_host_f64(got), oracle_ref[name],
                          f"no-alloc backward call {call} B={B} H={H} N={N} d={d} causal={causal}")
    st, site = fa2.fa2_get_device_status()
    assert st == 0, f"device status {st} at {site:#x}"
