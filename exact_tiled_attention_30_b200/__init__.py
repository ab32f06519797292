"""Exact tiled attention (FlashAttention-2 method) for B200 / sm_100a.

Thin Python binding of the C ABI declared in ``include/fa2.h``: every function
with an ``fa2_`` name marshals its arguments (device pointers, sizes, the
current CUDA stream) and calls the entry point of the same name in
``libfa2_b200.so``. All arithmetic runs in that library's CUDA kernels; there is
no fallback. If the library is missing the import fails loudly; build it with
``python -m exact_tiled_attention_30_b200.build``.

``attention_forward`` / ``attention_backward`` are conveniences that allocate
the outputs (and the backward workspace) with PyTorch and then call the C ABI.
"""
from __future__ import annotations

import ctypes
import os

__all__ = [
    "FA2Error", "LIB_PATH", "load_library", "fa2_forward", "fa2_backward", "fa2_backward_workspace_size",
    "fa2_backward_preprocess", "fa2_backward_main", "fa2_backward_dq_convert",
    "fa2_backward_ex", "fa2_backward_dq_strategy", "fa2_backward_main_dkdv", "fa2_backward_dq",
    "DQ_AUTO", "DQ_REDUCE", "DQ_SEPARATE",
    "fa2_status_string", "fa2_get_device_status", "fa2_clear_device_status",
    "attention_forward", "attention_backward", "STATUS",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libfa2_b200.so")

#: dQ strategies of fa2_backward_ex (fa2_dq_strategy in include/fa2.h)
DQ_AUTO, DQ_REDUCE, DQ_SEPARATE = 0, 1, 2

STATUS = {0: "FA2_OK", 1: "FA2_ERR_INVALID_ARG", 2: "FA2_ERR_UNSUPPORTED",
          3: "FA2_ERR_MISALIGNED", 4: "FA2_ERR_CUDA", 5: "FA2_ERR_TIMEOUT", 6: "FA2_ERR_CONFLICT"}


class FA2Error(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} failed: {STATUS.get(status, status)}")
        self.status = status


_lib = None


def load_library():
    """The ctypes handle of libfa2_b200.so. Raises if the library was not built:
    there is no CPU or PyTorch fallback for any entry point."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: the CUDA library must be built "
            "(python -m exact_tiled_attention_30_b200.build); there is no CPU fallback")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i = ctypes.c_void_p, ctypes.c_int
    lib.fa2_forward.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, ctypes.c_float, vp]
    lib.fa2_forward.restype = i
    lib.fa2_backward_workspace_size.argtypes = [i, i, i, i]
    lib.fa2_backward_workspace_size.restype = ctypes.c_size_t
    lib.fa2_backward.argtypes = [vp] * 9 + [i, i, i, i, i, ctypes.c_float, vp, ctypes.c_size_t, vp]
    lib.fa2_backward.restype = i
    lib.fa2_backward_preprocess.argtypes = [vp, vp, vp, i, i, i, i, vp, ctypes.c_size_t, vp]
    lib.fa2_backward_preprocess.restype = i
    lib.fa2_backward_main.argtypes = [vp] * 6 + [i, i, i, i, i, ctypes.c_float, vp,
                                                 ctypes.c_size_t, vp]
    lib.fa2_backward_main.restype = i
    lib.fa2_backward_dq_convert.argtypes = [vp, i, i, i, i, ctypes.c_float, vp, ctypes.c_size_t, vp]
    lib.fa2_backward_dq_convert.restype = i
    lib.fa2_backward_ex.argtypes = [vp] * 9 + [i, i, i, i, i, ctypes.c_float, vp, ctypes.c_size_t,
                                              i, vp]
    lib.fa2_backward_ex.restype = i
    lib.fa2_backward_dq_strategy.argtypes = [i, i, i, i, i]
    lib.fa2_backward_dq_strategy.restype = i
    lib.fa2_backward_main_dkdv.argtypes = [vp] * 6 + [i, i, i, i, i, ctypes.c_float, vp,
                                                      ctypes.c_size_t, vp]
    lib.fa2_backward_main_dkdv.restype = i
    lib.fa2_backward_dq.argtypes = [vp] * 5 + [i, i, i, i, i, ctypes.c_float, vp, ctypes.c_size_t, vp]
    lib.fa2_backward_dq.restype = i
    lib.fa2_forward_qk.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, ctypes.c_float, vp]
    lib.fa2_forward_qk.restype = i
    lib.fa2_backward_qk.argtypes = [vp] * 9 + [i, i, i, i, i, i, ctypes.c_float, vp, ctypes.c_size_t,
                                              vp]
    lib.fa2_backward_qk.restype = i
    lib.fa2_forward_backward_host_workspace_size.argtypes = [i, i, i, i, i]
    lib.fa2_forward_backward_host_workspace_size.restype = ctypes.c_size_t
    lib.fa2_forward_backward_host.argtypes = [vp] * 9 + [i, i, i, i, i, ctypes.c_float, i, vp,
                                                        ctypes.c_size_t, vp]
    lib.fa2_forward_backward_host.restype = i
    lib.fa2_status_string.argtypes = [i]
    lib.fa2_status_string.restype = ctypes.c_char_p
    lib.fa2_get_device_status.argtypes = [vp, ctypes.POINTER(i)]
    lib.fa2_get_device_status.restype = i
    lib.fa2_clear_device_status.argtypes = []
    lib.fa2_clear_device_status.restype = i
    _lib = lib
    return lib


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        import torch

        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(fn: str, status: int):
    if status != 0:
        raise FA2Error(fn, status)


def _bhnd(q):
    if q.dim() != 4:
        raise ValueError("expected a [B, H, N, d] tensor")
    return tuple(int(x) for x in q.shape)


def _require(t, name, dtype=None, shape=None):
    """Checks one tensor argument before its pointer goes to the library: a
    contiguous CUDA tensor on the current device (where the library launches),
    of the given dtype and shape. The C ABI sees only pointers and sizes, so a
    wrong shape or device would otherwise reach the kernels."""
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    import torch

    cur = torch.cuda.current_device()
    if t.device.index != cur:
        raise ValueError(f"{name} is on {t.device}; the library launches on the current "
                         f"device cuda:{cur}")


def _require_bf16(shape, *named):
    import torch

    for t, n in named:
        _require(t, n, torch.bfloat16, shape)


def _require_lse(lse, shape):
    import torch

    _require(lse, "lse", torch.float32, shape)


def fa2_forward(q, k, v, o, lse, causal: bool, scale: float, stream=None) -> None:
    """C ABI fa2_forward on torch tensors: q, k, v, o bf16 [B,H,N,d]; lse fp32 [B,H,N]."""
    B, H, N, d = _bhnd(q)
    _require_bf16((B, H, N, d), (q, "q"), (k, "k"), (v, "v"), (o, "o"))
    _require_lse(lse, (B, H, N))
    _check("fa2_forward", load_library().fa2_forward(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, N,
                                          d, int(bool(causal)), float(scale), _stream(stream)))


def fa2_backward_workspace_size(B: int, H: int, N: int, d: int) -> int:
    return int(load_library().fa2_backward_workspace_size(B, H, N, d))


def fa2_backward(q, k, v, o, lse, dout, dq, dk, dv, causal: bool, scale: float, workspace,
                 stream=None) -> None:
    """C ABI fa2_backward on torch tensors; workspace is a uint8 CUDA tensor."""
    B, H, N, d = _bhnd(q)
    _require_bf16((B, H, N, d), (q, "q"), (k, "k"), (v, "v"), (o, "o"), (dout, "dout"),
                  (dq, "dq"), (dk, "dk"), (dv, "dv"))
    _require_lse(lse, (B, H, N))
    _require(workspace, "workspace")
    nbytes = workspace.numel() * workspace.element_size()
    _check("fa2_backward", load_library().fa2_backward(
        _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv),
        B, H, N, d, int(bool(causal)), float(scale), _ptr(workspace), nbytes, _stream(stream)))


def _nbytes(t) -> int:
    return t.numel() * t.element_size()


def fa2_backward_preprocess(o, lse, dout, workspace, stream=None) -> None:
    """C ABI fa2_backward_preprocess (first of the three backward stages)."""
    B, H, N, d = _bhnd(o)
    _require_bf16((B, H, N, d), (o, "o"), (dout, "dout"))
    _require_lse(lse, (B, H, N))
    _require(workspace, "workspace")
    _check("fa2_backward_preprocess", load_library().fa2_backward_preprocess(
        _ptr(o), _ptr(lse), _ptr(dout), B, H, N, d, _ptr(workspace), _nbytes(workspace),
        _stream(stream)))


def fa2_backward_main(q, k, v, dout, dk, dv, causal: bool, scale: float, workspace,
                      stream=None) -> None:
    """C ABI fa2_backward_main (dK, dV and the fp32 dQ accumulator)."""
    B, H, N, d = _bhnd(q)
    _require_bf16((B, H, N, d), (q, "q"), (k, "k"), (v, "v"), (dout, "dout"), (dk, "dk"),
                  (dv, "dv"))
    _require(workspace, "workspace")
    _check("fa2_backward_main", load_library().fa2_backward_main(
        _ptr(q), _ptr(k), _ptr(v), _ptr(dout), _ptr(dk), _ptr(dv), B, H, N, d, int(bool(causal)),
        float(scale), _ptr(workspace), _nbytes(workspace), _stream(stream)))


def fa2_backward_dq_convert(dq, scale: float, workspace, stream=None) -> None:
    """C ABI fa2_backward_dq_convert (dq = bf16(scale * accumulator))."""
    B, H, N, d = _bhnd(dq)
    _require_bf16((B, H, N, d), (dq, "dq"))
    _require(workspace, "workspace")
    _check("fa2_backward_dq_convert", load_library().fa2_backward_dq_convert(
        _ptr(dq), B, H, N, d, float(scale), _ptr(workspace), _nbytes(workspace), _stream(stream)))


def fa2_backward_ex(q, k, v, o, lse, dout, dq, dk, dv, causal: bool, scale: float, workspace,
                    dq_strategy: int = DQ_AUTO, stream=None) -> None:
    """C ABI fa2_backward_ex: fa2_backward with an explicit dQ strategy."""
    B, H, N, d = _bhnd(q)
    _require_bf16((B, H, N, d), (q, "q"), (k, "k"), (v, "v"), (o, "o"), (dout, "dout"),
                  (dq, "dq"), (dk, "dk"), (dv, "dv"))
    _require_lse(lse, (B, H, N))
    _require(workspace, "workspace")
    _check("fa2_backward_ex", load_library().fa2_backward_ex(
        _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv),
        B, H, N, d, int(bool(causal)), float(scale), _ptr(workspace), _nbytes(workspace),
        int(dq_strategy), _stream(stream)))


def fa2_backward_dq_strategy(B: int, H: int, N: int, d: int, causal: bool) -> int:
    return int(load_library().fa2_backward_dq_strategy(B, H, N, d, int(bool(causal))))


def fa2_backward_main_dkdv(q, k, v, dout, dk, dv, causal: bool, scale: float, workspace,
                           stream=None) -> None:
    """C ABI fa2_backward_main_dkdv (dK, dV only; FA2_DQ_SEPARATE)."""
    B, H, N, d = _bhnd(q)
    _require_bf16((B, H, N, d), (q, "q"), (k, "k"), (v, "v"), (dout, "dout"), (dk, "dk"),
                  (dv, "dv"))
    _require(workspace, "workspace")
    _check("fa2_backward_main_dkdv", load_library().fa2_backward_main_dkdv(
        _ptr(q), _ptr(k), _ptr(v), _ptr(dout), _ptr(dk), _ptr(dv), B, H, N, d, int(bool(causal)),
        float(scale), _ptr(workspace), _nbytes(workspace), _stream(stream)))


def fa2_backward_dq(q, k, v, dout, dq, causal: bool, scale: float, workspace, stream=None) -> None:
    """C ABI fa2_backward_dq (query-parallel dQ kernel; FA2_DQ_SEPARATE)."""
    B, H, N, d = _bhnd(q)
    _require_bf16((B, H, N, d), (q, "q"), (k, "k"), (v, "v"), (dout, "dout"), (dq, "dq"))
    _require(workspace, "workspace")
    _check("fa2_backward_dq", load_library().fa2_backward_dq(
        _ptr(q), _ptr(k), _ptr(v), _ptr(dout), _ptr(dq), B, H, N, d, int(bool(causal)),
        float(scale), _ptr(workspace), _nbytes(workspace), _stream(stream)))


def fa2_status_string(status: int) -> str:
    return load_library().fa2_status_string(int(status)).decode()


def fa2_get_device_status(stream=None):
    """(status, site) after synchronising the stream; status 5 = a kernel timed out."""
    info = ctypes.c_int(0)
    st = load_library().fa2_get_device_status(_stream(stream), ctypes.byref(info))
    return int(st), int(info.value)


def fa2_clear_device_status() -> None:
    _check("fa2_clear_device_status", load_library().fa2_clear_device_status())


def fa2_forward_qk(q, k, v, o, lse, causal: bool, scale: float, stream=None) -> None:
    """C ABI fa2_forward_qk: q, o [B,H,Nq,d], k, v [B,H,Nk,d] bf16; lse fp32 [B,H,Nq].
    Causal masking is aligned to the bottom-right corner (query i sees keys
    j <= i + Nk - Nq)."""
    B, H, Nq, d = _bhnd(q)
    Nk = _bhnd(k)[2]
    _require_bf16((B, H, Nq, d), (q, "q"), (o, "o"))
    _require_bf16((B, H, Nk, d), (k, "k"), (v, "v"))
    _require_lse(lse, (B, H, Nq))
    _check("fa2_forward_qk", load_library().fa2_forward_qk(
        _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, Nq, Nk, d, int(bool(causal)),
        float(scale), _stream(stream)))


def fa2_backward_qk(q, k, v, o, lse, dout, dq, dk, dv, causal: bool, scale: float, workspace,
                    stream=None) -> None:
    """C ABI fa2_backward_qk (shapes as fa2_forward_qk; dq like q, dk and dv like k;
    workspace of fa2_backward_workspace_size(B, H, Nq, d) bytes)."""
    B, H, Nq, d = _bhnd(q)
    Nk = _bhnd(k)[2]
    _require_bf16((B, H, Nq, d), (q, "q"), (o, "o"), (dout, "dout"), (dq, "dq"))
    _require_bf16((B, H, Nk, d), (k, "k"), (v, "v"), (dk, "dk"), (dv, "dv"))
    _require_lse(lse, (B, H, Nq))
    _require(workspace, "workspace")
    _check("fa2_backward_qk", load_library().fa2_backward_qk(
        _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv),
        B, H, Nq, Nk, d, int(bool(causal)), float(scale), _ptr(workspace), _nbytes(workspace),
        _stream(stream)))


def attention_forward(q, k, v, causal: bool = False, scale: float | None = None, stream=None):
    """Allocates o and lse, runs fa2_forward (fa2_forward_qk when k and q differ in
    length) on q's device, returns (o, lse)."""
    import torch

    B, H, N, d = _bhnd(q)
    if scale is None:
        scale = d ** -0.5
    with torch.cuda.device(q.device):
        o = torch.empty_like(q)
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
        if k.shape[2] != N:
            fa2_forward_qk(q, k, v, o, lse, causal, scale, stream)
        else:
            fa2_forward(q, k, v, o, lse, causal, scale, stream)
    return o, lse


def attention_backward(q, k, v, o, lse, dout, causal: bool = False, scale: float | None = None,
                       stream=None, workspace=None, dq_strategy: int = DQ_AUTO):
    """Allocates dq, dk, dv (and the workspace unless given), runs fa2_backward_ex
    (fa2_backward_qk when k and q differ in length) on q's device."""
    import torch

    B, H, N, d = _bhnd(q)
    if scale is None:
        scale = d ** -0.5
    with torch.cuda.device(q.device):
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        if workspace is None:
            workspace = torch.empty(fa2_backward_workspace_size(B, H, N, d), dtype=torch.uint8,
                                    device=q.device)
        if k.shape[2] != N:  # different key length: fa2_backward_qk (dQ by reductions)
            fa2_backward_qk(q, k, v, o, lse, dout, dq, dk, dv, causal, scale, workspace, stream)
        else:
            fa2_backward_ex(q, k, v, o, lse, dout, dq, dk, dv, causal, scale, workspace,
                            dq_strategy, stream)
    return dq, dk, dv


def fa2_backward_noalloc(q, k, v, o, lse, dout, dq, dk, dv, causal: bool, scale: float,
                         stream=None) -> None:
    """C ABI fa2_backward_noalloc: the backward pass with its scratch in a fixed
    device array inside the library (FA2_NOALLOC_SCRATCH_BYTES = 64 MiB) instead
    of a workspace, for callers that cannot allocate device memory at that point.
    Raises FA2Error(FA2_ERR_UNSUPPORTED) when the sizes need more scratch than that.
    Calls on one stream are safe; calls that overlap on the GPU race on the array."""
    lib = load_library()
    fn = lib.fa2_backward_noalloc
    if fn.restype is not ctypes.c_int or fn.argtypes is None:
        vp, i = ctypes.c_void_p, ctypes.c_int
        fn.argtypes = [vp] * 9 + [i, i, i, i, i, ctypes.c_float, vp]
        fn.restype = i
    B, H, N, d = _bhnd(q)
    _require_bf16((B, H, N, d), (q, "q"), (k, "k"), (v, "v"), (o, "o"), (dout, "dout"),
                  (dq, "dq"), (dk, "dk"), (dv, "dv"))
    _require_lse(lse, (B, H, N))
    _check("fa2_backward_noalloc", fn(
        _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv),
        B, H, N, d, int(bool(causal)), float(scale), _stream(stream)))


def fa2_forward_backward_host_workspace_size(B: int, H: int, N: int, d: int,
                                             heads_per_chunk: int = 0) -> int:
    return int(load_library().fa2_forward_backward_host_workspace_size(B, H, N, d, heads_per_chunk))


def _require_host(t, name, dtype):
    if t.is_cuda or not t.is_contiguous() or t.dtype != dtype:
        raise ValueError(f"{name} must be a contiguous {dtype} host tensor")


def fa2_forward_backward_host(q, k, v, dout, o, lse, dq, dk, dv, causal: bool, scale: float,
                              workspace, heads_per_chunk: int = 0, stream=None) -> None:
    """C ABI fa2_forward_backward_host: q, k, v, dout and the outputs o, lse, dq,
    dk, dv are HOST tensors (page-locked for the copies to overlap); workspace is
    a CUDA uint8 tensor of fa2_forward_backward_host_workspace_size bytes."""
    import torch

    B, H, N, d = _bhnd(q)
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (dout, "dout"), (o, "o"), (dq, "dq"), (dk, "dk"),
                 (dv, "dv")):
        _require_host(t, n, torch.bfloat16)
        if tuple(t.shape) != (B, H, N, d):
            raise ValueError(f"{n} has shape {tuple(t.shape)}, expected {(B, H, N, d)}")
    _require_host(lse, "lse", torch.float32)
    if tuple(lse.shape) != (B, H, N):
        raise ValueError("lse must be [B, H, N]")
    _require(workspace, "workspace")
    _check("fa2_forward_backward_host", load_library().fa2_forward_backward_host(
        _ptr(q), _ptr(k), _ptr(v), _ptr(dout), _ptr(o), _ptr(lse), _ptr(dq), _ptr(dk), _ptr(dv),
        B, H, N, d, int(bool(causal)), float(scale), int(heads_per_chunk), _ptr(workspace),
        _nbytes(workspace), _stream(stream)))


def attention_forward_backward_host(q, k, v, dout, causal: bool = False, scale: float | None = None,
                                    heads_per_chunk: int = 0, workspace=None, out=None,
                                    stream=None):
    """Forward and backward of host tensors, copies pipelined with the kernels.
    Returns host (o, lse, dq, dk, dv), page-locked (or the tensors of `out`);
    they are complete once `stream` (default: the current stream) has passed
    the call."""
    import torch

    B, H, N, d = _bhnd(q)
    if scale is None:
        scale = d ** -0.5
    if out is None:
        pin = dict(dtype=torch.bfloat16, pin_memory=True)
        out = (torch.empty((B, H, N, d), **pin), torch.empty((B, H, N), dtype=torch.float32,
                                                            pin_memory=True),
               torch.empty((B, H, N, d), **pin), torch.empty((B, H, N, d), **pin),
               torch.empty((B, H, N, d), **pin))
    if workspace is None:
        workspace = torch.empty(fa2_forward_backward_host_workspace_size(B, H, N, d, heads_per_chunk),
                                dtype=torch.uint8, device="cuda")
    o, lse, dq, dk, dv = out
    fa2_forward_backward_host(q, k, v, dout, o, lse, dq, dk, dv, causal, scale, workspace,
                              heads_per_chunk, stream)
    return o, lse, dq, dk, dv


def _autograd_function():
    import torch

    class _Attention(torch.autograd.Function):
        """Exact attention with both passes on the C ABI (fa2_forward, fa2_backward)."""

        @staticmethod
        def forward(ctx, q, k, v, causal, scale):
            o, lse = attention_forward(q, k, v, causal=causal, scale=scale)
            ctx.save_for_backward(q, k, v, o, lse)
            ctx.causal, ctx.scale = causal, scale
            return o

        @staticmethod
        def backward(ctx, dout):
            q, k, v, o, lse = ctx.saved_tensors
            dq, dk, dv = attention_backward(q, k, v, o, lse, dout.contiguous(), causal=ctx.causal,
                                            scale=ctx.scale)
            return dq, dk, dv, None, None

    return _Attention


_ATTENTION_FN = None


def attention(q, k, v, causal: bool = False, scale: float | None = None):
    """softmax(scale * q k^T [causal]) v as a differentiable PyTorch op: the forward
    and backward passes run in this library's kernels (q, k, v: contiguous bf16
    CUDA tensors [B, H, N, d]; d in {64, 128}). The drop-in form of the method
    for code that trains through attention with autograd."""
    global _ATTENTION_FN
    if _ATTENTION_FN is None:
        _ATTENTION_FN = _autograd_function()
    if scale is None:
        scale = q.shape[-1] ** -0.5
    return _ATTENTION_FN.apply(q, k, v, bool(causal), float(scale))
