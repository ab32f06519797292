"""fp64 CPU oracle for exact attention (test infrastructure).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU legs of ``bench.py``
(``cpu_baseline`` and ``--impl reference``) may import this package. The CUDA
product path never touches it and shares no code with it.

The arithmetic lives in ``attn_oracle.cpp`` (plain fp64 loops, threads over
rows); this file only builds that library, widens bf16 inputs to fp64 and
marshals arrays. See the C++ file's header for the definition it follows and
the passages it cites.

parity: pinned by ``tests/test_oracle.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attn_oracle.cpp")
_LIB = os.path.join(_HERE, "liboracle_attn.so")
_lock = threading.Lock()
_lib = None

# x86-64-v3 (AVX2) keeps the build portable between hosts; fp contraction is off
# so every product and sum rounds separately, as written.
CXXFLAGS = ["-O3", "-march=x86-64-v3", "-ffp-contract=off", "-fno-fast-math", "-std=c++17",
            "-fPIC", "-shared", "-pthread"]


def build(force: bool = False) -> str:
    """Compile the oracle library in place (g++); returns its path."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.run(["g++", *CXXFLAGS, _SRC, "-o", tmp], check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _bind(lib):
    d = ctypes.POINTER(ctypes.c_double)
    i64 = ctypes.c_int64
    pi64 = ctypes.POINTER(ctypes.c_int64)
    lib.oracle_attention_forward.argtypes = [d, d, d, i64, i64, i64, ctypes.c_int,
                                             ctypes.c_double, pi64, i64, d, d, ctypes.c_int]
    lib.oracle_attention_forward.restype = ctypes.c_int
    lib.oracle_attention_backward.argtypes = [d, d, d, d, i64, i64, i64, ctypes.c_int,
                                              ctypes.c_double, d, d, d, d, d, ctypes.c_int]
    lib.oracle_attention_backward.restype = ctypes.c_int
    lib.oracle_attention_backward_rows.argtypes = [d, d, d, d, i64, i64, i64, ctypes.c_int,
                                                   ctypes.c_double, pi64, i64, pi64, i64,
                                                   d, d, d, ctypes.c_int]
    lib.oracle_attention_backward_rows.restype = ctypes.c_int
    lib.oracle_attention_forward_qk.argtypes = [d, d, d, i64, i64, i64, i64, ctypes.c_int,
                                                ctypes.c_double, pi64, i64, d, d, ctypes.c_int]
    lib.oracle_attention_forward_qk.restype = ctypes.c_int
    lib.oracle_attention_backward_qk.argtypes = [d, d, d, d, i64, i64, i64, i64, ctypes.c_int,
                                                 ctypes.c_double, d, d, d, d, d, ctypes.c_int]
    lib.oracle_attention_backward_qk.restype = ctypes.c_int
    lib.oracle_attention_backward_rows_qk.argtypes = [d, d, d, d, i64, i64, i64, i64, ctypes.c_int,
                                                      ctypes.c_double, pi64, i64, pi64, i64,
                                                      d, d, d, ctypes.c_int]
    lib.oracle_attention_backward_rows_qk.restype = ctypes.c_int
    lib.oracle_default_threads.restype = ctypes.c_int
    return lib


def _load():
    global _lib
    with _lock:
        if _lib is None:
            _lib = _bind(ctypes.CDLL(build()))
    return _lib


_override = threading.local()


def _active():
    lib = getattr(_override, "lib", None)
    return lib if lib is not None else _load()


class use_library:
    """Context manager: route this thread's oracle calls to another build of the
    same source (the mutation tests plant mistakes in a copy and check that the
    pins catch them)."""

    def __init__(self, path: str):
        self.lib = _bind(ctypes.CDLL(path))

    def __enter__(self):
        self.prev = getattr(_override, "lib", None)
        _override.lib = self.lib
        return self

    def __exit__(self, *exc):
        _override.lib = self.prev
        return False


def default_threads() -> int:
    return int(_active().oracle_default_threads())


def _f64(x) -> np.ndarray:
    """fp64 contiguous view; uint16 arrays are read as bf16 bit patterns and widened exactly."""
    x = np.asarray(x)
    if x.dtype == np.uint16:
        x = (x.astype(np.uint32) << np.uint32(16)).view(np.float32)
    return np.ascontiguousarray(x, dtype=np.float64)


def _ptr(a: np.ndarray, ctype=ctypes.c_double):
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def _heads(x: np.ndarray):
    """[..., N, d] -> ([n_heads, N, d] fp64, leading shape)."""
    x = _f64(x)
    lead = x.shape[:-2]
    return np.ascontiguousarray(x.reshape(-1, x.shape[-2], x.shape[-1])), lead


def attention_forward(q, k, v, causal: bool, scale: float, rows=None, nthreads: int = 0):
    """O and LSE of standard attention. q: [..., Nq, d], k, v: [..., Nk, d] (fp64 or
    bf16 bits); causal masking is aligned to the bottom-right corner (query i sees
    keys j <= i + Nk - Nq).

    Returns (o [..., R, d], lse [..., R]) with R = len(rows) or Nq.
    """
    qh, lead = _heads(q)
    kh, _ = _heads(k)
    vh, _ = _heads(v)
    nh, N, d = qh.shape
    Nk = kh.shape[1]
    if rows is None:
        rp, R = None, N
    else:
        rows_a = np.ascontiguousarray(rows, dtype=np.int64)
        rp, R = _ptr(rows_a, ctypes.c_int64), rows_a.size
    o = np.empty((nh, R, d))
    lse = np.empty((nh, R))
    rc = _active().oracle_attention_forward_qk(_ptr(qh), _ptr(kh), _ptr(vh), nh, N, Nk, d,
                                             int(causal), float(scale), rp, R, _ptr(o), _ptr(lse),
                                             int(nthreads))
    if rc != 0:
        raise ValueError("oracle_attention_forward rejected its arguments")
    return o.reshape(*lead, R, d), lse.reshape(*lead, R)


def attention_backward(q, k, v, dout, causal: bool, scale: float, nthreads: int = 0):
    """Full backward. Returns dict with o, lse, dq, dk, dv (fp64; o, lse, dq shaped
    like q, dk and dv like k)."""
    qh, lead = _heads(q)
    kh, _ = _heads(k)
    vh, _ = _heads(v)
    dh, _ = _heads(dout)
    nh, N, d = qh.shape
    Nk = kh.shape[1]
    out = {name: np.empty((nh, N, d)) for name in ("o", "dq")}
    out.update({name: np.empty((nh, Nk, d)) for name in ("dk", "dv")})
    out["lse"] = np.empty((nh, N))
    rc = _active().oracle_attention_backward_qk(_ptr(qh), _ptr(kh), _ptr(vh), _ptr(dh), nh, N, Nk,
                                              d, int(causal), float(scale), _ptr(out["o"]),
                                              _ptr(out["lse"]), _ptr(out["dq"]), _ptr(out["dk"]),
                                              _ptr(out["dv"]), int(nthreads))
    if rc != 0:
        raise ValueError("oracle_attention_backward rejected its arguments")
    res = {name: out[name].reshape(*lead, N, d) for name in ("o", "dq")}
    res.update({name: out[name].reshape(*lead, Nk, d) for name in ("dk", "dv")})
    res["lse"] = out["lse"].reshape(*lead, N)
    return res


def attention_backward_rows(q, k, v, dout, causal: bool, scale: float, qrows, krows,
                            nthreads: int = 0):
    """dQ at query rows qrows and dK, dV at key rows krows of every head given.

    Returns (dq [..., len(qrows), d], dk [..., len(krows), d], dv [..., len(krows), d]).
    """
    qh, lead = _heads(q)
    kh, _ = _heads(k)
    vh, _ = _heads(v)
    dh, _ = _heads(dout)
    nh, N, d = qh.shape
    Nk = kh.shape[1]
    qr = np.ascontiguousarray(qrows, dtype=np.int64)
    kr = np.ascontiguousarray(krows, dtype=np.int64)
    dq = np.empty((nh, qr.size, d))
    dk = np.empty((nh, kr.size, d))
    dv = np.empty((nh, kr.size, d))
    rc = _active().oracle_attention_backward_rows_qk(
        _ptr(qh), _ptr(kh), _ptr(vh), _ptr(dh), nh, N, Nk, d, int(causal), float(scale),
        _ptr(qr, ctypes.c_int64), qr.size, _ptr(kr, ctypes.c_int64), kr.size,
        _ptr(dq), _ptr(dk), _ptr(dv), int(nthreads))
    if rc != 0:
        raise ValueError("oracle_attention_backward_rows rejected its arguments")
    return (dq.reshape(*lead, qr.size, d), dk.reshape(*lead, kr.size, d),
            dv.reshape(*lead, kr.size, d))
