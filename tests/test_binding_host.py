"""The Python binding on the host, without a GPU: every fa2_* function checks its
tensor arguments (CUDA, contiguous, dtype, shape, on the current device) before
anything reaches the library, and marshals valid arguments into the C call of the
same name in the documented order. The library is replaced by a recorder, so
nothing is launched; the tensors are stand-ins that carry only what the binding
reads (shape, dtype, device, layout, address)."""
import ctypes
import math

import pytest
import torch

import exact_tiled_attention_30_b200 as fa2

B, H, N, NK, D = 2, 3, 200, 330, 64


class FakeCuda:
    """Stands in for a CUDA tensor: only what the binding reads."""

    _next = 0x100000

    def __init__(self, shape, dtype=torch.bfloat16, index=0, contiguous=True):
        self.shape = torch.Size(shape)
        self.dtype = dtype
        self.is_cuda = True
        self.device = torch.device("cuda", index)
        self._contiguous = contiguous
        FakeCuda._next += 0x100000
        self._ptr = FakeCuda._next

    def is_contiguous(self):
        return self._contiguous

    def dim(self):
        return len(self.shape)

    def data_ptr(self):
        return self._ptr

    def numel(self):
        return math.prod(self.shape)

    def element_size(self):
        return torch.empty((), dtype=self.dtype).element_size()


class Recorder:
    """Replaces the ctypes library: records (entry point, arguments)."""

    def __init__(self):
        self.calls = []

    def __getattr__(self, name):
        if not name.startswith("fa2_"):
            raise AttributeError(name)
        calls = self.calls

        def fn(*args):
            calls.append((name, args))
            return 0

        fn.restype, fn.argtypes = ctypes.c_int, []
        return fn


@pytest.fixture
def rec(monkeypatch):
    r = Recorder()
    monkeypatch.setattr(fa2, "load_library", lambda: r)
    monkeypatch.setattr(torch.cuda, "current_device", lambda: 0)
    return r


def tensors(nk=N):
    t = {n: FakeCuda((B, H, N, D)) for n in ("q", "o", "dout", "dq")}
    t.update({n: FakeCuda((B, H, nk, D)) for n in ("k", "v", "dk", "dv")})
    t["lse"] = FakeCuda((B, H, N), torch.float32)
    t["workspace"] = FakeCuda((4096,), torch.uint8)
    return t


# function, its tensor arguments in order, its other arguments, key length
CALLS = {
    "fa2_forward": (["q", "k", "v", "o", "lse"], [True, 0.125], N),
    "fa2_backward": (["q", "k", "v", "o", "lse", "dout", "dq", "dk", "dv"],
                     [True, 0.125, "workspace"], N),
    "fa2_backward_preprocess": (["o", "lse", "dout", "workspace"], [], N),
    "fa2_backward_main": (["q", "k", "v", "dout", "dk", "dv"], [False, 0.125, "workspace"], N),
    "fa2_backward_dq_convert": (["dq"], [0.125, "workspace"], N),
    "fa2_backward_ex": (["q", "k", "v", "o", "lse", "dout", "dq", "dk", "dv"],
                        [True, 0.125, "workspace", fa2.DQ_SEPARATE], N),
    "fa2_backward_main_dkdv": (["q", "k", "v", "dout", "dk", "dv"],
                               [True, 0.125, "workspace"], N),
    "fa2_backward_dq": (["q", "k", "v", "dout", "dq"], [True, 0.125, "workspace"], N),
    "fa2_forward_qk": (["q", "k", "v", "o", "lse"], [True, 0.125], NK),
    "fa2_backward_qk": (["q", "k", "v", "o", "lse", "dout", "dq", "dk", "dv"],
                        [True, 0.125, "workspace"], NK),
    "fa2_backward_noalloc": (["q", "k", "v", "o", "lse", "dout", "dq", "dk", "dv"],
                             [False, 0.125], N),
}


def invoke(name, t):
    names, extra, _ = CALLS[name]
    args = [t[n] for n in names] + [t[x] if isinstance(x, str) else x for x in extra]
    getattr(fa2, name)(*args, stream=7)


@pytest.mark.parametrize("name", sorted(CALLS))
def test_valid_arguments_are_marshalled_in_order(rec, name):
    names, extra, nk = CALLS[name]
    t = tensors(nk)
    invoke(name, t)
    assert len(rec.calls) == 1
    called, args = rec.calls[0]
    assert called == name
    ptrs = [t[n].data_ptr() for n in names if n != "workspace"]
    assert list(args[:len(ptrs)]) == ptrs
    assert args[-1] == 7  # the stream goes last
    sizes = list(args[len(ptrs):len(ptrs) + 5])
    if name.endswith("_qk"):
        assert sizes == [B, H, N, NK, D]
    elif name == "fa2_backward_preprocess":
        assert sizes[:4] == [B, H, N, D]
    else:
        assert sizes[:4] == [B, H, N, D]
    if "workspace" in names or "workspace" in extra:
        ws = t["workspace"]
        assert ws.data_ptr() in args and ws.numel() in args
    if True in extra or False in extra:
        causal = True in extra
        assert int(causal) in args[len(ptrs) + 4:len(ptrs) + 6]


def lse_takers():
    return sorted(n for n, (names, _, _) in CALLS.items() if "lse" in names)


@pytest.mark.parametrize("name", lse_takers())
def test_lse_of_the_wrong_length_is_rejected(rec, name):
    t = tensors(CALLS[name][2])
    t["lse"] = FakeCuda((B, H, N - 1), torch.float32)
    with pytest.raises(ValueError, match="lse"):
        invoke(name, t)
    assert rec.calls == []


@pytest.mark.parametrize("name", sorted(CALLS))
def test_tensor_on_another_device_is_rejected(rec, name):
    names = CALLS[name][0]
    for victim in names:
        t = tensors(CALLS[name][2])
        old = t[victim]
        t[victim] = FakeCuda(old.shape, old.dtype, index=1)
        with pytest.raises(ValueError, match="current device"):
            invoke(name, t)
    assert rec.calls == []


@pytest.mark.parametrize("name", sorted(CALLS))
def test_wrong_dtype_layout_or_shape_is_rejected(rec, name):
    names, _, nk = CALLS[name]
    for victim in (n for n in names if n not in ("workspace",)):
        old = tensors(nk)[victim]
        bad_dtype = torch.float16 if old.dtype == torch.bfloat16 else torch.float64
        wrong_rows = list(old.shape)
        wrong_rows[2] += 1
        for bad in (FakeCuda(old.shape, bad_dtype), FakeCuda(old.shape, old.dtype, contiguous=False),
                    FakeCuda(wrong_rows, old.dtype)):
            t = tensors(nk)
            t[victim] = bad
            if victim == names[0] and bad.shape != old.shape:
                continue  # the first tensor defines B, H, N, d
            with pytest.raises(ValueError):
                invoke(name, t)
    assert rec.calls == []


def test_host_buffer_entry_checks_its_tensors(rec):
    host = {n: torch.empty((B, H, N, D), dtype=torch.bfloat16)
            for n in ("q", "k", "v", "dout", "o", "dq", "dk", "dv")}
    lse = torch.empty((B, H, N), dtype=torch.float32)
    ws = FakeCuda((1 << 20,), torch.uint8)
    args = [host[n] for n in ("q", "k", "v", "dout", "o")] + [lse] + \
        [host[n] for n in ("dq", "dk", "dv")]
    fa2.fa2_forward_backward_host(*args, True, 0.125, ws, 4, stream=7)
    (called, cargs), = rec.calls
    assert called == "fa2_forward_backward_host"
    assert list(cargs[9:13]) == [B, H, N, D] and cargs[-1] == 7
    assert ws.data_ptr() in cargs and ws.numel() in cargs
    bad_lse = torch.empty((B, H, N + 1), dtype=torch.float32)
    with pytest.raises(ValueError, match="lse"):
        fa2.fa2_forward_backward_host(*args[:5], bad_lse, *args[6:], True, 0.125, ws, 4, stream=7)
    with pytest.raises(ValueError, match="current device"):
        fa2.fa2_forward_backward_host(*args, True, 0.125, FakeCuda((1 << 20,), torch.uint8, 1), 4,
                                      stream=7)
    assert len(rec.calls) == 1
