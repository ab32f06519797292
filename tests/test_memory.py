"""Memory is linear in the sequence length.

The reproduction page of the FlashAttention-2 paper notes, in its benchmark
figure captions, that standard PyTorch attention runs out of memory at 16k
tokens: it stores the N x N score and probability matrices. The tiled method
keeps them on chip, so what it holds in device memory grows like B*H*N*d. These
tests check that for this library: the backward workspace is an exact linear
function of N (CPU), and at the 16k-token benchmark configuration a forward and
backward allocate no device memory beyond the caller's inputs, outputs and that
workspace (GPU).
"""
import math

import pytest

A = 0x10000


def _lib():
    import exact_tiled_attention_30_b200 as m

    return m.load_library()


@pytest.mark.parametrize("d", [64, 128])
def test_workspace_is_linear_in_n(d):
    lib = _lib()
    B, H = 2, 3
    ws = {N: lib.fa2_backward_workspace_size(B, H, N, d) for N in (128, 256, 1024, 16384, 65536)}
    per_row = ws[256] - ws[128]
    # fp32 dQ accumulator (4 d bytes), D and LSE * log2 e (4 bytes each) per row of
    # every head, plus a 16-byte work counter
    assert per_row == B * H * 128 * (4 * d + 8)
    for N, size in ws.items():
        assert size == (N // 128) * per_row + 16
    # ragged lengths round up to the 128-row tile
    assert lib.fa2_backward_workspace_size(B, H, 1000, d) == ws[1024]
    # far below one N x N fp32 score matrix per head at 16k tokens
    assert ws[16384] * 100 < B * H * 16384 * 16384 * 4


def test_host_entry_workspace_does_not_grow_with_n_squared():
    lib = _lib()
    small = lib.fa2_forward_backward_host_workspace_size(1, 16, 4096, 128, 2)
    big = lib.fa2_forward_backward_host_workspace_size(1, 16, 16384, 128, 2)
    assert big == pytest.approx(4 * small, rel=1e-3)


@pytest.mark.gpu
def test_no_device_allocation_at_16k_tokens():
    """B=1 H=16 N=16384 d=128 causal: the library never allocates, so device free
    memory does not move across a forward + backward, and everything torch holds
    is the caller's inputs, outputs and workspace (~0.7 GB, against the 17 GB
    that one fp32 score matrix per head would take)."""
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import exact_tiled_attention_30_b200 as fa2

    fa2.load_library()
    B, H, N, d = 1, 16, 16384, 128
    scale = 1.0 / math.sqrt(d)
    g = torch.Generator(device="cuda").manual_seed(5)
    q, k, v, do = (torch.randn(B, H, N, d, device="cuda", dtype=torch.bfloat16, generator=g)
                   for _ in range(4))
    o, dq, dk, dv = (torch.empty_like(q) for _ in range(4))
    lse = torch.empty(B, H, N, device="cuda", dtype=torch.float32)
    ws = torch.empty(fa2.fa2_backward_workspace_size(B, H, N, d), dtype=torch.uint8, device="cuda")
    # first calls: one-time set-up (module load, kernel attributes)
    fa2.fa2_forward(q, k, v, o, lse, True, scale)
    fa2.fa2_backward(q, k, v, o, lse, do, dq, dk, dv, True, scale, ws)
    torch.cuda.synchronize()
    torch.cuda.reset_peak_memory_stats()
    held = torch.cuda.memory_allocated()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(3):
        fa2.fa2_forward(q, k, v, o, lse, True, scale)
        fa2.fa2_backward(q, k, v, o, lse, do, dq, dk, dv, True, scale, ws)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0, f"device free memory moved by {free0 - free1} bytes"
    assert torch.cuda.max_memory_allocated() == held
    tensors = 8 * B * H * N * d * 2 + B * H * N * 4 + ws.numel()
    assert held >= tensors and held < tensors + (64 << 20)
    assert held * 20 < B * H * N * N * 4
    st, site = fa2.fa2_get_device_status()
    assert st == 0, f"device status {fa2.fa2_status_string(st)} at site {site:#x}"
