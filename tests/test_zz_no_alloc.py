"""The entry point for callers that cannot allocate device memory.

mra_attention_fwd_noalloc serves code that must not call cudaMalloc (a host
framework's caching allocator owns the device, a plugin may not allocate, or
an allocation could block or fail mid-stream).  It keeps all scratch in one
static 16 MiB device array.  These tests call it through the C ABI and check
its output against mra_attention_fwd (bit for bit) and the oracle on the same
inputs, on two calls in a row (the second call finds the first call's
leftovers in the shared array), read its status word, and check that a call
allocates no device memory.  This file is named so that pytest collects it
last.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import resolution_block_sparse_b200 as mra
from resolution_block_sparse_b200 import _binding
from resolution_block_sparse_b200.workloads import random_inputs

BF16_TOL = 2e-2   # the bf16 output tolerance of the parity tests


def test_too_large_is_rejected_before_any_launch():
    # aligned fake pointers: the size check fails first, nothing is touched
    lib = mra.load_library()
    fake = ctypes.c_void_p(4096)
    st = lib.mra_attention_fwd_noalloc(fake, fake, fake, None, fake, 2, 12, 4096, 64, 4, 1, 2, 3,
                                       None)
    assert st == _binding.MRA_ERR_TOO_LARGE
    assert "scratch" in mra.mra_status_string(st)


@pytest.mark.gpu
@pytest.mark.parametrize("B,H,N,mode,first_n,diag_n,pad", [
    (2, 2, 1024, 0, 1, 1, [0, 50]),      # pool, cluster selection, attention
    (2, 2, 1024, 1, 2, 3, [17, 0]),
    (8, 8, 256, 0, 1, 1, [0, 40, 0, 0, 96, 0, 0, 0]),   # 64 heads of 8 x 8 blocks: the single-launch pass
])
def test_noalloc_matches_allocating_entry_point_twice(B, H, N, mode, first_n, diag_n, pad):
    """Two calls in a row on different inputs (the second finds the first
    call's leftovers in the shared array): each output equals the allocating
    entry point's bit for bit (same kernels, same inputs), matches the oracle
    within the bf16 tolerance, and the no-allocation status word reads 0."""
    assert torch.cuda.is_available()
    dev = torch.device("cuda:0")
    D, bpr = 64, 4
    outs = []
    for call, seed in enumerate((11, 12)):
        d = random_inputs(B, H, N, D, dtype=torch.bfloat16, seed=seed + N, pad_tokens=pad)
        q, k, v = (d[x].to(dev) for x in ("q", "k", "v"))
        mask = d["mask"].to(dev)
        ref = torch.empty_like(q)
        mra.mra_attention_fwd(q, k, v, mask, ref, bpr, mode, first_n, diag_n)
        got = torch.full_like(q, float("nan"))
        mra.mra_attention_fwd_noalloc(q, k, v, mask, got, bpr, mode, first_n, diag_n)
        torch.cuda.synchronize()
        g = got.float().cpu().numpy()
        assert np.all(np.isfinite(g)), f"call {call}: non-finite output"
        np.testing.assert_array_equal(got.view(torch.int16).cpu().numpy(), ref.view(torch.int16).cpu().numpy(),
                                      err_msg=f"call {call}: differs from mra_attention_fwd")
        want = oracle.forward(d["q"].double().numpy(), d["k"].double().numpy(), d["v"].double().numpy(),
                              d["mask"].double().numpy(), block_per_row=bpr, approx_mode=mode,
                              first_n=first_n, diag_n=diag_n, want_intermediates=False)["out"]
        err = float(np.max(np.abs(g - want)))
        assert err <= BF16_TOL, f"call {call}: max-abs error {err} against the oracle"
        assert mra.mra_get_noalloc_status() == 0
        outs.append(g)
    assert not np.array_equal(outs[0], outs[1])


@pytest.mark.gpu
def test_noalloc_call_allocates_nothing():
    """After a first call on the device (which looks up the array's address),
    a call changes neither the device's free memory nor torch's reserved pool."""
    dev = torch.device("cuda:0")
    d = random_inputs(2, 2, 1024, 64, dtype=torch.bfloat16, seed=21, pad_tokens=[0, 64])
    q, k, v = (d[x].to(dev) for x in ("q", "k", "v"))
    mask = d["mask"].to(dev)
    out = torch.empty_like(q)
    mra.mra_attention_fwd_noalloc(q, k, v, mask, out, 4, 0, 1, 1)
    torch.cuda.synchronize()
    free0, reserved0 = torch.cuda.mem_get_info(dev)[0], torch.cuda.memory_reserved(dev)
    for _ in range(3):
        mra.mra_attention_fwd_noalloc(q, k, v, mask, out, 4, 0, 1, 1)
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info(dev)[0] == free0
    assert torch.cuda.memory_reserved(dev) == reserved0
    assert mra.mra_get_noalloc_status() == 0


@pytest.mark.gpu
def test_noalloc_rejects_too_large_on_gpu():
    dev = torch.device("cuda:0")
    q = torch.zeros(2, 12, 4096, 64, dtype=torch.bfloat16, device=dev)
    with pytest.raises(mra.MraError) as e:
        mra.mra_attention_fwd_noalloc(q, q, q, None, torch.empty_like(q), 4, 1, 2, 3)
    assert e.value.status == _binding.MRA_ERR_TOO_LARGE
