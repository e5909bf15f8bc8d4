"""The entry point for callers that cannot allocate device memory.

mra_attention_fwd_noalloc serves code that must not call cudaMalloc (a host
framework's caching allocator owns the device, a plugin may not allocate, or
an allocation could block or fail mid-stream).  It keeps all scratch in one
static 16 MiB device array.  These tests call it through the C ABI and check
its output against mra_attention_fwd on the same inputs, on two calls in a
row (the second call finds the first call's leftovers in the shared array).
This file is named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

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
@pytest.mark.parametrize("mode,first_n,diag_n,pad", [(0, 1, 1, [0, 50]), (1, 2, 3, [17, 0])])
def test_noalloc_matches_allocating_entry_point_twice(mode, first_n, diag_n, pad):
    assert torch.cuda.is_available()
    dev = torch.device("cuda:0")
    B, H, N, D, bpr = 2, 2, 1024, 64, 4
    outs = []
    for call, seed in enumerate((11, 12)):          # two calls in a row, different inputs
        d = random_inputs(B, H, N, D, dtype=torch.bfloat16, seed=seed, pad_tokens=pad)
        q, k, v = (d[x].to(dev) for x in ("q", "k", "v"))
        mask = d["mask"].to(dev)
        ref = torch.empty_like(q)
        mra.mra_attention_fwd(q, k, v, mask, ref, bpr, mode, first_n, diag_n)
        got = torch.full_like(q, float("nan"))
        mra.mra_attention_fwd_noalloc(q, k, v, mask, got, bpr, mode, first_n, diag_n)
        torch.cuda.synchronize()
        g = got.float().cpu().numpy()
        r = ref.float().cpu().numpy()
        assert np.all(np.isfinite(g)), f"call {call}: non-finite output"
        err = float(np.max(np.abs(g - r)))
        assert err <= BF16_TOL, f"call {call}: max-abs difference {err}"
        outs.append(g)
    assert not np.array_equal(outs[0], outs[1])


@pytest.mark.gpu
def test_noalloc_rejects_too_large_on_gpu():
    dev = torch.device("cuda:0")
    q = torch.zeros(2, 12, 4096, 64, dtype=torch.bfloat16, device=dev)
    with pytest.raises(mra.MraError) as e:
        mra.mra_attention_fwd_noalloc(q, q, q, None, torch.empty_like(q), 4, 1, 2, 3)
    assert e.value.status == _binding.MRA_ERR_TOO_LARGE
