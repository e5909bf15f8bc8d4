"""Parity of the CUDA backward pass (gradients of the forward output with the
selection held fixed) with the fp64 oracle's backward on the same seeded
inputs: both modes, key masks, priors, D = 32 and 64, fp32 and bf16 inputs,
rows split across work items, and the full-mode low-resolution gradient, on
maps of up to 512 x 512 blocks.

Tolerance (max-abs error over each gradient, relative to max(1, its largest
magnitude)): 1e-4 for fp32 inputs (all arithmetic fp32); 2e-2 for bf16
inputs, whose forward pass (which supplies dout . out for every query) uses
bf16 attention weights in its tensor-core products.
"""
import numpy as np
import pytest
import torch

import oracle
import resolution_block_sparse_b200 as mra
from resolution_block_sparse_b200.workloads import random_inputs

pytestmark = pytest.mark.gpu

CASES = [
    # (B, H, N, D, dtype, bpr, mode, first_n, diag_n, pad)
    (1, 2, 256, 64, torch.float32, 2, 0, 1, 1, [40]),
    (1, 2, 256, 64, torch.float32, 2, 1, 1, 1, [40]),
    (2, 1, 320, 32, torch.float32, 3, 0, 2, 3, [0, 70]),
    (1, 2, 1024, 64, torch.float32, 20, 0, 0, 0, None),        # rows split across work items
    (2, 2, 512, 64, torch.bfloat16, 4, 0, 1, 1, [0, 33]),
    (2, 2, 512, 64, torch.bfloat16, 4, 1, 1, 1, [0, 33]),
    (1, 2, 2048, 64, torch.bfloat16, 40, 1, 1, 1, None),       # 2-item rows
    (1, 1, 4096, 64, torch.bfloat16, 4, 1, 2, 3, None),        # 16-item first-n rows
    (2, 1, 256, 64, torch.bfloat16, 2, 0, 0, 0, [256, 10]),    # a fully padded sequence
    (1, 2, 512, 64, torch.float32, 16, 0, 0, 0, [17]),         # saturated budget
    # maps above 128 x 128 blocks: the multi-kernel selection and the
    # low-resolution gradient over long rows of unselected blocks
    (1, 1, 8192, 64, torch.bfloat16, 4, 0, 1, 1, None),        # 256 x 256 blocks, full mode
    (1, 1, 8192, 32, torch.float32, 2, 0, 2, 3, [300]),        # fp32, padded, 256 x 256
    (1, 1, 16384, 64, torch.bfloat16, 8, 0, 1, 1, [500]),      # 512 x 512 blocks, full mode
    # 130 x 130 blocks: ragged last 64 x 64 pair tile in both directions
    (1, 2, 4160, 64, torch.bfloat16, 3, 0, 1, 1, [333]),
    (1, 1, 4160, 32, torch.float32, 3, 0, 2, 3, [70]),
]


@pytest.mark.parametrize("case", CASES, ids=[f"c{i}" for i in range(len(CASES))])
def test_backward_parity(case):
    B, H, N, D, dtype, bpr, mode, f, g, pad = case
    d = random_inputs(B, H, N, D, dtype=dtype, seed=700 + N + bpr, pad_tokens=pad, v_scale=1.0)
    dout = random_inputs(B, H, N, D, dtype=dtype, seed=800 + N)["q"]
    kw = dict(block_per_row=bpr, approx_mode=mode, first_n=f, diag_n=g)
    dev = torch.device("cuda")
    q, k, v, go = (x.to(dev) for x in (d["q"], d["k"], d["v"], dout))
    m = None if d["mask"] is None else d["mask"].to(dev)
    dq = torch.empty(B, H, N, D, dtype=torch.float32, device=dev)
    dk = torch.empty_like(dq)
    dv = torch.empty_like(dq)
    mra.mra_attention_bwd(q, k, v, m, go, dq, dk, dv, bpr, mode, f, g)
    torch.cuda.synchronize()
    assert mra.mra_get_device_status() == 0
    wide = [x.double() for x in (d["q"], d["k"], d["v"], dout)]   # exact widening of the input bytes
    ref = oracle.backward(wide[0], wide[1], wide[2], d["mask"], wide[3], **kw)
    tol = 1e-4 if dtype == torch.float32 else 2e-2
    for name, got, want in zip(("dq", "dk", "dv"), (dq, dk, dv), ref):
        got = got.cpu().double().numpy()
        err = np.abs(got - want).max()
        scale = max(1.0, np.abs(want).max())
        assert err <= tol * scale, f"{name}: max-abs error {err:.3e} > {tol} x {scale:.3f}"


def test_backward_rejects_misaligned_gradients():
    d = random_inputs(1, 1, 64, 64, dtype=torch.bfloat16, seed=1)
    dev = torch.device("cuda")
    q, k, v = (d[x].to(dev) for x in ("q", "k", "v"))
    buf = torch.empty(1 * 64 * 64 + 4, dtype=torch.float32, device=dev)
    dq = buf[1:1 + 64 * 64].view(1, 1, 64, 64)       # 4-byte offset: not 16-byte aligned
    dk = torch.empty(1, 1, 64, 64, dtype=torch.float32, device=dev)
    with pytest.raises(mra.MraError):
        mra.mra_attention_bwd(q, k, v, None, q, dq, dk, dk, 1, 0, 0, 0)
