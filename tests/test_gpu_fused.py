"""GPU parity of the single-launch forward pass for maps of at most 16 x 16
blocks (one CTA per (batch, head) does the whole pass; MRA_FUSED=1 forces it
wherever it fits), and of the multi-kernel path on the same cases
(MRA_FUSED=0), both against the oracle with the intermediates (pooled means,
low-resolution logits, selection)."""
import os

import numpy as np
import pytest
import torch

import mra_testlib as tl
import resolution_block_sparse_b200 as mra
from resolution_block_sparse_b200.workloads import WORKLOADS, make_inputs, random_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    mra.load_library()
    yield


@pytest.fixture
def multi_kernel():
    os.environ["MRA_FUSED"] = "0"
    yield
    del os.environ["MRA_FUSED"]


@pytest.fixture
def fused():
    os.environ["MRA_FUSED"] = "1"
    yield
    del os.environ["MRA_FUSED"]


CASES = [
    # (B, H, N, D, dtype, bpr, mode, first_n, diag_n, pad_tokens)
    (1, 1, 32, 64, torch.bfloat16, 1, 0, 0, 0, None),          # one block
    (2, 3, 288, 64, torch.bfloat16, 2, 0, 1, 1, [0, 70]),     # ragged mask
    (2, 3, 288, 64, torch.bfloat16, 2, 1, 1, 1, [0, 70]),
    (1, 2, 512, 32, torch.bfloat16, 3, 0, 2, 3, [100]),       # D = 32, 16 blocks
    (2, 2, 512, 64, torch.bfloat16, 16, 0, 0, 0, [0, 33]),    # saturated budget
    (2, 2, 512, 64, torch.bfloat16, 16, 1, 0, 0, [0, 33]),
    (1, 2, 512, 64, torch.bfloat16, 1, 1, 2, 3, None),        # oversubscribed priors
    (2, 1, 256, 64, torch.bfloat16, 2, 0, 0, 0, [256, 0]),    # fully padded sequence
    (1, 2, 320, 32, torch.float32, 2, 0, 1, 1, [40]),         # fp32
    (1, 2, 256, 64, torch.float32, 2, 1, 1, 2, [40]),
    (1, 2, 512, 32, torch.float32, 4, 0, 0, 0, None),
]


def _check(case):
    B, H, N, D, dtype, bpr, mode, f, g, pad = case
    inputs = random_inputs(B, H, N, D, dtype=dtype, seed=900 + N + bpr, pad_tokens=pad, v_scale=1.0)
    kw = dict(block_per_row=bpr, approx_mode=mode, first_n=f, diag_n=g)
    gpu = tl.run_gpu(inputs, **kw)
    launches = mra.mra_last_launch_count()
    tl.compare(inputs, gpu, tl.run_oracle(inputs, **kw))
    return gpu, launches


@pytest.mark.parametrize("case", CASES, ids=[f"c{i}" for i in range(len(CASES))])
def test_fused_parity(case, fused):
    _, launches = _check(case)
    assert launches == 1


@pytest.mark.parametrize("case", CASES, ids=[f"c{i}" for i in range(len(CASES))])
def test_multi_kernel_parity_on_small_maps(case, multi_kernel):
    _, launches = _check(case)
    assert launches >= 3


@pytest.mark.parametrize("index,launches", [(1, 4), (2, 1)])
def test_small_workloads_path_choice(index, launches):
    """By default the single-launch pass runs where it is faster: bf16 with at
    least 64 heads (N=512 x 96 heads); the two-head fp32 case keeps the
    multi-kernel path."""
    w = WORKLOADS[index]
    inputs = make_inputs(w)
    kw = dict(block_per_row=w.block_per_row, approx_mode=w.approx_mode, first_n=w.first_n, diag_n=w.diag_n)
    gpu = tl.run_gpu(inputs, **kw)
    assert mra.mra_last_launch_count() == launches
    tl.compare(inputs, gpu, tl.run_oracle(inputs, **kw))
