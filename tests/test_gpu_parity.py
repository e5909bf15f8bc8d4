"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Full-size cases are the five seeded workloads (resolution_block_sparse_b200.
workloads); the small cases span several blocks and ragged shapes, and cover
the method's degenerate cases (one block, saturated budget, oversubscribed
priors, fully padded sequences, rows without a selected block).
"""
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


@pytest.mark.parametrize("index", [1, 2, 3, 4, 5])
def test_workload_parity(index):
    w = WORKLOADS[index]
    inputs = make_inputs(w)
    kw = dict(block_per_row=w.block_per_row, approx_mode=w.approx_mode, first_n=w.first_n,
              diag_n=w.diag_n)
    gpu = tl.run_gpu(inputs, **kw)
    ora = tl.run_oracle(inputs, **kw)
    stats = tl.compare(inputs, gpu, ora)
    print(f"workload {index}: {stats}")
    if index == 3:
        # saturated budget: every block of every head selected
        assert gpu["sel"].shape[1] == w.nbr ** 2


SMALL = [
    # (B, H, N, D, dtype, bpr, mode, first_n, diag_n, pad_tokens, scale)
    (1, 1, 32, 64, torch.bfloat16, 1, 0, 0, 0, None, 1.0),          # one block
    (1, 2, 96, 64, torch.bfloat16, 1, 0, 0, 0, None, 1.0),          # 3 blocks, k=3
    (2, 3, 288, 64, torch.bfloat16, 2, 0, 1, 1, [0, 70], 1.0),      # ragged mask
    (2, 3, 288, 64, torch.bfloat16, 2, 1, 1, 1, [0, 70], 1.0),      # same, sparse
    (1, 2, 800, 32, torch.bfloat16, 3, 0, 2, 3, [100], 1.0),        # D=32, 25 blocks
    (1, 2, 800, 32, torch.bfloat16, 3, 1, 2, 3, [100], 1.0),
    (2, 2, 512, 64, torch.bfloat16, 16, 0, 0, 0, [0, 33], 1.0),     # saturated budget
    (2, 2, 512, 64, torch.bfloat16, 16, 1, 0, 0, [0, 33], 1.0),
    (1, 2, 1024, 64, torch.bfloat16, 1, 1, 2, 3, None, 1.0),        # oversubscribed priors
    (1, 2, 1024, 64, torch.bfloat16, 1, 0, 2, 3, None, 1.0),
    (2, 1, 256, 64, torch.bfloat16, 2, 0, 0, 0, [256, 0], 1.0),     # fully padded sequence
    (2, 1, 256, 64, torch.bfloat16, 2, 1, 0, 0, [256, 0], 1.0),
    (1, 2, 2048, 64, torch.bfloat16, 40, 0, 1, 1, None, 1.0),       # long rows: multi-chunk merge
    (1, 2, 2048, 64, torch.bfloat16, 40, 1, 1, 1, None, 1.0),
    (1, 2, 320, 32, torch.float32, 2, 0, 1, 1, [40], 1.0),          # fp32 D=32
    (1, 2, 320, 64, torch.float32, 2, 1, 1, 2, [40], 1.0),          # fp32 D=64
    (1, 2, 1024, 64, torch.float32, 20, 0, 0, 0, None, 1.0),        # fp32 multi-chunk
    (1, 2, 512, 64, torch.bfloat16, 4, 0, 0, 0, None, 3.0),         # peaked scores
    (1, 2, 512, 64, torch.bfloat16, 4, 1, 1, 1, [17], 3.0),
    (1, 1, 8192, 64, torch.bfloat16, 2, 0, 1, 0, None, 1.0),       # 32-item row: grouped merge
    (1, 1, 8192, 64, torch.bfloat16, 2, 1, 1, 0, [300], 1.0),
    (1, 1, 8192, 32, torch.float32, 2, 0, 1, 0, [300], 1.0),
    # 130 x 130 blocks: ragged 64-column tiles of the logit map and of the
    # low-resolution part (rows not 16-byte aligned), 5-word bitmap rows
    (1, 2, 4160, 64, torch.bfloat16, 3, 0, 1, 1, [333], 1.0),
    (1, 2, 4160, 64, torch.bfloat16, 3, 1, 2, 3, [333], 1.0),
    (1, 1, 4160, 32, torch.float32, 3, 0, 1, 1, [70], 1.0),
]


@pytest.mark.parametrize("case", SMALL, ids=[f"c{i}" for i in range(len(SMALL))])
def test_small_parity(case):
    B, H, N, D, dtype, bpr, mode, f, g, pad, scale = case
    # scale sharpens the scores (Q, K); V stays N(0, 1) so that outputs stay
    # in the range the bf16 tolerance is stated for
    inputs = random_inputs(B, H, N, D, dtype=dtype, seed=100 + N + bpr, scale=scale, pad_tokens=pad,
                           v_scale=1.0)
    kw = dict(block_per_row=bpr, approx_mode=mode, first_n=f, diag_n=g)
    gpu = tl.run_gpu(inputs, **kw)
    ora = tl.run_oracle(inputs, **kw)
    tl.compare(inputs, gpu, ora)


def test_fully_padded_sequence_outputs_zero():
    inputs = random_inputs(2, 2, 256, 64, dtype=torch.bfloat16, seed=3, pad_tokens=[256, 10])
    gpu = tl.run_gpu(inputs, block_per_row=2, approx_mode=0)
    assert np.all(gpu["out"][0] == 0.0)
    assert np.all(gpu["out"][1, :, -10:] == 0.0)


def test_plain_entry_points_match_ex():
    w = WORKLOADS[2]
    inputs = make_inputs(w)
    kw = dict(block_per_row=w.block_per_row, approx_mode=w.approx_mode, first_n=w.first_n,
              diag_n=w.diag_n)
    a = tl.run_gpu(inputs, want_intermediates=True, **kw)
    b = tl.run_gpu(inputs, want_intermediates=False, **kw)
    np.testing.assert_array_equal(a["out"], b["out"])   # deterministic, bit-identical


@pytest.mark.parametrize("index", [2, 4])
def test_host_entry_matches_device_entry(index):
    """The host entry computes in chunks of heads; every (batch, head) is
    independent, so its output is bit-identical to the device entry's."""
    w = WORKLOADS[index]
    inputs = make_inputs(w)
    kw = dict(block_per_row=w.block_per_row, approx_mode=w.approx_mode, first_n=w.first_n,
              diag_n=w.diag_n)
    dev = tl.run_gpu(inputs, want_intermediates=False, **kw)
    q, k, v = (inputs[x].pin_memory() for x in ("q", "k", "v"))
    m = None if inputs["mask"] is None else inputs["mask"].pin_memory()
    out = torch.empty_like(q).pin_memory()
    mra.mra_attention_fwd_host(q, k, v, m, out, w.block_per_row, w.approx_mode, w.first_n, w.diag_n)
    np.testing.assert_array_equal(out.float().numpy(), dev["out"])


@pytest.mark.parametrize("B,H,dtype", [(3, 5, torch.bfloat16), (1, 5, torch.float32), (1, 1, torch.bfloat16)])
def test_host_entry_ragged_chunks(B, H, dtype):
    """Head counts that do not divide into equal chunks (3 x 5 heads: chunks
    of 2, 2, 1 per batch entry; 1 x 5: five chunks of 1)."""
    N, D = 640, 64
    inputs = random_inputs(B, H, N, D, dtype=dtype, seed=B * 10 + H, pad_tokens=[37] * B)
    kw = dict(block_per_row=3, approx_mode=0, first_n=1, diag_n=1)
    dev = tl.run_gpu(inputs, want_intermediates=False, **kw)
    q, k, v = (inputs[x].pin_memory() for x in ("q", "k", "v"))
    out = torch.empty_like(q).pin_memory()
    mra.mra_attention_fwd_host(q, k, v, inputs["mask"].pin_memory(), out, 3, 0, 1, 1)
    np.testing.assert_array_equal(out.float().numpy(), dev["out"])
    tl.compare(inputs, dev, tl.run_oracle(inputs, **kw), check_intermediates=False)


def test_workspace_regrows_across_sizes():
    for N in (256, 4096, 512):
        inputs = random_inputs(1, 2, N, 64, dtype=torch.bfloat16, seed=N)
        gpu = tl.run_gpu(inputs, block_per_row=3, approx_mode=0, first_n=1)
        ora = tl.run_oracle(inputs, block_per_row=3, approx_mode=0, first_n=1)
        tl.compare(inputs, gpu, ora)


def test_invalid_arguments_do_not_launch():
    q = torch.zeros(1, 1, 64, 64, dtype=torch.bfloat16, device="cuda")
    out = torch.empty_like(q)
    with pytest.raises(mra.MraError) as e:
        mra.mra_attention_fwd(q[:, :, :48], q[:, :, :48], q[:, :, :48], None, out[:, :, :48], 1, 0, 0, 0)
    assert e.value.status == 1
    q48 = torch.zeros(1, 1, 64, 48, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(mra.MraError) as e:
        mra.mra_attention_fwd(q48, q48, q48, None, torch.empty_like(q48), 1, 0, 0, 0)
    assert e.value.status == 2


@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("N", [4096, 8192])
def test_exact_ties_take_smallest_indices(N, mode):
    """Every token has the same Q and the same K, so every low-resolution logit
    is equal, every key's x is exactly 0 and the keys differ only by the
    priors' tier: the k-th key sits among hundreds of exactly equal keys.  The
    selection takes the equal keys of smallest flat index r * nbr + c, on the
    single-kernel selection (N=4096, 128 x 128 blocks) and on the multi-kernel
    one (N=8192).  Near-tie tolerance does not apply: the sets must be equal."""
    d = random_inputs(1, 2, N, 64, dtype=torch.bfloat16, seed=77 + N + mode, v_scale=1.0)
    base = torch.linspace(-1.0, 1.0, 64)
    d["q"] = base.expand(1, 2, N, 64).to(torch.bfloat16).contiguous()
    d["k"] = (0.5 * base.flip(0)).expand(1, 2, N, 64).to(torch.bfloat16).contiguous()
    kw = dict(block_per_row=2, approx_mode=mode, first_n=1, diag_n=1)
    gpu = tl.run_gpu(d, **kw)
    ora = tl.run_oracle(d, **kw)
    for bh in range(2):
        np.testing.assert_array_equal(gpu["sel"][bh], ora["sel"][bh], err_msg=f"head {bh}")
    tl.compare(d, gpu, ora)
