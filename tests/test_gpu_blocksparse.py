"""GPU parity of block-sparse attention on given block lists (through the C
ABI) with the oracle's attention on the same selected set in sparse mode.

The GPU side builds its BigBird lists with the library's generator, the
oracle side with the oracle's; arbitrary block sets (empty rows, full rows
that span several work items, heads of different sizes) come from a seeded
generator.  Tolerances are the forward pass's: max-abs 2e-2 for bf16 inputs,
1e-4 for fp32 inputs.
"""
import numpy as np
import pytest
import torch

import mra_testlib as tl
import oracle
import resolution_block_sparse_b200 as mra
from resolution_block_sparse_b200._binding import MRA_DEV_COUNT
from resolution_block_sparse_b200.workloads import BIGBIRD, bigbird_random_blocks, random_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    mra.load_library()
    mra.mra_get_device_status()
    yield


def _pad_lists(lists, fill):
    cap = max(1, max(len(x) for x in lists))
    arr = np.full((len(lists), cap), fill, dtype=np.int32)
    for i, x in enumerate(lists):
        arr[i, :len(x)] = x
        if fill != -1 and len(x) < cap and len(x) > 0:
            arr[i, len(x):] = x[0]       # the oracle counts a repeated block once
    return arr


def _run(inputs, gpu_lists, ora_lists, *, skip_heads=()):
    q, k, v, mask = (inputs[x] for x in ("q", "k", "v", "mask"))
    B, H, N, D = q.shape
    dev = torch.device("cuda:0")
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    md = None if mask is None else mask.to(dev)
    out = torch.zeros_like(qd)
    idx = torch.from_numpy(_pad_lists(gpu_lists, -1)).to(dev)
    mra.mra_blocksparse_attention_fwd(qd, kd, vd, md, out, idx)
    torch.cuda.synchronize()
    # list kernel and attention, plus the group plan when the tcgen05 kernel runs
    assert mra.mra_last_launch_count() in (2, 3)
    status = mra.mra_get_device_status()
    got = out.float().cpu().numpy()
    want = oracle.attend_with_selection(q.double().numpy(), k.double().numpy(), v.double().numpy(),
                                        None if mask is None else mask.double().numpy(),
                                        _pad_lists(ora_lists, 0), approx_mode=1)
    got = got.reshape(B * H, N, D)
    want = want.reshape(B * H, N, D)
    keep = [h for h in range(B * H) if h not in skip_heads]
    err = float(np.max(np.abs(got[keep] - want[keep])))
    assert np.all(np.isfinite(got[keep]))
    assert err <= tl.OUT_TOL[q.dtype], err
    return status, err, got


def _bigbird_lists(BH, N, bs, r, seed):
    rb = bigbird_random_blocks(BH, N // bs, r, seed)
    gpu = [mra.mra_bigbird_block_list(N, bs, rb[h]) for h in range(BH)]
    ora = [oracle.bigbird_blocks(N, bs, rb[h]) for h in range(BH)]
    return gpu, ora


@pytest.mark.parametrize("B,H,N,D,dtype,bs,r,pad", [
    (2, 3, 1024, 64, torch.bfloat16, 64, 3, [0, 70]),
    (1, 2, 768, 32, torch.float32, 32, 1, [45]),
    (1, 2, 256, 64, torch.bfloat16, 64, 1, None),       # 4 blocks: full attention
    (1, 2, 2048, 64, torch.float32, 128, 2, [0]),       # 4x4 sub-blocks per BigBird block
    (2, 1, 4096, 32, torch.bfloat16, 64, 3, [1000, 3]),
])
def test_bigbird_parity(B, H, N, D, dtype, bs, r, pad):
    inputs = random_inputs(B, H, N, D, dtype=dtype, seed=300 + N + D, pad_tokens=pad)
    gpu, ora = _bigbird_lists(B * H, N, bs, r, seed=400 + N)
    status, err, _ = _run(inputs, gpu, ora)
    assert status == 0
    print(f"bigbird N={N} D={D} {dtype}: max-abs {err:.3e}")


def test_bigbird_workload_parity():
    w = BIGBIRD
    inputs = random_inputs(w.B, w.H, w.N, w.D, dtype=torch.bfloat16, seed=w.seed)
    gpu, ora = _bigbird_lists(w.B * w.H, w.N, w.block_size, w.num_random, w.seed)
    status, err, _ = _run(inputs, gpu, ora)
    assert status == 0
    print(f"{w.name}: max-abs {err:.3e}")


def _random_sets(BH, nbr, seed, p):
    rng = np.random.default_rng(seed)
    out = []
    for h in range(BH):
        m = rng.random((nbr, nbr)) < p[h % len(p)]
        m[h % nbr, :] = h % 2 == 0          # a full row in even heads, an empty one in odd heads
        out.append(np.flatnonzero(m.ravel()).astype(np.int32))
    return out


@pytest.mark.parametrize("B,H,N,D,dtype,p,pad", [
    (1, 4, 2048, 64, torch.bfloat16, [0.05, 0.3, 0.002, 0.9], [77]),
    (2, 2, 640, 32, torch.float32, [0.2, 0.5], [0, 200]),
    (1, 2, 1024, 64, torch.float32, [1.0, 0.0], None),   # every block / no block but one row
])
def test_arbitrary_block_sets(B, H, N, D, dtype, p, pad):
    inputs = random_inputs(B, H, N, D, dtype=dtype, seed=500 + N, pad_tokens=pad)
    sets = _random_sets(B * H, N // 32, 600 + N, p)
    empty = [h for h, s in enumerate(sets) if len(s) == 0]
    status, err, got = _run(inputs, sets, [s if len(s) else np.array([0], np.int32) for s in sets],
                            skip_heads=empty)
    assert status == 0
    for h in empty:                         # no key set anywhere: the output is 0
        assert np.all(got[h] == 0.0)


def test_invalid_list_flags_its_head_only():
    B, H, N, D = 1, 3, 512, 64
    inputs = random_inputs(B, H, N, D, dtype=torch.bfloat16, seed=700)
    gpu, ora = _bigbird_lists(B * H, N, 64, 1, seed=701)
    bad = gpu[1].copy()
    bad[[3, 4]] = bad[[4, 3]]                 # not ascending
    status, _, _ = _run(inputs, [gpu[0], bad, gpu[2]], ora, skip_heads=[1])
    assert status == MRA_DEV_COUNT
