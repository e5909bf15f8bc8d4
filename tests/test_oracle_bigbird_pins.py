"""Pins of the oracle's BigBird block pattern and of block-sparse attention on
a given block set.

Page "Transformers 中的 BigBird：面向超长序列的稀疏注意力模型完全指南": window
of 3 blocks, 2 global blocks, num_random_blocks >= 1 random blocks, full
attention for sequences of at most (5 + 2 * num_random_blocks) blocks.  The
pattern is checked by counting against its definition on every row, and the
attention on the pattern against torch's SDPA in fp64 with the same boolean
token mask (a library routine on the dense restatement).
"""
import numpy as np
import pytest
import torch

import oracle
from resolution_block_sparse_b200.workloads import random_inputs


def _rand(nb, r, seed):
    return np.random.default_rng(seed).integers(0, nb, size=(nb, r))


@pytest.mark.parametrize("N,bs,r", [(2048, 64, 3), (4096, 64, 2), (2048, 128, 1), (1024, 32, 2)])
def test_pattern_rows_by_definition(N, bs, r):
    nb = N // bs
    rb = _rand(nb, r, N + r)
    flat = oracle.bigbird_blocks(N, bs, rb)
    nbr = N // 32
    assert np.all(np.diff(flat) > 0)
    sel = np.zeros(nbr * nbr, bool)
    sel[flat] = True
    sel = sel.reshape(nbr, nbr)
    f = bs // 32
    coarse = sel[::f, ::f]
    # every 32-block inside one block_size block carries the coarse decision
    assert np.array_equal(np.kron(coarse, np.ones((f, f), bool)), sel)
    for i in range(nb):
        row = set(np.flatnonzero(coarse[i]))
        if i in (0, nb - 1):
            assert row == set(range(nb))                 # global rows attend to everything
            continue
        want = {0, nb - 1} | {j for j in (i - 1, i, i + 1) if 0 <= j < nb} | set(int(x) for x in rb[i])
        assert row == want
    assert coarse[:, 0].all() and coarse[:, nb - 1].all()   # everyone attends to the global blocks


def test_short_sequences_use_full_attention():
    bs, r = 64, 3
    nb = 5 + 2 * r
    flat = oracle.bigbird_blocks(nb * bs, bs, _rand(nb, r, 1))
    nbr = nb * bs // 32
    assert len(flat) == nbr * nbr
    flat = oracle.bigbird_blocks((nb + 1) * bs, bs, _rand(nb + 1, r, 2))
    assert len(flat) < ((nb + 1) * bs // 32) ** 2


def test_invalid_pattern_arguments():
    with pytest.raises(ValueError):
        oracle.bigbird_blocks(2048, 48, _rand(40, 2, 3))
    with pytest.raises(ValueError):
        oracle.bigbird_blocks(2048, 64, np.zeros((32, 0), int))
    with pytest.raises(ValueError):
        oracle.bigbird_blocks(2048, 64, np.full((32, 2), 32))


@pytest.mark.parametrize("pad", [None, [0, 100]])
def test_attention_on_pattern_equals_masked_dense(pad):
    B, H, N, D, bs, r = 2, 2, 1024, 16, 64, 2
    d = random_inputs(B, H, N, D, seed=91, pad_tokens=pad)
    nb = N // bs
    sels = [oracle.bigbird_blocks(N, bs, _rand(nb, r, 100 + h)) for h in range(B * H)]
    kmax = max(len(s_) for s_ in sels)
    # attend_with_selection takes a common count: pad each list with its own last index
    sel = np.stack([np.concatenate([s_, np.full(kmax - len(s_), s_[-1], np.int32)]) for s_ in sels])
    out = oracle.attend_with_selection(d["q"], d["k"], d["v"], d["mask"], sel, approx_mode=1)
    nbr = N // 32
    q, kk, v = (d[x].double() for x in ("q", "k", "v"))
    for bh in range(B * H):
        b, h = divmod(bh, H)
        blk = np.zeros(nbr * nbr, bool)
        blk[sels[bh]] = True
        tok = torch.as_tensor(np.kron(blk.reshape(nbr, nbr), np.ones((32, 32), bool)))
        if d["mask"] is not None:
            tok = tok & (d["mask"][b] > 0)[None, :]
        ref = torch.nn.functional.scaled_dot_product_attention(q[b, h], kk[b, h], v[b, h], attn_mask=tok)
        ref = torch.nan_to_num(ref, nan=0.0)
        if d["mask"] is not None:
            ref = ref * (d["mask"][b] > 0)[:, None]
        np.testing.assert_allclose(out[b, h], ref.numpy(), rtol=0, atol=1e-12)


def _golden_counts():
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "bigbird_keys_per_query.txt")
    rows = []
    for line in open(path):
        line = line.strip()
        if line and not line.startswith("#"):
            rows.append(tuple(int(x) for x in line.split()))
    return rows


@pytest.mark.parametrize("N,bs,r,g_keys,w_keys,r_keys,total", _golden_counts())
def test_keys_per_query_match_the_pages_count(N, bs, r, g_keys, w_keys, r_keys, total):
    """A middle block whose random blocks avoid its window and the global
    blocks attends to exactly the page's global + window + random keys."""
    nb = N // bs
    i = nb // 2
    rb = _rand(nb, r, 5)
    avoid = {0, nb - 1, i - 1, i, i + 1}
    free = [j for j in range(nb) if j not in avoid]
    rb[i] = free[:r]                      # distinct, outside window and globals
    flat = oracle.bigbird_blocks(N, bs, rb)
    nbr = N // 32
    f = bs // 32
    row = (i * f) * nbr                   # first 32-token row of block i
    cols = flat[(flat >= row) & (flat < row + nbr)] % nbr
    assert g_keys + w_keys + r_keys == total
    assert len(cols) * 32 == total
    # and a global row attends to the whole sequence
    cols0 = flat[flat < nbr] % nbr
    assert len(cols0) * 32 == N
