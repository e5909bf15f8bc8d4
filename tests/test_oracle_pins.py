"""Pins of the CPU oracle against what the MRA page and the mathematics fix.

Source: "深入解析 Transformers 中的 MRA 模型" (blog.gitcode.com), sections
"MraConfig：四个专属参数与完整默认值" and "源码级原理：MRA 两级注意力到底怎么算".
None of these tests compares the oracle with a copy of its own formula: the
expected values are the page's worked numbers, hand-evaluated closed forms,
brute-force counting, or a library routine (torch scaled_dot_product_attention
in fp64) on a special case that reduces to it.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle
from resolution_block_sparse_b200.workloads import random_inputs

pytestmark = pytest.mark.filterwarnings("ignore")
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def dense_attention_fp64(q, k, v, mask):
    """Masked dense softmax(QK^T/sqrt(D))V via torch's SDPA in fp64; padded
    queries and rows without a valid key are set to 0."""
    q, k, v = (torch.as_tensor(np.asarray(x, dtype=np.float64)) for x in (q, k, v))
    B, H, N, D = q.shape
    if mask is None:
        return torch.nn.functional.scaled_dot_product_attention(q, k, v).numpy()
    m = torch.as_tensor(np.asarray(mask, dtype=np.float64)) > 0
    attn_mask = m[:, None, None, :].expand(B, H, N, N)
    out = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=attn_mask)
    out = torch.nan_to_num(out, nan=0.0)
    out = out * m[:, None, :, None]
    return out.numpy()


# ---------------------------------------------------------------- num_block
def test_num_block_matches_page_example():
    rows = []
    with open(os.path.join(GOLDEN, "num_block.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if line:
                rows.append([int(x) for x in line.split()])
    assert rows, "golden file is empty"
    for N, bpr, expected, dense in rows:
        assert oracle.num_block(N, bpr) == expected, (N, bpr)
        assert (N // 32) ** 2 == dense


# ---------------------------------------------------------------- pooling
def test_block_counts_and_pool_closed_form():
    B, H, N, D = 2, 1, 96, 4
    x = np.zeros((B, H, N, D))
    t = np.arange(N, dtype=np.float64)
    x[:, :, :, 0] = t              # dimension 0 carries the token index
    x[:, :, :, 1] = 1.0            # dimension 1 is constant
    mask = np.ones((B, N))
    mask[1, 32:64] = 0.0           # batch 1: block 1 empty
    mask[1, 88:96] = 0.0           # batch 1: block 2 keeps tokens 64..87
    cnt = oracle.block_counts(mask, B, N)
    np.testing.assert_array_equal(cnt, [[32, 32, 32], [32, 0, 24]])
    pooled = oracle.pool(x, mask)
    np.testing.assert_allclose(pooled[:, :, 0], [[15.5, 47.5, 79.5], [15.5, 0.0, 75.5]], rtol=0, atol=1e-12)
    np.testing.assert_allclose(pooled[:, :, 1], [[1, 1, 1], [1, 0, 1]], rtol=0, atol=1e-12)
    np.testing.assert_array_equal(pooled[:, :, 2:], 0.0)
    # no mask: plain block means
    pooled_all = oracle.pool(x, None)
    np.testing.assert_allclose(pooled_all[1, :, 0], [15.5, 47.5, 79.5], atol=1e-12)


# ---------------------------------------------------------------- low-res logits
def test_lowres_logits_closed_form():
    D = 4
    qhat = np.zeros((1, 3, D))
    khat = np.zeros((1, 3, D))
    qhat[0, 0, 0] = 1.0
    qhat[0, 1, 1] = 1.0
    qhat[0, 2, 2] = 1.0
    khat[0, 0, 1] = 2.0
    khat[0, 1, 2] = 3.0
    khat[0, 2, 0] = 5.0
    logit = oracle.lowres_logits(qhat, khat)
    expected = np.zeros((3, 3))
    expected[0, 2] = 5.0 / 2.0     # q-block 0 against k-block 2, / sqrt(4)
    expected[1, 0] = 2.0 / 2.0
    expected[2, 1] = 3.0 / 2.0
    np.testing.assert_allclose(logit[0], expected, atol=1e-15)


# ---------------------------------------------------------------- keys
def test_row_max_penalties_and_priors_closed_form():
    # 4 blocks, block 3 empty; logits chosen by hand
    logit = np.array([[[1.0, 3.0, 2.0, 9.0],
                       [0.5, 0.0, -1.0, 7.0],
                       [2.0, 2.0, 4.0, 8.0],
                       [0.0, 0.0, 0.0, 0.0]]])
    cnt = np.array([[32.0, 32.0, 32.0, 0.0]])
    mlo = oracle.row_max(logit, cnt, 1, 1)
    # the empty column 3 does not take part in the row max
    np.testing.assert_array_equal(mlo[0], [3.0, 0.5, 4.0, 0.0])
    key = oracle.selection_keys(logit, mlo, cnt, 1, 1, first_n=1, diag_n=3)
    P, E = 5e3, 1e4
    expected = np.array([
        # row 0: first-n on every column; band covers c in {0, 1}
        [1 - 3 + 2 * P, 3 - 3 + 2 * P, 2 - 3 + P, 9 - 3 + P - E],
        # row 1: first-n on column 0; band covers c in {0, 1, 2}
        [0.5 - 0.5 + 2 * P, 0 - 0.5 + P, -1 - 0.5 + P, 7 - 0.5 - E],
        # row 2: band covers c in {1, 2, 3}
        [2 - 4 + P, 2 - 4 + P, 4 - 4 + P, 8 - 4 + P - E],
        # row 3 is empty: -E on every cell, -E again on the empty column;
        # first-n on column 0, band covers c in {2, 3}
        [0 + P - E, 0 - E, 0 + P - E, 0 + P - 2 * E],
    ])
    np.testing.assert_allclose(key[0], expected, atol=1e-9)


def test_diagonal_band_widths():
    nbr = 6
    logit = np.zeros((1, nbr, nbr))
    cnt = np.full((1, nbr), 32.0)
    mlo = np.zeros((1, nbr))
    for g, offsets in [(1, {0}), (2, {-1, 0}), (3, {-1, 0, 1}), (4, {-2, -1, 0, 1})]:
        key = oracle.selection_keys(logit, mlo, cnt, 1, 1, first_n=0, diag_n=g)[0]
        band = {(r, c) for r in range(nbr) for c in range(nbr) if (c - r) in offsets}
        got = {(r, c) for r in range(nbr) for c in range(nbr) if key[r, c] > 1.0}
        assert got == band, g


# ---------------------------------------------------------------- selection
def brute_force_topk(key_flat, k):
    """Rank by counting: x is selected iff fewer than k entries precede it in
    the order (larger key first, smaller index first on equal keys)."""
    n = key_flat.size
    sel = []
    for x in range(n):
        ahead = 0
        for y in range(n):
            if key_flat[y] > key_flat[x] or (key_flat[y] == key_flat[x] and y < x):
                ahead += 1
        if ahead < k:
            sel.append(x)
    return np.array(sel, dtype=np.int32)


@pytest.mark.parametrize("nbr,k,seed", [(4, 5, 0), (6, 12, 1), (8, 16, 2), (8, 64, 3), (5, 1, 4)])
def test_select_matches_brute_force(nbr, k, seed):
    rng = np.random.default_rng(seed)
    # coarse values so that ties are frequent
    key = np.round(rng.normal(size=(3, nbr, nbr)) * 2) / 2
    sel = oracle.select(key, k)
    for h in range(3):
        np.testing.assert_array_equal(sel[h], brute_force_topk(key[h].reshape(-1), k))


def test_tie_rule_on_all_zero_queries():
    # q = 0 makes every low-res logit 0: every key ties, the k smallest flat
    # indices win; priors lift their blocks above the tie.
    d = random_inputs(1, 1, 256, 16, seed=5)
    q = np.zeros((1, 1, 256, 16))
    res = oracle.forward(q, d["k"], d["v"], None, block_per_row=2, approx_mode=1)
    np.testing.assert_array_equal(res["sel"][0], np.arange(16))
    res = oracle.forward(q, d["k"], d["v"], None, block_per_row=2, approx_mode=1, diag_n=1)
    diag = [r * 8 + r for r in range(8)]
    rest = [i for i in range(64) if i not in diag][:8]
    np.testing.assert_array_equal(res["sel"][0], sorted(diag + rest))


def test_priors_present_when_they_fit():
    d = random_inputs(2, 2, 512, 32, seed=7)
    nbr = 16
    f, g = 2, 3
    res = oracle.forward(d["q"], d["k"], d["v"], None, block_per_row=7, approx_mode=0,
                         first_n=f, diag_n=g)
    k = res["k"]
    prior = {r * nbr + c for r in range(nbr) for c in range(nbr)
             if (r < f or c < f) or abs(r - c) <= 1}
    assert len(prior) <= k
    for h in range(4):
        assert prior <= set(res["sel"][h].tolist())


def test_oversubscribed_priors_keep_double_priors_first():
    d = random_inputs(1, 2, 512, 32, seed=8)
    nbr = 16
    f, g = 2, 3
    res = oracle.forward(d["q"], d["k"], d["v"], None, block_per_row=2, approx_mode=1,
                         first_n=f, diag_n=g)
    k = res["k"]
    first = {r * nbr + c for r in range(nbr) for c in range(nbr) if (r < f or c < f)}
    band = {r * nbr + c for r in range(nbr) for c in range(nbr) if abs(r - c) <= 1}
    assert len(first | band) > k
    for h in range(2):
        s = set(res["sel"][h].tolist())
        assert (first & band) <= s          # 2 biases beat 1
        assert s <= (first | band)          # no unbiased block beats a biased one


def test_row_argmax_selected():
    d = random_inputs(2, 3, 512, 32, seed=9, pad_tokens=[0, 40])
    res = oracle.forward(d["q"], d["k"], d["v"], d["mask"], block_per_row=1, approx_mode=0)
    nbr = 16
    cnt = res["cnt"]
    for bh in range(6):
        b = bh // 3
        valid_c = np.where(cnt[b] > 0)[0]
        s = set(res["sel"][bh].tolist())
        for r in range(nbr):
            if cnt[b, r] == 0:
                continue
            best = valid_c[np.argmax(res["logit"][bh, r, valid_c])]
            assert r * nbr + best in s


# ---------------------------------------------------------------- attention
@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("pad", [None, [0, 45], [70, 33]])
def test_saturated_budget_equals_dense(mode, pad):
    B, H, N, D = 2, 2, 128, 16
    d = random_inputs(B, H, N, D, seed=11, pad_tokens=pad)
    nbr = N // 32
    res = oracle.forward(d["q"], d["k"], d["v"], d["mask"], block_per_row=nbr, approx_mode=mode)
    assert res["k"] == nbr * nbr
    ref = dense_attention_fp64(d["q"], d["k"], d["v"], d["mask"])
    np.testing.assert_allclose(res["out"], ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("bpr,f,g", [(1, 0, 0), (2, 1, 1), (1, 2, 3)])
@pytest.mark.parametrize("pad", [None, [0, 45]])
def test_block_constant_qk_full_mode_equals_dense(bpr, f, g, pad):
    """With Q and K constant inside every 32-token block, every score of block
    pair (r, c) equals the low-resolution logit, so full mode must reproduce
    dense attention whatever the budget selects."""
    B, H, N, D = 2, 2, 192, 16
    gen = torch.Generator().manual_seed(21)
    nbr = N // 32
    qb = torch.randn(B, H, nbr, 1, D, generator=gen).expand(B, H, nbr, 32, D).reshape(B, H, N, D)
    kb = torch.randn(B, H, nbr, 1, D, generator=gen).expand(B, H, nbr, 32, D).reshape(B, H, N, D)
    v = torch.randn(B, H, N, D, generator=gen)
    mask = None
    if pad is not None:
        mask = torch.ones(B, N)
        for b, p in enumerate(pad):
            if p:
                mask[b, N - p:] = 0
    res = oracle.forward(qb.numpy(), kb.numpy(), v.numpy(), None if mask is None else mask.numpy(),
                         block_per_row=bpr, approx_mode=0, first_n=f, diag_n=g)
    assert res["k"] < nbr * nbr
    ref = dense_attention_fp64(qb, kb, v, None if mask is None else mask.numpy())
    np.testing.assert_allclose(res["out"], ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("mode", [0, 1])
def test_rows_sum_to_one(mode):
    B, H, N, D = 2, 2, 256, 16
    d = random_inputs(B, H, N, D, seed=13, pad_tokens=[0, 50])
    v = np.ones((B, H, N, D))
    res = oracle.forward(d["q"], d["k"], v, d["mask"], block_per_row=1, approx_mode=mode,
                         first_n=1)
    out = res["out"]
    mask = d["mask"].numpy()
    nbr = N // 32
    for b in range(B):
        for h in range(H):
            sel = set(res["sel"][b * H + h].tolist())
            for i in range(N):
                if mask[b, i] == 0:
                    assert np.all(out[b, h, i] == 0)
                    continue
                r = i // 32
                has_valid_sel = any((r * nbr + c) in sel and mask[b, c * 32:(c + 1) * 32].sum() > 0
                                    for c in range(nbr))
                if mode == 0 or has_valid_sel:
                    np.testing.assert_allclose(out[b, h, i], 1.0, atol=1e-12)
                else:
                    assert np.all(out[b, h, i] == 0)


def test_one_hot_value_probe_measures_block_mass():
    """V = one-hot of the key's block: out_i[c] is the attention mass that
    query i puts on block c.  Unselected blocks carry cnt_c * e^{l_rc} (pooled
    block means computed here with numpy), selected ones sum e^{s_ij}."""
    B, H, N, D = 1, 1, 256, 8
    d = random_inputs(B, H, N, D, seed=17, pad_tokens=[40])
    q = d["q"].double().numpy()
    k = d["k"].double().numpy()
    mask = d["mask"].double().numpy()
    nbr = N // 32
    v = np.zeros((B, H, N, D))
    for j in range(N):
        v[0, 0, j, j // 32] = 1.0
    res = oracle.forward(q, k, v, mask, block_per_row=2, approx_mode=0)
    sel = set(res["sel"][0].tolist())
    m = mask[0]
    cnt = np.array([m[c * 32:(c + 1) * 32].sum() for c in range(nbr)])
    qh = np.array([(q[0, 0, c * 32:(c + 1) * 32] * m[c * 32:(c + 1) * 32, None]).sum(0) / max(cnt[c], 1)
                   for c in range(nbr)])
    kh = np.array([(k[0, 0, c * 32:(c + 1) * 32] * m[c * 32:(c + 1) * 32, None]).sum(0) / max(cnt[c], 1)
                   for c in range(nbr)])
    for i in [0, 37, 100, 190]:
        r = i // 32
        mass = np.zeros(nbr)
        for c in range(nbr):
            if (r * nbr + c) in sel:
                js = [j for j in range(c * 32, (c + 1) * 32) if m[j] > 0]
                mass[c] = sum(math.exp(q[0, 0, i] @ k[0, 0, j] / math.sqrt(D)) for j in js)
            elif cnt[c] > 0:
                mass[c] = cnt[c] * math.exp(qh[r] @ kh[c] / math.sqrt(D))
        np.testing.assert_allclose(res["out"][0, 0, i, :nbr], mass / mass.sum(), rtol=1e-11, atol=1e-14)


@pytest.mark.parametrize("mode", [0, 1])
def test_blockwise_equals_substituted_logit_dense(mode):
    """Dense restatement: out_i = softmax over keys j of s'_ij, with s'_ij the
    exact score on selected blocks, the block logit on unselected ones (full
    mode) or -inf (sparse mode), and padded keys removed."""
    B, H, N, D = 1, 2, 256, 16
    d = random_inputs(B, H, N, D, seed=19, pad_tokens=[20])
    res = oracle.forward(d["q"], d["k"], d["v"], d["mask"], block_per_row=2, approx_mode=mode,
                         first_n=1, diag_n=1)
    q, k, v = (d[x].double().numpy() for x in ("q", "k", "v"))
    m = d["mask"].numpy()[0]
    nbr = N // 32
    for h in range(H):
        S = q[0, h] @ k[0, h].T / math.sqrt(D)
        L = res["logit"][h]
        sel = np.zeros((nbr, nbr), bool)
        sel.flat[res["sel"][h]] = True
        blk_sel = np.kron(sel, np.ones((32, 32), bool))
        if mode == 0:
            Sp = np.where(blk_sel, S, np.kron(L, np.ones((32, 32))))
        else:
            Sp = np.where(blk_sel, S, -np.inf)
        Sp[:, m == 0] = -np.inf
        with np.errstate(invalid="ignore"):
            mx = Sp.max(axis=1, keepdims=True)
            W = np.exp(Sp - mx)
            W = np.nan_to_num(W)
            den = W.sum(axis=1, keepdims=True)
            out = np.where(den > 0, (W @ v[0, h]) / np.where(den > 0, den, 1), 0.0)
        out[m == 0] = 0.0
        np.testing.assert_allclose(res["out"][0, h], out, rtol=0, atol=1e-12)


def test_invalid_arguments_rejected():
    d = random_inputs(1, 1, 64, 8, seed=1)
    with pytest.raises(ValueError):
        oracle.forward(d["q"][:, :, :48], d["k"][:, :, :48], d["v"][:, :, :48], None,
                       block_per_row=1)
    with pytest.raises(ValueError):
        oracle.forward(d["q"], d["k"], d["v"], None, block_per_row=0)
    with pytest.raises(ValueError):
        oracle.forward(d["q"], d["k"], d["v"], None, block_per_row=1, approx_mode=2)
