"""Pins of the oracle's MraSelfAttention layer (projection, head split, the
forward pass per head, head merge).

Source: "深入解析 Transformers 中的 MRA 模型" (blog.gitcode.com): the layer is
BERT's self-attention with mra2_attention inside; heads below 32 are padded
for the kernels and cut back.  The expected values come from torch's own
multi-head attention (fp64) where the budget selects every block, from the
oracle's forward pass where the layer reduces to it, and from a head
permutation invariant.
"""
import numpy as np
import pytest
import torch

import oracle


def _weights(hidden, seed, scale=None):
    g = torch.Generator("cpu").manual_seed(seed)
    s = scale if scale is not None else hidden ** -0.5
    w = torch.randn(3 * hidden, hidden, generator=g, dtype=torch.float64) * s
    b = torch.randn(3 * hidden, generator=g, dtype=torch.float64) * 0.1
    return w.numpy(), b.numpy()


@pytest.mark.parametrize("B,N,hidden,H,pad", [
    (2, 128, 64, 4, [0, 40]),      # d = 16 (padded to 32 by the kernels)
    (1, 96, 96, 2, None),          # d = 48
    (2, 64, 128, 2, [10, 0]),      # d = 64
])
def test_saturated_layer_equals_torch_multihead_attention(B, N, hidden, H, pad):
    g = torch.Generator("cpu").manual_seed(7)
    x = torch.randn(B, N, hidden, generator=g, dtype=torch.float64)
    w, b = _weights(hidden, 8)
    mask = None
    if pad is not None:
        mask = torch.ones(B, N, dtype=torch.float64)
        for i, p in enumerate(pad):
            if p:
                mask[i, N - p:] = 0
    got = oracle.self_attention(x.numpy(), w, b, None if mask is None else mask.numpy(), H,
                                block_per_row=N // 32, approx_mode=1)
    mha = torch.nn.MultiheadAttention(hidden, H, bias=True, batch_first=True, dtype=torch.float64)
    with torch.no_grad():
        mha.in_proj_weight.copy_(torch.from_numpy(w))
        mha.in_proj_bias.copy_(torch.from_numpy(b))
        mha.out_proj.weight.copy_(torch.eye(hidden, dtype=torch.float64))
        mha.out_proj.bias.zero_()
        kpm = None if mask is None else (mask == 0)
        want, _ = mha(x, x, x, key_padding_mask=kpm, need_weights=False)
    want = want.numpy()
    if mask is not None:
        valid = mask.numpy() > 0
        np.testing.assert_allclose(got[valid], want[valid], rtol=0, atol=1e-12)
        assert np.all(got[~valid] == 0.0)          # padded queries: 0 (a reading)
    else:
        np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


def test_one_identity_head_is_the_forward_pass():
    B, N, hidden = 1, 256, 32
    g = torch.Generator("cpu").manual_seed(9)
    x = torch.randn(B, N, hidden, generator=g, dtype=torch.float64).numpy()
    eye = np.eye(hidden)
    w = np.concatenate([eye, 2 * eye, -eye])
    got = oracle.self_attention(x, w, None, None, 1, block_per_row=2, approx_mode=0, first_n=1, diag_n=1)
    q = x[:, None]
    want = oracle.forward(q, 2 * q, -q, None, block_per_row=2, approx_mode=0, first_n=1, diag_n=1)["out"]
    np.testing.assert_array_equal(got, want[:, 0])


def test_head_permutation_permutes_the_output():
    B, N, hidden, H = 1, 256, 64, 4
    d = hidden // H
    g = torch.Generator("cpu").manual_seed(11)
    x = torch.randn(B, N, hidden, generator=g, dtype=torch.float64).numpy()
    w, b = _weights(hidden, 12)
    perm = np.array([2, 0, 3, 1])
    rows = np.concatenate([j * hidden + np.concatenate([np.arange(p * d, (p + 1) * d) for p in perm])
                           for j in range(3)])
    kw = dict(block_per_row=2, approx_mode=0, first_n=1, diag_n=1)
    base = oracle.self_attention(x, w, b, None, H, **kw)
    permuted = oracle.self_attention(x, w[rows], b[rows], None, H, **kw)
    for i, p in enumerate(perm):
        np.testing.assert_array_equal(permuted[..., i * d:(i + 1) * d], base[..., p * d:(p + 1) * d])
