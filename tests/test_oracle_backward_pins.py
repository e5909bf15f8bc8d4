"""Pins of the CPU oracle's backward pass (gradients of the forward output with
the selected set held fixed).

Source: "深入解析 Transformers 中的 MRA 模型" (blog.gitcode.com), section
"源码级原理：MRA 两级注意力到底怎么算": step three (the sampled-dense products
are autograd functions whose backward reuses the kernels through transposed
indices), step four (sparse mode uses the low-resolution branch only to pick
blocks, under no_grad; full mode's low-resolution output is part of the
result).  None of these tests restates the oracle's gradient formulas: the
expected values come from torch autograd in fp64 on a dense formulation of
the same forward pass, from autograd of plain dense attention where the
budget selects every block, and from central finite differences of the
oracle's own forward pass.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from resolution_block_sparse_b200.workloads import random_inputs

pytestmark = pytest.mark.filterwarnings("ignore")


def _dense_substituted_grads(q, k, v, mask, sel, mode, dout):
    """Gradients by torch autograd (fp64) of the dense restatement of the
    forward: out_i = sum_j softmax_j(s'_ij) v_j with s'_ij = q_i.k_j/sqrt(D)
    on selected blocks, the block logit qhat_b.khat_c/sqrt(D) of the masked
    block means on unselected ones (full mode) or -inf (sparse mode), padded
    keys removed, padded queries and rows without a key set to 0.  The block
    means are differentiable torch ops, so the gradient reaches every token
    through them; the selection sel [BH, k] is a constant."""
    B, H, N, D = q.shape
    nbr = N // 32
    qt, kt, vt = (torch.tensor(np.asarray(x, dtype=np.float64), requires_grad=True) for x in (q, k, v))
    m = torch.ones(B, N, dtype=torch.float64) if mask is None else torch.as_tensor(
        np.asarray(mask, dtype=np.float64))
    mb = m.reshape(B, 1, nbr, 32, 1)
    cnt = mb.sum(dim=3)                                            # [B,1,nbr,1]
    safe = torch.where(cnt > 0, cnt, torch.ones_like(cnt))

    def means(x):
        return (x.reshape(B, H, nbr, 32, D) * mb).sum(dim=3) / safe   # [B,H,nbr,D]

    scale = 1.0 / math.sqrt(D)
    S = qt @ kt.transpose(-1, -2) * scale                           # [B,H,N,N]
    L = means(qt) @ means(kt).transpose(-1, -2) * scale             # [B,H,nbr,nbr]
    selb = torch.zeros(B * H, nbr * nbr, dtype=torch.bool)
    selb[torch.arange(B * H).unsqueeze(1), torch.as_tensor(np.asarray(sel, dtype=np.int64))] = True
    selb = selb.reshape(B, H, nbr, nbr)
    sel_tok = selb.repeat_interleave(32, dim=2).repeat_interleave(32, dim=3)
    L_tok = L.repeat_interleave(32, dim=2).repeat_interleave(32, dim=3)
    neg = torch.full_like(S, -math.inf)
    Sp = torch.where(sel_tok, S, L_tok if mode == 0 else neg)
    keyok = (m > 0)[:, None, None, :].expand(B, H, N, N)
    Sp = torch.where(keyok, Sp, neg)
    rowok = torch.isfinite(Sp).any(dim=-1, keepdim=True)
    P = torch.softmax(torch.where(rowok, Sp, torch.zeros_like(Sp)), dim=-1)
    P = torch.where(rowok & torch.isfinite(Sp), P, torch.zeros_like(P))
    out = (P @ vt) * (m > 0)[:, None, :, None]
    (out * torch.as_tensor(np.asarray(dout, dtype=np.float64))).sum().backward()
    return qt.grad.numpy(), kt.grad.numpy(), vt.grad.numpy(), out.detach().numpy()


@pytest.mark.parametrize("mode,pad,bpr,f,g", [
    (0, [20, 0], 2, 1, 1),
    (1, [20, 0], 2, 1, 1),
    (0, None, 1, 0, 0),
    (0, [64, 40], 3, 2, 3),     # a wholly padded block, oversubscribed priors
    (1, [0, 33], 3, 2, 3),
])
def test_backward_equals_autograd_of_dense_restatement(mode, pad, bpr, f, g):
    B, H, N, D = 2, 2, 256, 16
    d = random_inputs(B, H, N, D, seed=31, pad_tokens=pad)
    dout = random_inputs(B, H, N, D, seed=32)["q"]
    kw = dict(block_per_row=bpr, approx_mode=mode, first_n=f, diag_n=g)
    res = oracle.forward(d["q"], d["k"], d["v"], d["mask"], **kw)
    dq, dk, dv = oracle.backward(d["q"], d["k"], d["v"], d["mask"], dout, **kw)
    eq, ek, ev, out = _dense_substituted_grads(d["q"], d["k"], d["v"], d["mask"], res["sel"], mode, dout)
    np.testing.assert_allclose(out, res["out"], rtol=0, atol=1e-12)   # the restatement is the forward
    for got, want in ((dq, eq), (dk, ek), (dv, ev)):
        np.testing.assert_allclose(got, want, rtol=0, atol=1e-11)


@pytest.mark.parametrize("pad", [None, [0, 45]])
def test_saturated_budget_backward_equals_dense_attention_autograd(pad):
    """A budget that selects every block makes the forward plain softmax
    attention, in either mode; its gradient is autograd of SDPA in fp64."""
    B, H, N, D = 2, 2, 128, 16
    d = random_inputs(B, H, N, D, seed=41, pad_tokens=pad)
    dout = random_inputs(B, H, N, D, seed=42)["q"]
    dq, dk, dv = oracle.backward(d["q"], d["k"], d["v"], d["mask"], dout, block_per_row=N // 32,
                                 approx_mode=0)
    qt, kt, vt = (d[x].double().clone().requires_grad_(True) for x in ("q", "k", "v"))
    if d["mask"] is None:
        out = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt)
    else:
        m = d["mask"].double() > 0
        am = m[:, None, None, :].expand(B, H, N, N)
        out = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=am)
        out = torch.nan_to_num(out, nan=0.0) * m[:, None, :, None]
    (out * dout.double()).sum().backward()
    for got, want in ((dq, qt.grad), (dk, kt.grad), (dv, vt.grad)):
        np.testing.assert_allclose(got, want.numpy(), rtol=0, atol=1e-11)


@pytest.mark.parametrize("mode", [0, 1])
def test_backward_matches_finite_differences(mode):
    """Central differences of the oracle's forward (loss = sum out * dout) at
    random coordinates, where the perturbation leaves the selection as is."""
    B, H, N, D = 1, 1, 128, 8
    d = random_inputs(B, H, N, D, seed=51, pad_tokens=[10])
    base = {x: d[x].double().numpy() for x in ("q", "k", "v")}
    mask = d["mask"].numpy()
    dout = random_inputs(B, H, N, D, seed=52)["q"].double().numpy()
    kw = dict(block_per_row=2, approx_mode=mode, first_n=1, diag_n=1)
    grads = dict(zip(("q", "k", "v"), oracle.backward(base["q"], base["k"], base["v"], mask, dout, **kw)))
    sel0 = oracle.forward(base["q"], base["k"], base["v"], mask, **kw)["sel"]
    rng = np.random.default_rng(53)
    h = 1e-6
    checked = 0
    for name in ("q", "k", "v"):
        for _ in range(12):
            idx = (0, 0, int(rng.integers(N - 10)), int(rng.integers(D)))
            vals = []
            for sgn in (1, -1):
                x = {n: a.copy() for n, a in base.items()}
                x[name][idx] += sgn * h
                r = oracle.forward(x["q"], x["k"], x["v"], mask, **kw)
                if not np.array_equal(r["sel"], sel0):
                    break
                vals.append(float((r["out"] * dout).sum()))
            if len(vals) < 2:
                continue
            fd = (vals[0] - vals[1]) / (2 * h)
            assert abs(fd - grads[name][idx]) <= 1e-6 * max(1.0, abs(fd)), (name, idx, fd, grads[name][idx])
            checked += 1
    assert checked >= 30


def test_sparse_mode_gradient_ignores_the_low_resolution_branch():
    """Sparse mode: only selected blocks reach the output, so the gradients
    of K and V vanish on every key block that no row selected."""
    B, H, N, D = 1, 1, 256, 8
    d = random_inputs(B, H, N, D, seed=61)
    dout = random_inputs(B, H, N, D, seed=62)["q"]
    kw = dict(block_per_row=1, approx_mode=1, first_n=0, diag_n=0)
    res = oracle.forward(d["q"], d["k"], d["v"], None, **kw)
    _, dk, dv = oracle.backward(d["q"], d["k"], d["v"], None, dout, **kw)
    nbr = N // 32
    cols = set(int(s) % nbr for s in res["sel"][0])
    for c in range(nbr):
        if c not in cols:
            assert np.all(dv[0, 0, 32 * c:32 * (c + 1)] == 0.0)
            assert np.all(dk[0, 0, 32 * c:32 * (c + 1)] == 0.0)
