"""Seeded synthetic inputs for the MRA-2 forward pass.

This module draws random numbers and builds masks; it holds none of the
method's arithmetic.  The same host tensors feed the CUDA path and the CPU
oracle.

The five workloads follow the shapes of the MRA page ("深入解析 Transformers 中
的 MRA 模型", sections "MraConfig：四个专属参数与完整默认值" and "快速上手"):
32-token blocks, head size 64 (768 hidden / 12 heads), block_per_row budgets of
2-8, sequence lengths from 256 to 16384.  Every generator is
``torch.Generator('cpu').manual_seed(1000 + workload index)`` and draws, in
order, Q, K, V and then the mask, in fp32, before the cast to the workload's
dtype.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    index: int
    name: str
    B: int
    H: int
    N: int
    D: int
    dtype: str            # "f32" or "bf16"
    block_per_row: int
    approx_mode: int      # 0 = full, 1 = sparse
    first_n: int
    diag_n: int
    values: str           # "normal", "normal_half", "gmm64"
    padded: bool          # key padding mask on the last U[0, 25%] tokens

    @property
    def nbr(self) -> int:
        return self.N // 32

    @property
    def num_block(self) -> int:
        return min(self.nbr * self.block_per_row, self.nbr * self.nbr)

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    def describe(self) -> str:
        mode = "full" if self.approx_mode == 0 else "sparse"
        return (f"mra2_fwd {self.dtype} B={self.B} H={self.H} N={self.N} D={self.D} "
                f"block_per_row={self.block_per_row} num_block={self.num_block}/{self.nbr ** 2} "
                f"{mode} first_n={self.first_n} diag_n={self.diag_n} values={self.values}"
                f"{' padded' if self.padded else ''}")


WORKLOADS = {
    1: Workload(1, "f32_n256", 1, 2, 256, 32, "f32", 2, 0, 0, 0, "normal", False),
    2: Workload(2, "bf16_n512_padded", 8, 12, 512, 64, "bf16", 4, 0, 0, 0, "normal_half", True),
    3: Workload(3, "bf16_n2048_saturated", 4, 12, 2048, 64, "bf16", 64, 0, 0, 0, "normal", False),
    4: Workload(4, "bf16_n4096_sparse", 2, 12, 4096, 64, "bf16", 4, 1, 2, 3, "normal", False),
    5: Workload(5, "bf16_n16384_gmm", 1, 16, 16384, 64, "bf16", 8, 0, 1, 1, "gmm64", False),
}


def _gmm(gen: torch.Generator, B: int, H: int, N: int, D: int, centres: torch.Tensor) -> torch.Tensor:
    """Tokens from a 64-component mixture: each 32-token run picks one centre
    uniformly; token = centre + 0.3 * N(0, I)."""
    runs = N // 32
    comp = torch.randint(0, centres.shape[1], (B, H, runs), generator=gen)
    # centres is [B*H, 64, D]: one set of centres per (batch, head)
    idx = comp.reshape(B * H, runs)
    chosen = centres[torch.arange(B * H).unsqueeze(1), idx]          # [BH, runs, D]
    base = chosen.repeat_interleave(32, dim=1)                        # [BH, N, D]
    noise = torch.randn(B * H, N, D, generator=gen)
    return (base + 0.3 * noise).reshape(B, H, N, D)


def padding_mask(gen: torch.Generator, B: int, N: int) -> torch.Tensor:
    """Per sequence, u ~ U[0,1); the last 32*round(0.25*u*N/32) tokens are padding."""
    u = torch.rand(B, generator=gen)
    mask = torch.ones(B, N, dtype=torch.float32)
    for b in range(B):
        pad = 32 * int(round(0.25 * float(u[b]) * N / 32))
        if pad > 0:
            mask[b, N - pad:] = 0.0
    return mask


def make_inputs(w: Workload, seed: Optional[int] = None):
    """Return dict(q, k, v, mask) as host tensors; q/k/v in the workload dtype,
    mask float32 [B, N] of 0/1 or None."""
    gen = torch.Generator("cpu").manual_seed(1000 + w.index if seed is None else seed)
    B, H, N, D = w.B, w.H, w.N, w.D
    if w.values == "gmm64":
        centres = torch.randn(B * H, 64, D, generator=gen)
        q = _gmm(gen, B, H, N, D, centres)
        k = _gmm(gen, B, H, N, D, centres)
        v = torch.randn(B, H, N, D, generator=gen)
    else:
        scale = 4.0 / math.sqrt(D) if w.values == "normal_half" else 1.0
        q = torch.randn(B, H, N, D, generator=gen) * scale
        k = torch.randn(B, H, N, D, generator=gen) * scale
        v = torch.randn(B, H, N, D, generator=gen) * scale
    mask = padding_mask(gen, B, N) if w.padded else None
    dt = w.torch_dtype
    return {"q": q.to(dt).contiguous(), "k": k.to(dt).contiguous(), "v": v.to(dt).contiguous(),
            "mask": mask}


def random_inputs(B: int, H: int, N: int, D: int, dtype=torch.float32, seed: int = 0,
                  scale: float = 1.0, pad_tokens=None, v_scale=None):
    """Generic seeded inputs for tests.  Q and K are N(0, scale^2), V is
    N(0, v_scale^2) (v_scale defaults to scale).  pad_tokens: None, or a list
    of B counts of trailing padded tokens (any count, not only whole blocks)."""
    gen = torch.Generator("cpu").manual_seed(seed)
    vs = scale if v_scale is None else v_scale
    q = (torch.randn(B, H, N, D, generator=gen) * scale).to(dtype).contiguous()
    k = (torch.randn(B, H, N, D, generator=gen) * scale).to(dtype).contiguous()
    v = (torch.randn(B, H, N, D, generator=gen) * vs).to(dtype).contiguous()
    mask = None
    if pad_tokens is not None:
        mask = torch.ones(B, N, dtype=torch.float32)
        for b, p in enumerate(pad_tokens):
            if p > 0:
                mask[b, N - p:] = 0.0
    return {"q": q, "k": k, "v": v, "mask": mask}


# BigBird block-sparse workload (page "Transformers 中的 BigBird：面向超长序列的
# 稀疏注意力模型完全指南": block size 64 and 3 random blocks per query block by
# default, sequences up to 4096 tokens), run through the block-list attention
# entry point.  Q, K, V are N(0, 1) bf16 from random_inputs(seed=2000).
@dataclasses.dataclass(frozen=True)
class BigBirdWorkload:
    name: str
    B: int
    H: int
    N: int
    D: int
    block_size: int
    num_random: int
    seed: int


BIGBIRD = BigBirdWorkload("bigbird_b2_h12_n4096_d64_bs64_r3", 2, 12, 4096, 64, 64, 3, 2000)


def bigbird_random_blocks(BH: int, nb: int, r: int, seed: int):
    """Random blocks of the BigBird pattern, drawn per (batch*head, block row):
    int32 [BH, nb, r], uniform on [0, nb) (a draw may repeat a window or global
    block; the pattern counts it once)."""
    gen = torch.Generator("cpu").manual_seed(seed)
    return torch.randint(0, nb, (BH, nb, r), generator=gen, dtype=torch.int64).to(torch.int32).numpy()


# MraSelfAttention layer workload: the metric's attention (B=2, N=4096, 12
# heads of 64, sparse, 4 blocks per row, priors 2 and 3) behind its Q/K/V
# projection from hidden 768 (the page's MraConfig defaults).  x ~ N(0, 1),
# weights N(0, 1/hidden), bias N(0, 0.01), bf16 x and weights.
@dataclasses.dataclass(frozen=True)
class LayerWorkload:
    name: str
    B: int
    N: int
    hidden: int
    H: int
    block_per_row: int
    approx_mode: int
    first_n: int
    diag_n: int
    seed: int


LAYER = LayerWorkload("mra_self_attention_b2_n4096_hidden768_h12_sparse_bpr4_f2_g3", 2, 4096, 768, 12, 4, 1, 2, 3,
                      3000)


def layer_inputs(lw: LayerWorkload, seed: Optional[int] = None):
    """x bf16 [B, N, hidden], w_qkv bf16 [3*hidden, hidden], b_qkv fp32 [3*hidden]."""
    gen = torch.Generator("cpu").manual_seed(lw.seed if seed is None else seed)
    x = torch.randn(lw.B, lw.N, lw.hidden, generator=gen).to(torch.bfloat16)
    w = (torch.randn(3 * lw.hidden, lw.hidden, generator=gen) * lw.hidden ** -0.5).to(torch.bfloat16)
    b = torch.randn(3 * lw.hidden, generator=gen) * 0.1
    return x, w, b
