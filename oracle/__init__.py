"""CPU oracle of the MRA-2 forward pass and its gradient (fp64, plain C,
OpenMP over heads).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import this package.  The
product path (``resolution_block_sparse_b200`` and its CUDA library) never
imports, links or runs it; the two share no code.

Source of the arithmetic: the page "深入解析 Transformers 中的 MRA 模型"
(blog.gitcode.com), sections "MraConfig：四个专属参数与完整默认值" and
"源码级原理：MRA 两级注意力到底怎么算" (steps one to four).  The C source
``mra_oracle.c`` cites the step each function follows.

What pins each function (tests marked ``not gpu``):

* ``num_block``            - the page's worked example (512 tokens, 4 blocks per
                             row -> 64 of 256), ``tests/golden/num_block.txt``.
* ``block_counts``/``pool``- closed forms on one-hot and masked inputs.
* ``lowres_logits``        - closed forms (orthogonal one-hot blocks; a
                             transposed operand fails).
* ``row_max``/``selection_keys`` - closed forms for penalties and priors; the
                             row-argmax invariant.
* ``select``               - brute-force rank counting on tiny maps; the
                             priors-present invariant; the tie rule.
* ``forward`` (hi-res part)- a budget that selects every block equals dense
                             softmax attention computed by torch's
                             scaled_dot_product_attention in fp64.
* ``forward`` (low-res part) - block-constant Q and K make full mode equal
                             dense attention for any budget; probes with
                             one-hot V measure the count weighting.
* ``backward``             - torch autograd (fp64) of a dense restatement of
                             the forward (exact scores on selected blocks,
                             block logits of differentiable block means on
                             unselected ones in full mode, -inf in sparse
                             mode); autograd of SDPA where the budget selects
                             every block; central finite differences of
                             ``forward`` with the selection unchanged
                             (``tests/test_oracle_backward_pins.py``).
* ``bigbird_blocks``       - the BigBird page's pattern rules checked row by
                             row by counting; attention on the pattern
                             (``attend_with_selection``, sparse mode) against
                             SDPA with the same token mask in fp64
                             (``tests/test_oracle_bigbird_pins.py``).  Which
                             two blocks are global, the clipped window and
                             the union of repeated blocks are readings.
* ``self_attention``       - a budget that selects every block equals torch's
                             multi-head attention (fp64, identity output
                             projection) on the same weights; permuting the
                             heads of the weights permutes the output's head
                             slices; one head with identity weights is the
                             forward pass itself (``tests/test_oracle_layer_pins.py``).
* padded-query outputs (0), the empty-row output (0), the prior band offsets
  and the exact bias arithmetic are readings of the page, not fixed by it:
  **parity unpinned** beyond internal consistency.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mra_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libmra_oracle.so")
_lock = threading.Lock()
_lib = None

BLOCK = 32


def build(force: bool = False) -> str:
    """Compile the oracle's shared library in place (gcc -O2 -fopenmp)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c99", "-o", tmp, _SRC, "-lm"]
        )
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _bind(path: str):
    lib = ctypes.CDLL(path)
    dp = ctypes.POINTER(ctypes.c_double)
    ip = ctypes.POINTER(ctypes.c_int32)
    c_int, c_long = ctypes.c_int, ctypes.c_long
    lib.mra_oracle_num_block.restype = c_long
    lib.mra_oracle_num_block.argtypes = [c_long, c_long]
    lib.mra_oracle_block_counts.restype = None
    lib.mra_oracle_block_counts.argtypes = [dp, c_int, c_int, dp]
    lib.mra_oracle_pool.restype = None
    lib.mra_oracle_pool.argtypes = [dp, dp, c_int, c_int, c_int, c_int, dp]
    lib.mra_oracle_lowres_logits.restype = None
    lib.mra_oracle_lowres_logits.argtypes = [dp, dp, c_int, c_int, c_int, dp]
    lib.mra_oracle_row_max.restype = None
    lib.mra_oracle_row_max.argtypes = [dp, dp, c_int, c_int, c_int, dp]
    lib.mra_oracle_selection_keys.restype = None
    lib.mra_oracle_selection_keys.argtypes = [dp, dp, dp, c_int, c_int, c_int, c_int, c_int, dp]
    lib.mra_oracle_select.restype = None
    lib.mra_oracle_select.argtypes = [dp, c_int, c_int, c_long, ip]
    lib.mra_oracle_forward.restype = c_int
    lib.mra_oracle_forward.argtypes = [dp, dp, dp, dp] + [c_int] * 8 + [dp, ip, dp, dp, dp, dp, c_int]
    lib.mra_oracle_backward.restype = c_int
    lib.mra_oracle_backward.argtypes = [dp, dp, dp, dp, dp] + [c_int] * 8 + [dp, dp, dp, c_int]
    lib.mra_oracle_attend_with_selection.restype = c_int
    lib.mra_oracle_attend_with_selection.argtypes = [dp, dp, dp, dp] + [c_int] * 5 + [ip, c_long, dp, c_int]
    return lib


_active = None      # a library bound by use_variant(), for planted-mistake tests


def _load():
    global _lib
    if _active is not None:
        return _active
    with _lock:
        if _lib is None:
            build()
            _lib = _bind(_LIB_PATH)
    return _lib


def compile_variant(source_text: str, out_dir: str) -> str:
    """Compile a modified copy of the oracle source (used only by tests that
    plant a mistake in the oracle to show that a pin catches it)."""
    src = os.path.join(out_dir, "mra_oracle_variant.c")
    lib = os.path.join(out_dir, "libmra_oracle_variant.so")
    with open(src, "w") as f:
        f.write(source_text)
    subprocess.check_call(["gcc", "-O1", "-fopenmp", "-fPIC", "-shared", "-std=c99", "-o", lib, src, "-lm"])
    return lib


def source_text() -> str:
    with open(_SRC) as f:
        return f.read()


class use_variant:
    """Context manager: route every oracle call through the library at path."""

    def __init__(self, path: str):
        self.lib = _bind(path)

    def __enter__(self):
        global _active
        self.prev = _active
        _active = self.lib
        return self

    def __exit__(self, *exc):
        global _active
        _active = self.prev
        return False


def _d(a):
    """Contiguous fp64 numpy view (None stays None) and its pointer."""
    if a is None:
        return None, None
    a = np.ascontiguousarray(np.asarray(a, dtype=np.float64))
    return a, a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _i32(a):
    a = np.ascontiguousarray(np.asarray(a, dtype=np.int32))
    return a, a.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))


def _out(shape, dtype=np.float64):
    a = np.zeros(shape, dtype=dtype)
    ct = ctypes.c_double if dtype == np.float64 else ctypes.c_int32
    return a, a.ctypes.data_as(ctypes.POINTER(ct))


def num_block(N: int, block_per_row: int) -> int:
    return int(_load().mra_oracle_num_block(N, block_per_row))


def block_counts(mask, B: int, N: int):
    m, mp = _d(mask)
    out, op = _out((B, N // BLOCK))
    _load().mra_oracle_block_counts(mp, B, N, op)
    return out


def pool(x, mask):
    """x: [B,H,N,D]; mask: [B,N] or None -> [B*H, nbr, D]."""
    B, H, N, D = x.shape
    xa, xp = _d(x)
    m, mp = _d(mask)
    out, op = _out((B * H, N // BLOCK, D))
    _load().mra_oracle_pool(xp, mp, B, H, N, D, op)
    return out


def lowres_logits(qhat, khat):
    BH, nbr, D = qhat.shape
    qa, qp = _d(qhat)
    ka, kp = _d(khat)
    out, op = _out((BH, nbr, nbr))
    _load().mra_oracle_lowres_logits(qp, kp, BH, nbr, D, op)
    return out


def row_max(logit, cnt, B: int, H: int):
    nbr = logit.shape[-1]
    la, lp = _d(logit)
    ca, cp = _d(cnt)
    out, op = _out((B * H, nbr))
    _load().mra_oracle_row_max(lp, cp, B, H, nbr, op)
    return out


def selection_keys(logit, mlo, cnt, B: int, H: int, first_n: int, diag_n: int):
    nbr = logit.shape[-1]
    la, lp = _d(logit)
    ma, mp = _d(mlo)
    ca, cp = _d(cnt)
    out, op = _out((B * H, nbr, nbr))
    _load().mra_oracle_selection_keys(lp, mp, cp, B, H, nbr, first_n, diag_n, op)
    return out


def select(key, k: int):
    """key: [BH, nbr, nbr] -> [BH, k] selected flat indices, ascending."""
    BH, nbr, _ = key.shape
    ka, kp = _d(key)
    out, op = _out((BH, k), np.int32)
    _load().mra_oracle_select(kp, BH, nbr, k, op)
    return out


def forward(q, k, v, mask=None, *, block_per_row: int, approx_mode: int = 0, first_n: int = 0,
            diag_n: int = 0, nthreads: int = 0, want_intermediates: bool = True):
    """The whole forward pass in fp64.

    q, k, v: [B,H,N,D] (any float dtype, widened exactly to fp64); mask: [B,N]
    of 0/1 or None.  approx_mode 0 = full, 1 = sparse.  Returns a dict with
    ``out`` [B,H,N,D] and, when asked, ``sel`` [BH,k], ``key`` and ``logit``
    [BH,nbr,nbr], ``pooled`` [3,BH,nbr,D], ``cnt`` [B,nbr].
    """
    B, H, N, D = q.shape
    nbr = N // BLOCK
    kk = num_block(N, block_per_row) if (N % BLOCK == 0 and N >= BLOCK) else 0
    qa, qp = _d(q)
    ka, kp = _d(k)
    va, vp = _d(v)
    ma, mp = _d(mask)
    out, op = _out((B, H, N, D))
    res = {"out": out, "k": kk}
    if want_intermediates:
        sel, sp = _out((B * H, kk), np.int32)
        key, keyp = _out((B * H, nbr, nbr))
        logit, lp = _out((B * H, nbr, nbr))
        pooled, pp = _out((3, B * H, nbr, D))
        cnt, cp = _out((B, nbr))
        res.update(sel=sel, key=key, logit=logit, pooled=pooled, cnt=cnt)
    else:
        sp = keyp = lp = pp = cp = None
    rc = _load().mra_oracle_forward(qp, kp, vp, mp, B, H, N, D, block_per_row, approx_mode,
                                    first_n, diag_n, op, sp, keyp, lp, pp, cp, nthreads)
    if rc != 0:
        raise ValueError("oracle rejected the arguments")
    return res


def attend_with_selection(q, k, v, mask, sel, *, approx_mode: int = 0, nthreads: int = 0):
    """Attention (steps three and four) for a given selected set sel [BH, k]."""
    B, H, N, D = q.shape
    qa, qp = _d(q)
    ka, kp = _d(k)
    va, vp = _d(v)
    ma, mp = _d(mask)
    sa, sp = _i32(sel)
    out, op = _out((B, H, N, D))
    rc = _load().mra_oracle_attend_with_selection(qp, kp, vp, mp, B, H, N, D, approx_mode, sp,
                                                  sa.shape[-1], op, nthreads)
    if rc != 0:
        raise ValueError("oracle rejected the arguments")
    return out


def backward(q, k, v, mask, dout, *, block_per_row: int, approx_mode: int = 0, first_n: int = 0,
             diag_n: int = 0, nthreads: int = 0):
    """Gradients (dq, dk, dv) [B,H,N,D] fp64 of the forward output with the
    selection held fixed, for the incoming gradient dout [B,H,N,D]."""
    B, H, N, D = q.shape
    qa, qp = _d(q)
    ka, kp = _d(k)
    va, vp = _d(v)
    ma, mp = _d(mask)
    ga, gp = _d(dout)
    dq, dqp = _out((B, H, N, D))
    dk, dkp = _out((B, H, N, D))
    dv, dvp = _out((B, H, N, D))
    rc = _load().mra_oracle_backward(qp, kp, vp, mp, gp, B, H, N, D, block_per_row, approx_mode,
                                     first_n, diag_n, dqp, dkp, dvp, nthreads)
    if rc != 0:
        raise ValueError("oracle rejected the arguments")
    return dq, dk, dv


def bigbird_blocks(N: int, block_size: int, rand_blocks):
    """Selected 32-token blocks (sorted flat indices r * nbr + c, nbr = N / 32)
    of one head under the BigBird block-sparse pattern.

    Page "Transformers 中的 BigBird：面向超长序列的稀疏注意力模型完全指南",
    sections on the attention mechanism and the usage notes: three kinds of
    attention combined - a window of 3 blocks, 2 global blocks that attend to
    every block and that every block attends to, and num_random_blocks random
    blocks per query block (at least one); the sequence length a multiple of
    the block size; sequences of at most (5 + 2 * num_random_blocks) blocks
    use full attention.  Readings (the page does not fix them): the global
    blocks are the first and the last block; the window of block i is
    {i - 1, i, i + 1} inside the sequence; attention runs over the union of
    the blocks (a block chosen twice counts once); the random blocks are an
    input (rand_blocks [nb][r] of block indices, drawn by the caller).
    Each block_size block (a multiple of 32) maps to the 32-token blocks it
    covers."""
    import numpy as np

    if block_size % BLOCK != 0 or N % block_size != 0:
        raise ValueError("block_size must be a multiple of 32 and divide N")
    rand_blocks = np.asarray(rand_blocks, dtype=np.int64)
    nb = N // block_size
    r = rand_blocks.shape[1] if rand_blocks.ndim == 2 else 0
    if r < 1 or rand_blocks.shape[0] != nb:
        raise ValueError("rand_blocks must be [nb][r] with r >= 1")
    if rand_blocks.min() < 0 or rand_blocks.max() >= nb:
        raise ValueError("random block out of range")
    full = nb <= 5 + 2 * r
    sel = np.zeros((nb, nb), dtype=bool)
    for i in range(nb):
        if full or i == 0 or i == nb - 1:
            sel[i, :] = True
            continue
        sel[i, [0, nb - 1]] = True
        sel[i, max(0, i - 1):min(nb, i + 2)] = True
        sel[i, rand_blocks[i]] = True
    f = block_size // BLOCK
    fine = np.kron(sel, np.ones((f, f), dtype=bool))
    return np.flatnonzero(fine.ravel()).astype(np.int32)


def self_attention(x, w_qkv, b_qkv, mask, H: int, *, block_per_row: int, approx_mode: int = 0,
                   first_n: int = 0, diag_n: int = 0, nthreads: int = 0):
    """The MraSelfAttention layer in fp64: x [B,N,hidden], w_qkv
    [3*hidden, hidden] (query, key, value weights stacked, each [out][in]),
    b_qkv [3*hidden] or None, mask [B,N] or None.  Returns [B,N,hidden].

    Page "深入解析 Transformers 中的 MRA 模型", the architecture paragraph
    (BERT-style self-attention: linear query, key and value maps of the
    hidden states, H heads of size hidden/H) and the engineering notes after
    step four (heads below 32 are zero-padded for the kernels and cut back:
    read as leaving the result unchanged, so here the heads keep their own
    size d and the scores their 1/sqrt(d)).  Feature h*d + e of a projection
    is element e of head h; the merged output puts head h's output at
    features h*d .. h*d + d - 1."""
    x = np.asarray(x, dtype=np.float64)
    w = np.asarray(w_qkv, dtype=np.float64)
    B, N, hidden = x.shape
    if hidden % H != 0 or w.shape != (3 * hidden, hidden):
        raise ValueError("hidden must divide by H and w_qkv be [3*hidden, hidden]")
    d = hidden // H
    proj = x @ w.T                                            # [B, N, 3*hidden]
    if b_qkv is not None:
        proj = proj + np.asarray(b_qkv, dtype=np.float64)
    heads = [proj[:, :, j * hidden:(j + 1) * hidden].reshape(B, N, H, d).transpose(0, 2, 1, 3)
             for j in range(3)]                               # [B, H, N, d] each
    out = forward(heads[0], heads[1], heads[2], mask, block_per_row=block_per_row, approx_mode=approx_mode,
                  first_n=first_n, diag_n=diag_n, nthreads=nthreads, want_intermediates=False)["out"]
    return np.ascontiguousarray(out.transpose(0, 2, 1, 3).reshape(B, N, hidden))
