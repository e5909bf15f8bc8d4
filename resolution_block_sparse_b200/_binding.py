"""ctypes binding of the C ABI in include/mra.h (argument marshalling only).

Every function here forwards to ``libmra_b200.so``; none computes any step of
the method itself.  Loading fails loudly when the library is missing: there
is no fallback path.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmra_b200.so")

(MRA_OK, MRA_ERR_INVALID_ARG, MRA_ERR_UNSUPPORTED, MRA_ERR_CUDA, MRA_ERR_ALLOC,
 MRA_ERR_DEVICE_TIMEOUT, MRA_ERR_TOO_LARGE) = range(7)
MRA_NOALLOC_SCRATCH_BYTES = 16 << 20
MRA_FULL, MRA_SPARSE = 0, 1
MRA_DTYPE_BF16, MRA_DTYPE_F32 = 0, 1
MRA_DEV_KEY_RANGE, MRA_DEV_COUNT, MRA_DEV_TIMEOUT = 1, 2, 4

EXPORTED = (
    "mra_attention_fwd", "mra_attention_fwd_f32", "mra_attention_fwd_ex", "mra_attention_fwd_host",
    "mra_num_block", "mra_status_string", "mra_get_device_status", "mra_profile_enable",
    "mra_profile_read", "mra_last_launch_count", "mra_attention_fwd_noalloc", "mra_attention_bwd",
    "mra_attention_bwd_f32", "mra_blocksparse_attention_fwd", "mra_bigbird_block_list",
    "mra_self_attention_fwd", "mra_qkv_projection", "mra_get_noalloc_status", "mra_status_from_device",
)

_lock = threading.Lock()
_lib = None


class MraError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {status_string(status)} (status {status})")
        self.status = status


def load_library(path: str = LIB_PATH):
    """Load libmra_b200.so and declare its signatures (raises if missing)."""
    global _lib
    with _lock:
        if _lib is not None and path == LIB_PATH:
            return _lib
        if not os.path.exists(path):
            raise RuntimeError(
                f"CUDA library not built: {path} is missing "
                "(run `python -m resolution_block_sparse_b200.build`)")
        lib = ctypes.CDLL(path)
        vp, ip, c_int = ctypes.c_void_p, ctypes.c_int, ctypes.c_int
        fwd_args = [vp, vp, vp, vp, vp] + [c_int] * 8 + [vp]
        lib.mra_attention_fwd.argtypes = fwd_args
        lib.mra_attention_fwd.restype = c_int
        lib.mra_attention_fwd_f32.argtypes = fwd_args
        lib.mra_attention_fwd_f32.restype = c_int
        lib.mra_attention_fwd_noalloc.argtypes = fwd_args
        lib.mra_attention_fwd_noalloc.restype = c_int
        lib.mra_attention_fwd_ex.argtypes = [vp, vp, vp, vp, vp] + [c_int] * 9 + [vp, vp, vp, vp]
        lib.mra_attention_fwd_ex.restype = c_int
        lib.mra_attention_fwd_host.argtypes = [vp, vp, vp, vp, vp] + [c_int] * 9 + [vp]
        lib.mra_attention_fwd_host.restype = c_int
        for name in ("mra_attention_bwd", "mra_attention_bwd_f32"):
            fn = getattr(lib, name)
            fn.argtypes = [vp] * 8 + [c_int] * 8 + [vp]
            fn.restype = c_int
        lib.mra_blocksparse_attention_fwd.argtypes = [vp] * 5 + [c_int] * 4 + [vp, c_int, c_int, vp]
        lib.mra_blocksparse_attention_fwd.restype = c_int
        lib.mra_bigbird_block_list.argtypes = [c_int, c_int, c_int, vp, vp, c_int, ctypes.POINTER(c_int)]
        lib.mra_bigbird_block_list.restype = c_int
        lib.mra_self_attention_fwd.argtypes = [vp] * 5 + [c_int] * 8 + [vp]
        lib.mra_self_attention_fwd.restype = c_int
        lib.mra_qkv_projection.argtypes = [vp] * 4 + [c_int] * 4 + [vp]
        lib.mra_qkv_projection.restype = c_int
        lib.mra_num_block.argtypes = [c_int, c_int]
        lib.mra_num_block.restype = ctypes.c_size_t
        lib.mra_status_string.argtypes = [c_int]
        lib.mra_status_string.restype = ctypes.c_char_p
        lib.mra_get_device_status.argtypes = [vp]
        lib.mra_get_noalloc_status.argtypes = [vp]
        lib.mra_get_noalloc_status.restype = c_int
        lib.mra_status_from_device.argtypes = [c_int]
        lib.mra_status_from_device.restype = c_int
        lib.mra_get_device_status.restype = c_int
        lib.mra_profile_enable.argtypes = [c_int]
        lib.mra_profile_enable.restype = None
        lib.mra_profile_read.argtypes = [ctypes.POINTER(ctypes.c_char_p), ctypes.POINTER(c_int),
                                         ctypes.POINTER(ctypes.c_double), c_int]
        lib.mra_profile_read.restype = c_int
        lib.mra_last_launch_count.argtypes = []
        lib.mra_last_launch_count.restype = c_int
        if path == LIB_PATH:
            _lib = lib
        return lib


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _check(status: int, where: str):
    if status != MRA_OK:
        raise MraError(status, where)


def _shape(q):
    if q.dim() != 4:
        raise ValueError("q, k, v must be [B, H, N, D]")
    return tuple(int(x) for x in q.shape)


def _mode(approx_mode):
    if isinstance(approx_mode, str):
        return {"full": MRA_FULL, "sparse": MRA_SPARSE}[approx_mode]
    return int(approx_mode)


def mra_attention_fwd(q, k, v, key_mask, out, block_per_row, approx_mode, first_n, diag_n,
                      stream=None):
    """bf16 forward on device tensors [B,H,N,D]; key_mask float32 [B,N] or None."""
    B, H, N, D = _shape(q)
    st = load_library().mra_attention_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(key_mask), _ptr(out),
                                          B, H, N, D, block_per_row, _mode(approx_mode), first_n,
                                          diag_n, _stream(stream))
    _check(st, "mra_attention_fwd")
    return out


def mra_attention_fwd_f32(q, k, v, key_mask, out, block_per_row, approx_mode, first_n, diag_n,
                          stream=None):
    """fp32 forward on device tensors [B,H,N,D]."""
    B, H, N, D = _shape(q)
    st = load_library().mra_attention_fwd_f32(_ptr(q), _ptr(k), _ptr(v), _ptr(key_mask), _ptr(out),
                                              B, H, N, D, block_per_row, _mode(approx_mode),
                                              first_n, diag_n, _stream(stream))
    _check(st, "mra_attention_fwd_f32")
    return out


def mra_attention_fwd_noalloc(q, k, v, key_mask, out, block_per_row, approx_mode, first_n,
                              diag_n, stream=None):
    """bf16 forward that allocates no device memory (static 16 MiB scratch);
    raises MraError(MRA_ERR_TOO_LARGE) when the problem does not fit."""
    B, H, N, D = _shape(q)
    st = load_library().mra_attention_fwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(key_mask),
                                                  _ptr(out), B, H, N, D, block_per_row,
                                                  _mode(approx_mode), first_n, diag_n,
                                                  _stream(stream))
    _check(st, "mra_attention_fwd_noalloc")
    return out


def mra_attention_bwd(q, k, v, key_mask, dout, dq, dk, dv, block_per_row, approx_mode, first_n, diag_n,
                      stream=None):
    """Backward on device tensors: q, k, v, dout [B,H,N,D] (bf16 or fp32);
    dq, dk, dv fp32 [B,H,N,D] are written."""
    B, H, N, D = _shape(q)
    lib = load_library()
    fn = lib.mra_attention_bwd if q.dtype == torch.bfloat16 else lib.mra_attention_bwd_f32
    st = fn(_ptr(q), _ptr(k), _ptr(v), _ptr(key_mask), _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv), B, H, N, D,
            block_per_row, _mode(approx_mode), first_n, diag_n, _stream(stream))
    _check(st, "mra_attention_bwd")
    return dq, dk, dv


def mra_attention_fwd_ex(q, k, v, key_mask, out, block_per_row, approx_mode, first_n, diag_n,
                         sel_idx=None, lowres_logit=None, pooled=None, stream=None):
    """Forward that also fills the optional intermediate tensors (device)."""
    B, H, N, D = _shape(q)
    dtype = MRA_DTYPE_BF16 if q.dtype == torch.bfloat16 else MRA_DTYPE_F32
    st = load_library().mra_attention_fwd_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(key_mask), _ptr(out),
                                             B, H, N, D, block_per_row, _mode(approx_mode), first_n,
                                             diag_n, dtype, _ptr(sel_idx), _ptr(lowres_logit),
                                             _ptr(pooled), _stream(stream))
    _check(st, "mra_attention_fwd_ex")
    return out


def mra_attention_fwd_host(q, k, v, key_mask, out, block_per_row, approx_mode, first_n, diag_n,
                           stream=None):
    """Forward on HOST tensors (pinned for asynchronous copies); synchronises."""
    B, H, N, D = _shape(q)
    dtype = MRA_DTYPE_BF16 if q.dtype == torch.bfloat16 else MRA_DTYPE_F32
    st = load_library().mra_attention_fwd_host(_ptr(q), _ptr(k), _ptr(v), _ptr(key_mask), _ptr(out),
                                               B, H, N, D, block_per_row, _mode(approx_mode),
                                               first_n, diag_n, dtype, _stream(stream))
    _check(st, "mra_attention_fwd_host")
    return out


def mra_blocksparse_attention_fwd(q, k, v, key_mask, out, block_idx, stream=None):
    """Attention on given 32x32 blocks: block_idx int32 [B*H, cap_sel] on the
    device, ascending flat indices r * (N/32) + c per head, -1 padded."""
    B, H, N, D = _shape(q)
    if block_idx.dtype != torch.int32 or block_idx.dim() != 2 or block_idx.shape[0] != B * H:
        raise ValueError("block_idx must be int32 [B*H, cap_sel]")
    if not block_idx.is_contiguous():
        raise ValueError("block_idx must be contiguous")
    dtype = MRA_DTYPE_BF16 if q.dtype == torch.bfloat16 else MRA_DTYPE_F32
    st = load_library().mra_blocksparse_attention_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(key_mask), _ptr(out),
                                                      B, H, N, D, _ptr(block_idx), int(block_idx.shape[1]),
                                                      dtype, _stream(stream))
    _check(st, "mra_blocksparse_attention_fwd")
    return out


def mra_bigbird_block_list(N: int, block_size: int, rand_blocks):
    """The BigBird pattern of one head (host): rand_blocks int [nb, r] ->
    int32 numpy array of ascending flat 32-token block indices."""
    import numpy as np

    rb = np.ascontiguousarray(np.asarray(rand_blocks), dtype=np.int32)
    if rb.ndim != 2:
        raise ValueError("rand_blocks must be [nb, r]")
    nbr = N // 32 if N > 0 else 0
    out = np.empty(max(1, nbr * nbr), dtype=np.int32)
    count = ctypes.c_int(0)
    st = load_library().mra_bigbird_block_list(N, block_size, int(rb.shape[1]), rb.ctypes.data_as(ctypes.c_void_p),
                                               out.ctypes.data_as(ctypes.c_void_p), int(out.size), ctypes.byref(count))
    _check(st, "mra_bigbird_block_list")
    return out[:count.value].copy()


def _layer_shape(x, w_qkv, H):
    if x.dim() != 3 or x.dtype != torch.bfloat16 or w_qkv.dtype != torch.bfloat16:
        raise ValueError("x must be bf16 [B, N, hidden] and w_qkv bf16 [3*hidden, hidden]")
    B, N, hidden = (int(s) for s in x.shape)
    if tuple(w_qkv.shape) != (3 * hidden, hidden):
        raise ValueError("w_qkv must be [3*hidden, hidden]")
    return B, N, hidden


def mra_self_attention_fwd(x, w_qkv, b_qkv, key_mask, out, H, block_per_row, approx_mode, first_n, diag_n,
                           stream=None):
    """The MraSelfAttention layer on device tensors: x bf16 [B, N, hidden],
    w_qkv bf16 [3*hidden, hidden], b_qkv fp32 [3*hidden] or None, key_mask
    fp32 [B, N] or None; out bf16 [B, N, hidden] is written."""
    B, N, hidden = _layer_shape(x, w_qkv, H)
    st = load_library().mra_self_attention_fwd(_ptr(x), _ptr(w_qkv), _ptr(b_qkv), _ptr(key_mask), _ptr(out), B,
                                               N, hidden, H, block_per_row, _mode(approx_mode), first_n, diag_n,
                                               _stream(stream))
    _check(st, "mra_self_attention_fwd")
    return out


def mra_qkv_projection(x, w_qkv, b_qkv, qkv, H, stream=None):
    """The layer's projection alone: qkv bf16 [3, B, H, N, Dp] (Dp = 32 if
    hidden/H <= 32 else 64) gets the head-split, zero-padded Q (scaled by
    sqrt(Dp/d)), K and V."""
    B, N, hidden = _layer_shape(x, w_qkv, H)
    st = load_library().mra_qkv_projection(_ptr(x), _ptr(w_qkv), _ptr(b_qkv), _ptr(qkv), B, N, hidden, H,
                                           _stream(stream))
    _check(st, "mra_qkv_projection")
    return qkv


def mra_num_block(N: int, block_per_row: int) -> int:
    return int(load_library().mra_num_block(N, block_per_row))


def status_string(status: int) -> str:
    try:
        return load_library().mra_status_string(status).decode()
    except RuntimeError:
        return f"status {status}"


mra_status_string = status_string


def mra_get_device_status(stream=None) -> int:
    return int(load_library().mra_get_device_status(_stream(stream)))


def mra_get_noalloc_status(stream=None) -> int:
    """Reads and clears the status word of the no-allocation entry point."""
    return int(load_library().mra_get_noalloc_status(_stream(stream)))


def mra_status_from_device(word: int) -> int:
    """mra_status for a device status word (host-side mapping)."""
    return int(load_library().mra_status_from_device(int(word)))


def mra_profile_enable(enable: bool) -> None:
    load_library().mra_profile_enable(1 if enable else 0)


def mra_profile_read(max_phases: int = 16):
    """{phase: (launches, total_ms)} since the previous read."""
    names = (ctypes.c_char_p * max_phases)()
    launches = (ctypes.c_int * max_phases)()
    ms = (ctypes.c_double * max_phases)()
    n = load_library().mra_profile_read(names, launches, ms, max_phases)
    return {names[i].decode(): (launches[i], ms[i]) for i in range(n)}


def mra_last_launch_count() -> int:
    return int(load_library().mra_last_launch_count())


def mra2_attention(q, k, v, key_mask=None, *, block_per_row: int = 4, approx_mode="full",
                   first_n: int = 0, diag_n: int = 0, stream=None):
    """Allocate the output and run the forward pass on device tensors."""
    out = torch.empty_like(q)
    fn = mra_attention_fwd if q.dtype == torch.bfloat16 else mra_attention_fwd_f32
    return fn(q, k, v, key_mask, out, block_per_row, approx_mode, first_n, diag_n, stream)
