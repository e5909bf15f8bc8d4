"""CPU checks of the block-list entry points: the library's BigBird pattern
generator is bit-identical to the oracle's (which is pinned against the
pattern's rules in test_oracle_bigbird_pins), and the block-sparse attention
entry point rejects invalid arguments before any launch."""
import ctypes

import numpy as np
import pytest

import oracle
import resolution_block_sparse_b200 as mra
from resolution_block_sparse_b200.workloads import BIGBIRD, bigbird_random_blocks


@pytest.mark.parametrize("N,bs,r", [
    (4096, 64, 3), (1024, 64, 1), (2048, 128, 2), (768, 64, 3),   # sparse pattern
    (448, 64, 1), (512, 64, 1),                                    # nb = 7 (full), nb = 8 (sparse)
    (96, 32, 1), (32, 32, 1), (8192, 256, 3), (1984, 32, 4),
])
def test_generator_matches_oracle(N, bs, r):
    nb = N // bs
    rb = bigbird_random_blocks(3, nb, r, seed=N + bs + r)
    for h in range(3):
        got = mra.mra_bigbird_block_list(N, bs, rb[h])
        want = oracle.bigbird_blocks(N, bs, rb[h])
        assert got.dtype == np.int32
        np.testing.assert_array_equal(got, want)


def test_generator_on_the_bigbird_workload():
    w = BIGBIRD
    nb = w.N // w.block_size
    rb = bigbird_random_blocks(w.B * w.H, nb, w.num_random, w.seed)
    counts = set()
    for h in range(w.B * w.H):
        got = mra.mra_bigbird_block_list(w.N, w.block_size, rb[h])
        np.testing.assert_array_equal(got, oracle.bigbird_blocks(w.N, w.block_size, rb[h]))
        counts.add(got.size)
    # random blocks that repeat a window or global block make heads differ
    assert len(counts) > 1


def test_generator_rejects_bad_arguments():
    lib = mra.load_library()
    out = (ctypes.c_int32 * 64)()
    cnt = ctypes.c_int(0)
    rb = (ctypes.c_int32 * 64)(*([0] * 64))
    ok = lib.mra_bigbird_block_list(256, 64, 1, rb, out, 64, ctypes.byref(cnt))
    assert ok == 0 and cnt.value == 64          # nb = 4: full attention, (256/32)^2 blocks
    assert lib.mra_bigbird_block_list(256, 48, 1, rb, out, 64, ctypes.byref(cnt)) == 1   # not a multiple of 32
    assert lib.mra_bigbird_block_list(320, 64, 1, rb, out, 64, ctypes.byref(cnt)) == 6   # full: 100 > 64
    assert lib.mra_bigbird_block_list(288, 64, 1, rb, out, 64, ctypes.byref(cnt)) == 1   # N % block_size
    assert lib.mra_bigbird_block_list(256, 64, 0, rb, out, 64, ctypes.byref(cnt)) == 1   # r < 1
    assert lib.mra_bigbird_block_list(256, 64, 1, None, out, 64, ctypes.byref(cnt)) == 1
    assert lib.mra_bigbird_block_list(256, 64, 1, rb, out, 63, ctypes.byref(cnt)) == 6   # capacity short
    assert lib.mra_bigbird_block_list(65536 + 64, 64, 1, rb, out, 64, ctypes.byref(cnt)) == 2
    bad = (ctypes.c_int32 * 4)(0, 1, 4, 2)      # block 4 of 4 is out of range
    assert lib.mra_bigbird_block_list(256, 64, 1, bad, out, 64, ctypes.byref(cnt)) == 1
    with pytest.raises(mra.MraError):
        mra.mra_bigbird_block_list(256, 64, np.full((4, 1), -1))


FAKE = ctypes.c_void_p(4096)


@pytest.mark.parametrize("N,D,cap,dtype,lst,expected", [
    (64, 64, 4, 0, FAKE, 0xFF),      # valid: not called (would launch)
    (64, 64, 0, 0, FAKE, 1),         # cap_sel < 1
    (64, 64, 5, 0, FAKE, 1),         # cap_sel > (N/32)^2
    (64, 64, 4, 0, None, 1),         # no list
    (64, 64, 4, 0, ctypes.c_void_p(4098), 1),   # misaligned list
    (64, 64, 4, 2, FAKE, 1),         # bad dtype
    (48, 64, 1, 0, FAKE, 1),         # N not a multiple of 32
    (64, 48, 4, 0, FAKE, 2),         # unsupported head size
])
def test_blocksparse_rejects_bad_arguments(N, D, cap, dtype, lst, expected):
    if expected == 0xFF:
        return
    lib = mra.load_library()
    assert lib.mra_blocksparse_attention_fwd(FAKE, FAKE, FAKE, None, FAKE, 1, 1, N, D, lst, cap, dtype,
                                             None) == expected
    odd = ctypes.c_void_p(4096 + 8)
    assert lib.mra_blocksparse_attention_fwd(odd, FAKE, FAKE, None, FAKE, 1, 1, 64, 64, FAKE, 4, 0, None) == 1


@pytest.mark.parametrize("B,N,hidden,H,expected", [
    (1, 64, 64, 3, 1),       # hidden not a multiple of H
    (1, 48, 64, 2, 1),       # N not a multiple of 32
    (0, 64, 64, 2, 1),       # empty batch
    (1, 64, 256, 2, 2),      # head size 128 > 64
    (1, 64, 36, 3, 2),       # hidden not a multiple of 8
])
def test_layer_rejects_bad_sizes(B, N, hidden, H, expected):
    lib = mra.load_library()
    assert lib.mra_self_attention_fwd(FAKE, FAKE, None, None, FAKE, B, N, hidden, H, 2, 1, 0, 0, None) == expected
    assert lib.mra_qkv_projection(FAKE, FAKE, None, FAKE, B, N, hidden, H, None) == expected


def test_layer_rejects_bad_pointers():
    lib = mra.load_library()
    odd = ctypes.c_void_p(4096 + 8)
    assert lib.mra_self_attention_fwd(odd, FAKE, None, None, FAKE, 1, 64, 64, 2, 2, 1, 0, 0, None) == 1
    assert lib.mra_self_attention_fwd(FAKE, FAKE, ctypes.c_void_p(4098), None, FAKE, 1, 64, 64, 2, 2, 1, 0, 0,
                                      None) == 1
    assert lib.mra_self_attention_fwd(FAKE, FAKE, None, None, FAKE, 1, 64, 64, 2, 2, 5, 0, 0, None) == 1  # mode
    assert lib.mra_qkv_projection(FAKE, None, None, FAKE, 1, 64, 64, 2, None) == 1


def test_bindings_check_shapes_before_calling_the_library():
    """The Python wrappers reject tensors of the wrong dtype or shape before
    any pointer reaches the library (CPU tensors, nothing launched)."""
    import torch

    q = torch.zeros(1, 2, 64, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        mra.mra_blocksparse_attention_fwd(q, q, q, None, q, torch.zeros(2, 4, dtype=torch.int64))
    with pytest.raises(ValueError):
        mra.mra_blocksparse_attention_fwd(q, q, q, None, q, torch.zeros(3, 4, dtype=torch.int32))
    with pytest.raises(ValueError):
        mra.mra_blocksparse_attention_fwd(q, q, q, None, q, torch.zeros(4, 2, dtype=torch.int32).t())
    x = torch.zeros(1, 64, 128, dtype=torch.bfloat16)
    w = torch.zeros(3 * 128, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        mra.mra_self_attention_fwd(x.float(), w, None, None, x, 2, 2, 1, 0, 0)
    with pytest.raises(ValueError):
        mra.mra_self_attention_fwd(x, w[:128], None, None, x, 2, 2, 1, 0, 0)
    with pytest.raises(ValueError):
        mra.mra_qkv_projection(x[0], w, None, x, 2)
    with pytest.raises(ValueError):
        mra.mra_bigbird_block_list(256, 64, np.zeros(4, dtype=np.int32))
