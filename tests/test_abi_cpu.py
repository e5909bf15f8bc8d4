"""CPU checks of the C ABI: the library loads, exports every declared symbol,
and rejects invalid arguments before touching any pointer or the GPU."""
import ctypes
import glob
import os
import re

import pytest

import oracle
import resolution_block_sparse_b200 as mra
from resolution_block_sparse_b200 import _binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        names.update(re.findall(r"MRA_API\s+[\w\s\*]*?\b(mra_\w+)\s*\(", text))
    return names


def test_library_exports_every_declared_symbol():
    lib = mra.load_library()
    names = declared_symbols()
    assert {"mra_attention_fwd", "mra_attention_fwd_f32", "mra_attention_fwd_ex",
            "mra_num_block"} <= names
    for n in names:
        assert hasattr(lib, n), n
    assert names == set(_binding.EXPORTED) | (names - set(_binding.EXPORTED))
    assert set(_binding.EXPORTED) <= names


def test_num_block_matches_oracle_and_page_example():
    assert mra.mra_num_block(512, 4) == 64
    for N, bpr in [(256, 2), (512, 4), (2048, 64), (4096, 4), (16384, 8), (64, 4), (32, 1)]:
        assert mra.mra_num_block(N, bpr) == oracle.num_block(N, bpr)
    assert mra.mra_num_block(100, 4) == 0
    assert mra.mra_num_block(512, 0) == 0


def test_status_strings():
    for s in range(6):
        assert isinstance(mra.mra_status_string(s), str)
    assert mra.mra_status_string(99) == "unknown status"


FAKE = ctypes.c_void_p(4096)   # aligned, never dereferenced: validation fails first


@pytest.mark.parametrize("B,H,N,D,bpr,mode,f,g,expected", [
    (1, 1, 48, 64, 1, 0, 0, 0, 1),      # N not a multiple of 32
    (1, 1, 0, 64, 1, 0, 0, 0, 1),       # empty sequence
    (0, 1, 64, 64, 1, 0, 0, 0, 1),      # empty batch
    (1, 1, 64, 64, 0, 0, 0, 0, 1),      # block_per_row < 1
    (1, 1, 64, 64, 1, 2, 0, 0, 1),      # bad mode
    (1, 1, 64, 64, 1, 0, 3, 0, 1),      # first_n > N/32
    (1, 1, 64, 64, 1, 0, 0, -1, 1),     # negative prior
    (1, 1, 64, 48, 1, 0, 0, 0, 2),      # unsupported head size
    (1, 1, 65536 + 32, 64, 1, 0, 0, 0, 2),   # above the maximum length
])
def test_invalid_sizes_rejected_without_launch(B, H, N, D, bpr, mode, f, g, expected):
    lib = mra.load_library()
    for fn in (lib.mra_attention_fwd, lib.mra_attention_fwd_f32):
        assert fn(FAKE, FAKE, FAKE, None, FAKE, B, H, N, D, bpr, mode, f, g, None) == expected


def test_null_and_misaligned_pointers_rejected():
    lib = mra.load_library()
    assert lib.mra_attention_fwd(None, FAKE, FAKE, None, FAKE, 1, 1, 64, 64, 1, 0, 0, 0, None) == 1
    odd = ctypes.c_void_p(4096 + 8)
    assert lib.mra_attention_fwd(odd, FAKE, FAKE, None, FAKE, 1, 1, 64, 64, 1, 0, 0, 0, None) == 1
    assert lib.mra_attention_fwd_ex(FAKE, FAKE, FAKE, None, FAKE, 1, 1, 64, 64, 1, 0, 0, 0, 7,
                                    None, None, None, None) in (1,)


def test_missing_library_fails_loudly(tmp_path):
    with pytest.raises(RuntimeError):
        _binding.load_library(str(tmp_path / "absent.so"))
