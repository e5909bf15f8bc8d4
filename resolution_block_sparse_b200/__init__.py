"""B200-native MRA-2 approximate self-attention (forward and backward passes),
and block-sparse attention on given block patterns (BigBird among them).

The compute path lives in the CUDA library ``libmra_b200.so`` behind the C-ABI
declared in ``include/mra.h``; this package is a thin ctypes binding to it
(``_binding``) plus the seeded synthetic inputs used by tests and benchmarks
(``workloads``).  Importing the package does not load the library; the first
call does, and raises if it has not been built.
"""
from ._binding import (  # noqa: F401
    EXPORTED,
    MRA_DTYPE_BF16,
    MRA_DTYPE_F32,
    MRA_FULL,
    MRA_SPARSE,
    MraError,
    load_library,
    mra2_attention,
    mra_attention_bwd,
    mra_attention_fwd,
    mra_attention_fwd_ex,
    mra_attention_fwd_f32,
    mra_attention_fwd_host,
    mra_attention_fwd_noalloc,
    mra_bigbird_block_list,
    mra_blocksparse_attention_fwd,
    mra_get_device_status,
    mra_get_noalloc_status,
    mra_last_launch_count,
    mra_num_block,
    mra_profile_enable,
    mra_profile_read,
    mra_qkv_projection,
    mra_self_attention_fwd,
    mra_status_from_device,
    mra_status_string,
)
