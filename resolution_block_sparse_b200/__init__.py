"""B200-native MRA-2 approximate self-attention (forward pass).

The compute path lives in the CUDA library ``libmra_b200.so`` behind the C-ABI
declared in ``include/mra.h``; this package is a thin ctypes binding to it.
"""
