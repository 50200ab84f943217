"""B200-native Reformer LSH self-attention.

The computation lives in ``liblsh.so`` (hand-written sm_100a CUDA behind the C
ABI of ``include/lsh.h``); this package is the Python binding (``_lib``, same
names as the C ABI), a buffer-owning driver (``attention``) and the seeded
synthetic workloads (``workloads``).
"""
from ._lib import (LSH_BF16, LSH_F32, LshError, LshLibraryMissing, lsh_attn_bwd, lsh_attn_fwd,
                   lsh_bwd_workspace_size, lsh_device_status, lsh_fwd_workspace_size, lsh_hash,
                   lsh_launch_count, lsh_problem, lsh_sort, lsh_sort_workspace_size, make_problem)

__all__ = ["LSH_BF16", "LSH_F32", "LshError", "LshLibraryMissing", "lsh_attn_bwd", "lsh_attn_fwd",
           "lsh_bwd_workspace_size", "lsh_device_status", "lsh_fwd_workspace_size", "lsh_hash",
           "lsh_launch_count", "lsh_problem", "lsh_sort", "lsh_sort_workspace_size",
           "make_problem"]
