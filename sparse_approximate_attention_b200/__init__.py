"""B200-native (sm_100a) approximate-attention prefill layer of Spava / APB-V.

The compute lives in libspava.so (C ABI, include/spava.h); this package holds
its ctypes binding (``spava``), the in-tree build step (``build``) and the
seeded synthetic input generators (``workloads``).
"""
from .spava import (Problem, SpavaError, attn_fwd, compress, device_error, gather_passing,  # noqa: F401
                    layer_fwd, lib, lse_merge, score, select_topk, workspace_size)
