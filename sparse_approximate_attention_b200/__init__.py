"""B200-native (sm_100a) approximate-attention prefill layer of Spava / APB-V.

The compute lives in libspava.so (C ABI, include/spava.h); this package holds
its ctypes binding (``spava``), the in-tree build step (``build``) and the
seeded synthetic input generators (``workloads``).
"""
from .spava import (Problem, SpavaError, attn_fwd, compress, debug_attn_abort, debug_wait_timeout, device_error,  # noqa: F401
                    gather_passing, layer_fwd, layer_fwd_noalloc, lib, lse_merge, score, score_variant, select_topk,
                    workspace_size)
