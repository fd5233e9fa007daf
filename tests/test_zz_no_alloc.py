"""The layer entry point that allocates nothing (spava_layer_fwd_noalloc).

Some callers only receive input and output pointers from a host framework
that owns the device allocator, so they cannot hand the layer a workspace.
This entry point keeps the intermediates in a fixed 64 MiB array inside the
library instead.  These tests call it through the C ABI and check it against
the workspace entry point (spava_layer_fwd), within the layer's tolerances,
on two calls in a row with different problems, so that whatever the first
call leaves in the shared array cannot leak into the second.  They pass alone
in a fresh process and after the other tests."""
import ctypes

import numpy as np
import pytest
import torch

import sparse_approximate_attention_b200 as spava
from sparse_approximate_attention_b200 import workloads as W

pytestmark = pytest.mark.gpu

O_TOL, LSE_TOL = 2e-2, 1e-3


def _noalloc(p, Q, K, V, O, lse):
    f = spava.lib().spava_layer_fwd_noalloc
    f.argtypes = [ctypes.c_void_p] * 7
    f.restype = ctypes.c_int
    return f(ctypes.addressof(p._c), Q.data_ptr(), K.data_ptr(), V.data_ptr(), O.data_ptr(),
             lse.data_ptr(), torch.cuda.current_stream().cuda_stream)


def _case(wl):
    inp = W.make_inputs(wl)
    p = spava.Problem.from_workload(wl)
    Q, K, V = (inp[k].cuda() for k in ("Q", "K", "V"))
    return p, Q, K, V


def test_noalloc_matches_workspace_entry_on_calls_in_a_row():
    """Three calls in a row on different problems: a larger one, a smaller
    one, then one with lp = 0 (no compression: attention reads no passing
    rows from the shared array), the last through the Python wrapper."""
    cases = [W.Workload("frames_small", 2, 256, [1024, 777, 1024, 300], 128, 256, 8, 2, 128,
                        generator="frames", seed=77),
             W.workloads()["tiny"],
             W.Workload("no_passing", 2, 40, [300, 129, 256, 77], 20, 0, 4, 2, 128, seed=78)]
    for n_call, wl in enumerate(cases):
        p, Q, K, V = _case(wl)
        n = Q.shape[0]
        O_ref, lse_ref = spava.layer_fwd(p, Q, K, V)
        O = torch.full_like(Q, float("nan"))
        lse = torch.full((wl.num_q_heads, n), float("nan"), device="cuda")
        if n_call < 2:
            assert _noalloc(p, Q, K, V, O, lse) == 0
        else:
            spava.layer_fwd_noalloc(p, Q, K, V, O, lse)
        torch.cuda.synchronize()
        assert spava.device_error() == 0
        assert torch.isfinite(O.float()).all() and torch.isfinite(lse).all()
        assert (O.float() - O_ref.float()).abs().max().item() <= O_TOL
        assert (lse - lse_ref).abs().max().item() <= LSE_TOL


def test_noalloc_rejects_problems_beyond_its_array():
    wl = W.workloads()["longvideo_256k_lp4096"]      # needs ~190 MB of intermediates
    p = spava.Problem.from_workload(wl)
    assert p.sizes()["workspace_bytes"] > 64 << 20
    f = spava.lib().spava_layer_fwd_noalloc
    f.argtypes = [ctypes.c_void_p] * 7
    f.restype = ctypes.c_int
    code = f(ctypes.addressof(p._c), None, None, None, None, None, None)
    assert code == 3                                 # SPAVA_ERR_WORKSPACE, nothing launched
    assert spava.lib().spava_status_string(code) == b"SPAVA_ERR_WORKSPACE"
