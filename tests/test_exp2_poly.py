"""The softmax's FMA-pipe 2^x (exp2_poly2 in csrc/ptx.cuh): its coefficients
are the committed least-squares fit, its float32 error stays within the
stated bound, and on the GPU it matches CUDA's exp2f within that bound."""
import os
import re

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "sparse_approximate_attention_b200", "csrc")
REL_BOUND = 1.2e-4   # below bf16's 2^-9: the value is rounded to bf16 for P anyway


def _kernel_coefficients():
    """c0..c3 as written in exp2_poly2 (Horner: ((c3 f + c2) f + c1) f + c0)."""
    txt = open(os.path.join(CSRC, "ptx.cuh")).read()
    body = txt[txt.index("exp2_poly2(float2 x)"):]
    body = body[:body.index("\n}\n")]
    vals = [float(v) for v in re.findall(r"make_float2\(([0-9.e-]+)f, \1f\)", body)]
    c3, c2, c1, c0 = vals[-4:]   # the last four constants of the function body
    return np.array([c0, c1, c2, c3])


def _fit():
    import importlib.util
    spec = importlib.util.spec_from_file_location("fit_exp2_poly", os.path.join(CSRC, "fit_exp2_poly.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod.fit()


def _poly32(x):
    """exp2_poly2 restated in float32 numpy arithmetic (round-half-even split,
    Horner with fused steps approximated by float32 products and sums)."""
    c0, c1, c2, c3 = (np.float32(v) for v in _kernel_coefficients())
    x = np.asarray(x, dtype=np.float32)
    i = np.rint(x).astype(np.float32)
    f = (x - i).astype(np.float32)
    p = ((c3 * f + c2) * f + c1) * f + c0
    out = np.ldexp(p.astype(np.float64), i.astype(np.int64)).astype(np.float32)
    return np.where(x < -126, np.float32(0), out)


def test_coefficients_are_the_committed_fit():
    got = _kernel_coefficients()
    want = _fit()
    assert np.array_equal(got.astype(np.float32), want.astype(np.float32)), (got, want)


def test_polynomial_error_bound_on_the_reduced_range():
    f = np.linspace(-0.5, 0.5, 200001)
    c = _fit()
    p = c[0] + f * (c[1] + f * (c[2] + f * c[3]))
    assert np.abs(p / np.exp2(f) - 1).max() <= 1.15e-4
    x = np.linspace(-30, 8, 400001).astype(np.float32)
    rel = np.abs(_poly32(x).astype(np.float64) / np.exp2(x.astype(np.float64)) - 1)
    assert rel.max() <= REL_BOUND


@pytest.mark.gpu
def test_gpu_matches_exp2f_within_the_bound():
    import sparse_approximate_attention_b200 as spava
    x = torch.cat([torch.linspace(-125.0, 8.0, 2_000_002, dtype=torch.float32),
                   torch.tensor([0.0, -0.0, 1.0, -1.0, 0.5, -0.5, 7.999, -124.9], dtype=torch.float32)])
    x = x[: x.numel() // 2 * 2].cuda()
    y = spava.debug_exp2_poly(x)
    ref = torch.exp2(x)   # CUDA's exp2f
    torch.cuda.synchronize()
    rel = ((y.double() - ref.double()).abs() / ref.double()).max().item()
    assert rel <= REL_BOUND, rel
    low = torch.tensor([-126.5, -127.0, -200.0, -float("inf"), -1e30, -130.0], dtype=torch.float32).cuda()
    assert torch.all(spava.debug_exp2_poly(low) == 0)
    edge = torch.linspace(-126.0, -125.0, 1000, dtype=torch.float32).cuda()
    assert (spava.debug_exp2_poly(edge).double() - torch.exp2(edge).double()).abs().max().item() <= 2.0 ** -124
