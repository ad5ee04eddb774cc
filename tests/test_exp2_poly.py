"""The FMA-pipe exponential used for part of the prefill softmax: its coefficients (read from the
source) meet the stated relative-error bound against the exact 2^x, on CPU; on the GPU the device
routine is compared with the exact value through the C ABI test entry point."""
import ctypes
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "paged_kv_cache_446_b200", "csrc", "common.cuh")
BOUND = 3e-6


def coefficients():
    text = open(SRC).read()
    body = text[text.index("exp2_poly2"):]
    names = ["kC0", "kC1", "kC2", "kC3", "kC4"]
    return [np.float32(re.search(rf"{n} = ([0-9.e+-]+)f", body).group(1)) for n in names]


def poly_on_half_interval(f):
    c = coefficients()
    p = c[4]
    for j in (3, 2, 1, 0):
        p = (p * f + c[j]).astype(np.float32)
    return p


def test_polynomial_relative_error_bound():
    f = np.linspace(-0.5, 0.5, 400001).astype(np.float32)
    rel = np.abs(poly_on_half_interval(f).astype(np.float64) / np.exp2(f.astype(np.float64)) - 1.0)
    assert rel.max() < BOUND, rel.max()


@pytest.mark.gpu
def test_device_exp2_against_exact():
    import torch
    from paged_kv_cache_446_b200 import pkv
    lib = ctypes.CDLL(pkv.LIB_PATH)
    fn = lib.pkv_selftest_exp2
    fn.restype = ctypes.c_int
    fn.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p]
    x = torch.linspace(-126.0, 127.0, 2_000_001, dtype=torch.float32, device="cuda")
    x = torch.cat([x, torch.tensor([-0.5, 0.5, 0.0, -1e-7, 1e-7, -125.75, 126.5], device="cuda")])
    y = torch.empty_like(x)
    assert fn(x.data_ptr(), y.data_ptr(), x.numel(), torch.cuda.current_stream().cuda_stream) == 0
    torch.cuda.synchronize()
    exact = torch.exp2(x.double())
    rel = ((y.double() - exact).abs() / exact).max().item()
    assert rel < BOUND, rel
    # below the clamp the result is at most 2^-126 (never wraps to a large or negative value)
    z = torch.tensor([-130.0, -200.0, -1e30, float("-inf")], device="cuda")
    w = torch.empty_like(z)
    assert fn(z.data_ptr(), w.data_ptr(), z.numel(), torch.cuda.current_stream().cuda_stream) == 0
    torch.cuda.synchronize()
    assert bool(((w >= 0) & (w <= 2.0 ** -125)).all()), w
