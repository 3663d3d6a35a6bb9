"""The FMA-pipe exponential (exp2_fma in csrc/tc_common.cuh): its polynomial
is the one the committed fit produces (CPU), and on the GPU it agrees with
CUDA's exp2f within the fit's relative error bound."""

import os
import re

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _coeffs_in_source():
    src = open(os.path.join(ROOT, "kv_cache_selection_b200", "csrc", "tc_common.cuh")).read()
    body = src[src.index("float exp2_fma(float x)"):]
    body = body[:body.index("return")]
    return [float(v) for v in re.findall(r"(-?\d+\.\d*)f", body)]


def test_polynomial_is_the_committed_fit():
    from kv_cache_selection_b200 import fit_exp2
    coeffs, rel = fit_exp2.fit()
    nums = _coeffs_in_source()
    # clamp, the two magic constants, then Horner from the highest degree down
    assert nums[0] == -126.0 and nums[1] == 12582912.0 and nums[2] == 12582912.0
    horner = nums[3:]
    assert horner == [coeffs[3], coeffs[2], coeffs[1], coeffs[0]]
    assert rel < 7.6e-5


def test_polynomial_error_in_numpy():
    """The same range reduction and polynomial in float32 numpy, against the
    float64 exponential: bound 7.6e-5 relative over [-125, 127]."""
    from kv_cache_selection_b200 import fit_exp2
    c, _ = fit_exp2.fit()
    c = np.asarray(c, dtype=np.float32)
    x = np.linspace(-125, 127, 200001).astype(np.float32)
    t = x + np.float32(12582912.0)
    j = t - np.float32(12582912.0)
    f = x - j
    p = ((c[3] * f + c[2]) * f + c[1]) * f + c[0]
    bits = (p.view(np.uint32).astype(np.uint64) + (t.view(np.uint32).astype(np.uint64) << 23)) & 0xFFFFFFFF
    y = bits.astype(np.uint32).view(np.float32).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    assert np.max(np.abs(y - ref) / ref) < 7.6e-5


@pytest.mark.gpu
@pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")
def test_exp2_fma_against_cuda_exp2f():
    from kv_cache_selection_b200 import statekv as S
    x = torch.cat([torch.linspace(-125.0, 127.0, 1 << 20, device="cuda"),
                   torch.tensor([0.0, -0.5, 0.5, -1.0, 1.0, -124.5, 8.0], device="cuda")])
    y = torch.empty_like(x)
    assert S.lib.statekv_selftest_exp2(x.data_ptr(), y.data_ptr(), x.numel(),
                                       torch.cuda.current_stream().cuda_stream) == 0
    ref = torch.exp2(x)  # CUDA's exp2f
    torch.cuda.synchronize()
    rel = ((y.double() - ref.double()).abs() / ref.double()).max().item()
    assert rel < 8e-5, rel
    # below the range: a tiny non-negative value, never NaN or a negative number
    lo = torch.tensor([-125.2, -125.7, -126.0, -126.3, -127.0, -200.0, float("-inf")], device="cuda")
    ylo = torch.empty_like(lo)
    assert S.lib.statekv_selftest_exp2(lo.data_ptr(), ylo.data_ptr(), lo.numel(),
                                       torch.cuda.current_stream().cuda_stream) == 0
    torch.cuda.synchronize()
    assert torch.all(ylo >= 0) and torch.all(ylo <= 2.0 ** -124)
