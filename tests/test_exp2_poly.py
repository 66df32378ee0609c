"""The forward kernel's FMA-pipe exp2 (Cody-Waite range reduction and a
degree-3 polynomial).

CPU: the coefficients written in fa_fwd.cuh are the fp32-rounded Remez
minimax polynomial that csrc/exp2_poly.py computes, and that polynomial,
evaluated as the kernel evaluates it (fp32 Horner with fused multiply-adds),
is within 7.5e-5 relative error of 2^f on [-1/2, 1/2]; an independent
check compares it with the Taylor series' leading coefficients.
GPU: the kernel's function, run through a test hook of the library, agrees
with CUDA's exp2 within that bound (plus the fp32 rounding of the final
scaling) over the inputs the softmax feeds it, and the clamp at -125 holds.
"""

import importlib.util
import math
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "exact_attention_118_b200", "csrc")
BOUND = 7.5e-5


def _gen():
    spec = importlib.util.spec_from_file_location("exp2_poly", os.path.join(CSRC, "exp2_poly.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _kernel_coefficients():
    with open(os.path.join(CSRC, "fa_fwd.cuh")) as f:
        text = f.read()
    m = re.search(r"constexpr float c0 = ([0-9.e+-]+)f, c1 = ([0-9.e+-]+)f, c2 = ([0-9.e+-]+)f, "
                  r"c3 = ([0-9.e+-]+)f;", text)
    assert m, "coefficients not found in fa_fwd.cuh"
    return [float(np.float32(float(g))) for g in m.groups()]


def test_kernel_coefficients_are_the_generated_ones():
    gen = _gen()
    assert _kernel_coefficients() == gen.fp32_coefficients()


def test_polynomial_error_bound_in_fp32():
    gen = _gen()
    err = gen.max_rel_error_fp32(_kernel_coefficients())
    assert err <= BOUND, err


def test_polynomial_is_close_to_the_taylor_series():
    # A minimax cubic for 2^f on a short interval stays near the Taylor
    # polynomial sum (f ln 2)^k / k!: this catches a swapped or mis-scaled
    # coefficient even if the generator itself were wrong.
    c = _kernel_coefficients()
    taylor = [math.log(2) ** k / math.factorial(k) for k in range(4)]
    for ck, tk in zip(c, taylor):
        assert abs(ck - tk) <= 0.02 * tk + 2e-4, (c, taylor)
    assert abs(c[0] - 1.0) < 1e-3


@pytest.mark.gpu
def test_device_exp2_matches_cuda_exp2():
    import torch

    import exact_attention_118_b200 as fa

    g = torch.Generator(device="cuda")
    g.manual_seed(7)
    x = torch.cat([
        torch.rand(1 << 20, device="cuda", generator=g) * 133.0 - 125.0,  # [-125, 8]
        torch.rand(1 << 16, device="cuda", generator=g) - 0.5,            # around 0
        torch.arange(-125, 9, device="cuda", dtype=torch.float32),       # integers (f = 0)
        torch.arange(-125, 8, device="cuda", dtype=torch.float32) + 0.5,  # ties of the rounding
        torch.tensor([-1e4, -300.0, -126.0, -125.5], device="cuda"),      # below the clamp
    ]).contiguous()
    y = torch.empty_like(x)
    st = fa.fa_selftest_exp2_fma(x.data_ptr(), y.data_ptr(), x.numel(), torch.cuda.current_stream().cuda_stream)
    assert st == fa.FA_OK
    torch.cuda.synchronize()
    ref = torch.exp2(torch.clamp(x, min=-125.0).double())
    rel = ((y.double() - ref).abs() / ref).max().item()
    assert rel <= BOUND + 2 ** -23, rel
    assert torch.isfinite(y).all().item() and (y > 0).all().item()
    # odd n: the last element alone
    y1 = torch.empty(1, device="cuda")
    x1 = torch.tensor([3.25], device="cuda")
    assert fa.fa_selftest_exp2_fma(x1.data_ptr(), y1.data_ptr(), 1, torch.cuda.current_stream().cuda_stream) == 0
    torch.cuda.synchronize()
    assert abs(y1.item() / 2 ** 3.25 - 1) <= BOUND + 2 ** -23
