"""The forward kernel's FMA-pipe 2^x: its polynomial is the Remez fit that
exact_io_aware_69_b200/fit_exp2.py computes, and its float32 evaluation stays within
the stated bound of the true 2^x. The GPU test holds the compiled routine against
CUDA's exp2f."""
import os
import re

import numpy as np
import pytest

from exact_io_aware_69_b200 import fit_exp2

HEADER = os.path.join(os.path.dirname(fit_exp2.__file__), "csrc", "sm100.cuh")


def _header_coefficients():
    text = open(HEADER).read()
    found = dict(re.findall(r"constexpr float kExp2C(\d) = ([0-9.e+-]+)f;", text))
    return [float(found[str(k)]) for k in range(len(found))]


def test_header_holds_the_fitted_coefficients():
    got = _header_coefficients()
    want = fit_exp2.coefficients()
    assert len(got) == fit_exp2.DEGREE + 1
    assert np.array_equal(np.float32(got), np.float32(want))


def test_fit_is_equioscillating_minimax():
    """Remez's optimum: the relative error reaches its maximum, with alternating sign,
    at degree + 2 points of [-1/2, 1/2] (Chebyshev's alternation theorem)."""
    c = fit_exp2.fit()
    xs = np.linspace(-0.5, 0.5, 200001)
    err = np.polyval(c[::-1], xs) / 2.0 ** xs - 1.0
    emax = np.abs(err).max()
    # local extrema of |err| at (nearly) the maximum level, alternating in sign
    idx = [i for i in range(1, len(xs) - 1) if abs(err[i]) >= abs(err[i - 1]) and abs(err[i]) >= abs(err[i + 1])]
    idx = [0] + idx + [len(xs) - 1]
    top = [i for i in idx if abs(err[i]) > 0.999 * emax]
    assert len(top) >= fit_exp2.DEGREE + 2
    signs = np.sign(err[top])
    assert np.all(signs[1:] != signs[:-1])
    assert emax < 3e-6


def test_float32_evaluation_error_bound():
    assert fit_exp2.max_rel_error() < 3e-6


def test_float32_evaluation_special_points():
    x = np.array([0.0, 1.0, -1.0, 8.0, -8.0, 0.5, -0.5, 3.25, -17.75], np.float32)
    y = fit_exp2.eval_f32(x)
    assert np.allclose(y, np.exp2(x.astype(np.float64)), rtol=3e-6, atol=0)
    # clamped far below: 2^-125 (never zero, never a wrapped exponent)
    z = fit_exp2.eval_f32(np.array([-126.0, -200.0, -1e30], np.float32))
    assert np.all(z > 0) and np.allclose(z, 2.0 ** -125, rtol=3e-6)


def test_a_wrong_coefficient_is_caught():
    """The bound check is sharp enough to see a perturbed coefficient."""
    c = fit_exp2.coefficients()
    c[2] *= 1.001
    assert fit_exp2.max_rel_error(c) > 1e-5


@pytest.mark.gpu
def test_device_exp2_against_cuda_exp2f():
    import torch

    from exact_io_aware_69_b200 import fa

    lib = fa.load()
    x = torch.linspace(-124.0, 8.0, 1 << 20, device="cuda", dtype=torch.float32)
    x = torch.cat([x, torch.tensor([0.0, 1.0, -1.0, 0.5, -0.5, 7.999, -0.0, 2.5], device="cuda")])
    y = torch.empty_like(x)
    assert lib.fa_selftest_exp2(x.data_ptr(), y.data_ptr(), x.numel(), None) == fa.FA_OK
    assert fa.device_status() == fa.FA_OK
    ref = torch.exp2(x.double())
    rel = ((y.double() - ref) / ref).abs().max().item()
    assert rel < 3e-6, rel
    # the same steps emulated on the host give the same float32 results up to the
    # last-bit differences of fused and unfused multiply-adds
    host = fit_exp2.eval_f32(x.cpu().numpy())
    assert np.allclose(y.cpu().numpy(), host, rtol=2e-7, atol=0)
    # below the clamp: 2^-125, never zero
    lo = torch.tensor([-126.0, -1000.0], device="cuda")
    ylo = torch.empty_like(lo)
    assert lib.fa_selftest_exp2(lo.data_ptr(), ylo.data_ptr(), 2, None) == fa.FA_OK
    assert torch.allclose(ylo.double(), torch.full_like(ylo.double(), 2.0 ** -125), rtol=3e-6)
