"""Accuracy of the kernels' two exponential paths, through streamkl_eval_exp2: the FMA-pipe
polynomial (this library's own: Cody-Waite range reduction and a Remez-fitted degree-4
polynomial) against fp64 exp2 and against CUDA's ex2.approx, over the whole argument range
the kernels give it (x <= 0)."""
import numpy as np
import pytest
import torch

from attention_kl_divergence_02_b200 import binding

pytestmark = pytest.mark.gpu

FIT_REL = 2.7e-6          # worst relative error of the fit (fp32 Horner, host)


def _grid():
    x = np.concatenate([np.linspace(-126.0, 0.0, 1 << 20), -np.logspace(-8, np.log10(126), 4096),
                        np.array([0.0, -0.0, -0.5, 0.5 - 1.0, -1.0, -1e-30, -125.999, -126.0])])
    return torch.tensor(x.astype(np.float32), device="cuda")


def test_polynomial_relative_error_within_the_fit():
    x = _grid()
    rc, y = binding.streamkl_eval_exp2(1, x)
    assert rc == binding.OK
    xs, ys = x.cpu().double().numpy(), y.cpu().double().numpy()
    ref = np.exp2(xs)
    rel = np.abs(ys / ref - 1.0)
    assert rel.max() <= 1.05 * FIT_REL, (rel.max(), xs[rel.argmax()])
    assert ys[xs == 0.0].min() == ys[xs == 0.0].max() and abs(ys[xs == 0.0][0] - 1.0) <= FIT_REL


def test_polynomial_agrees_with_the_exponential_unit():
    x = _grid()
    rc0, y0 = binding.streamkl_eval_exp2(0, x)
    rc1, y1 = binding.streamkl_eval_exp2(1, x)
    assert rc0 == binding.OK and rc1 == binding.OK
    xs = x.cpu().double().numpy()
    a, b = y0.cpu().double().numpy(), y1.cpu().double().numpy()
    ok = xs >= -125.0                        # both normal there (ex2.approx flushes subnormals)
    assert np.abs(b[ok] / a[ok] - 1.0).max() <= 4e-6
    # the exponential unit itself, for the record of what the polynomial stands beside
    assert np.abs(a[ok] / np.exp2(xs[ok]) - 1.0).max() <= 1e-6


def test_polynomial_below_the_clamp_and_arguments():
    x = torch.tensor([-126.5, -150.0, -1e4, -np.inf], dtype=torch.float32, device="cuda")
    rc, y = binding.streamkl_eval_exp2(1, x)
    assert rc == binding.OK
    ys = y.cpu().double().numpy()
    assert np.all(ys >= 0.0) and np.all(ys <= 2.0 ** -125)   # tiny, never wrapped or negative
    assert binding.streamkl_eval_exp2(2, x)[0] == binding.ERR_INVALID_ARG
    with pytest.raises(ValueError):
        binding.streamkl_eval_exp2(1, x.double())
    assert binding.streamkl_device_status() == binding.OK
