"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI and the fp64
oracle on the same seeded bf16 inputs, and compare within the stated tolerances:

    |dKL|  <= 2e-3 * max(1, |KL|)      |dLSE| <= 1e-3      rel-L2(dQ), rel-L2(dK) <= 1e-2

(the last per (batch, head) slice)."""
import numpy as np
import torch

import oracle
from attention_kl_divergence_02_b200 import binding, inputs

KL_TOL = 2e-3
LSE_TOL = 1e-3
GRAD_TOL = 1e-2


def gpu_inputs(w):
    t = inputs.make(w, device="cuda")
    return t


def host64(t):
    return inputs.to_f64(t)


def run_fwd(t, w):
    kl, l1, l2 = binding.fwd(t["q1"], t["k1"], t["q2"], t["k2"], scale=w.scale, causal=w.causal)
    assert binding.streamkl_device_status() == binding.OK
    return kl.cpu().double().numpy(), l1.cpu().double().numpy(), l2.cpu().double().numpy()


def check_fwd(got, want, where=""):
    kl, l1, l2 = got
    okl, ol1, ol2 = want
    assert np.all(np.isfinite(kl)) and np.all(np.isfinite(l1)) and np.all(np.isfinite(l2)), where
    ekl = np.abs(kl - okl) / np.maximum(1.0, np.abs(okl))
    e1 = np.abs(l1 - ol1)
    e2 = np.abs(l2 - ol2)
    assert ekl.max() <= KL_TOL, "%s KL err %.3g at %s" % (where, ekl.max(), np.unravel_index(ekl.argmax(), ekl.shape))
    assert e1.max() <= LSE_TOL, "%s LSE1 err %.3g" % (where, e1.max())
    assert e2.max() <= LSE_TOL, "%s LSE2 err %.3g" % (where, e2.max())
    return ekl.max(), e1.max(), e2.max()


def rel_l2(a, b, axes):
    num = np.sqrt(((a - b) ** 2).sum(axis=axes))
    den = np.sqrt((b ** 2).sum(axis=axes))
    return num / np.maximum(den, 1e-300)


def check_grad(got, want, where="", zero_atol=0.0):
    """got/want [B,H,N,d]: relative L2 error per (b, h) slice.  A slice whose exact gradient
    is identically zero (e.g. rows that see a single key) has no relative error; there the
    largest entry must stay below ``zero_atol`` (rounding noise of the fp32 statistics)."""
    assert np.all(np.isfinite(got)), where
    zero = np.sqrt((want ** 2).sum(axis=(2, 3))) == 0
    if zero.any():
        assert np.abs(got).max(axis=(2, 3))[zero].max() <= zero_atol, "%s nonzero gradient %.3g" % (
            where, np.abs(got).max(axis=(2, 3))[zero].max())
    e = np.where(zero, 0.0, rel_l2(got, want, axes=(2, 3)))
    assert e.max() <= GRAD_TOL, "%s rel-L2 %.3g at %s" % (where, e.max(), np.unravel_index(e.argmax(), e.shape))
    return e.max()
