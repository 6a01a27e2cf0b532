"""The 64K-context workload (B1 H32 NQ=NK=65536 d128, causal, shared keys) at full size,
in the launch configuration the library uses, checked on samples the oracle can afford.

Materialising P1 and P2 here would take 512 GiB; the GPU path keeps only the 12 bytes per
row of saved state.  The oracle works on a few sampled heads, each sliced out and widened
to fp64 on its own:
  * KL, LSE1, LSE2 and dQ (P1 fixed) on sampled rows, from the oracle's own row statistics;
  * dK on sampled keys, from the GPU's row statistics (KL, LSE1, LSE2 of all 65536 rows
    of the head -- too many for the fp64 oracle), which the first check spot-verifies: that
    part of the check is only partly independent;
  * dK on keys among the last 256, fully independent: under the causal mask only the last
    256 rows see them, so the oracle computes those rows' statistics itself and every other
    row's statistics are NaN (any use of them would show).
"""
import numpy as np
import pytest
import torch

import oracle
from attention_kl_divergence_02_b200 import binding, inputs

from parity import GRAD_TOL, KL_TOL, LSE_TOL, rel_l2

pytestmark = pytest.mark.gpu


def test_long64k_forward_and_mode1_backward_sampled():
    w = inputs.WORKLOADS["long64k"]
    t = inputs.make(w, device="cuda")
    kl, l1, l2 = binding.fwd(t["q1"], t["k1"], t["q2"], t["k2"], scale=w.scale, causal=True)
    dq, dk = binding.bwd(1, t["q1"], t["k1"], t["q2"], t["k2"], kl, l1, l2, t["dkl"], scale=w.scale,
                         causal=True)
    torch.cuda.synchronize()
    assert binding.streamkl_device_status() == binding.OK
    rng = np.random.default_rng(64)
    N, d = w.NQ, w.d
    for h in (0, 13, 31):
        sl = lambda x: inputs.to_f64(x[:, h:h + 1])
        q1, q2, k = sl(t["q1"]), sl(t["q2"]), sl(t["k1"])
        g = inputs.to_f64(t["dkl"][:, h:h + 1])
        rows = np.unique(np.concatenate([[0, 1, N - 1], rng.choice(N, 24, replace=False)]))
        okl, ol1, ol2 = oracle.fwd_rows(q1, k, q2, k, rows, scale=w.scale, causal=True)
        gkl = kl[0, h].cpu().double().numpy()[rows]
        assert np.max(np.abs(gkl - okl) / np.maximum(1, np.abs(okl))) <= KL_TOL
        assert np.max(np.abs(l1[0, h].cpu().double().numpy()[rows] - ol1)) <= LSE_TOL
        assert np.max(np.abs(l2[0, h].cpu().double().numpy()[rows] - ol2)) <= LSE_TOL
        odq = oracle.bwd_dq_rows(1, q1, k, q2, k, g, rows, scale=w.scale, causal=True)
        gdq = dq[0, h].float().cpu().double().numpy()[rows]
        assert rel_l2(gdq[None, None], odq[None, None], axes=(2, 3)).max() <= GRAD_TOL
        keys = np.unique(np.concatenate([[0, N - 1], rng.choice(N, 16, replace=False)]))
        stats = [x[:, h:h + 1].cpu().double().numpy() for x in (kl, l1, l2)]
        odk = oracle.bwd_dk_keys_stats(1, q1, k, q2, k, g, *stats, keys, scale=w.scale, causal=True)
        gdk = dk[0, h].float().cpu().double().numpy()[keys]
        assert rel_l2(gdk[None, None], odk[None, None], axes=(2, 3)).max() <= GRAD_TOL
        # the last keys: seen only by the last 256 rows, whose statistics the oracle computes
        tail = np.arange(N - 256, N)
        tkl, tl1, tl2 = oracle.fwd_rows(q1, k, q2, k, tail, scale=w.scale, causal=True)
        own = [np.full((1, 1, N), np.nan) for _ in range(3)]
        for a, v in zip(own, (tkl, tl1, tl2)):
            a[0, 0, tail] = v
        last = np.array([N - 256, N - 200, N - 129, N - 128, N - 17, N - 1])
        odk2 = oracle.bwd_dk_keys_stats(1, q1, k, q2, k, g, *own, last, scale=w.scale, causal=True)
        assert np.all(np.isfinite(odk2))
        gdk2 = dk[0, h].float().cpu().double().numpy()[last]
        assert rel_l2(gdk2[None, None], odk2[None, None], axes=(2, 3)).max() <= GRAD_TOL
    assert bool(torch.isfinite(kl).all()) and bool(torch.isfinite(dq.float()).all())
    assert kl.min().item() >= -2e-3
