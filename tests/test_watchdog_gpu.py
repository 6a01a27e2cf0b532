"""Failure detection on the GPU without a fault: every pipeline wait of the library is
bounded (a 2 s limit, then STREAMKL_ERR_TIMEOUT in the device status word and an abort
flag that stops the CTA's other waits).  streamkl_selftest_watchdog runs that machinery on
a barrier that nothing completes; the wait must run out, report the timeout to the host,
stop the second waiter early, and leave the context usable for the real kernels."""
import numpy as np
import pytest
import torch

import oracle
from attention_kl_divergence_02_b200 import binding, inputs

from parity import KL_TOL, LSE_TOL

pytestmark = pytest.mark.gpu

LIMIT_NS = 2_000_000_000
STAGGER_NS = 500_000_000


def test_waits_pass_when_the_barrier_completes():
    rc, ns = binding.streamkl_selftest_watchdog(0)
    assert rc == binding.OK
    assert max(ns) < 100_000_000
    assert binding.streamkl_device_status() == binding.OK


def test_starved_wait_times_out_and_stops_the_other_waiter():
    rc, ns = binding.streamkl_selftest_watchdog(1)
    assert rc == binding.ERR_TIMEOUT, binding.status_string(rc)
    # the first wait ran out its own limit ...
    assert LIMIT_NS <= ns[0] < LIMIT_NS + 500_000_000
    # ... the second, started 0.5 s later, gave up when the first raised the abort flag,
    # well before its own limit
    assert ns[1] < LIMIT_NS - STAGGER_NS + 200_000_000
    # the status word was read and cleared by the self-test
    assert binding.streamkl_device_status() == binding.OK


def test_context_usable_after_a_timeout():
    rc, _ = binding.streamkl_selftest_watchdog(1)
    assert rc == binding.ERR_TIMEOUT
    w = inputs.WORKLOADS["tiny"]
    t = inputs.make(w, device="cuda")
    kl, l1, l2 = binding.fwd(t["q1"], t["k1"], t["q2"], t["k2"], scale=w.scale, causal=w.causal)
    assert binding.streamkl_device_status() == binding.OK
    okl, ol1, ol2 = oracle.fwd(*[inputs.to_f64(t[k]) for k in ("q1", "k1", "q2", "k2")],
                               scale=w.scale, causal=w.causal)
    gkl = kl.double().cpu().numpy()
    assert np.max(np.abs(gkl - okl) / np.maximum(1, np.abs(okl))) <= KL_TOL
    assert np.max(np.abs(l1.double().cpu().numpy() - ol1)) <= LSE_TOL
    assert np.max(np.abs(l2.double().cpu().numpy() - ol2)) <= LSE_TOL


def test_exponential_probe_rates_are_plausible():
    """The exp2 throughput probe bench.py divides by: both paths run, count their work and
    land in a plausible band (tens of exp2 per clock per SM at most)."""
    import torch
    for kind in (0, 1):
        rc, n = binding.streamkl_probe_exp2(kind, 200)
        assert rc == binding.OK and n == 4 * binding.streamkl_num_sms() * 256 * 8 * 200
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        rc, n = binding.streamkl_probe_exp2(kind, 4000)
        b.record()
        torch.cuda.synchronize()
        per_clk_sm = n / (a.elapsed_time(b) * 1e-3) / binding.streamkl_num_sms() / 2.0e9
        assert 2.0 < per_clk_sm < 64.0, (kind, per_clk_sm)
    assert binding.streamkl_probe_exp2(2, 10)[0] == binding.ERR_INVALID_ARG
    assert binding.streamkl_probe_exp2(0, 0)[0] == binding.ERR_INVALID_ARG
    assert binding.streamkl_device_status() == binding.OK


def test_clock_probe_reads_a_plausible_clock_beside_a_kernel():
    """The clock probe, on a stream of its own beside a forward, records monotone time and
    cycle stamps at about the requested interval and an SM clock between 0.3 and 2.2 GHz;
    the forward beside it still matches the oracle."""
    w = inputs.variant(inputs.WORKLOADS["headline"], Hq=2, Hkv=2, NQ=4096, NK=4096)
    t = inputs.make(w, device="cuda")
    kl, l1, l2 = (torch.empty((w.B, w.Hq, w.NQ), device="cuda") for _ in range(3))
    samples = torch.zeros(2 + 2 * 400, dtype=torch.int64, device="cuda")
    side = torch.cuda.Stream()
    for bad in (torch.zeros(800, dtype=torch.float32, device="cuda"),
                torch.zeros(4, dtype=torch.int64, device="cuda"), torch.zeros(800, dtype=torch.int64)):
        with pytest.raises(ValueError):
            binding.streamkl_probe_clock(20_000_000, 100_000, bad, side)
    assert binding.streamkl_probe_clock(20_000_000, 100_000, samples, side) == binding.OK
    for _ in range(5):
        binding.fwd(t["q1"], t["k1"], t["q2"], t["k2"], scale=w.scale, causal=True, out=(kl, l1, l2))
    torch.cuda.synchronize()
    h = samples.cpu().tolist()
    n = h[0]
    assert 100 <= n <= 400, n
    ts = [h[2 + 2 * i] for i in range(n)]
    cs = [h[3 + 2 * i] for i in range(n)]
    assert all(b > a for a, b in zip(ts, ts[1:])) and all(b > a for a, b in zip(cs, cs[1:]))
    assert 19e6 <= ts[-1] - ts[0] <= 21e6
    gaps = sorted(b - a for a, b in zip(ts, ts[1:]))
    assert 90_000 <= gaps[len(gaps) // 2] <= 150_000
    mhz = (cs[-1] - cs[0]) / (ts[-1] - ts[0]) * 1e3
    assert 300 < mhz < 2200, mhz
    assert binding.streamkl_device_status() == binding.OK
    rows = np.arange(0, w.B * w.Hq * w.NQ, 97)
    okl, ol1, _ = oracle.fwd_rows(*[inputs.to_f64(t[k]) for k in ("q1", "k1", "q2", "k2")], rows,
                                  scale=w.scale, causal=True)
    gkl = kl.double().cpu().numpy().reshape(-1)[rows]
    assert np.max(np.abs(gkl - okl) / np.maximum(1, np.abs(okl))) <= KL_TOL
    assert np.max(np.abs(l1.double().cpu().numpy().reshape(-1)[rows] - ol1)) <= LSE_TOL
