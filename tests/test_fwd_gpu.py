"""Forward parity: the CUDA path (through the C ABI) against the fp64 oracle."""
import math

import numpy as np
import pytest
import torch

import oracle
from attention_kl_divergence_02_b200 import binding, inputs

from parity import check_fwd, host64, run_fwd

pytestmark = pytest.mark.gpu


def both(w):
    t = inputs.make(w, device="cuda")
    got = run_fwd(t, w)
    want = oracle.fwd(host64(t["q1"]), host64(t["k1"]), host64(t["q2"]), host64(t["k2"]),
                      scale=w.scale, causal=w.causal)
    return got, want, t


def test_tiny_workload():
    w = inputs.WORKLOADS["tiny"]
    got, want, _ = both(w)
    check_fwd(got, want, "tiny")


CASES = [
    # B, Hq, Hkv, NQ, NK, d, causal, shared
    (1, 2, 2, 640, 640, 128, False, False),
    (1, 2, 2, 640, 640, 128, True, False),
    (1, 2, 2, 640, 640, 128, True, True),
    (2, 4, 2, 300, 333, 64, False, False),     # GQA, ragged rows and keys
    (1, 3, 1, 129, 129, 64, True, True),       # one row past a tile, causal
    (1, 2, 2, 257, 257, 128, True, False),     # one row past a 256-row CTA block
    (1, 1, 1, 1, 1, 128, False, True),         # single key, single row
    (1, 1, 1, 1, 1000, 64, False, False),      # single row, ragged keys
    (1, 2, 1, 200, 1, 64, False, False),       # single key
    (1, 1, 1, 40, 40, 128, True, True),        # smaller than one tile
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "B%dHq%dHkv%dNQ%dNK%dd%d%s%s" % (
    c[0], c[1], c[2], c[3], c[4], c[5], "c" if c[6] else "", "s" if c[7] else ""))
def test_shapes(case):
    B, Hq, Hkv, NQ, NK, d, causal, shared = case
    w = inputs.custom(B, Hq, Hkv, NQ, NK, d, causal, shared, seed=NQ + NK + d)
    got, want, _ = both(w)
    check_fwd(got, want, str(case))


def test_peaked_and_flat_rows():
    """Per-head scaled queries (the grouped-query recipe) at a reduced size: peaked rows
    (large scale) and flat rows (small scale) in one call."""
    w = inputs.custom(2, 8, 2, 384, 1000, 64, False, False, seed=11, head_scaled=True)
    got, want, _ = both(w)
    check_fwd(got, want, "peaked")


def test_score_jumps_above_the_running_maximum():
    """Rows whose scores jump far above the maximum of the keys before them, in a later key
    tile, so the online rescale must carry the earlier sums down by that much: row 0 jumps by
    ~131 binary orders (2^-131 underflows fp32 -- the earlier keys must drop out, not turn
    into NaN), row 1 by ~78, row 2 by ~49; the other rows see moderate scores from the same
    keys.  Both distributions against the oracle, shared keys and distinct ones."""
    for shared in (True, False):
        w = inputs.custom(1, 1, 1, 256, 1024, 128, False, shared, seed=21)
        t = inputs.make(w, device="cpu")
        q1 = t["q1"].float()
        keys = {"k1": t["k1"].float() * 0.1}
        if not shared:
            keys["k2"] = t["k2"].float() * 0.1
        for key, row, c in ((700, 0, 8.0), (900, 1, 4.8), (950, 2, 3.0)):
            # a key along the row's query, scaled so that scale * <q1, k> = c * 128 * scale
            # nats = 16.3 * c binary orders above the earlier keys' near-zero scores
            qr = q1[0, 0, row]
            for name in keys:
                keys[name][0, 0, key] = c * 128.0 * qr / float(qr @ qr)
        t["k1"] = keys["k1"].to(torch.bfloat16)
        t["k2"] = t["k1"] if shared else keys["k2"].to(torch.bfloat16)
        t = {k: v.cuda() for k, v in t.items()}
        if shared:
            t["k2"] = t["k1"]
        got = run_fwd(t, w)
        want = oracle.fwd(host64(t["q1"]), host64(t["k1"]), host64(t["q2"]), host64(t["k2"]),
                          scale=w.scale, causal=False)
        check_fwd(got, want, "score jumps, shared=%s" % shared)
        # the jumps are as large as intended: LSE1 of rows 0-2 far above the others
        assert got[1][0, 0, 0] > 80 and got[1][0, 0, 1] > 45 and got[1][0, 0, 2] > 28


def test_identical_inputs_give_zero_kl():
    w = inputs.custom(1, 2, 2, 300, 300, 128, True, True, seed=3)
    t = inputs.make(w, device="cuda")
    kl, l1, l2 = binding.fwd(t["q1"], t["k1"], t["q1"], t["k1"], scale=w.scale, causal=True)
    torch.cuda.synchronize()
    # the two distributions take part of their exponentials on different units (exponential
    # unit vs FMA-pipe polynomial), so the identity holds to fp32 rounding, not bitwise
    assert (l1 - l2).abs().max().item() <= 1e-5
    assert kl.abs().max().item() <= 1e-5


def test_causal_row_zero_and_nonnegative():
    w = inputs.custom(1, 4, 4, 512, 512, 128, True, False, seed=5)
    t = inputs.make(w, device="cuda")
    kl, l1, l2 = binding.fwd(t["q1"], t["k1"], t["q2"], t["k2"], scale=w.scale, causal=True)
    kl = kl.cpu()
    assert torch.all(kl[:, :, 0].abs() <= 1e-6)
    assert kl.min() >= -2e-3
    s00 = (t["q1"][0, :, 0].float() * t["k1"][0, :, 0].float()).sum(-1) * w.scale
    assert torch.allclose(l1[0, :, 0].cpu(), s00.cpu(), atol=1e-3)


def test_deterministic():
    w = inputs.custom(1, 4, 4, 512, 512, 128, True, True, seed=6)
    t = inputs.make(w, device="cuda")
    a = binding.fwd(t["q1"], t["k1"], t["q2"], t["k2"], scale=w.scale, causal=True)
    b = binding.fwd(t["q1"], t["k1"], t["q2"], t["k2"], scale=w.scale, causal=True)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_non_default_scale_and_stream():
    w = inputs.custom(1, 2, 2, 256, 384, 128, False, False, seed=8)
    t = inputs.make(w, device="cuda")
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        got = binding.fwd(t["q1"], t["k1"], t["q2"], t["k2"], scale=0.3, causal=False, stream=s)
    s.synchronize()
    want = oracle.fwd(host64(t["q1"]), host64(t["k1"]), host64(t["q2"]), host64(t["k2"]), scale=0.3)
    check_fwd(tuple(x.cpu().double().numpy() for x in got), want, "scale0.3")


def test_no_extra_device_memory():
    """The forward allocates nothing: torch's allocator sees no growth and the free device
    memory reported by the driver does not drop across the call."""
    w = inputs.custom(1, 8, 8, 2048, 2048, 128, True, True, seed=9)
    t = inputs.make(w, device="cuda")
    out = tuple(torch.empty((1, 8, 2048), device="cuda") for _ in range(3))
    binding.fwd(t["q1"], t["k1"], t["q2"], t["k2"], causal=True, out=out)  # warm
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    alloc0 = torch.cuda.memory_allocated()
    binding.fwd(t["q1"], t["k1"], t["q2"], t["k2"], causal=True, out=out)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert torch.cuda.memory_allocated() == alloc0
    assert free1 >= free0


@pytest.mark.parametrize("name", ["b2h8n4k", "headline", "gqa"])
def test_full_size_sampled(name):
    """Full-size workloads in the launch configuration the benchmark times; the oracle
    checks 64 seeded random rows per (batch, head)."""
    base = inputs.WORKLOADS[name]
    for causal in ((False, True) if name == "b2h8n4k" else (base.causal,)):
        w = inputs.variant(base, causal=causal)
        t = inputs.make(w, device="cuda")
        kl, l1, l2 = run_fwd(t, w)
        rng = np.random.default_rng(123)
        rows = []
        for bh in range(w.B * w.Hq):
            rows += list(bh * w.NQ + rng.choice(w.NQ, size=64, replace=False))
        rows += [0, w.NQ - 1, w.B * w.Hq * w.NQ - 1]
        rows = np.array(sorted(set(rows)))
        want = oracle.fwd_rows(host64(t["q1"]), host64(t["k1"]), host64(t["q2"]), host64(t["k2"]),
                               rows, scale=w.scale, causal=w.causal)
        got = tuple(x.reshape(-1)[rows] for x in (kl, l1, l2))
        check_fwd(got, want, "%s causal=%s" % (name, causal))
        assert np.all(kl >= -2e-3)


def test_reverse_kl_by_swapping_the_distributions():
    """KL(P2||P1) through the same call with the two distributions' arguments swapped."""
    w = inputs.custom(1, 2, 2, 300, 300, 128, True, False, seed=41)
    t = inputs.make(w, device="cuda")
    got = binding.fwd(t["q2"], t["k2"], t["q1"], t["k1"], scale=w.scale, causal=True)
    assert binding.streamkl_device_status() == binding.OK
    want = oracle.fwd(host64(t["q2"]), host64(t["k2"]), host64(t["q1"]), host64(t["k1"]),
                      scale=w.scale, causal=True)
    check_fwd(tuple(x.cpu().double().numpy() for x in got), want, "reverse KL")
