"""One-pass symmetric divergence (streamkl_fwd_sym): KL(P1||P2) and KL(P2||P1) from a single
pass over the keys, through the C ABI, against the fp64 oracle in both directions (the oracle's
reverse direction and the sum are pinned against materialised softmaxes on the CPU)."""
import numpy as np
import pytest

import oracle
from attention_kl_divergence_02_b200 import binding, inputs

from parity import check_fwd, host64

pytestmark = pytest.mark.gpu

CASES = [
    # B, Hq, Hkv, NQ, NK, d, causal, shared
    (1, 2, 2, 640, 640, 128, True, True),
    (1, 2, 2, 300, 1000, 128, False, False),
    (2, 4, 2, 333, 300, 64, False, False),     # GQA, ragged
    (1, 3, 1, 129, 129, 64, True, True),
    (1, 2, 2, 100, 700, 128, False, True),     # one query tile, several key tiles
    (1, 1, 1, 20, 500, 128, False, False),     # at most 32 rows
    (1, 2, 2, 5, 900, 128, False, True),       # at most 8 rows: keys as MMA rows
    (1, 2, 2, 8, 8, 64, True, False),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "B%dHq%dHkv%dNQ%dNK%dd%d%s%s" % (
    c[0], c[1], c[2], c[3], c[4], c[5], "c" if c[6] else "", "s" if c[7] else ""))
def test_both_directions_match_oracle(case):
    B, Hq, Hkv, NQ, NK, d, causal, shared = case
    w = inputs.custom(B, Hq, Hkv, NQ, NK, d, causal, shared, seed=31 + NQ + NK + d)
    t = inputs.make(w, device="cuda")
    kl12, kl21, l1, l2 = (x.cpu().double().numpy()
                          for x in binding.fwd_sym(t["q1"], t["k1"], t["q2"], t["k2"], scale=w.scale,
                                                   causal=w.causal))
    assert binding.streamkl_device_status() == binding.OK
    h = {k: host64(v) for k, v in t.items()}
    o12, ol1, ol2 = oracle.fwd(h["q1"], h["k1"], h["q2"], h["k2"], scale=w.scale, causal=w.causal)
    o21, _, _ = oracle.fwd(h["q2"], h["k2"], h["q1"], h["k1"], scale=w.scale, causal=w.causal)
    check_fwd((kl12, l1, l2), (o12, ol1, ol2), "sym 12 %s" % (case,))
    check_fwd((kl21, l2, l1), (o21, ol2, ol1), "sym 21 %s" % (case,))
    sym = kl12 + kl21
    assert np.all(sym >= -4e-3)


def test_agrees_with_the_one_direction_forward():
    w = inputs.custom(1, 4, 4, 512, 512, 128, True, True, seed=77)
    t = inputs.make(w, device="cuda")
    kl12, kl21, l1, l2 = binding.fwd_sym(t["q1"], t["k1"], t["q2"], t["k2"], causal=True)
    a, b1, b2 = binding.fwd(t["q1"], t["k1"], t["q2"], t["k2"], causal=True)
    r, _, _ = binding.fwd(t["q2"], t["k2"], t["q1"], t["k1"], causal=True)
    assert binding.streamkl_device_status() == binding.OK
    for x, y in ((kl12, a), (l1, b1), (l2, b2), (kl21, r)):
        assert (x - y).abs().max().item() <= 1e-4
