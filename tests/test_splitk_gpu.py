"""Split-K forward (streamkl_fwd_splitk): the key tiles cut into ranges folded by separate
CTAs, then merged exactly.  Checked through the C ABI against the fp64 oracle on the same
seeded inputs, at small sizes that span several key ranges and ragged tiles, at the full
decode workload (B1 H16 NQ=1 NK=131072 d128, every row), and against the unsplit forward."""
import numpy as np
import pytest
import torch

import oracle
from attention_kl_divergence_02_b200 import binding, inputs

from parity import check_fwd, host64

pytestmark = pytest.mark.gpu


def _oracle(t, w):
    return oracle.fwd(host64(t["q1"]), host64(t["k1"]), host64(t["q2"]), host64(t["k2"]),
                      scale=w.scale, causal=w.causal)


def _split(t, w, splits):
    out = binding.fwd_splitk(t["q1"], t["k1"], t["q2"], t["k2"], scale=w.scale, causal=w.causal,
                             splits=splits)
    assert binding.streamkl_device_status() == binding.OK
    return tuple(x.cpu().double().numpy() for x in out)


CASES = [
    # B, Hq, Hkv, NQ, NK, d, causal, shared, splits
    (2, 4, 2, 1, 5000, 128, False, False, 0),      # decoding shape, library's choice
    (2, 4, 2, 1, 5000, 128, False, False, 3),      # uneven ranges (40 tiles -> 14, 14, 12)
    (1, 2, 2, 1, 300, 64, False, True, 64),        # more ranges asked than tiles (3)
    (1, 3, 1, 17, 3000, 64, False, True, 5),       # GQA, a few rows
    (1, 2, 2, 300, 1000, 128, False, False, 4),    # two query tiles per block, ragged rows
    (1, 2, 2, 700, 700, 128, True, True, 3),       # causal: early blocks own empty ranges
    (1, 1, 1, 5, 1, 128, False, True, 8),          # one key: one range, no workspace
    # row counts at the layout boundaries: 9 (first past the keys-as-rows kernel), 32 (the
    # last with rows copied into all four lane quarters), 33 (one 128-row query tile)
    (1, 2, 2, 9, 2000, 128, False, True, 0),
    (1, 2, 2, 32, 1500, 64, False, False, 3),
    (1, 2, 2, 33, 1500, 128, False, True, 2),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "B%dHq%dHkv%dNQ%dNK%dd%d%s%s_s%d" % (
    c[0], c[1], c[2], c[3], c[4], c[5], "c" if c[6] else "", "sh" if c[7] else "", c[8]))
def test_matches_oracle(case):
    B, Hq, Hkv, NQ, NK, d, causal, shared, splits = case
    w = inputs.custom(B, Hq, Hkv, NQ, NK, d, causal, shared, seed=7 + NQ + NK)
    t = inputs.make(w, device="cuda")
    check_fwd(_split(t, w, splits), _oracle(t, w), "splitk %s" % (case,))


FEW_ROWS = [
    # B, Hq, Hkv, NQ, NK, d, causal, shared, splits  (at most 8 query rows: keys as MMA rows)
    (1, 3, 3, 2, 700, 128, False, True, 0),
    (2, 4, 2, 8, 1000, 64, False, False, 0),      # GQA, distinct keys
    (1, 2, 2, 5, 5, 128, True, True, 1),          # causal (NQ == NK), one tile
    (1, 2, 2, 8, 8, 64, True, False, 3),          # causal, more ranges asked than tiles
    (1, 1, 1, 3, 129, 128, False, False, 1),      # one range, a ragged second key tile
    (1, 4, 1, 7, 4000, 128, False, True, 5),      # GQA 4:1, shared keys
    (1, 2, 2, 1, 300, 64, False, True, 0),
]


@pytest.mark.parametrize("case", FEW_ROWS, ids=lambda c: "B%dHq%dHkv%dNQ%dNK%dd%d%s%s_s%d" % (
    c[0], c[1], c[2], c[3], c[4], c[5], "c" if c[6] else "", "sh" if c[7] else "", c[8]))
def test_few_rows_matches_oracle(case):
    """At most 8 query rows: split and unsplit forward against the oracle."""
    B, Hq, Hkv, NQ, NK, d, causal, shared, splits = case
    w = inputs.custom(B, Hq, Hkv, NQ, NK, d, causal, shared, seed=11 + NQ + NK + d)
    t = inputs.make(w, device="cuda")
    want = _oracle(t, w)
    check_fwd(_split(t, w, splits), want, "few rows split %s" % (case,))
    got = binding.fwd(t["q1"], t["k1"], t["q2"], t["k2"], scale=w.scale, causal=w.causal)
    assert binding.streamkl_device_status() == binding.OK
    check_fwd(tuple(x.cpu().double().numpy() for x in got), want, "few rows unsplit %s" % (case,))


def test_matches_unsplit_forward():
    w = inputs.custom(2, 4, 4, 64, 4096, 128, False, True, seed=11)
    t = inputs.make(w, device="cuda")
    ref = tuple(x.cpu().double().numpy()
                for x in binding.fwd(t["q1"], t["k1"], t["q2"], t["k2"], scale=w.scale))
    for splits in (2, 5, 32):
        got = _split(t, w, splits)
        for a, b in zip(got, ref):
            assert np.max(np.abs(a - b)) <= 1e-4


def test_decode_workload_every_row():
    """Full decode workload in the configuration the benchmark times (library's choice of
    ranges); the oracle computes all 16 rows."""
    w = inputs.WORKLOADS["decode"]
    t = inputs.make(w, device="cuda")
    assert binding.streamkl_fwd_splits(w.B, w.Hq, w.NQ, w.NK) > 1
    check_fwd(_split(t, w, 0), _oracle(t, w), "decode")


def test_workspace_too_small_is_refused_before_launch():
    w = inputs.custom(1, 2, 2, 1, 4096, 128, False, True, seed=3)
    t = inputs.make(w, device="cuda")
    need = binding.streamkl_fwd_splitk_workspace_bytes(1, 2, 1, 4096, 4)
    assert need == 4 * 5 * 2 * 4
    ws = torch.empty(need // 4 - 4, dtype=torch.float32, device="cuda")
    out = tuple(torch.empty((1, 2, 1), device="cuda") for _ in range(3))
    rc = binding.streamkl_fwd_splitk(t["q1"], t["k1"], t["q2"], t["k2"], 1, 2, 2, 1, 4096, 128,
                                     w.scale, 0, 4, *out, ws, ws.numel() * 4)
    assert rc == binding.ERR_INVALID_ARG


@pytest.mark.parametrize("NQ,NK,causal,d", [(1, 1000, False, 128), (31, 777, False, 64),
                                            (32, 4096, False, 128), (33, 500, False, 128),
                                            (20, 20, True, 128), (7, 7, True, 64)])
def test_few_rows_plain_forward(NQ, NK, causal, d):
    """The unsplit forward at 32 query rows or fewer, where every warp of the warpgroup folds
    a quarter of each key tile and the four partial states are merged in the CTA."""
    w = inputs.custom(2, 2, 1, NQ, NK, d, causal, True, seed=100 + NQ)
    t = inputs.make(w, device="cuda")
    got = tuple(x.cpu().double().numpy()
                for x in binding.fwd(t["q1"], t["k1"], t["q2"], t["k2"], scale=w.scale,
                                     causal=causal))
    assert binding.streamkl_device_status() == binding.OK
    check_fwd(got, _oracle(t, w), "few rows NQ=%d NK=%d" % (NQ, NK))
