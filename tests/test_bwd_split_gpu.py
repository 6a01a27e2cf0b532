"""The backward for few query tiles and many keys: when one CTA per 128-row query tile would
leave SMs idle, the library splits each tile's key tiles into ranges (one CTA each); dK is
reduced as always and dQ, instead of being written once from TMEM, is added into an fp32
workspace and converted afterwards.  Checked through the C ABI against the fp64 oracle on
shapes that take that path (the workspace size shows it), including a causal one whose
ranges past the diagonal see no keys at all, and a prefill-chunk shape at full size against
sampled rows and keys."""
import numpy as np
import pytest
import torch

import oracle
from attention_kl_divergence_02_b200 import binding, inputs

from parity import GRAD_TOL, check_grad, host64, rel_l2

pytestmark = pytest.mark.gpu


def dk_bytes(w):
    return w.B * w.Hkv * ((w.NK + 127) // 128 * 128) * w.d * 4


def splits_in_use(w):
    return binding.streamkl_bwd_workspace_bytes(w.B, w.Hq, w.Hkv, w.NQ, w.NK, w.d) > dk_bytes(w)


CASES = [
    # B, Hq, Hkv, NQ, NK, d, causal, shared
    (1, 2, 2, 128, 4096, 128, False, False),
    (1, 1, 1, 200, 3000, 64, False, True),      # two query tiles, ragged rows
    (1, 2, 1, 64, 5000, 128, False, True),      # GQA, ragged keys
    (1, 1, 1, 640, 640, 128, True, True),       # causal: late ranges of early tiles are empty
    (2, 2, 2, 130, 1900, 64, False, False),
    (1, 4, 2, 200, 4000, 64, False, False),     # two query heads per CTA, key ranges
    (1, 4, 2, 384, 384, 64, True, True),        # the same, causal
]


@pytest.mark.parametrize("mode", [1, 2])
@pytest.mark.parametrize("case", CASES, ids=lambda c: "B%dHq%dHkv%dNQ%dNK%dd%d%s%s" % (
    c[0], c[1], c[2], c[3], c[4], c[5], "c" if c[6] else "", "s" if c[7] else ""))
def test_split_backward_matches_oracle(case, mode):
    B, Hq, Hkv, NQ, NK, d, causal, shared = case
    w = inputs.custom(B, Hq, Hkv, NQ, NK, d, causal, shared, seed=NQ + 3 * NK + d)
    assert splits_in_use(w)
    t = inputs.make(w, device="cuda")
    t["dkl"] = torch.rand(t["dkl"].shape, generator=torch.Generator().manual_seed(NQ)).cuda() + 0.25
    kl, l1, l2 = binding.fwd(t["q1"], t["k1"], t["q2"], t["k2"], scale=w.scale, causal=causal)
    dq, dk = binding.bwd(mode, t["q1"], t["k1"], t["q2"], t["k2"], kl, l1, l2, t["dkl"],
                         scale=w.scale, causal=causal)
    assert binding.streamkl_device_status() == binding.OK
    h = {k: host64(v) for k, v in t.items()}
    odq, odk = oracle.bwd(mode, h["q1"], h["k1"], h["q2"], h["k2"], h["dkl"], scale=w.scale,
                          causal=causal)
    check_grad(dq.cpu().double().numpy(), odq, "split dQ %s mode %d" % (case, mode), zero_atol=1e-6)
    check_grad(dk.cpu().double().numpy(), odk, "split dK %s mode %d" % (case, mode), zero_atol=1e-6)


def test_prefill_chunk_full_size_sampled():
    """B1 H16 NQ=512 NK=65536 d128 (a chunk of queries against a long context), mode 1, in
    the launch configuration the benchmark times: dQ on sampled rows and dK on sampled keys."""
    w = inputs.WORKLOADS["chunk"]
    assert splits_in_use(w)
    t = inputs.make(w, device="cuda")
    kl, l1, l2 = binding.fwd(t["q1"], t["k1"], t["q2"], t["k2"], scale=w.scale)
    dq, dk = binding.bwd(1, t["q1"], t["k1"], t["q2"], t["k2"], kl, l1, l2, t["dkl"], scale=w.scale)
    torch.cuda.synchronize()
    assert binding.streamkl_device_status() == binding.OK
    rng = np.random.default_rng(5)
    for hd in (0, 9):
        sl = lambda x: host64(x[:, hd:hd + 1])
        q1, q2, k = sl(t["q1"]), sl(t["q2"]), sl(t["k1"])
        g = host64(t["dkl"][:, hd:hd + 1])
        rows = np.unique(np.concatenate([[0, w.NQ - 1], rng.choice(w.NQ, 14, replace=False)]))
        odq = oracle.bwd_dq_rows(1, q1, k, q2, k, g, rows, scale=w.scale)
        gdq = dq[0, hd].float().cpu().double().numpy()[rows]
        assert rel_l2(gdq[None, None], odq[None, None], axes=(2, 3)).max() <= GRAD_TOL
        keys = np.unique(np.concatenate([[0, w.NK - 1], rng.choice(w.NK, 14, replace=False)]))
        odk = oracle.bwd_dk_keys(1, q1, k, q2, k, g, keys, scale=w.scale)
        gdk = dk[0, hd].float().cpu().double().numpy()[keys]
        assert rel_l2(gdk[None, None], odk[None, None], axes=(2, 3)).max() <= GRAD_TOL
