"""Backward parity (both settings): the CUDA path through the C ABI against the fp64 oracle.
Relative L2 error of dQ and dK per (batch, head) slice <= 1e-2."""
import numpy as np
import pytest
import torch

import oracle
from attention_kl_divergence_02_b200 import binding, inputs

from parity import GRAD_TOL, check_grad, host64, rel_l2

pytestmark = pytest.mark.gpu


def gpu_bwd(t, w, mode, workspace=None):
    kl, l1, l2 = binding.fwd(t["q1"], t["k1"], t["q2"], t["k2"], scale=w.scale, causal=w.causal)
    dq, dk = binding.bwd(mode, t["q1"], t["k1"], t["q2"], t["k2"], kl, l1, l2, t["dkl"],
                         scale=w.scale, causal=w.causal, workspace=workspace)
    assert binding.streamkl_device_status() == binding.OK
    return dq.cpu().double().numpy(), dk.cpu().double().numpy()


def host(t):
    return {k: host64(v) for k, v in t.items()}


@pytest.mark.parametrize("mode", [1, 2])
def test_tiny_workload(mode):
    w = inputs.WORKLOADS["tiny"]
    t = inputs.make(w, device="cuda")
    dq, dk = gpu_bwd(t, w, mode)
    h = host(t)
    odq, odk = oracle.bwd(mode, h["q1"], h["k1"], h["q2"], h["k2"], h["dkl"], scale=w.scale,
                          causal=w.causal)
    check_grad(dq, odq, "tiny dQ mode %d" % mode)
    check_grad(dk, odk, "tiny dK mode %d" % mode)


CASES = [
    # B, Hq, Hkv, NQ, NK, d, causal, shared
    (1, 2, 2, 640, 640, 128, False, False),
    (1, 2, 2, 640, 640, 128, True, False),
    (1, 2, 2, 640, 640, 128, True, True),
    (2, 4, 2, 300, 333, 64, False, False),     # GQA, ragged rows and keys
    (1, 4, 1, 200, 520, 64, False, True),      # GQA 4:1, shared keys
    (1, 3, 1, 129, 129, 64, True, True),
    (1, 2, 2, 257, 257, 128, True, False),
    (1, 1, 1, 1, 1, 128, False, True),
    (1, 1, 1, 40, 40, 128, True, True),
    (1, 2, 1, 3, 700, 128, False, False),
    # d = 64 with an even KV-group size: two query heads per CTA (their dK partials summed on
    # chip); causal with a ragged last tile, 4:1 shared keys, and two KV groups with B = 2
    (1, 4, 2, 333, 333, 64, True, False),
    (1, 8, 2, 257, 257, 64, True, True),
    (2, 4, 2, 130, 1000, 64, False, False),
    (1, 8, 1, 200, 700, 64, False, False),     # 8:1: four head pairs share one KV head
]


@pytest.mark.parametrize("mode", [1, 2])
@pytest.mark.parametrize("case", CASES, ids=lambda c: "B%dHq%dHkv%dNQ%dNK%dd%d%s%s" % (
    c[0], c[1], c[2], c[3], c[4], c[5], "c" if c[6] else "", "s" if c[7] else ""))
def test_shapes(case, mode):
    B, Hq, Hkv, NQ, NK, d, causal, shared = case
    w = inputs.custom(B, Hq, Hkv, NQ, NK, d, causal, shared, seed=NQ * 7 + NK + d)
    t = inputs.make(w, device="cuda")
    # non-uniform upstream gradient
    t["dkl"] = torch.rand(t["dkl"].shape, generator=torch.Generator().manual_seed(1)).cuda() + 0.5
    dq, dk = gpu_bwd(t, w, mode)
    h = host(t)
    odq, odk = oracle.bwd(mode, h["q1"], h["k1"], h["q2"], h["k2"], h["dkl"], scale=w.scale,
                          causal=w.causal)
    # natural size of a gradient entry is scale * g * |q| * |k|; fp32 rounding of the saved
    # statistics leaves noise around 1e-7 of that where the exact gradient is zero
    zero_atol = 1e-6 * w.scale * float(h["dkl"].max()) * max(np.abs(h["q1"]).max(), np.abs(h["q2"]).max()) \
        * max(np.abs(h["k1"]).max(), np.abs(h["k2"]).max())
    check_grad(dq, odq, "%s dQ mode %d" % (case, mode), zero_atol)
    check_grad(dk, odk, "%s dK mode %d" % (case, mode), zero_atol)


def test_workspace_contents_do_not_matter():
    w = inputs.custom(1, 2, 2, 384, 384, 128, True, True, seed=4)
    t = inputs.make(w, device="cuda")
    n = binding.streamkl_bwd_workspace_bytes(1, 2, 2, 384, 384, 128) // 4
    ws = torch.full((n,), float("nan"), device="cuda")
    a = gpu_bwd(t, w, 1, workspace=ws)
    ws.fill_(1e30)
    b = gpu_bwd(t, w, 1, workspace=ws)
    for x, y in zip(a, b):
        assert np.all(np.isfinite(x))
        assert rel_l2(x, y, axes=(2, 3)).max() < 1e-3


def test_identical_distributions_give_zero_gradient():
    """P1 = P2 has zero gradient in both settings; on the GPU it vanishes to the rounding of
    the fp32 statistics (the two sides take some exponentials on different units), i.e.
    far below the gradient of the same call with distinct distributions."""
    w = inputs.custom(1, 2, 2, 256, 256, 128, True, True, seed=12)
    t = inputs.make(w, device="cuda")
    for mode in (1, 2):
        kl, l1, l2 = binding.fwd(t["q1"], t["k1"], t["q2"], t["k2"], causal=True)
        dq_ref, dk_ref = binding.bwd(mode, t["q1"], t["k1"], t["q2"], t["k2"], kl, l1, l2, t["dkl"], causal=True)
        kl, l1, l2 = binding.fwd(t["q1"], t["k1"], t["q1"], t["k1"], causal=True)
        dq, dk = binding.bwd(mode, t["q1"], t["k1"], t["q1"], t["k1"], kl, l1, l2, t["dkl"], causal=True)
        torch.cuda.synchronize()
        assert dq.abs().max().item() <= 1e-4 * dq_ref.abs().max().item()
        assert dk.abs().max().item() <= 1e-4 * dk_ref.abs().max().item()


def test_extra_memory_is_only_the_workspace():
    w = inputs.custom(1, 8, 8, 2048, 2048, 128, True, True, seed=9)
    t = inputs.make(w, device="cuda")
    kl, l1, l2 = binding.fwd(t["q1"], t["k1"], t["q2"], t["k2"], causal=True)
    n = binding.streamkl_bwd_workspace_bytes(1, 8, 8, 2048, 2048, 128) // 4
    ws = torch.empty(n, device="cuda")
    out = (torch.empty_like(t["q1"]), torch.empty_like(t["k1"]))
    binding.bwd(1, t["q1"], t["k1"], t["q2"], t["k2"], kl, l1, l2, t["dkl"], causal=True, out=out, workspace=ws)
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    alloc0 = torch.cuda.memory_allocated()
    binding.bwd(1, t["q1"], t["k1"], t["q2"], t["k2"], kl, l1, l2, t["dkl"], causal=True, out=out, workspace=ws)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert torch.cuda.memory_allocated() == alloc0
    assert free1 >= free0


def sampled_check(name, mode, causal=None, heads_for_dk=1, rows_per_head=32, keys_per_head=48):
    base = inputs.WORKLOADS[name]
    w = base if causal is None else inputs.variant(base, causal=causal)
    t = inputs.make(w, device="cuda")
    dq, dk = gpu_bwd(t, w, mode)
    h = host(t)
    rng = np.random.default_rng(7 + mode)
    d = w.d
    # dQ: sampled rows of every (b, head); each oracle row needs only its own row
    rows = np.concatenate([bh * w.NQ + rng.choice(w.NQ, rows_per_head, replace=False)
                           for bh in range(w.B * w.Hq)])
    odq = oracle.bwd_dq_rows(mode, h["q1"], h["k1"], h["q2"], h["k2"], h["dkl"], rows,
                             scale=w.scale, causal=w.causal)
    gdq = dq.reshape(-1, d)[rows]
    e = rel_l2(gdq.reshape(w.B * w.Hq, rows_per_head, d)[None], odq.reshape(w.B * w.Hq, rows_per_head, d)[None], axes=(2, 3))
    assert e.max() <= GRAD_TOL, "%s dQ rel-L2 %.3g" % (name, e.max())
    # dK: sampled keys of the first (and, with heads_for_dk = 2, the last) (b, KV head): the
    # first and last planes of the backward's grouped plane schedule
    units = [0] if heads_for_dk < 2 else [0, w.B * w.Hkv - 1]
    keys = np.concatenate([u * w.NK + rng.choice(w.NK, keys_per_head, replace=False) for u in units])
    odk = oracle.bwd_dk_keys(mode, h["q1"], h["k1"], h["q2"], h["k2"], h["dkl"], keys,
                             scale=w.scale, causal=w.causal)
    gdk = dk.reshape(-1, d)[keys]
    e = rel_l2(gdk.reshape(len(units), keys_per_head, d)[None], odk.reshape(len(units), keys_per_head, d)[None], axes=(2, 3))
    assert e.max() <= GRAD_TOL, "%s dK rel-L2 %.3g" % (name, e.max())
    assert np.all(np.isfinite(dq)) and np.all(np.isfinite(dk))


@pytest.mark.parametrize("causal", [False, True])
def test_full_size_b2h8n4k_mode1(causal):
    sampled_check("b2h8n4k", 1, causal=causal, heads_for_dk=2)


@pytest.mark.parametrize("mode", [1, 2])
def test_full_size_headline(mode):
    sampled_check("headline", mode, heads_for_dk=2)


def test_full_size_gqa_mode2():
    sampled_check("gqa", 2, heads_for_dk=2, rows_per_head=16, keys_per_head=32)


SIGN_CASES = [
    # B, Hq, Hkv, NQ, NK, d, causal, shared
    (1, 2, 2, 300, 700, 128, False, False),
    (1, 1, 1, 640, 640, 128, True, True),      # key ranges per query tile (few query tiles)
    (2, 4, 2, 129, 260, 64, False, True),
]


@pytest.mark.parametrize("mode", [1, 2])
@pytest.mark.parametrize("kind", ["signed", "zeros"])
@pytest.mark.parametrize("case", SIGN_CASES, ids=lambda c: "NQ%dNK%dd%d%s" % (c[3], c[4], c[5], "c" if c[6] else ""))
def test_upstream_gradient_signs_and_zeros(case, kind, mode):
    """g of both signs takes the path that multiplies by g (a warp with any g < 0 cannot fold
    log2 g into the exponent); g = 0 on every third row must give those rows exactly zero
    dQ (their dS is zeroed, not computed from log2 0 = -inf)."""
    B, Hq, Hkv, NQ, NK, d, causal, shared = case
    w = inputs.custom(B, Hq, Hkv, NQ, NK, d, causal, shared, seed=NQ + NK + d + 1)
    t = inputs.make(w, device="cuda")
    gen = torch.Generator().manual_seed(17)
    if kind == "signed":
        g = torch.randn(t["dkl"].shape, generator=gen)
    else:
        g = torch.rand(t["dkl"].shape, generator=gen) + 0.25
        g[..., ::3] = 0.0
    t["dkl"] = g.cuda()
    dq, dk = gpu_bwd(t, w, mode)
    h = host(t)
    odq, odk = oracle.bwd(mode, h["q1"], h["k1"], h["q2"], h["k2"], h["dkl"], scale=w.scale,
                          causal=w.causal)
    zero_atol = 1e-6 * w.scale * float(np.abs(h["dkl"]).max()) * max(np.abs(h["q1"]).max(), np.abs(h["q2"]).max()) \
        * max(np.abs(h["k1"]).max(), np.abs(h["k2"]).max())
    check_grad(dq, odq, "%s %s dQ mode %d" % (case, kind, mode), zero_atol)
    check_grad(dk, odk, "%s %s dK mode %d" % (case, kind, mode), zero_atol)
    if kind == "zeros":
        assert np.abs(dq[..., ::3, :]).max() == 0.0


def test_binding_refuses_mismatched_tensors_before_launch():
    """The Python wrappers check every tensor the kernels would read or write (dtype, shape,
    contiguity, device) and the workspace size before calling the library."""
    w = inputs.custom(1, 2, 2, 128, 128, 64, False, True, seed=3)
    t = inputs.make(w, device="cuda")
    kl, l1, l2 = binding.fwd(t["q1"], t["k1"], t["q2"], t["k2"])
    with pytest.raises(ValueError):
        binding.fwd(t["q1"], t["k1"], t["q2"], t["k2"], out=(kl, l1, torch.empty(1, 2, 64, device="cuda")))
    with pytest.raises(ValueError):
        binding.bwd(1, t["q1"], t["k1"], t["q2"], t["k2"], kl, l1, l2, t["dkl"].half())
    with pytest.raises(ValueError):
        binding.bwd(1, t["q1"], t["k1"], t["q2"], t["k2"], kl, l1, l2, t["dkl"],
                    out=(torch.empty_like(t["q1"]), torch.empty(1, 2, 64, 64, dtype=torch.bfloat16, device="cuda")))
    need = binding.streamkl_bwd_workspace_bytes(1, 2, 2, 128, 128, 64)
    with pytest.raises(ValueError):
        binding.bwd(1, t["q1"], t["k1"], t["q2"], t["k2"], kl, l1, l2, t["dkl"],
                    workspace=torch.empty(need // 4 - 1, device="cuda"))
    # keys that disagree with the queries: a smaller batch, another head dim, a KV head count
    # that does not divide the query heads -- each would size a tensor map past an allocation
    bf = dict(dtype=torch.bfloat16, device="cuda")
    for k in (torch.zeros(2, 2, 128, 64, **bf), torch.zeros(1, 2, 128, 32, **bf),
              torch.zeros(1, 3, 128, 64, **bf)):
        for call in (lambda: binding.fwd(t["q1"], k, t["q2"], k),
                     lambda: binding.fwd_splitk(t["q1"], k, t["q2"], k),
                     lambda: binding.bwd(1, t["q1"], k, t["q2"], k, kl, l1, l2, t["dkl"])):
            with pytest.raises(ValueError):
                call()
    w2 = inputs.custom(1, 2, 2, 1, 1024, 64, False, True, seed=4)     # 8 key tiles: a real split
    t2 = inputs.make(w2, device="cuda")
    assert binding.streamkl_fwd_splitk_workspace_bytes(1, 2, 1, 1024, 2) > 4
    with pytest.raises(ValueError):
        binding.fwd_splitk(t2["q1"], t2["k1"], t2["q2"], t2["k2"], splits=2,
                           workspace=torch.empty(1, device="cuda"))
    assert binding.streamkl_device_status() == binding.OK


@pytest.mark.parametrize("mode", [1, 2])
def test_reverse_kl_backward_by_swapping_the_distributions(mode):
    """The gradient of KL(P2||P1): the same calls with the two distributions' arguments
    swapped (forward, then backward with the swapped saved state), against the oracle's
    backward on the swapped inputs.  Mode 1 then holds P2 fixed and trains (Q1, K1); mode 2
    holds P1 fixed and trains (Q2, K2)."""
    w = inputs.custom(1, 2, 2, 300, 300, 128, True, False, seed=43)
    t = inputs.make(w, device="cuda")
    t["dkl"] = torch.rand(t["dkl"].shape, generator=torch.Generator().manual_seed(5)).cuda() + 0.5
    kl, l2, l1 = binding.fwd(t["q2"], t["k2"], t["q1"], t["k1"], scale=w.scale, causal=True)
    dq, dk = binding.bwd(mode, t["q2"], t["k2"], t["q1"], t["k1"], kl, l2, l1, t["dkl"],
                         scale=w.scale, causal=True)
    assert binding.streamkl_device_status() == binding.OK
    h = host(t)
    odq, odk = oracle.bwd(mode, h["q2"], h["k2"], h["q1"], h["k1"], h["dkl"], scale=w.scale,
                          causal=True)
    check_grad(dq.cpu().double().numpy(), odq, "reverse KL dQ mode %d" % mode)
    check_grad(dk.cpu().double().numpy(), odk, "reverse KL dK mode %d" % mode)
