"""streamkl_bwd_noalloc: the backward for callers that may not allocate device memory (a
framework allocator that owns the GPU, a fixed memory budget, no room for cudaMalloc's
synchronisation).  It keeps the dK accumulator in the library's built-in 32 MiB buffer
instead of a caller workspace.  Checked here through the C ABI against streamkl_bwd with a
torch-allocated workspace, on two calls in a row (the buffer keeps the previous call's
contents, which must not leak into the next result)."""
import numpy as np
import pytest
import torch

from attention_kl_divergence_02_b200 import binding, inputs

from parity import GRAD_TOL, rel_l2

pytestmark = pytest.mark.gpu


def _fwd(t, w):
    return binding.fwd(t["q1"], t["k1"], t["q2"], t["k2"], scale=w.scale, causal=w.causal)


def _with_workspace(mode, t, w, stats):
    dq, dk = torch.empty_like(t["q1"]), torch.empty_like(t["k1"])
    ws = torch.empty(binding.streamkl_bwd_workspace_bytes(w.B, w.Hq, w.Hkv, w.NQ, w.NK, w.d) // 4, device="cuda")
    rc = binding.streamkl_bwd(mode, t["q1"], t["k1"], t["q2"], t["k2"], *stats, t["dkl"], w.B, w.Hq,
                              w.Hkv, w.NQ, w.NK, w.d, w.scale, w.causal, dq, dk, ws,
                              ws.numel() * 4)
    assert rc == binding.OK
    return dq, dk


def _no_alloc(mode, t, w, stats):
    dq, dk = torch.empty_like(t["q1"]), torch.empty_like(t["k1"])
    rc = binding.streamkl_bwd_noalloc(mode, t["q1"], t["k1"], t["q2"], t["k2"], *stats, t["dkl"],
                                      w.B, w.Hq, w.Hkv, w.NQ, w.NK, w.d, w.scale, w.causal, dq, dk)
    assert rc == binding.OK, binding.last_cuda_error()
    return dq, dk


def _close(a, b):
    a = a.float().cpu().numpy()[None] if a.dim() == 3 else a.float().cpu().numpy()
    b = b.float().cpu().numpy()[None] if b.dim() == 3 else b.float().cpu().numpy()
    assert np.all(np.isfinite(a))
    return rel_l2(a.astype(np.float64), b.astype(np.float64), axes=(2, 3)).max()


CASES = [
    # B, Hq, Hkv, NQ, NK, d, causal, shared
    (1, 2, 2, 640, 640, 128, True, True),
    (2, 4, 2, 300, 333, 64, False, False),
    (1, 4, 4, 16384, 16384, 128, True, True),   # workspace exactly the 32 MiB buffer
]


@pytest.mark.parametrize("mode", [1, 2])
@pytest.mark.parametrize("case", CASES, ids=lambda c: "B%dHq%dNQ%dNK%dd%d" % (c[0], c[1], c[3], c[4], c[5]))
def test_matches_workspace_backward_twice(case, mode):
    B, Hq, Hkv, NQ, NK, d, causal, shared = case
    w = inputs.custom(B, Hq, Hkv, NQ, NK, d, causal, shared, seed=31 + NQ + d)
    assert binding.streamkl_bwd_workspace_bytes(B, Hq, Hkv, NQ, NK, d) <= binding.NOALLOC_SCRATCH_BYTES
    t = inputs.make(w, device="cuda")
    t["dkl"] = torch.rand(t["dkl"].shape, generator=torch.Generator().manual_seed(3)).cuda() + 0.5
    stats = _fwd(t, w)
    ref_dq, ref_dk = _with_workspace(mode, t, w, stats)
    for _ in range(2):
        dq, dk = _no_alloc(mode, t, w, stats)
        torch.cuda.synchronize()
        assert _close(dq, ref_dq) <= GRAD_TOL
        assert _close(dk, ref_dk) <= GRAD_TOL
    assert binding.streamkl_device_status() == binding.OK


def test_rejects_problems_larger_than_the_buffer():
    # 33 MiB of dK accumulator: refused on the host before any launch
    B, Hq, NQ, d = 1, 33, 2048, 128
    assert binding.streamkl_bwd_workspace_bytes(B, Hq, Hq, NQ, NQ, d) > binding.NOALLOC_SCRATCH_BYTES
    fake = 1 << 20
    rc = binding.streamkl_bwd_noalloc(1, fake, fake, fake, fake, fake, fake, fake, fake, B, Hq, Hq,
                                      NQ, NQ, d, 0.088, 1, fake, fake, stream=0)
    assert rc == binding.ERR_UNSUPPORTED
    assert "32" in binding.last_cuda_error() or "scratch" in binding.last_cuda_error()
