"""The library's calls inside a CUDA graph: a captured forward (plain, split-K with its merge
launched as a programmatic dependent, few rows) and backward (workspace memset, kernel,
converts) replay to the same bits as the eager calls, and again after the inputs change in
place (a graph replays on whatever the captured buffers hold)."""
import numpy as np
import pytest
import torch

import oracle
from attention_kl_divergence_02_b200 import binding, inputs

from parity import check_fwd, host64

pytestmark = pytest.mark.gpu


def _capture(fn):
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn()                      # warm-up outside the graph (library load, attributes)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    return g


@pytest.mark.parametrize("case", [
    # B, Hq, Hkv, NQ, NK, d, causal, shared, split
    (1, 4, 4, 1, 4096, 128, False, True, True),       # decode shape: few-row kernel + merge
    (1, 2, 2, 64, 3000, 64, False, False, True),      # split-K query-row kernel + merge
    (1, 2, 2, 640, 640, 128, True, True, False),      # plain forward
])
def test_forward_replays_bit_exact(case):
    B, Hq, Hkv, NQ, NK, d, causal, shared, split = case
    w = inputs.custom(B, Hq, Hkv, NQ, NK, d, causal, shared, seed=31 + NQ)
    t = inputs.make(w, device="cuda")
    out = tuple(torch.empty((B, Hq, NQ), device="cuda") for _ in range(3))
    need = binding.streamkl_fwd_splitk_workspace_bytes(B, Hq, NQ, NK, 0)
    ws = torch.empty(max(4, need) // 4, device="cuda")

    def call():
        if split:
            binding.fwd_splitk(t["q1"], t["k1"], t["q2"], t["k2"], scale=w.scale, causal=causal,
                               splits=0, out=out, workspace=ws)
        else:
            binding.fwd(t["q1"], t["k1"], t["q2"], t["k2"], scale=w.scale, causal=causal, out=out)

    call()
    torch.cuda.synchronize()
    eager = [x.clone() for x in out]
    g = _capture(call)
    for x in out:
        x.fill_(float("nan"))
    g.replay()
    torch.cuda.synchronize()
    assert binding.streamkl_device_status() == binding.OK
    for a, b in zip(out, eager):
        assert torch.equal(a, b)
    # new inputs in the captured buffers: the replay computes on them
    t["q2"].copy_(t["q2"].flip(2))
    g.replay()
    torch.cuda.synchronize()
    want = oracle.fwd(host64(t["q1"]), host64(t["k1"]), host64(t["q2"]), host64(t["k2"]),
                      scale=w.scale, causal=causal)
    check_fwd(tuple(x.cpu().double().numpy() for x in out), want, "graph replay %s" % (case,))


def test_backward_replays_to_the_eager_result():
    """The dK partial sums are fp32 reductions in L2 in no fixed order, so a replay matches the
    eager call to the last bf16 bits, not bitwise."""
    w = inputs.custom(1, 4, 2, 300, 300, 64, True, False, seed=41)   # two heads per CTA
    t = inputs.make(w, device="cuda")
    kl, l1, l2 = binding.fwd(t["q1"], t["k1"], t["q2"], t["k2"], scale=w.scale, causal=True)
    out = (torch.empty_like(t["q1"]), torch.empty_like(t["k1"]))
    ws = torch.empty(binding.streamkl_bwd_workspace_bytes(1, 4, 2, 300, 300, 64) // 4, device="cuda")

    def call():
        binding.bwd(1, t["q1"], t["k1"], t["q2"], t["k2"], kl, l1, l2, t["dkl"], scale=w.scale,
                    causal=True, out=out, workspace=ws)

    call()
    torch.cuda.synchronize()
    eager = [x.clone() for x in out]
    g = _capture(call)
    for x in out:
        x.zero_()
    g.replay()
    g.replay()                    # the captured memset re-zeroes the workspace every replay
    torch.cuda.synchronize()
    assert binding.streamkl_device_status() == binding.OK
    for a, b in zip(out, eager):
        a, b = a.double(), b.double()
        assert float((a - b).norm() / b.norm()) <= 1e-3
