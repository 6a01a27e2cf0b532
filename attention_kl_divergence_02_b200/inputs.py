"""Seeded synthetic inputs for the StreamKL workloads.

This module draws random tensors and nothing else: it holds none of the method's
arithmetic, and both the CUDA path's tests and the CPU oracle's tests take their inputs
from it.  Every tensor is drawn in fp32 on the CPU from one ``torch.Generator`` seeded
per workload, then rounded to bf16; the oracle reads the same bf16 values, widened to
double.

Draw order: Q1, K1, [K2 when the keys are distinct], noise; then Q2 = a*Q1 + b*noise in
fp32 before rounding.  The grouped-query workload instead draws Q1, K1, K2, Q2 and two
per-head factors c1, c2 ~ U(0.5, 2) that multiply Q1[:, h] and Q2[:, h].

The upstream gradient g (``dkl``, one value per query row) is the mean reduction:
1/NQ for the 256-row workload, 1/(B*Hq*NQ) elsewhere.
"""
from dataclasses import dataclass, field, replace
import math

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    NQ: int
    NK: int
    d: int
    causal: bool
    shared_k: bool
    modes: tuple
    seed: int
    q2_a: float = 1.0          # Q2 = q2_a * Q1 + q2_b * noise
    q2_b: float = 0.5
    head_scaled: bool = False  # grouped-query workload: independent Q1, Q2 with per-head scales
    g_per_row_mean: bool = False  # g = 1/NQ (else 1/(B*Hq*NQ))
    note: str = field(default="", compare=False)

    @property
    def scale(self):
        return 1.0 / math.sqrt(self.d)

    def pairs(self):
        """Unmasked (row, key) pairs as counted for FLOPs: halved when causal."""
        p = self.B * self.Hq * self.NQ * self.NK
        return p / 2 if self.causal else p

    def fwd_flops(self):
        return 4.0 * self.d * self.pairs()

    def bwd_flops(self):
        return 8.0 * self.d * self.pairs()


WORKLOADS = {
    "tiny": Workload("tiny", 1, 1, 1, 256, 256, 64, False, True, (1,), 0, 1.0, 0.3,
                     g_per_row_mean=True,
                     note="B1 H1 N256 d64 non-causal shared K; Q2 = Q1 + 0.3 N"),
    "b2h8n4k": Workload("b2h8n4k", 2, 8, 8, 4096, 4096, 128, True, False, (1,), 1, 1.0, 0.5,
                        note="B2 H8 N4096 d128, distinct K1 K2; Q2 = Q1 + 0.5 N (causal and non-causal)"),
    "headline": Workload("headline", 1, 32, 32, 16384, 16384, 128, True, True, (1, 2), 2, 0.8, 0.6,
                         note="B1 H32 N16384 d128 causal shared K; Q2 = 0.8 Q1 + 0.6 N"),
    "long64k": Workload("long64k", 1, 32, 32, 65536, 65536, 128, True, True, (1,), 3, 1.0, 0.5,
                        note="B1 H32 N65536 d128 causal shared K; Q2 = Q1 + 0.5 N"),
    "gqa": Workload("gqa", 4, 32, 8, 2048, 32768, 64, False, False, (2,), 4, head_scaled=True,
                    note="B4 Hq32 Hkv8 NQ2048 NK32768 d64 non-causal distinct K; per-head Q scale U(0.5,2)"),
    "chunk": Workload("chunk", 1, 16, 16, 512, 65536, 128, False, True, (1, 2), 6, 1.0, 0.5,
                      note="B1 H16 NQ512 NK65536 d128 non-causal shared K (a chunk of queries "
                           "against a long context: 64 query tiles for 148 SMs, the case the "
                           "key-range backward is for); Q2 = Q1 + 0.5 N"),
    "decode": Workload("decode", 1, 16, 16, 1, 131072, 128, False, True, (), 5, 1.0, 0.5,
                       note="B1 H16 NQ1 NK131072 d128 non-causal shared K (one query row per head "
                            "against a long key sequence: 16 query blocks for 148 SMs, the case "
                            "the split-K forward is for); Q2 = Q1 + 0.5 N"),
}


def custom(B, Hq, Hkv, NQ, NK, d, causal, shared_k, seed, q2_a=1.0, q2_b=0.5, modes=(1, 2),
           head_scaled=False, name="custom"):
    """A workload with the same recipe at another shape (tests use small ones)."""
    return Workload(name, B, Hq, Hkv, NQ, NK, d, bool(causal), bool(shared_k), tuple(modes),
                    seed, q2_a, q2_b, head_scaled)


def variant(w, **kw):
    return replace(w, **kw)


def make(w, device="cpu"):
    """Draw the workload's tensors.  Returns a dict of bf16 tensors q1, k1, q2, k2
    ([B,H,N,d]; k2 is k1 itself when the keys are shared) and the fp32 per-row dkl."""
    gen = torch.Generator(device="cpu")
    gen.manual_seed(int(w.seed))
    qs = (w.B, w.Hq, w.NQ, w.d)
    ks = (w.B, w.Hkv, w.NK, w.d)
    q1 = torch.randn(qs, generator=gen, dtype=torch.float32)
    k1 = torch.randn(ks, generator=gen, dtype=torch.float32)
    if w.head_scaled:
        k2 = k1 if w.shared_k else torch.randn(ks, generator=gen, dtype=torch.float32)
        q2 = torch.randn(qs, generator=gen, dtype=torch.float32)
        c1 = torch.rand((w.Hq,), generator=gen, dtype=torch.float32) * 1.5 + 0.5
        c2 = torch.rand((w.Hq,), generator=gen, dtype=torch.float32) * 1.5 + 0.5
        q1 = q1 * c1.view(1, -1, 1, 1)
        q2 = q2 * c2.view(1, -1, 1, 1)
    else:
        k2 = k1 if w.shared_k else torch.randn(ks, generator=gen, dtype=torch.float32)
        noise = torch.randn(qs, generator=gen, dtype=torch.float32)
        q2 = w.q2_a * q1 + w.q2_b * noise
        del noise
    q1 = q1.to(torch.bfloat16)
    q2 = q2.to(torch.bfloat16)
    k1b = k1.to(torch.bfloat16)
    k2b = k1b if w.shared_k else k2.to(torch.bfloat16)
    g = 1.0 / w.NQ if w.g_per_row_mean else 1.0 / (w.B * w.Hq * w.NQ)
    dkl = torch.full((w.B, w.Hq, w.NQ), g, dtype=torch.float32)
    out = {"q1": q1, "k1": k1b, "q2": q2, "k2": k2b, "dkl": dkl}
    if device != "cpu":
        moved = {}
        for k, v in out.items():
            moved[k] = v.to(device)
        if w.shared_k:
            moved["k2"] = moved["k1"]
        out = moved
    return out


def to_f64(t):
    """bf16/fp32 torch tensor -> float64 numpy (exact widening)."""
    return t.detach().to("cpu").to(torch.float64).numpy()
