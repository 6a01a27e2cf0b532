"""Materialised fp64 brute force of the attention KL (small inputs only).

TEST INFRASTRUCTURE ONLY.  This is the computation the StreamKL pages describe as the
thing being replaced ("Definição do Problema" of the StreamKL technical summary,
gist.science, Portuguese): both attention distributions P1, P2 are built as full
N_Q x N_K matrices and the KL is reduced element-wise.  It shares nothing with the C
oracle or the CUDA path; tests use it as an independent cross-check.
"""
import numpy as np


def _expand_heads(k, hq):
    """[B,Hkv,NK,d] -> [B,Hq,NK,d]: query head h reads KV head h // (Hq/Hkv)."""
    hkv = k.shape[1]
    return np.repeat(k, hq // hkv, axis=1)


def _mask(nq, nk, causal):
    m = np.ones((nq, nk), dtype=bool)
    if causal:
        m &= np.arange(nk)[None, :] <= np.arange(nq)[:, None]
    return m


def log_softmax_masked(s, mask):
    s = np.where(mask, s, -np.inf)
    mx = s.max(axis=-1, keepdims=True)
    z = np.log(np.exp(s - mx).sum(axis=-1, keepdims=True)) + mx
    return s - z, z[..., 0]


def materialise(q1, k1, q2, k2, scale=None, causal=False):
    """Returns (S1, S2, logP1, logP2, LSE1, LSE2, mask), each [B,Hq,NQ,NK] or [B,Hq,NQ]."""
    q1, k1, q2, k2 = (np.asarray(x, dtype=np.float64) for x in (q1, k1, q2, k2))
    d = q1.shape[-1]
    scale = 1.0 / np.sqrt(d) if scale is None else float(scale)
    hq = q1.shape[1]
    K1, K2 = _expand_heads(k1, hq), _expand_heads(k2, hq)
    S1 = scale * np.einsum("bhid,bhjd->bhij", q1, K1)
    S2 = scale * np.einsum("bhid,bhjd->bhij", q2, K2)
    mask = _mask(q1.shape[2], k1.shape[2], causal)
    lp1, lse1 = log_softmax_masked(S1, mask)
    lp2, lse2 = log_softmax_masked(S2, mask)
    return S1, S2, lp1, lp2, lse1, lse2, mask


def fwd(q1, k1, q2, k2, scale=None, causal=False):
    """KL(P1||P2) per row, LSE1, LSE2 from the materialised matrices."""
    _, _, lp1, lp2, lse1, lse2, mask = materialise(q1, k1, q2, k2, scale, causal)
    p1 = np.where(mask, np.exp(lp1), 0.0)
    with np.errstate(invalid="ignore"):  # masked entries: (-inf) - (-inf), discarded below
        diff = np.where(mask, lp1 - lp2, 0.0)
    return (p1 * diff).sum(-1), lse1, lse2
