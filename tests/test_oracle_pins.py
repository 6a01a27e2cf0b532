"""Pins of the fp64 oracle to facts other than itself (no GPU).

Each test checks the oracle against something it does not compute itself: hand-derived
closed forms, library routines (scipy, torch autograd on a materialised loss), the
materialised brute force, finite differences, and invariants of the definition.  Each is
chosen so that a dropped term, a wrong sign, a wrong index or a transposed operand in the
oracle fails at least one of them.
"""
import math
import os

import numpy as np
import pytest
import scipy.special as sp
import torch

import oracle
from oracle import brute

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rnd(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


def make(B, Hq, Hkv, NQ, NK, d, seed, qscale=1.0, shared=False):
    q1 = rnd((B, Hq, NQ, d), seed, qscale)
    k1 = rnd((B, Hkv, NK, d), seed + 1)
    q2 = q1 + 0.5 * rnd((B, Hq, NQ, d), seed + 2, qscale)
    k2 = k1.copy() if shared else rnd((B, Hkv, NK, d), seed + 3)
    return q1, k1, q2, k2


def read_golden(name):
    vals = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *rest = line.split()
            vals[key] = [float(x) for x in rest]
    return vals


# ---------------------------------------------------------------- closed forms
def test_two_key_golden():
    g = read_golden("two_key_closed_form.txt")
    q1 = np.array(g["q1"]).reshape(1, 1, 1, 1)
    q2 = np.array(g["q2"]).reshape(1, 1, 1, 1)
    k = np.array(g["k"]).reshape(1, 1, 2, 1)
    kl, l1, l2 = oracle.fwd(q1, k, q2, k, scale=1.0)
    assert kl[0, 0, 0] == pytest.approx(g["kl"][0], abs=1e-15)
    assert l1[0, 0, 0] == pytest.approx(g["lse1"][0], abs=1e-15)
    assert l2[0, 0, 0] == pytest.approx(g["lse2"][0], abs=1e-15)
    # causal 2x2: row 0 sees key 0 only, row 1 both keys
    Q1 = np.concatenate([q1, q1], axis=2)
    Q2 = np.concatenate([q2, q2], axis=2)
    kl, l1, l2 = oracle.fwd(Q1, k, Q2, k, scale=1.0, causal=True)
    assert kl[0, 0, 0] == 0.0 and l1[0, 0, 0] == 0.0 and l2[0, 0, 0] == 0.0
    assert kl[0, 0, 1] == pytest.approx(g["kl"][0], abs=1e-15)


def test_materialised_bytes_golden():
    g = read_golden("materialised_bytes.txt")
    heads, ctx, bpe, mats = g["heads"][0], g["context"][0], g["bytes_per_entry"][0], g["matrices"][0]
    assert mats * heads * ctx * ctx * bpe == g["bytes"][0]
    assert g["bytes"][0] / 2**30 == g["gib"][0]


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_bernoulli_two_keys(seed):
    """With two valid keys both distributions are Bernoulli(sigmoid(delta_t))."""
    d = 16
    q1, k1, q2, k2 = make(1, 2, 2, 3, 2, d, seed, qscale=2.0)
    kl, l1, l2 = oracle.fwd(q1, k1, q2, k2)
    sc = 1 / math.sqrt(d)
    for h in range(2):
        for i in range(3):
            s1 = sc * k1[0, h] @ q1[0, h, i]
            s2 = sc * k2[0, h] @ q2[0, h, i]
            p = 1 / (1 + math.exp(-(s1[1] - s1[0])))
            q = 1 / (1 + math.exp(-(s2[1] - s2[0])))
            want = p * math.log(p / q) + (1 - p) * math.log((1 - p) / (1 - q))
            assert kl[0, h, i] == pytest.approx(want, rel=1e-10, abs=1e-14)
            assert l1[0, h, i] == pytest.approx(max(s1) + math.log1p(math.exp(min(s1) - max(s1))), rel=1e-13)


def test_uniform_p1_when_q1_zero():
    """Q1 = 0 makes P1 uniform on the n valid keys: KL = LSE2 - ln n - mean_j s2_j."""
    d = 32
    _, k1, q2, k2 = make(1, 2, 1, 40, 40, d, 3)
    q1 = np.zeros_like(q2)
    for causal in (False, True):
        kl, l1, l2 = oracle.fwd(q1, k1, q2, k2, causal=causal)
        for h in range(2):
            for i in (0, 1, 17, 39):
                n = i + 1 if causal else 40
                s2 = (k2[0, 0, :n] @ q2[0, h, i]) / math.sqrt(d)
                assert l1[0, h, i] == pytest.approx(math.log(n), rel=1e-13)
                assert l2[0, h, i] == pytest.approx(sp.logsumexp(s2), rel=1e-12)
                want = sp.logsumexp(s2) - math.log(n) - s2.mean()
                assert kl[0, h, i] == pytest.approx(want, rel=1e-10, abs=1e-13)


def test_identical_keys_give_uniform():
    d = 64
    q1, _, q2, _ = make(1, 1, 1, 8, 20, d, 4)
    key = rnd((d,), 9)
    k = np.tile(key, (1, 1, 20, 1))
    kl, l1, l2 = oracle.fwd(q1, k, q2, k)
    s1 = q1[0, 0] @ key / 8.0
    s2 = q2[0, 0] @ key / 8.0
    np.testing.assert_allclose(kl[0, 0], 0.0, atol=1e-13)
    np.testing.assert_allclose(l1[0, 0], s1 + math.log(20), rtol=1e-13)
    np.testing.assert_allclose(l2[0, 0], s2 + math.log(20), rtol=1e-13)


# ---------------------------------------------------------------- library routines
@pytest.mark.parametrize("causal", [False, True])
def test_against_scipy_rel_entr(causal):
    d, n = 64, 48
    q1, k1, q2, k2 = make(2, 4, 2, n, n, d, 5, qscale=1.5)
    kl, l1, l2 = oracle.fwd(q1, k1, q2, k2, causal=causal)
    for b in range(2):
        for h in range(4):
            hk = h // 2
            S1 = q1[b, h] @ k1[b, hk].T / 8.0
            S2 = q2[b, h] @ k2[b, hk].T / 8.0
            for i in range(n):
                m = i + 1 if causal else n
                P1 = sp.softmax(S1[i, :m])
                P2 = sp.softmax(S2[i, :m])
                assert kl[b, h, i] == pytest.approx(sp.rel_entr(P1, P2).sum(), rel=1e-9, abs=1e-13)
                assert l1[b, h, i] == pytest.approx(sp.logsumexp(S1[i, :m]), rel=1e-12)
                assert l2[b, h, i] == pytest.approx(sp.logsumexp(S2[i, :m]), rel=1e-12)


def test_against_torch_kl_div_rectangular_gqa():
    d = 64
    B, Hq, Hkv, NQ, NK = 2, 6, 3, 17, 53
    q1, k1, q2, k2 = make(B, Hq, Hkv, NQ, NK, d, 6, qscale=2.0)
    kl, l1, l2 = oracle.fwd(q1, k1, q2, k2, scale=0.3)
    t = lambda a: torch.from_numpy(a)
    K1 = t(k1).repeat_interleave(Hq // Hkv, dim=1)
    K2 = t(k2).repeat_interleave(Hq // Hkv, dim=1)
    S1 = 0.3 * t(q1) @ K1.transpose(-1, -2)
    S2 = 0.3 * t(q2) @ K2.transpose(-1, -2)
    lp1 = torch.log_softmax(S1, -1)
    lp2 = torch.log_softmax(S2, -1)
    want = torch.nn.functional.kl_div(lp2, lp1, log_target=True, reduction="none").sum(-1)
    np.testing.assert_allclose(kl, want.numpy(), rtol=1e-9, atol=1e-13)
    np.testing.assert_allclose(l1, torch.logsumexp(S1, -1).numpy(), rtol=1e-12)
    np.testing.assert_allclose(l2, torch.logsumexp(S2, -1).numpy(), rtol=1e-12)


# ---------------------------------------------------------------- brute force and recurrence
@pytest.mark.parametrize("causal", [False, True])
def test_brute_force_and_streaming_recurrence(causal):
    d = 64
    q1, k1, q2, k2 = make(1, 2, 1, 70, 70, d, 7, qscale=1.5, shared=True)
    kl, l1, l2 = oracle.fwd(q1, k1, q2, k2, causal=causal)
    bk, b1, b2 = brute.fwd(q1, k1, q2, k2, causal=causal)
    np.testing.assert_allclose(kl, bk, rtol=1e-10, atol=1e-13)
    np.testing.assert_allclose(l1, b1, rtol=1e-12)
    np.testing.assert_allclose(l2, b2, rtol=1e-12)
    for tile in (1, 7, 16, 64, 128):
        sk, s1, s2 = oracle.fwd_streaming(q1, k1, q2, k2, causal=causal, tile=tile)
        np.testing.assert_allclose(sk, kl, rtol=1e-9, atol=1e-12)
        np.testing.assert_allclose(s1, l1, rtol=1e-12)
        np.testing.assert_allclose(s2, l2, rtol=1e-12)


def test_streaming_recurrence_needs_the_rescale():
    """The online form is exact only with the exp(m_old - m_new) correction: with an
    increasing score sequence (later tiles hold larger maxima) the uncorrected sums
    that the simplified listing of the agents-report write-up implies would be wrong, so
    agreement here shows the correction is applied."""
    d = 1
    n = 40
    q = np.ones((1, 1, 1, d))
    k = np.linspace(0, 8, n).reshape(1, 1, n, d)
    kl, l1, _ = oracle.fwd(q, k, 0.5 * q, k, scale=1.0)
    sk, s1, _ = oracle.fwd_streaming(q, k, 0.5 * q, k, scale=1.0, tile=4)
    assert sk[0, 0, 0] == pytest.approx(kl[0, 0, 0], rel=1e-12)
    assert s1[0, 0, 0] == pytest.approx(sp.logsumexp(k[0, 0, :, 0]), rel=1e-13)


# ---------------------------------------------------------------- invariants
def test_kl_nonnegative_and_zero_on_identity():
    d = 128
    for seed, qs in ((8, 1.0), (9, 4.0)):
        q1, k1, q2, k2 = make(1, 2, 2, 33, 65, d, seed, qscale=qs)
        kl, _, _ = oracle.fwd(q1, k1, q2, k2)
        assert kl.min() >= -1e-12
        assert kl.max() > 1e-3
        kl0, a, b = oracle.fwd(q1, k1, q1, k1)
        assert np.all(kl0 == 0.0) and np.array_equal(a, b)


def test_reverse_and_symmetric_kl_against_brute_force():
    """Swapping the two distributions' arguments gives KL(P2||P1); the sum of both
    directions equals sum_j (p1 - p2)(log p1 - log p2), computed here from materialised
    softmaxes (scipy), and is non-negative."""
    d = 64
    q1, k1, q2, k2 = make(1, 2, 2, 17, 40, d, 21)
    fwd12, _, _ = oracle.fwd(q1, k1, q2, k2)
    fwd21, _, _ = oracle.fwd(q2, k2, q1, k1)
    s1 = np.einsum("bhid,bhjd->bhij", q1, k1) / 8.0
    s2 = np.einsum("bhid,bhjd->bhij", q2, k2) / 8.0
    lp1 = s1 - sp.logsumexp(s1, axis=-1, keepdims=True)
    lp2 = s2 - sp.logsumexp(s2, axis=-1, keepdims=True)
    rev = (np.exp(lp2) * (lp2 - lp1)).sum(-1)
    sym = ((np.exp(lp1) - np.exp(lp2)) * (lp1 - lp2)).sum(-1)
    np.testing.assert_allclose(fwd21, rev, rtol=1e-10, atol=1e-13)
    np.testing.assert_allclose(fwd12 + fwd21, sym, rtol=1e-10, atol=1e-13)
    assert sym.min() >= -1e-12
    assert np.abs(fwd12 - fwd21).max() > 1e-4          # the two directions differ


def test_causal_row_zero():
    d = 64
    q1, k1, q2, k2 = make(1, 3, 3, 9, 9, d, 10)
    kl, l1, l2 = oracle.fwd(q1, k1, q2, k2, causal=True)
    assert np.all(kl[:, :, 0] == 0.0)
    np.testing.assert_allclose(l1[0, :, 0], np.einsum("hd,hd->h", q1[0, :, 0], k1[0, :, 0]) / 8.0,
                               rtol=1e-14)


def test_row_shift_invariance():
    """Adding a vector c to every key shifts row i's scores by scale*q_i.c: KL unchanged,
    LSE shifted by exactly that amount."""
    d = 64
    q1, k1, q2, k2 = make(1, 2, 2, 12, 30, d, 11)
    c = rnd((d,), 12)
    kl, l1, l2 = oracle.fwd(q1, k1, q2, k2)
    klc, l1c, l2c = oracle.fwd(q1, k1 + c, q2, k2 + c)
    np.testing.assert_allclose(klc, kl, rtol=1e-8, atol=1e-12)
    np.testing.assert_allclose((l1c - l1)[0], q1[0] @ c / 8.0, rtol=1e-9, atol=1e-12)
    np.testing.assert_allclose((l2c - l2)[0], q2[0] @ c / 8.0, rtol=1e-9, atol=1e-12)


def test_fwd_rows_matches_full():
    d = 64
    q1, k1, q2, k2 = make(2, 4, 2, 50, 50, d, 13)
    for causal in (False, True):
        kl, l1, l2 = oracle.fwd(q1, k1, q2, k2, causal=causal)
        rows = np.array([0, 7, 49, 50, 123, 399])
        rk, r1, r2 = oracle.fwd_rows(q1, k1, q2, k2, rows, causal=causal)
        np.testing.assert_array_equal(rk, kl.reshape(-1)[rows])
        np.testing.assert_array_equal(r1, l1.reshape(-1)[rows])
        np.testing.assert_array_equal(r2, l2.reshape(-1)[rows])


# ---------------------------------------------------------------- backward
def torch_grads(mode, q1, k1, q2, k2, g, scale, causal):
    """Autograd of sum_i g_i KL_i on the materialised fp64 loss, fixed side detached."""
    t = lambda a, rg: torch.tensor(a, dtype=torch.float64, requires_grad=rg)
    Q1, Q2 = t(q1, mode == 2), t(q2, mode == 1)
    K1, K2 = t(k1, mode == 2), t(k2, mode == 1)
    rep = q1.shape[1] // k1.shape[1]
    S1 = scale * Q1 @ K1.repeat_interleave(rep, 1).transpose(-1, -2)
    S2 = scale * Q2 @ K2.repeat_interleave(rep, 1).transpose(-1, -2)
    if causal:
        n = q1.shape[2]
        m = torch.ones(n, n, dtype=torch.bool).tril()
        S1 = S1.masked_fill(~m, -math.inf)
        S2 = S2.masked_fill(~m, -math.inf)
    lp1 = torch.log_softmax(S1, -1)
    lp2 = torch.log_softmax(S2, -1)
    if mode == 1:
        lp1 = lp1.detach()
    else:
        lp2 = lp2.detach()
    p1 = lp1.exp()
    diff = torch.where(p1 > 0, lp1 - lp2, torch.zeros_like(lp1))
    kl = (p1 * diff).sum(-1)
    (kl * torch.tensor(g)).sum().backward()
    if mode == 1:
        return Q2.grad.numpy(), K2.grad.numpy()
    return Q1.grad.numpy(), K1.grad.numpy()


@pytest.mark.parametrize("mode", [1, 2])
@pytest.mark.parametrize("causal", [False, True])
def test_bwd_against_torch_autograd(mode, causal):
    d = 64
    B, Hq, Hkv, N = 2, 4, 2, 37
    q1, k1, q2, k2 = make(B, Hq, Hkv, N, N, d, 20 + mode, qscale=1.5)
    g = np.random.default_rng(5).uniform(0.1, 1.0, (B, Hq, N))
    dq, dk = oracle.bwd(mode, q1, k1, q2, k2, g, scale=0.2, causal=causal)
    tq, tk = torch_grads(mode, q1, k1, q2, k2, g, 0.2, causal)
    np.testing.assert_allclose(dq, tq, rtol=1e-9, atol=1e-13)
    np.testing.assert_allclose(dk, tk, rtol=1e-9, atol=1e-13)


def _loss(q1, k1, q2, k2, g, causal):
    kl, _, _ = oracle.fwd(q1, k1, q2, k2, causal=causal)
    return float((kl * g).sum())


@pytest.mark.parametrize("mode", [1, 2])
def test_bwd_central_finite_differences(mode):
    """Central differences (h = 1e-5) of sum g*KL on 20 random entries each of the free Q
    and K.  Holding the other distribution's inputs fixed makes the derivative of the
    full loss equal the mode's gradient."""
    d, N = 64, 256
    q1, k1, q2, k2 = make(1, 1, 1, N, N, d, 30, shared=True)
    k2 = k2.copy()  # separate storage: perturbing the free K leaves the fixed one alone
    g = np.full((1, 1, N), 1.0 / N)
    dq, dk = oracle.bwd(mode, q1, k1, q2, k2, g)
    rng = np.random.default_rng(31 + mode)
    h = 1e-5
    for which in ("q", "k"):
        base = {"q1": q1, "k1": k1, "q2": q2, "k2": k2}
        name = which + ("2" if mode == 1 else "1")
        grad = dq if which == "q" else dk
        arr = base[name]
        for _ in range(20):
            idx = tuple(rng.integers(0, s) for s in arr.shape)
            plus, minus = arr.copy(), arr.copy()
            plus[idx] += h
            minus[idx] -= h
            fp = _loss(**{**base, name: plus}, g=g, causal=False)
            fm = _loss(**{**base, name: minus}, g=g, causal=False)
            fd = (fp - fm) / (2 * h)
            assert fd == pytest.approx(grad[idx], rel=1e-6, abs=1e-11)


@pytest.mark.parametrize("mode", [1, 2])
def test_bwd_invariants(mode):
    d = 64
    q1, k1, q2, k2 = make(1, 4, 2, 40, 40, d, 40)
    g = np.random.default_rng(1).uniform(0.5, 1.5, (1, 4, 40))
    for causal in (False, True):
        dq, dk = oracle.bwd(mode, q1, k1, q2, k2, g, causal=causal)
        # every row of dS sums to zero -> the key gradients of a KV head sum to zero
        np.testing.assert_allclose(dk.sum(axis=2), 0.0, atol=1e-12)
        # ... and dQ does not change when a constant vector is added to every key
        c = rnd((d,), 41)
        kk1, kk2 = (k1 + c, k2) if mode == 2 else (k1, k2 + c)
        dqc, _ = oracle.bwd(mode, q1, kk1, q2, kk2, g, causal=causal)
        np.testing.assert_allclose(dqc, dq, rtol=1e-7, atol=1e-12)
        # identical distributions: no gradient
        dq0, dk0 = oracle.bwd(mode, q1, k1, q1, k1, g, causal=causal)
        assert np.abs(dq0).max() < 1e-14 and np.abs(dk0).max() < 1e-14


@pytest.mark.parametrize("mode", [1, 2])
def test_sampled_rows_and_keys_match_full(mode):
    d = 64
    B, Hq, Hkv, N = 2, 4, 2, 45
    q1, k1, q2, k2 = make(B, Hq, Hkv, N, N, d, 50)
    g = np.random.default_rng(2).uniform(0.5, 1.5, (B, Hq, N))
    for causal in (False, True):
        dq, dk = oracle.bwd(mode, q1, k1, q2, k2, g, causal=causal)
        rows = np.array([0, 3, 44, 45, 200, 359])
        np.testing.assert_allclose(oracle.bwd_dq_rows(mode, q1, k1, q2, k2, g, rows, causal=causal),
                                   dq.reshape(-1, d)[rows], rtol=1e-12, atol=1e-16)
        keys = np.array([0, 9, 44, 45, 100, 179])
        np.testing.assert_allclose(oracle.bwd_dk_keys(mode, q1, k1, q2, k2, g, keys, causal=causal),
                                   dk.reshape(-1, d)[keys], rtol=1e-10, atol=1e-16)


def test_bad_arguments_rejected():
    q = np.zeros((1, 3, 4, 8))
    k = np.zeros((1, 2, 4, 8))
    with pytest.raises(ValueError):
        oracle.fwd(q, k, q, k)          # Hq % Hkv != 0
    q = np.zeros((1, 2, 4, 8))
    k = np.zeros((1, 2, 5, 8))
    with pytest.raises(ValueError):
        oracle.fwd(q, k, q, k, causal=True)  # causal needs NQ == NK


@pytest.mark.parametrize("mode", [1, 2])
def test_dk_with_given_statistics_matches_recomputed(mode):
    """The variant that takes row statistics as inputs, fed the oracle's own statistics,
    gives the self-contained dK (it differs only in where LSE and KL come from)."""
    d = 64
    B, Hq, Hkv, N = 1, 4, 2, 60
    q1, k1, q2, k2 = make(B, Hq, Hkv, N, N, d, 60)
    g = np.random.default_rng(3).uniform(0.5, 1.5, (B, Hq, N))
    for causal in (False, True):
        kl, l1, l2 = oracle.fwd(q1, k1, q2, k2, causal=causal)
        keys = np.array([0, 5, 59, 60, 111, 119])
        a = oracle.bwd_dk_keys(mode, q1, k1, q2, k2, g, keys, causal=causal)
        b = oracle.bwd_dk_keys_stats(mode, q1, k1, q2, k2, g, kl, l1, l2, keys, causal=causal)
        np.testing.assert_allclose(b, a, rtol=1e-12, atol=1e-16)
