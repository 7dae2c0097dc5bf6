"""Pins for the f64 oracle: each test checks it against something other than itself.

- library special cases: torch SDPA (f64, CPU) with is_causal, with an explicit band
  mask, with GQA by repeat_interleave; torch autograd through SDPA for gradients;
- brute force on tiny shapes, with the full softmax Jacobian instead of the Delta
  shortcut;
- central finite differences of L = sum(O * dO);
- the page's mask written out (tests/golden/mask_*.txt);
- invariants and closed forms of the definition.
"""
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rnd(shape, seed, sigma=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(*shape, generator=g, dtype=torch.float64) * sigma)


def qkv(B, Hq, Hkv, T, D, seed=0, sq=1.0, sk=1.0):
    q = rnd((B, Hq, T, D), seed, sq)
    k = rnd((B, Hkv, T, D), seed + 1, sk)
    v = rnd((B, Hkv, T, D), seed + 2)
    dO = rnd((B, Hq, T, D), seed + 3)
    return q, k, v, dO


def band_mask(T, W):
    """Boolean [T, T] mask from torch's triangle routines: keep k <= q, and when
    W > 0 also k > q - W."""
    m = torch.ones(T, T, dtype=torch.bool).tril()
    if W > 0:
        m = m & torch.ones(T, T, dtype=torch.bool).triu(diagonal=-(W - 1))
    return m


def sdpa_ref(q, k, v, scale, W=0, softcap=0.0):
    """Attention through torch's own SDPA. Softcap enters as an additive bias
    (cap*tanh(S/cap) - S) so that SDPA's softmax sees the capped scores."""
    G = q.shape[1] // k.shape[1]
    kr = k.repeat_interleave(G, dim=1)
    vr = v.repeat_interleave(G, dim=1)
    T = q.shape[2]
    if softcap == 0.0 and W == 0:
        return F.scaled_dot_product_attention(q, kr, vr, is_causal=True, scale=scale)
    mask = band_mask(T, W)
    if softcap == 0.0:
        return F.scaled_dot_product_attention(q, kr, vr, attn_mask=mask, scale=scale)
    S = scale * q @ kr.transpose(-1, -2)
    bias = softcap * torch.tanh(S / softcap) - S
    bias = bias.masked_fill(~mask, float("-inf"))
    return F.scaled_dot_product_attention(q, kr, vr, attn_mask=bias, scale=scale)


def sdpa_grads(q, k, v, dO, scale, W=0, softcap=0.0):
    q = q.clone().requires_grad_(True)
    k = k.clone().requires_grad_(True)
    v = v.clone().requires_grad_(True)
    o = sdpa_ref(q, k, v, scale, W, softcap)
    o.backward(dO)
    return o.detach(), q.grad, k.grad, v.grad


CASES = [
    # B, Hq, Hkv, T, D, W, C
    (1, 1, 1, 1, 4, 0, 0.0),
    (2, 2, 2, 37, 8, 0, 0.0),
    (1, 4, 2, 33, 16, 0, 0.0),
    (1, 6, 2, 40, 8, 7, 0.0),
    (2, 3, 1, 29, 8, 1, 0.0),
    (1, 2, 1, 31, 8, 0, 3.0),
    (1, 4, 4, 45, 8, 9, 2.0),
    (1, 3, 3, 20, 8, 25, 0.0),  # W > T
]


@pytest.mark.parametrize("B,Hq,Hkv,T,D,W,C", CASES)
def test_fwd_bwd_match_torch_sdpa_autograd(B, Hq, Hkv, T, D, W, C):
    q, k, v, dO = qkv(B, Hq, Hkv, T, D, seed=T + D, sq=2.0 if C else 1.0, sk=2.0 if C else 1.0)
    scale = 1.0 / math.sqrt(D)
    o_ref, dq_ref, dk_ref, dv_ref = sdpa_grads(q, k, v, dO, scale, W, C)
    o, lse = oracle.attn_fwd(q, k, v, scale, W, C)
    np.testing.assert_allclose(o, o_ref.numpy(), rtol=1e-12, atol=1e-12)
    dq, dk, dv, delta, lse2 = oracle.attn_bwd(q, k, v, dO, scale, W, C)
    np.testing.assert_allclose(dq, dq_ref.numpy(), rtol=1e-10, atol=1e-11)
    np.testing.assert_allclose(dk, dk_ref.numpy(), rtol=1e-10, atol=1e-11)
    np.testing.assert_allclose(dv, dv_ref.numpy(), rtol=1e-10, atol=1e-11)
    np.testing.assert_array_equal(lse, lse2)


@pytest.mark.parametrize("W,C", [(0, 0.0), (5, 0.0), (0, 4.0), (6, 3.0)])
def test_lse_matches_torch_logsumexp(W, C):
    q, k, _, _ = qkv(1, 2, 1, 23, 8, seed=11, sq=2.0, sk=2.0)
    scale = 0.3
    _, lse = oracle.attn_fwd(q, k, k, scale, W, C)
    S = scale * q @ k.repeat_interleave(2, dim=1).transpose(-1, -2)
    if C:
        S = C * torch.tanh(S / C)
    S = S.masked_fill(~band_mask(23, W), float("-inf"))
    np.testing.assert_allclose(lse, torch.logsumexp(S, dim=-1).numpy(), rtol=1e-13, atol=1e-13)


# ----------------------------------------------------------------- brute force

def brute(q, k, v, dO, scale, W, C):
    """Tiny shapes only: explicit loops, softmax Jacobian J_ab = P_a (delta_ab - P_b)."""
    q, k, v, dO = (x.numpy() for x in (q, k, v, dO))
    B, Hq, T, D = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    o = np.zeros_like(q)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for b in range(B):
        for h in range(Hq):
            g = h // G
            for i in range(T):
                keys = [j for j in range(T) if (j <= i and (W == 0 or j > i - W))]
                raw = {j: scale * sum(q[b, h, i, d] * k[b, g, j, d] for d in range(D)) for j in keys}
                s = {j: (C * math.tanh(raw[j] / C) if C else raw[j]) for j in keys}
                z = sum(math.exp(s[j]) for j in keys)
                P = {j: math.exp(s[j]) / z for j in keys}
                for j in keys:
                    o[b, h, i] += P[j] * v[b, g, j]
                    dv[b, g, j] += P[j] * dO[b, h, i]
                dP = {j: sum(dO[b, h, i, d] * v[b, g, j, d] for d in range(D)) for j in keys}
                for a in keys:
                    dsa = sum(P[a] * ((1.0 if a == c else 0.0) - P[c]) * dP[c] for c in keys)
                    if C:
                        dsa *= 1.0 - math.tanh(raw[a] / C) ** 2
                    dq[b, h, i] += scale * dsa * k[b, g, a]
                    dk[b, g, a] += scale * dsa * q[b, h, i]
    return o, dq, dk, dv


@pytest.mark.parametrize("T,D,W,C,Hq,Hkv", [(5, 3, 0, 0.0, 2, 1), (6, 2, 2, 0.0, 1, 1),
                                             (6, 3, 3, 1.5, 4, 2), (4, 1, 1, 0.0, 2, 2),
                                             (7, 2, 0, 0.7, 3, 1)])
def test_bruteforce_jacobian(T, D, W, C, Hq, Hkv):
    q, k, v, dO = qkv(1, Hq, Hkv, T, D, seed=3 * T + D, sq=1.5, sk=1.5)
    scale = 0.9
    o_b, dq_b, dk_b, dv_b = brute(q, k, v, dO, scale, W, C)
    o, _ = oracle.attn_fwd(q, k, v, scale, W, C)
    dq, dk, dv, _, _ = oracle.attn_bwd(q, k, v, dO, scale, W, C)
    for a, b in ((o, o_b), (dq, dq_b), (dk, dk_b), (dv, dv_b)):
        np.testing.assert_allclose(a, b, rtol=1e-11, atol=1e-12)


# ----------------------------------------------------- central finite differences

@pytest.mark.parametrize("W,C", [(0, 0.0), (4, 0.0), (0, 2.5), (3, 1.2)])
def test_central_finite_differences(W, C):
    B, Hq, Hkv, T, D = 1, 4, 2, 9, 3
    q, k, v, dO = qkv(B, Hq, Hkv, T, D, seed=40 + W, sq=1.3, sk=1.3)
    scale = 0.8
    dq, dk, dv, _, _ = oracle.attn_bwd(q, k, v, dO, scale, W, C)
    grads = {"q": dq, "k": dk, "v": dv}
    base = {"q": q.numpy().copy(), "k": k.numpy().copy(), "v": v.numpy().copy()}
    dOn = dO.numpy()
    h = 1e-6

    def loss(x):
        o, _ = oracle.attn_fwd(x["q"], x["k"], x["v"], scale, W, C)
        return float(np.sum(o * dOn))

    for name in ("q", "k", "v"):
        arr = base[name]
        for idx in np.ndindex(arr.shape):
            xp = {n: a.copy() for n, a in base.items()}
            xm = {n: a.copy() for n, a in base.items()}
            xp[name][idx] += h
            xm[name][idx] -= h
            fd = (loss(xp) - loss(xm)) / (2 * h)
            assert abs(fd - grads[name][idx]) <= 1e-7 * (1.0 + abs(fd)), (name, idx, fd, grads[name][idx])


# --------------------------------------------------------------- mask (the page)

def read_mask(path):
    rows = {}
    with open(path) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            q, ks = line.split(":")
            rows[int(q)] = [int(x) for x in ks.split()]
    return rows


@pytest.mark.parametrize("fname,T,W", [("mask_T6_W3.txt", 6, 3), ("mask_T5_W0.txt", 5, 0)])
def test_mask_matches_page(fname, T, W):
    rows = read_mask(os.path.join(GOLDEN, fname))
    q, k, _, _ = qkv(1, 1, 1, T, 4, seed=5)
    P = oracle.attn_probs(q, k, 0.5, W, 0.0)[0, 0]
    for i in range(T):
        nz = [j for j in range(T) if P[i, j] != 0.0]
        assert nz == rows[i], (i, nz, rows[i])


# --------------------------------------------------------- invariants, closed forms

def test_probability_rows_sum_to_one_and_respect_mask():
    q, k, _, _ = qkv(2, 4, 2, 30, 8, seed=9, sq=2.0, sk=2.0)
    for W, C in ((0, 0.0), (6, 0.0), (0, 3.0), (11, 5.0)):
        P = oracle.attn_probs(q, k, 0.4, W, C)
        np.testing.assert_allclose(P.sum(-1), 1.0, rtol=0, atol=1e-14)
        allowed = band_mask(30, W).numpy()
        assert np.all(P[..., ~allowed] == 0.0)
        assert np.all(P[..., allowed] > 0.0)


def test_ones_value_gives_ones_output():
    q, k, _, _ = qkv(1, 2, 2, 25, 8, seed=2)
    v = torch.ones(1, 2, 25, 8, dtype=torch.float64)
    o, _ = oracle.attn_fwd(q, k, v, 0.35, 4, 2.0)
    np.testing.assert_allclose(o, 1.0, rtol=0, atol=1e-14)


def test_window_at_least_T_is_full_causal_bitwise():
    q, k, v, dO = qkv(1, 4, 2, 27, 8, seed=4)
    ref = oracle.attn_fwd(q, k, v, 0.3, 0, 1.5)
    refb = oracle.attn_bwd(q, k, v, dO, 0.3, 0, 1.5)
    for W in (27, 28, 1000):
        o, lse = oracle.attn_fwd(q, k, v, 0.3, W, 1.5)
        np.testing.assert_array_equal(o, ref[0])
        np.testing.assert_array_equal(lse, ref[1])
        for a, b in zip(oracle.attn_bwd(q, k, v, dO, 0.3, W, 1.5), refb):
            np.testing.assert_array_equal(a, b)


def test_huge_softcap_reproduces_no_cap():
    q, k, v, dO = qkv(1, 2, 1, 21, 8, seed=6)
    C = 1e8
    o0, l0 = oracle.attn_fwd(q, k, v, 0.35, 0, 0.0)
    o1, l1 = oracle.attn_fwd(q, k, v, 0.35, 0, C)
    smax = float((q.abs().sum(-1).max() * k.abs().sum(-1).max()) * 0.35)
    bound = 4.0 * (smax ** 3) / (3 * C * C) + 1e-13  # cap*tanh(s/cap) = s - s^3/(3 cap^2) + ...
    np.testing.assert_allclose(o1, o0, rtol=0, atol=bound)
    np.testing.assert_allclose(l1, l0, rtol=0, atol=bound)
    g0 = oracle.attn_bwd(q, k, v, dO, 0.35, 0, 0.0)
    g1 = oracle.attn_bwd(q, k, v, dO, 0.35, 0, C)
    for a, b in zip(g0[:3], g1[:3]):
        np.testing.assert_allclose(a, b, rtol=0, atol=1e-10)


def test_small_softcap_changes_result():
    """A cap in the tanh regime must move the output (guards a dropped cap term)."""
    q, k, v, _ = qkv(1, 1, 1, 16, 8, seed=8, sq=3.0, sk=3.0)
    o0, _ = oracle.attn_fwd(q, k, v, 0.5, 0, 0.0)
    o1, _ = oracle.attn_fwd(q, k, v, 0.5, 0, 2.0)
    assert np.max(np.abs(o0 - o1)) > 1e-2


def test_gqa_equals_repeated_kv_heads():
    B, Hq, Hkv, T, D = 2, 6, 2, 19, 8
    G = Hq // Hkv
    q, k, v, dO = qkv(B, Hq, Hkv, T, D, seed=12)
    kr = k.repeat_interleave(G, dim=1)
    vr = v.repeat_interleave(G, dim=1)
    for W, C in ((0, 0.0), (5, 2.0)):
        o, lse = oracle.attn_fwd(q, k, v, 0.4, W, C)
        o2, lse2 = oracle.attn_fwd(q, kr, vr, 0.4, W, C)
        np.testing.assert_allclose(o, o2, rtol=0, atol=1e-14)
        np.testing.assert_allclose(lse, lse2, rtol=0, atol=1e-14)
        dq, dk, dv, _, _ = oracle.attn_bwd(q, k, v, dO, 0.4, W, C)
        dq2, dk2, dv2, _, _ = oracle.attn_bwd(q, kr, vr, dO, 0.4, W, C)
        np.testing.assert_allclose(dq, dq2, rtol=0, atol=1e-13)
        np.testing.assert_allclose(dk, dk2.reshape(B, Hkv, G, T, D).sum(2), rtol=0, atol=1e-12)
        np.testing.assert_allclose(dv, dv2.reshape(B, Hkv, G, T, D).sum(2), rtol=0, atol=1e-12)


def test_key_shift_invariance():
    """Adding one vector c to every key adds q.c to a whole score row: P, O and dQ
    are unchanged (rows of the softmax gradient sum to zero) and LSE moves by
    scale*q.c. Holds without a cap."""
    q, k, v, dO = qkv(1, 2, 1, 22, 8, seed=13)
    c = rnd((8,), 99)
    k2 = k + c
    o, lse = oracle.attn_fwd(q, k, v, 0.3, 6, 0.0)
    o2, lse2 = oracle.attn_fwd(q, k2, v, 0.3, 6, 0.0)
    np.testing.assert_allclose(o2, o, rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse2 - lse, 0.3 * (q @ c).numpy(), rtol=0, atol=1e-12)
    dq, dk, dv, _, _ = oracle.attn_bwd(q, k, v, dO, 0.3, 6, 0.0)
    dq2, dk2, dv2, _, _ = oracle.attn_bwd(q, k2, v, dO, 0.3, 6, 0.0)
    np.testing.assert_allclose(dq2, dq, rtol=0, atol=1e-12)
    np.testing.assert_allclose(dv2, dv, rtol=0, atol=1e-12)


def test_delta_identity():
    q, k, v, dO = qkv(2, 4, 2, 24, 8, seed=14)
    for W, C in ((0, 0.0), (7, 2.0)):
        o, _ = oracle.attn_fwd(q, k, v, 0.5, W, C)
        _, _, _, delta, _ = oracle.attn_bwd(q, k, v, dO, 0.5, W, C)
        np.testing.assert_allclose(delta, oracle.rowdot(o, dO), rtol=1e-12, atol=1e-13)
        # and the library form
        np.testing.assert_allclose(delta, (torch.from_numpy(o) * dO).sum(-1).numpy(),
                                   rtol=1e-12, atol=1e-13)


def test_closed_form_single_token_and_window_one():
    q, k, v, dO = qkv(1, 4, 2, 1, 8, seed=15)
    o, lse = oracle.attn_fwd(q, k, v, 0.7, 0, 0.0)
    np.testing.assert_allclose(o, v.repeat_interleave(2, dim=1).numpy(), rtol=0, atol=1e-15)
    np.testing.assert_allclose(lse, 0.7 * (q * k.repeat_interleave(2, 1)).sum(-1).numpy(),
                               rtol=1e-14, atol=1e-14)
    # W = 1: every query sees only itself
    q, k, v, dO = qkv(1, 4, 2, 17, 8, seed=16)
    o, lse = oracle.attn_fwd(q, k, v, 0.7, 1, 2.0)
    np.testing.assert_allclose(o, v.repeat_interleave(2, dim=1).numpy(), rtol=0, atol=1e-15)
    s = 0.7 * (q * k.repeat_interleave(2, 1)).sum(-1)
    np.testing.assert_allclose(lse, (2.0 * torch.tanh(s / 2.0)).numpy(), rtol=1e-13, atol=1e-13)
    dq, dk, dv, _, _ = oracle.attn_bwd(q, k, v, dO, 0.7, 1, 2.0)
    assert np.max(np.abs(dq)) < 1e-14 and np.max(np.abs(dk)) < 1e-14
    np.testing.assert_allclose(dv, dO.reshape(1, 2, 2, 17, 8).sum(2).numpy(), rtol=0, atol=1e-14)


def test_closed_form_zero_query_uniform_average():
    T, D = 26, 8
    _, k, v, _ = qkv(1, 1, 1, T, D, seed=17)
    q = torch.zeros(1, 1, T, D, dtype=torch.float64)
    for W in (0, 5):
        o, lse = oracle.attn_fwd(q, k, v, 0.6, W, 0.0)
        for i in range(T):
            lo = max(0, i - W + 1) if W else 0
            np.testing.assert_allclose(o[0, 0, i], v[0, 0, lo:i + 1].mean(0).numpy(), rtol=0, atol=1e-14)
            assert abs(lse[0, 0, i] - math.log(i + 1 - lo)) < 1e-14


def test_closed_form_constant_value():
    q, k, _, dO = qkv(1, 2, 1, 20, 8, seed=18)
    v = torch.full((1, 1, 20, 8), 0.0, dtype=torch.float64) + torch.arange(8.0, dtype=torch.float64)
    o, _ = oracle.attn_fwd(q, k, v, 0.5, 0, 3.0)
    np.testing.assert_allclose(o, np.broadcast_to(np.arange(8.0), o.shape), rtol=0, atol=1e-13)
    dq, dk, dv, _, _ = oracle.attn_bwd(q, k, v, dO, 0.5, 0, 3.0)
    assert np.max(np.abs(dq)) < 1e-12 and np.max(np.abs(dk)) < 1e-12


# ------------------------------------------- Delta from the stored (rounded) O

def test_rounding_matches_torch_conversions():
    g = torch.Generator().manual_seed(21)
    x = torch.cat([torch.randn(20000, generator=g, dtype=torch.float64) * 10 ** torch.randint(-6, 6, (20000,),
                                                                                                 generator=g),
                   torch.tensor([0.0, -0.0, 1.0, 1.00390625, 1.01171875, 1.0078125, 65504.0, 3.3e38, -2.5e-40,
                                 1e-45, float("inf"), -float("inf")], dtype=torch.float64)])
    np.testing.assert_array_equal(oracle.round_to(x, "f32"), x.to(torch.float32).double().numpy())
    np.testing.assert_array_equal(oracle.round_to(x, "bf16"),
                                  x.to(torch.float32).to(torch.bfloat16).double().numpy())


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_delta_from_rounded_output(dtype):
    q, k, v, dO = qkv(1, 4, 2, 30, 8, seed=22)
    for W, C in ((0, 0.0), (7, 2.0)):
        o, _ = oracle.attn_fwd(q, k, v, 0.5, W, C)
        tdt = torch.float32 if dtype == "f32" else torch.bfloat16
        o_stored = torch.from_numpy(o).to(torch.float32).to(tdt).double()
        want = (o_stored * dO).sum(-1).numpy()
        _, _, _, delta, _ = oracle.attn_bwd(q, k, v, dO, 0.5, W, C, o_round=dtype)
        np.testing.assert_allclose(delta, want, rtol=1e-12, atol=1e-12)
        # the gradient moves only through Delta: dV is unchanged, and dQ moves by
        # -scale * dDelta_i * sum_j P_ij cap'_ij K_j
        ex = oracle.attn_bwd(q, k, v, dO, 0.5, W, C)
        rd = oracle.attn_bwd(q, k, v, dO, 0.5, W, C, o_round=dtype)
        np.testing.assert_array_equal(rd[2], ex[2])
        P = oracle.attn_probs(q, k, 0.5, W, C)
        kr = k.repeat_interleave(2, dim=1).numpy()
        S = 0.5 * np.einsum("bhid,bhjd->bhij", q.numpy(), kr)
        cg = (1 - np.tanh(S / C) ** 2) if C else 1.0
        U = np.einsum("bhij,bhjd->bhid", P * cg, kr)
        np.testing.assert_allclose(rd[0] - ex[0], -0.5 * (rd[3] - ex[3])[..., None] * U, rtol=1e-9, atol=1e-13)


# ---------------------------------------------------------------- attention sinks
# A sink is a learned logit per query head in the softmax denominator with no
# value vector (ARCHITECTURES.md family table, GPT-OSS row; "Vague 2" item 10;
# SMALL_MODELS_RESEARCH.md section 2.4).

def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def test_sink_minus_infinity_is_plain_softmax_bitwise():
    q, k, v, dO = _rand((2, 4, 9, 8), 1), _rand((2, 2, 9, 8), 2), _rand((2, 2, 9, 8), 3), _rand((2, 4, 9, 8), 4)
    sink = np.full(4, -np.inf)
    o, lse = oracle.attn_fwd(q, k, v, 0.3, 4, 2.0)
    o2, lse2, _ = oracle.attn_fwd_ext(q, k, v, 0.3, 4, 2.0, sink=sink)
    assert np.array_equal(o, o2) and np.array_equal(lse, lse2)
    g = oracle.attn_bwd(q, k, v, dO, 0.3, 4, 2.0)
    g2 = oracle.attn_bwd_ext(q, k, v, dO, 0.3, 4, 2.0, sink=sink)
    for a, b in zip(g[:3] + g[3:], g2[:3] + g2[4:]):
        assert np.array_equal(a, b)
    assert np.all(g2[3] == 0.0)


def _augment_with_sink_key(q, k, v, dO, sink, scale, c=0.75):
    """The sink as a real key: one extra feature (query h: sink_h / (scale * c),
    keys: c for a new key at position 0, 0 elsewhere) and a zero value vector, so
    every query's score with the new key is sink_h and it adds nothing to O."""
    B, Hq, T, D = q.shape
    Hkv = k.shape[1]
    qa = np.zeros((B, Hq, T + 1, D + 1)); ka = np.zeros((B, Hkv, T + 1, D + 1))
    va = np.zeros((B, Hkv, T + 1, D + 1)); doa = np.zeros((B, Hq, T + 1, D + 1))
    qa[:, :, 1:, :D] = q
    qa[:, :, :, D] = (sink / (scale * c))[None, :, None]
    ka[:, :, 1:, :D] = k
    ka[:, :, 0, D] = c
    va[:, :, 1:, :D] = v   # the new key's value and every value's extra feature are 0
    doa[:, :, 1:, :D] = dO  # the new position 0 is not a real query: no upstream gradient
    return qa, ka, va, doa


@pytest.mark.parametrize("Hq,Hkv", [(2, 2), (4, 2)])
def test_sink_equals_an_extra_zero_value_key(Hq, Hkv):
    B, T, D, scale = 2, 11, 6, 0.4
    q, k, v, dO = _rand((B, Hq, T, D), 5), _rand((B, Hkv, T, D), 6), _rand((B, Hkv, T, D), 7), _rand((B, Hq, T, D), 8)
    sink = np.linspace(-1.0, 1.5, Hq)
    o, lse, _ = oracle.attn_fwd_ext(q, k, v, scale, 0, 0.0, sink=sink)
    qa, ka, va, doa = _augment_with_sink_key(q, k, v, dO, sink, scale)
    oa, lsea = oracle.attn_fwd(qa, ka, va, scale)
    np.testing.assert_allclose(o, oa[:, :, 1:, :D], rtol=0, atol=1e-12)
    assert np.all(oa[:, :, 1:, D] == 0.0)
    np.testing.assert_allclose(lse, lsea[:, :, 1:], rtol=0, atol=1e-12)
    dq, dk, dv, dsink, _, _ = oracle.attn_bwd_ext(q, k, v, dO, scale, 0, 0.0, sink=sink)
    dqa, dka, dva, _, _ = oracle.attn_bwd(qa, ka, va, doa, scale)
    np.testing.assert_allclose(dq, dqa[:, :, 1:, :D], rtol=0, atol=1e-11)
    np.testing.assert_allclose(dk, dka[:, :, 1:, :D], rtol=0, atol=1e-11)
    np.testing.assert_allclose(dv, dva[:, :, 1:, :D], rtol=0, atol=1e-11)
    # d/d sink_h: through the extra query feature, d s_sink / d qa_extra = scale * c
    np.testing.assert_allclose(dsink, dqa[:, :, 1:, D].sum(axis=(0, 2)) / (scale * 0.75), rtol=0, atol=1e-11)


def test_sink_closed_form_single_key():
    # T = 1: s = scale * q.k = 0.5 * 2 = 1; P(key) = e / (e + e^sigma), sigma = ln 3
    q = np.array([1.0, 0.0]).reshape(1, 1, 1, 2)
    k = np.array([2.0, 0.0]).reshape(1, 1, 1, 2)
    v = np.array([4.0, -2.0]).reshape(1, 1, 1, 2)
    o, lse, ml = oracle.attn_fwd_ext(q, k, v, 0.5, sink=np.array([math.log(3.0)]))
    p = math.e / (math.e + 3.0)
    np.testing.assert_allclose(o.ravel(), [4.0 * p, -2.0 * p], rtol=1e-15)
    np.testing.assert_allclose(lse.ravel(), [math.log(math.e + 3.0)], rtol=1e-15)
    assert ml.ravel()[0] == 1.0
    # dO = (1, 0): loss = O_0 = 4 p(sigma); d/dsigma = -4 p (1 - p)
    dO = np.array([1.0, 0.0]).reshape(1, 1, 1, 2)
    _, _, _, dsink, _, _ = oracle.attn_bwd_ext(q, k, v, dO, 0.5, sink=np.array([math.log(3.0)]))
    np.testing.assert_allclose(dsink, [-4.0 * p * (1.0 - p)], rtol=1e-13)


@pytest.mark.parametrize("W,C", [(0, 0.0), (3, 0.0), (0, 1.5), (4, 2.0)])
def test_dsink_central_finite_differences(W, C):
    B, Hq, Hkv, T, D, scale = 2, 4, 2, 10, 5, 0.6
    q, k, v, dO = _rand((B, Hq, T, D), 9), _rand((B, Hkv, T, D), 10), _rand((B, Hkv, T, D), 11), _rand((B, Hq, T, D), 12)
    sink = np.array([0.2, -0.7, 1.1, 0.0])
    _, _, _, dsink, _, _ = oracle.attn_bwd_ext(q, k, v, dO, scale, W, C, sink=sink)
    h = 1e-6
    for i in range(Hq):
        sp, sm = sink.copy(), sink.copy()
        sp[i] += h
        sm[i] -= h
        lp = np.sum(oracle.attn_fwd_ext(q, k, v, scale, W, C, sink=sp)[0] * dO)
        lm = np.sum(oracle.attn_fwd_ext(q, k, v, scale, W, C, sink=sm)[0] * dO)
        np.testing.assert_allclose(dsink[i], (lp - lm) / (2 * h), rtol=1e-6, atol=1e-9)


# ---------------------------------------------------------------- max logit
# The per-head maximum attention logit that QK-Clip monitors (ARCHITECTURES.md
# "Vague 3" item 12; family table, Kimi K2 row).

def test_max_logit_hand_example():
    # D = 1, scale 1: q = (1, 2, -1), k = (3, -1, 0.5). Allowed scores (i, j):
    # causal (0,0)=3 (1,0)=6 (1,1)=-2 (2,0)=-3 (2,1)=1 (2,2)=-0.5 -> max 6;
    # window 1 keeps the diagonal 3, -2, -0.5 -> max 3; a cap of 2 maps them to
    # 2 tanh(6/2) and 2 tanh(3/2).
    q = np.array([1.0, 2.0, -1.0]).reshape(1, 1, 3, 1)
    k = np.array([3.0, -1.0, 0.5]).reshape(1, 1, 3, 1)
    v = np.ones((1, 1, 3, 1))
    assert oracle.attn_fwd_ext(q, k, v, 1.0)[2].ravel()[0] == 6.0
    assert oracle.attn_fwd_ext(q, k, v, 1.0, 1)[2].ravel()[0] == 3.0
    np.testing.assert_allclose(oracle.attn_fwd_ext(q, k, v, 1.0, 0, 2.0)[2].ravel()[0], 2 * math.tanh(3.0), rtol=1e-15)
    np.testing.assert_allclose(oracle.attn_fwd_ext(q, k, v, 1.0, 1, 2.0)[2].ravel()[0], 2 * math.tanh(1.5), rtol=1e-15)
    # the sink is not a logit of the max
    assert oracle.attn_fwd_ext(q, k, v, 1.0, sink=np.array([50.0]))[2].ravel()[0] == 6.0


def test_max_logit_is_attained_by_an_allowed_pair_and_bounds_the_rest():
    B, Hq, Hkv, T, D, scale, W = 2, 4, 2, 13, 6, 0.5, 5
    q, k, v = _rand((B, Hq, T, D), 13), _rand((B, Hkv, T, D), 14), _rand((B, Hkv, T, D), 15)
    ml = oracle.attn_fwd_ext(q, k, v, scale, W)[2]
    kk = np.repeat(k, Hq // Hkv, axis=1)
    s = scale * np.einsum("bhid,bhjd->bhij", q, kk)
    i, j = np.arange(T)[:, None], np.arange(T)[None, :]
    allowed = (j <= i) & (j > i - W)
    s_allowed = np.where(allowed, s, -np.inf)
    assert np.all(s_allowed <= ml[:, :, None, None] + 0.0)
    hits = np.isclose(s_allowed, ml[:, :, None, None], rtol=0, atol=1e-12) & allowed
    assert np.all(hits.any(axis=(2, 3)))


# ---------------------------------------------------------------- decode
# One new query per (b, hq) against a KV cache (INFERENCE_RESEARCH.md section 2).

@pytest.mark.parametrize("W,C,use_sink", [(0, 0.0, False), (5, 0.0, False), (0, 2.0, True), (4, 1.5, True)])
def test_decode_equals_last_row_of_the_forward(W, C, use_sink):
    B, Hq, Hkv, T, Tmax, D, scale = 2, 4, 2, 13, 16, 6, 0.45
    qf, kc, vc = _rand((B, Hq, T, D), 21), _rand((B, Hkv, Tmax, D), 22), _rand((B, Hkv, Tmax, D), 23)
    sink = np.array([0.5, -0.3, 1.2, 0.1]) if use_sink else None
    o, lse = oracle.attn_decode(qf[:, :, T - 1], kc, vc, scale, T, W, C, sink=sink)
    ro, rl, _ = oracle.attn_fwd_ext(qf, kc[:, :, :T], vc[:, :, :T], scale, W, C, sink=sink)
    np.testing.assert_array_equal(o, ro[:, :, T - 1])
    np.testing.assert_array_equal(lse, rl[:, :, T - 1])


def test_decode_per_entry_lengths_and_cache_tail_ignored():
    B, Hq, Hkv, Tmax, D, scale = 3, 2, 1, 12, 5, 0.5
    q, kc, vc = _rand((B, Hq, D), 24), _rand((B, Hkv, Tmax, D), 25), _rand((B, Hkv, Tmax, D), 26)
    lens = [12, 1, 7]
    o, lse = oracle.attn_decode(q, kc, vc, scale, Tmax, seq_lens=lens)
    kc2, vc2 = kc.copy(), vc.copy()
    for b, n in enumerate(lens):
        kc2[b, :, n:] = 1e6   # positions past the entry's length are never read
        vc2[b, :, n:] = np.nan
        ob, lb = oracle.attn_decode(q[b:b + 1], kc[b:b + 1], vc[b:b + 1], scale, n)
        np.testing.assert_array_equal(o[b:b + 1], ob)
        np.testing.assert_array_equal(lse[b:b + 1], lb)
    o2, lse2 = oracle.attn_decode(q, kc2, vc2, scale, Tmax, seq_lens=lens)
    np.testing.assert_array_equal(o, o2)
    # length 1 sees only position 0: o = v[0], lse = the one score
    np.testing.assert_allclose(o[1], np.repeat(vc[1, :, 0], Hq // Hkv, axis=0), rtol=1e-15)
    np.testing.assert_allclose(lse[1], scale * (q[1] @ kc[1, 0, 0]), rtol=1e-14)


# ---------------------------------------------------------------- d_k != d_v
# Decompressed multi-head latent attention: q.k over d_k = nope + rope, values of
# d_v ("Vague 3" item 13; family table, DeepSeek V3 row).

@pytest.mark.parametrize("B,Hq,Hkv,T,Dk,Dv,W,C", [
    (1, 2, 2, 23, 12, 8, 0, 0.0),
    (2, 4, 2, 31, 24, 16, 5, 0.0),
    (1, 2, 1, 19, 8, 12, 0, 3.0),   # d_v > d_k too
    (1, 3, 3, 27, 12, 8, 7, 2.0),
])
def test_dk_ne_dv_matches_torch_sdpa_autograd(B, Hq, Hkv, T, Dk, Dv, W, C):
    sig = 2.0 if C else 1.0
    q, k = rnd((B, Hq, T, Dk), 31, sig), rnd((B, Hkv, T, Dk), 32, sig)
    v, dO = rnd((B, Hkv, T, Dv), 33), rnd((B, Hq, T, Dv), 34)
    scale = 1.0 / math.sqrt(Dk)
    o_ref, dq_ref, dk_ref, dv_ref = sdpa_grads(q, k, v, dO, scale, W, C)
    o, lse, _ = oracle.attn_fwd_ext(q, k, v, scale, W, C)
    assert o.shape == (B, Hq, T, Dv)
    np.testing.assert_allclose(o, o_ref.numpy(), rtol=1e-12, atol=1e-12)
    dq, dk, dv, _, _, lse2 = oracle.attn_bwd_ext(q, k, v, dO, scale, W, C)
    np.testing.assert_allclose(dq, dq_ref.numpy(), rtol=1e-10, atol=1e-11)
    np.testing.assert_allclose(dk, dk_ref.numpy(), rtol=1e-10, atol=1e-11)
    np.testing.assert_allclose(dv, dv_ref.numpy(), rtol=1e-10, atol=1e-11)
    np.testing.assert_array_equal(lse, lse2)


def test_dk_ne_dv_value_columns_are_independent():
    # o's value columns come from v's alone: cutting v (and dO) to its first
    # columns gives the first columns of o and dv, and the same dq, dk when dO
    # is zero on the columns cut
    B, Hq, Hkv, T, Dk, Dv = 1, 2, 1, 17, 8, 12
    q, k = rnd((B, Hq, T, Dk), 35), rnd((B, Hkv, T, Dk), 36)
    v, dO = rnd((B, Hkv, T, Dv), 37), rnd((B, Hq, T, Dv), 38)
    dO[..., 5:] = 0.0
    o, lse, _ = oracle.attn_fwd_ext(q, k, v, 0.3)
    o5, lse5, _ = oracle.attn_fwd_ext(q, k, v[..., :5], 0.3)
    np.testing.assert_array_equal(o[..., :5], o5)
    np.testing.assert_array_equal(lse, lse5)
    g = oracle.attn_bwd_ext(q, k, v, dO, 0.3)
    g5 = oracle.attn_bwd_ext(q, k, v[..., :5], dO[..., :5], 0.3)
    np.testing.assert_allclose(g[0], g5[0], rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(g[1], g5[1], rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(g[2][..., :5], g5[2], rtol=1e-13, atol=1e-14)
