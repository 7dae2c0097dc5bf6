"""GPU parity of d_k != d_v (decompressed multi-head latent attention: q.k over
d_k = 192, values of d_v = 128; ARCHITECTURES.md "Vague 3" item 13) through the C
ABI against the oracle, with GQA, a window, a cap and ragged lengths: the f32
CUDA-core path at the f32 bar (1e-4 absolute), the bf16 tensor-core forward and
backward at the bf16 bar (2e-2 + 1e-2 |ref|)."""
import math

import pytest
import torch

import oracle
import causal_flash_attention_attn_b200 as fa
from parity_util import check_close

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,Hq,Hkv,T,W,C", [(1, 4, 2, 150, 0, 0.0), (2, 2, 1, 97, 40, 0.0), (1, 2, 2, 130, 0, 20.0)])
def test_dk192_dv128_matches_oracle(B, Hq, Hkv, T, W, C):
    Dk, Dv = 192, 128
    g = torch.Generator(device="cpu").manual_seed(T + W)
    q = torch.randn(B, Hq, T, Dk, generator=g)
    k = torch.randn(B, Hkv, T, Dk, generator=g)
    v = torch.randn(B, Hkv, T, Dv, generator=g)
    dO = torch.randn(B, Hq, T, Dv, generator=g)
    dev = torch.device("cuda:0")
    qd, kd, vd, dOd = (x.to(dev) for x in (q, k, v, dO))
    sc = 1.0 / math.sqrt(Dk)
    o = torch.full((B, Hq, T, Dv), float("nan"), device=dev)
    lse = torch.full((B, Hq, T), float("nan"), device=dev)
    s = fa.forge_attn_fwd_dkv(qd, kd, vd, o, lse, B, Hq, Hkv, T, Dk, Dv, sc, W, C, fa.FORGE_DTYPE_F32)
    assert s == fa.FORGE_OK, fa.forge_attn_status_string(s)
    nbytes = fa.forge_attn_bwd_workspace_size_dkv(B, Hq, Hkv, T, Dk, Dv, fa.FORGE_DTYPE_F32)
    ws = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    dq, dk, dv = (torch.full_like(x, float("nan")) for x in (qd, kd, vd))
    s = fa.forge_attn_bwd_dkv(qd, kd, vd, o, lse, dOd, dq, dk, dv, B, Hq, Hkv, T, Dk, Dv, sc, W, C,
                              fa.FORGE_DTYPE_F32, ws, nbytes)
    assert s == fa.FORGE_OK, fa.forge_attn_status_string(s)
    torch.cuda.synchronize()
    assert fa.forge_attn_check() == fa.FORGE_OK
    ro, rl, _ = oracle.attn_fwd_ext(q, k, v, sc, W, C)
    rdq, rdk, rdv, _, _, _ = oracle.attn_bwd_ext(q, k, v, dO, sc, W, C, o_round="f32")
    for name, a, b in (("o", o, ro), ("lse", lse, rl), ("dq", dq, rdq), ("dk", dk, rdk), ("dv", dv, rdv)):
        check_close(name, a.cpu(), b, "f32")


@pytest.mark.parametrize("B,Hq,Hkv,T,W,C", [(2, 4, 2, 300, 0, 0.0), (1, 2, 1, 257, 100, 0.0), (1, 4, 4, 200, 0, 20.0)])
def test_dk192_dv128_bf16_forward_matches_oracle(B, Hq, Hkv, T, W, C):
    """The tensor-core forward (single query tile per CTA, K/V ring slots sized
    for d_k) at the bf16 bar."""
    Dk, Dv = 192, 128
    g = torch.Generator(device="cpu").manual_seed(1000 + T + W)
    sig = 2.0 if C else 1.0
    q = (torch.randn(B, Hq, T, Dk, generator=g) * sig).to(torch.bfloat16)
    k = (torch.randn(B, Hkv, T, Dk, generator=g) * sig).to(torch.bfloat16)
    v = torch.randn(B, Hkv, T, Dv, generator=g).to(torch.bfloat16)
    dev = torch.device("cuda:0")
    qd, kd, vd = (x.to(dev) for x in (q, k, v))
    sc = 1.0 / math.sqrt(Dk)
    o = torch.full((B, Hq, T, Dv), float("nan"), device=dev).to(torch.bfloat16)
    lse = torch.full((B, Hq, T), float("nan"), device=dev)
    s = fa.forge_attn_fwd_dkv(qd, kd, vd, o, lse, B, Hq, Hkv, T, Dk, Dv, sc, W, C, fa.FORGE_DTYPE_BF16)
    assert s == fa.FORGE_OK, fa.forge_attn_status_string(s)
    torch.cuda.synchronize()
    assert fa.forge_attn_check() == fa.FORGE_OK
    ro, rl, _ = oracle.attn_fwd_ext(q, k, v, sc, W, C)
    check_close("o", o.cpu(), ro, "bf16")
    check_close("lse", lse.cpu(), rl, "bf16")


@pytest.mark.parametrize("B,Hq,Hkv,T,W,C", [
    (2, 4, 2, 300, 0, 0.0),     # GQA, ragged last tile
    (1, 2, 1, 257, 100, 0.0),   # window
    (1, 4, 4, 200, 0, 20.0),    # cap in the tanh regime
    (1, 8, 1, 520, 0, 0.0),     # eight query heads per KV head, several key tiles
    (1, 2, 2, 64, 0, 0.0),      # shorter than one tile
    (2, 2, 1, 1, 0, 0.0),       # one token
    (1, 2, 1, 700, 129, 5.0),   # window and a small cap over many tiles
])
def test_dk192_dv128_bf16_backward_matches_oracle(B, Hq, Hkv, T, W, C):
    """The tensor-core backward (a dK/dV kernel and a dQ kernel) after the
    tensor-core forward, every output NaN-filled first, against the oracle with
    Delta from its own O rounded to bf16 (the o the forward returns)."""
    Dk, Dv = 192, 128
    g = torch.Generator(device="cpu").manual_seed(2000 + T + W)
    sig = 2.0 if C else 1.0
    q = (torch.randn(B, Hq, T, Dk, generator=g) * sig).to(torch.bfloat16)
    k = (torch.randn(B, Hkv, T, Dk, generator=g) * sig).to(torch.bfloat16)
    v = torch.randn(B, Hkv, T, Dv, generator=g).to(torch.bfloat16)
    dO = torch.randn(B, Hq, T, Dv, generator=g).to(torch.bfloat16)
    dev = torch.device("cuda:0")
    qd, kd, vd, dOd = (x.to(dev) for x in (q, k, v, dO))
    sc = 1.0 / math.sqrt(Dk)
    o = torch.full((B, Hq, T, Dv), float("nan"), device=dev).to(torch.bfloat16)
    lse = torch.full((B, Hq, T), float("nan"), device=dev)
    s = fa.forge_attn_fwd_dkv(qd, kd, vd, o, lse, B, Hq, Hkv, T, Dk, Dv, sc, W, C, fa.FORGE_DTYPE_BF16)
    assert s == fa.FORGE_OK, fa.forge_attn_status_string(s)
    nbytes = fa.forge_attn_bwd_workspace_size_dkv(B, Hq, Hkv, T, Dk, Dv, fa.FORGE_DTYPE_BF16)
    ws = torch.full((nbytes,), 255, dtype=torch.uint8, device=dev)
    dq, dk, dv = (torch.full_like(x, float("nan")) for x in (qd, kd, vd))
    s = fa.forge_attn_bwd_dkv(qd, kd, vd, o, lse, dOd, dq, dk, dv, B, Hq, Hkv, T, Dk, Dv, sc, W, C,
                              fa.FORGE_DTYPE_BF16, ws, nbytes)
    assert s == fa.FORGE_OK, fa.forge_attn_status_string(s)
    torch.cuda.synchronize()
    assert fa.forge_attn_check() == fa.FORGE_OK
    rdq, rdk, rdv, _, _, _ = oracle.attn_bwd_ext(q, k, v, dO, sc, W, C, o_round="bf16")
    for name, a, b in (("dq", dq, rdq), ("dk", dk, rdk), ("dv", dv, rdv)):
        check_close(name, a.cpu(), b, "bf16")


def test_dk192_dv128_bf16_backward_deterministic():
    """Neither kernel reduces across CTAs: two runs agree bit for bit."""
    Dk, Dv, B, Hq, Hkv, T = 192, 128, 1, 4, 2, 333
    g = torch.Generator(device="cpu").manual_seed(77)
    dev = torch.device("cuda:0")
    q = torch.randn(B, Hq, T, Dk, generator=g).to(torch.bfloat16).to(dev)
    k = torch.randn(B, Hkv, T, Dk, generator=g).to(torch.bfloat16).to(dev)
    v = torch.randn(B, Hkv, T, Dv, generator=g).to(torch.bfloat16).to(dev)
    dO = torch.randn(B, Hq, T, Dv, generator=g).to(torch.bfloat16).to(dev)
    o, lse = fa.attention_fwd(q, k, v)
    a = fa.attention_bwd(q, k, v, o, lse, dO)
    b = fa.attention_bwd(q, k, v, o, lse, dO)
    torch.cuda.synchronize()
    for x, y in zip(a, b):
        assert torch.equal(x, y)
