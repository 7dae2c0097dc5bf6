"""GPU parity where the (batch, head) pairs outnumber the 65535 blocks that grid y
allows. The f32 CUDA-core kernels take one block row per (b, query head) or
(b, KV head) pair, and the decode split kernels one per (b, KV head); past 65535
pairs the launches spread them over grid y and z. Heads (and decode entries) are
independent, so a sample that spans both z slices is compared with the oracle,
and a one-token sequence adds its closed forms for every head: the only allowed
key is the query's own, so o = v, lse = the scaled score, dv = dO and dq = dk = 0
(Forge config schema, forge-studio RESEARCH.md section 2: B, n_heads up to what
the sizes allow; the header's limit is B * Hq <= 2^24)."""
import math

import numpy as np
import pytest
import torch

import oracle
import causal_flash_attention_attn_b200 as fa
from parity_util import check_close

pytestmark = pytest.mark.gpu

PAIRS = 65537                      # two more than grid y takes
SAMPLE = [0, 1, 65533, 65534, 65535, 65536]  # pairs 65535 and 65536 sit in the second z slice


def _fwd_bwd(q, k, v, dO, scale):
    dev = torch.device("cuda:0")
    qd, kd, vd, dOd = (x.to(dev) for x in (q, k, v, dO))
    o, lse = fa.attention_fwd(qd, kd, vd, scale)
    dq, dk, dv = fa.attention_bwd(qd, kd, vd, o, lse, dOd, scale)
    torch.cuda.synchronize()
    assert fa.forge_attn_check() == fa.FORGE_OK
    return o.cpu(), lse.cpu(), dq.cpu(), dk.cpu(), dv.cpu()


def test_f32_one_token_closed_forms_on_every_head():
    g = torch.Generator(device="cpu").manual_seed(11)
    q, k, v, dO = (torch.randn(1, PAIRS, 1, 64, generator=g) for _ in range(4))
    sc = 1.0 / 8.0
    o, lse, dq, dk, dv = _fwd_bwd(q, k, v, dO, sc)
    assert torch.equal(o, v)       # one key with probability exactly 1
    assert torch.equal(dv, dO)
    s = sc * (q.double() * k.double()).sum(-1)
    check_close("lse", lse, s.numpy(), "f32")
    check_close("dq", dq, np.zeros(dq.shape), "f32")
    check_close("dk", dk, np.zeros(dk.shape), "f32")


def test_f32_sampled_heads_match_oracle():
    g = torch.Generator(device="cpu").manual_seed(12)
    T, D = 3, 64
    q, k, v, dO = (torch.randn(1, PAIRS, T, D, generator=g) for _ in range(4))
    sc = 1.0 / math.sqrt(D)
    o, lse, dq, dk, dv = _fwd_bwd(q, k, v, dO, sc)
    idx = torch.tensor(SAMPLE)
    qs, ks, vs, dOs = (x[:, idx] for x in (q, k, v, dO))
    ro, rl = oracle.attn_fwd(qs, ks, vs, sc)
    rdq, rdk, rdv, _, _ = oracle.attn_bwd(qs, ks, vs, dOs, sc, o_round="f32")
    for name, got, ref in (("o", o, ro), ("lse", lse, rl), ("dq", dq, rdq), ("dk", dk, rdk), ("dv", dv, rdv)):
        check_close(name, got[:, idx], ref, "f32")


DECODE = [
    # name, B, Hq, Hkv, D: B * Hkv > 65535; the warp-pipelined kernel (G 4, D 128)
    # and the CTA-wide one (G 8, D 256)
    ("warp_g4_d128", 16385, 16, 4, 128),
    ("cta_g8_d256", 65536, 8, 1, 256),
]


@pytest.mark.parametrize("case", DECODE, ids=[c[0] for c in DECODE])
def test_decode_sampled_entries_match_oracle(case):
    name, B, Hq, Hkv, D = case
    T, Tmax = 5, 8
    g = torch.Generator(device="cpu").manual_seed(13)
    q = torch.randn(B, Hq, D, generator=g).to(torch.bfloat16)
    kc = torch.randn(B, Hkv, Tmax, D, generator=g).to(torch.bfloat16)
    vc = torch.randn(B, Hkv, Tmax, D, generator=g).to(torch.bfloat16)
    dev = torch.device("cuda:0")
    sc = 1.0 / math.sqrt(D)
    o, lse = fa.attention_decode(q.to(dev), kc.to(dev), vc.to(dev), T=T, scale=sc)
    torch.cuda.synchronize()
    assert fa.forge_attn_check() == fa.FORGE_OK
    # entries whose KV heads include pairs on both sides of 65535 (pair = b * Hkv + kv head)
    ents = sorted({p // Hkv for p in SAMPLE if p < B * Hkv} | {B - 1})
    e = torch.tensor(ents)
    ro, rl = oracle.attn_decode(q[e], kc[e], vc[e], sc, T)
    check_close("o", o.cpu()[e], ro, "bf16")
    check_close("lse", lse.cpu()[e], rl, "bf16")
