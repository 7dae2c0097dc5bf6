"""GPU parity of the KV-cache decode (one query per entry and head against the
cache, INFERENCE_RESEARCH.md section 2) through the C ABI against the oracle, on
the three head dims, bf16 and f32, GQA, windows, caps, sinks and per-entry
lengths, through both split kernels (the warp-pipelined one for groups whose
queries fit a lane's registers, the CTA-wide one for the others). Tolerances
are those of the other parity tests."""
import math

import numpy as np
import pytest
import torch

import oracle
import causal_flash_attention_attn_b200 as fa
from parity_util import check_close

pytestmark = pytest.mark.gpu

CASES = [
    # name, dtype, B, Hq, Hkv, T, Tmax, D, window, softcap, sink, lens
    ("bf16_d128_gqa7", "bf16", 2, 14, 2, 1000, 1024, 128, 0, 0.0, False, None),
    ("bf16_d128_win", "bf16", 1, 8, 8, 3000, 3072, 128, 700, 0.0, False, None),
    ("bf16_d64_cap_sink", "bf16", 3, 4, 2, 500, 512, 64, 0, 30.0, True, None),
    ("bf16_d256_lens", "bf16", 3, 8, 4, 900, 960, 256, 0, 0.0, False, [900, 1, 77]),
    ("bf16_d128_g16_lens_win", "bf16", 2, 16, 1, 2048, 2048, 128, 100, 0.0, True, [2048, 129]),
    ("f32_d128", "f32", 2, 4, 2, 333, 400, 128, 0, 0.0, False, None),
    ("f32_d256_win_lens", "f32", 2, 2, 1, 260, 300, 256, 50, 0.0, False, [260, 10]),
    # groups of 4 query heads at head dims 128 and 256 (the warp-pipelined kernel),
    # ragged lengths; 8 heads at 256 (the CTA-wide kernel)
    ("bf16_d128_g4_lens", "bf16", 3, 16, 4, 1500, 1536, 128, 0, 0.0, False, [1500, 3, 1029]),
    ("bf16_d256_g4_cap_sink", "bf16", 2, 8, 2, 700, 768, 256, 0, 25.0, True, None),
    ("bf16_d256_g8_win", "bf16", 1, 8, 1, 800, 800, 256, 300, 0.0, False, None),
    ("f32_d64_mha_lens", "f32", 2, 3, 3, 450, 512, 64, 0, 0.0, False, [450, 33]),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_decode_matches_oracle(case):
    name, dtype, B, Hq, Hkv, T, Tmax, D, W, C, use_sink, lens = case
    g = torch.Generator(device="cpu").manual_seed(hash(name) % (2 ** 31))
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    sig = 2.0 if C > 0 else 1.0
    q = (torch.randn(B, Hq, D, generator=g) * sig).to(tdt)
    kc = (torch.randn(B, Hkv, Tmax, D, generator=g) * sig).to(tdt)
    vc = torch.randn(B, Hkv, Tmax, D, generator=g).to(tdt)
    sink = torch.tensor(np.linspace(-0.5, 3.0, Hq), dtype=torch.float32) if use_sink else None
    dev = torch.device("cuda:0")
    sc = 1.0 / math.sqrt(D)
    sl = torch.tensor(lens, dtype=torch.int32, device=dev) if lens is not None else None
    o, lse = fa.attention_decode(q.to(dev), kc.to(dev), vc.to(dev), T=T, scale=sc, window=W, softcap=C,
                                 seq_lens=sl, sink=None if sink is None else sink.to(dev))
    torch.cuda.synchronize()
    assert fa.forge_attn_check() == fa.FORGE_OK
    ro, rl = oracle.attn_decode(q, kc, vc, sc, T, W, C, sink=sink, seq_lens=lens)
    check_close("o", o.cpu(), ro, dtype)
    check_close("lse", lse.cpu(), rl, dtype)


def test_decode_length_beyond_T_is_reported():
    dev = torch.device("cuda:0")
    q = torch.randn(2, 2, 64, device=dev).to(torch.bfloat16)
    kc = torch.randn(2, 2, 256, 64, device=dev).to(torch.bfloat16)
    sl = torch.tensor([100, 200], dtype=torch.int32, device=dev)
    fa.attention_decode(q, kc, kc, T=150, seq_lens=sl)
    assert fa.forge_attn_check() == fa.FORGE_ERR_INVALID_ARG
    assert fa.forge_attn_check() == fa.FORGE_OK
