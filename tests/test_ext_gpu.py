"""GPU parity of the extended entry points through the C ABI against the oracle:
attention sinks (ARCHITECTURES.md family table, GPT-OSS row; "Vague 2" item 10)
and the per-head max logit QK-Clip monitors ("Vague 3" item 12), on the
two-tile forward (head dims 64, 128), the single-tile forward (256) and the f32
path, with windows, caps, GQA and ragged lengths. Tolerances are those of the
other parity tests."""
import math

import numpy as np
import pytest
import torch

import oracle
import causal_flash_attention_attn_b200 as fa
from causal_flash_attention_attn_b200 import inputs
from parity_util import check_close

pytestmark = pytest.mark.gpu

CASES = [
    # name, dtype, B, Hq, Hkv, T, D, window, softcap
    ("bf16_d128", "bf16", 2, 4, 2, 300, 128, 0, 0.0),
    ("bf16_d128_win_cap", "bf16", 1, 4, 1, 385, 128, 100, 5.0),
    ("bf16_d64", "bf16", 2, 2, 2, 257, 64, 0, 0.0),
    ("bf16_d256_cap", "bf16", 1, 2, 1, 200, 256, 64, 50.0),
    ("f32_d64", "f32", 1, 2, 2, 130, 64, 0, 0.0),
    ("f32_d128_win", "f32", 1, 4, 2, 100, 128, 30, 0.0),
]


def _workload(name, dtype, B, Hq, Hkv, T, D, W, C, seed):
    return inputs.Workload(name, dtype, B, Hq, Hkv, T, D, window=W, softcap=C, seed=seed,
                           sigma_q=2.0 if C > 0 else 1.0, sigma_k=2.0 if C > 0 else 1.0)


def _sinks(Hq):
    # spread over the scores' range so that the sink takes a visible share
    return torch.tensor(np.linspace(-1.0, 2.5, Hq), dtype=torch.float32)


def _run_ext(w, sink, want_max=True):
    dev = torch.device("cuda:0")
    q, k, v, dO = (x.to(dev) for x in inputs.make_inputs(w))
    dt = fa.dtype_code(q.dtype)
    sc = 1.0 / math.sqrt(w.D)
    o = torch.full_like(q, float("nan"))
    lse = torch.full((w.B, w.Hq, w.T), float("nan"), device=dev)
    ml = torch.full((w.B, w.Hq), 123.0, device=dev) if want_max else None
    sk = sink.to(dev) if sink is not None else None
    s = fa.forge_attn_fwd_ext(q, k, v, o, lse, w.B, w.Hq, w.Hkv, w.T, w.D, sc, w.window, w.softcap, sk, ml, dt)
    assert s == fa.FORGE_OK, fa.forge_attn_status_string(s)
    nbytes = fa.forge_attn_bwd_workspace_size(w.B, w.Hq, w.Hkv, w.T, w.D, dt)
    ws = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    dq, dk, dv = (torch.full_like(x, float("nan")) for x in (q, k, v))
    dsink = torch.full((w.Hq,), float("nan"), device=dev) if sk is not None else None
    s = fa.forge_attn_bwd_ext(q, k, v, o, lse, dO, dq, dk, dv, w.B, w.Hq, w.Hkv, w.T, w.D, sc, w.window, w.softcap,
                              sk, dsink, dt, ws, nbytes)
    assert s == fa.FORGE_OK, fa.forge_attn_status_string(s)
    torch.cuda.synchronize()
    assert fa.forge_attn_check() == fa.FORGE_OK
    return (q.cpu(), k.cpu(), v.cpu(), dO.cpu()), (o.cpu(), lse.cpu(), None if ml is None else ml.cpu(), dq.cpu(),
                                                   dk.cpu(), dv.cpu(), None if dsink is None else dsink.cpu())


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_sink_and_max_logit_match_oracle(case):
    name, dtype, B, Hq, Hkv, T, D, W, C = case
    w = _workload(name, dtype, B, Hq, Hkv, T, D, W, C, seed=41)
    sink = _sinks(Hq)
    (q, k, v, dO), (o, lse, ml, dq, dk, dv, dsink) = _run_ext(w, sink)
    sc = 1.0 / math.sqrt(D)
    ro, rl, rml = oracle.attn_fwd_ext(q, k, v, sc, W, C, sink=sink)
    rdq, rdk, rdv, rds, rdelta, rlse = oracle.attn_bwd_ext(q, k, v, dO, sc, W, C, sink=sink, o_round=dtype)
    check_close("o", o, ro, dtype)
    check_close("lse", lse, rl, dtype)
    check_close("max_logit", ml, rml, dtype)
    check_close("dq", dq, rdq, dtype)
    check_close("dk", dk, rdk, dtype)
    check_close("dv", dv, rdv, dtype)
    if dtype == "f32":
        check_close("dsink", dsink, rds, dtype)
    else:
        # dsink is a sum over all B*T rows of exp(sink - lse) * Delta, terms of
        # both signs that largely cancel; each Delta carries the bf16 rounding of
        # o, so the bf16 bar (2e-2 + 1e-2 * magnitude) applies to the magnitude of
        # the summands, sum |terms|, as in the usual error bound of a sum.
        terms = np.exp(sink.double().numpy()[None, :, None] - rlse) * rdelta
        mag = np.abs(terms).sum(axis=(0, 2))
        err = np.abs(dsink.double().numpy() - rds)
        assert np.all(err <= 2e-2 + 1e-2 * mag), (err, mag, rds)
    # the sink visibly changes the result (the case is not trivially sink-free)
    ro0, _ = oracle.attn_fwd(q, k, v, sc, W, C)
    assert np.abs(ro - ro0).max() > 0.05


@pytest.mark.parametrize("case", [CASES[0], CASES[3], CASES[4]], ids=["bf16_d128", "bf16_d256", "f32_d64"])
def test_without_sink_equals_plain_entry_points_bitwise(case):
    """sink = NULL with a max-logit request computes o and lse exactly as
    forge_attn_fwd, and forge_attn_bwd_ext with NULLs exactly as forge_attn_bwd
    (dk, dv bit for bit; dq is summed over key tiles with f32 atomics, so the
    order of those additions may move its bf16 rounding by one unit)."""
    name, dtype, B, Hq, Hkv, T, D, W, C = case
    w = _workload(name, dtype, B, Hq, Hkv, T, D, W, C, seed=43)
    (q, k, v, dO), (o, lse, ml, dq, dk, dv, _) = _run_ext(w, None)
    dev = torch.device("cuda:0")
    qd, kd, vd, dOd = (x.to(dev) for x in (q, k, v, dO))
    sc = 1.0 / math.sqrt(D)
    o2, lse2 = fa.attention_fwd(qd, kd, vd, sc, W, C)
    dq2, dk2, dv2 = fa.attention_bwd(qd, kd, vd, o2, lse2, dOd, sc, W, C)
    torch.cuda.synchronize()
    for a, b in ((o, o2), (lse, lse2), (dk, dk2), (dv, dv2)):
        assert torch.equal(a, b.cpu())
    tol = 2.0 ** -7 if dtype == "bf16" else 1e-6
    assert torch.allclose(dq.float(), dq2.cpu().float(), rtol=tol, atol=1e-6)
    _, _, rml = oracle.attn_fwd_ext(q, k, v, sc, W, C)
    check_close("max_logit", ml, rml, dtype)

