"""forge_attn_bwd_noalloc: the backward for callers that cannot allocate device
memory (hosts that only receive device buffers from another runtime, or processes
whose memory pool owns the whole device). Its scratch is a fixed 32 MiB array in
the library that every call shares.

Checked through the C ABI against forge_attn_bwd with a fresh caller workspace:
dk and dv bit for bit (each is summed inside one CTA in a fixed order, so the two
entry points must agree exactly), dq within the bf16 / f32 bar (its reductions
run in a varying order) and against the f64 oracle. Calls come two in a row on
one shape, and as a larger shape followed by a smaller one with another padded
length and head count, so that nothing one call leaves in the shared array can
reach the next call's results. Kept in its own file, collected last."""
import math

import numpy as np
import pytest
import torch

import causal_flash_attention_attn_b200 as fa
import oracle
from causal_flash_attention_attn_b200 import inputs

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda:0")


def _close(name, a, b, dtype):
    a = a.double().cpu().numpy() if hasattr(a, "detach") else np.asarray(a, np.float64)
    b = b.double().cpu().numpy() if hasattr(b, "detach") else np.asarray(b, np.float64)
    assert np.all(np.isfinite(a)), name
    err = np.abs(a - b)
    if dtype == "f32":
        assert err.max() <= 1e-4, f"{name}: {err.max():.3e}"
    else:
        assert np.all(err <= 2e-2 + 1e-2 * np.abs(b)), f"{name}: {err.max():.3e}"


def _setup(w):
    q, k, v, dO = inputs.make_inputs(w)
    qd, kd, vd, dOd = (x.to(DEV) for x in (q, k, v, dO))
    o, lse = fa.attention_fwd(qd, kd, vd, w.sm_scale, w.window, w.softcap)
    return (q, k, v, dO), (qd, kd, vd, dOd, o, lse)


def _noalloc(w, dev_inputs):
    qd, kd, vd, dOd, o, lse = dev_inputs
    dq, dk, dv = (torch.full_like(x, float("nan")) for x in (qd, kd, vd))
    s = fa.forge_attn_bwd_noalloc(qd, kd, vd, o, lse, dOd, dq, dk, dv, w.B, w.Hq, w.Hkv, w.T, w.D, w.sm_scale,
                                  w.window, w.softcap, fa.dtype_code(qd.dtype))
    assert s == fa.FORGE_OK, fa.forge_attn_status_string(s)
    torch.cuda.synchronize()
    assert fa.forge_attn_check() == fa.FORGE_OK
    return dq, dk, dv


def _workspace_bwd(w, dev_inputs):
    """forge_attn_bwd with a fresh caller workspace (filled with 0xFF first)."""
    qd, kd, vd, dOd, o, lse = dev_inputs
    dt = fa.dtype_code(qd.dtype)
    dq, dk, dv = (torch.full_like(x, float("nan")) for x in (qd, kd, vd))
    n = fa.forge_attn_bwd_workspace_size(w.B, w.Hq, w.Hkv, w.T, w.D, dt)
    ws = torch.full((n,), 255, dtype=torch.uint8, device=DEV)
    s = fa.forge_attn_bwd(qd, kd, vd, o, lse, dOd, dq, dk, dv, w.B, w.Hq, w.Hkv, w.T, w.D, w.sm_scale, w.window,
                          w.softcap, dt, ws, n)
    assert s == fa.FORGE_OK, fa.forge_attn_status_string(s)
    torch.cuda.synchronize()
    assert fa.forge_attn_check() == fa.FORGE_OK
    return dq, dk, dv


def _check_against_both(w, host_inputs, dev_inputs, got):
    dq, dk, dv = got
    rdq, rdk, rdv = _workspace_bwd(w, dev_inputs)
    assert torch.equal(dk, rdk), f"{w.name}: dk differs from forge_attn_bwd"
    assert torch.equal(dv, rdv), f"{w.name}: dv differs from forge_attn_bwd"
    _close(w.name + " dq vs forge_attn_bwd", dq, rdq, w.dtype)
    q, k, v, dO = host_inputs
    odq, odk, odv, _, _ = oracle.attn_bwd(q, k, v, dO, w.sm_scale, w.window, w.softcap, o_round=w.dtype)
    _close(w.name + " dq vs oracle", dq, odq, w.dtype)
    _close(w.name + " dk vs oracle", dk, odk, w.dtype)
    _close(w.name + " dv vs oracle", dv, odv, w.dtype)


@pytest.mark.parametrize("w", [
    inputs.Workload("noalloc_bf16", "bf16", 2, 4, 2, 300, 128, window=0, seed=31),
    inputs.Workload("noalloc_bf16_win_cap", "bf16", 1, 4, 1, 257, 64, window=100, softcap=5.0, seed=32,
                    sigma_q=2.0, sigma_k=2.0),
    inputs.Workload("noalloc_f32", "f32", 1, 2, 2, 200, 64, seed=33),
])
def test_noalloc_matches_workspace_backward_twice(w):
    host, dev = _setup(w)
    for _ in range(2):
        _check_against_both(w, host, dev, _noalloc(w, dev))


def test_noalloc_larger_call_then_smaller_call():
    # the first call fills more rows of the array (B*Hq = 8, padded length 384)
    # than the second reads (B*Hq = 2, padded length 256), with another layout
    big = inputs.Workload("noalloc_big", "bf16", 2, 4, 2, 300, 128, seed=34)
    small = inputs.Workload("noalloc_small", "bf16", 1, 2, 1, 130, 128, window=50, seed=35)
    hb, db = _setup(big)
    _noalloc(big, db)
    hs, ds = _setup(small)
    _check_against_both(small, hs, ds, _noalloc(small, ds))


def test_noalloc_rejects_problems_beyond_its_scratch():
    # 2 x 28 x 4096 x 128 needs ~117 MB of scratch: rejected, nothing launched
    A = 0x10000
    s = fa.forge_attn_bwd_noalloc(A, A, A, A, A, A, A, A, A, 2, 28, 4, 4096, 128, 0.088, 0, 0.0,
                                  fa.FORGE_DTYPE_BF16)
    assert s == fa.FORGE_ERR_WORKSPACE
    assert "32 MiB" in fa.forge_attn_last_cuda_error()
