"""Helpers shared by the GPU parity tests: run the CUDA path and the oracle on the
same seeded inputs and compare with the path's stated tolerances:
max-abs 1e-4 on the f32 path (the Forge pages' own CPU-vs-GPU bar), and
|gpu - ref| <= 2e-2 + 1e-2 * |ref| elementwise for bf16 inputs with f32
accumulation."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import causal_flash_attention_attn_b200 as fa

ATOL_F32 = 1e-4
ATOL_BF16, RTOL_BF16 = 2e-2, 1e-2


def check_close(name, gpu, ref, dtype):
    gpu = gpu.detach().double().cpu().numpy() if hasattr(gpu, "detach") else np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    assert gpu.shape == ref.shape, (name, gpu.shape, ref.shape)
    assert np.all(np.isfinite(gpu)), f"{name}: non-finite values"
    err = np.abs(gpu - ref)
    if dtype == "f32":
        worst = float(err.max()) if err.size else 0.0
        assert worst <= ATOL_F32, f"{name}: max abs err {worst:.3e} > {ATOL_F32}"
        return worst
    bound = ATOL_BF16 + RTOL_BF16 * np.abs(ref)
    ratio = err / bound
    worst = float(ratio.max()) if ratio.size else 0.0
    if worst > 1.0:
        idx = np.unravel_index(int(np.argmax(ratio)), ratio.shape)
        raise AssertionError(f"{name}: err {err[idx]:.3e} at {idx} (gpu {gpu[idx]:.5f}, ref {ref[idx]:.5f}) "
                             f"exceeds {ATOL_BF16} + {RTOL_BF16}*|ref|; max abs err {err.max():.3e}")
    return float(err.max()) if err.size else 0.0


def run_gpu(q, k, v, dO, scale, window, softcap):
    dev = torch.device("cuda:0")
    qd, kd, vd, dOd = (x.to(dev) for x in (q, k, v, dO))
    o, lse = fa.attention_fwd(qd, kd, vd, scale, window, softcap)
    dq, dk, dv = fa.attention_bwd(qd, kd, vd, o, lse, dOd, scale, window, softcap)
    torch.cuda.synchronize()
    assert fa.forge_attn_check() == fa.FORGE_OK
    return o.cpu(), lse.cpu(), dq.cpu(), dk.cpu(), dv.cpu()


def groups_to_check(B, Hkv):
    """(b, kv head) pairs compared at full size: group 0 at b = 0 and the last
    group at b = B - 1 (every query head of the group, every row)."""
    pairs = [(0, 0)]
    if (B - 1, Hkv - 1) != (0, 0):
        pairs.append((B - 1, Hkv - 1))
    return pairs


# Lines the terminal summary prints after the run (tests/conftest.py): the bf16
# gradients' distance from the exact gradient, which no test asserts.
REPORT: list[str] = []


def bar_ratio(gpu, ref):
    """(max |gpu - ref|, max of |gpu - ref| / (2e-2 + 1e-2 |ref|)) over all elements."""
    gpu = gpu.detach().double().cpu().numpy() if hasattr(gpu, "detach") else np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    err = np.abs(gpu - ref)
    if not err.size:
        return 0.0, 0.0
    return float(err.max()), float((err / (ATOL_BF16 + RTOL_BF16 * np.abs(ref))).max())


def compare_all(q, k, v, dO, scale, window, softcap, dtype, gpu=None, subset=False, exact_report=None):
    """Compare o, lse, dq, dk, dv of the CUDA path against the oracle.

    The backward is compared with the oracle's Delta taken from its own O rounded
    to the call's dtype (the o a forward call of that dtype returns, which the
    backward consumes). With exact_report = a label (bf16 only), the gradients'
    distance from the exact gradient (Delta from the unrounded O) is also
    measured, as a ratio to the bf16 bar, and added to REPORT without an assert.
    subset=True compares the complete KV groups 0 at b = 0 and the last at b = B - 1."""
    if gpu is None:
        gpu = run_gpu(q, k, v, dO, scale, window, softcap)
    o, lse, dq, dk, dv = gpu
    B, Hq, T, D = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    if not subset:
        slices = [(slice(None), slice(None), slice(None), "")]
    else:
        slices = [(slice(b, b + 1), slice(h * G, (h + 1) * G), slice(h, h + 1), f"[b={b},kv={h}]")
                  for b, h in groups_to_check(B, Hkv)]
    worst = {"dq": (0.0, 0.0), "dk": (0.0, 0.0), "dv": (0.0, 0.0)}
    for bs, hs, ks_, tag in slices:
        qs, ks, vs, ds = q[bs, hs], k[bs, ks_], v[bs, ks_], dO[bs, hs]
        ro, rl = oracle.attn_fwd(qs, ks, vs, scale, window, softcap)
        rdq, rdk, rdv, _, _ = oracle.attn_bwd(qs, ks, vs, ds, scale, window, softcap, o_round=dtype)
        check_close("o" + tag, o[bs, hs], ro, dtype)
        check_close("lse" + tag, lse[bs, hs], rl, dtype)
        check_close("dq" + tag, dq[bs, hs], rdq, dtype)
        check_close("dk" + tag, dk[bs, ks_], rdk, dtype)
        check_close("dv" + tag, dv[bs, ks_], rdv, dtype)
        if exact_report and dtype == "bf16":
            edq, edk, edv, _, _ = oracle.attn_bwd(qs, ks, vs, ds, scale, window, softcap, o_round=None)
            for name, g, r in (("dq", dq[bs, hs], edq), ("dk", dk[bs, ks_], edk), ("dv", dv[bs, ks_], edv)):
                a, rr = bar_ratio(g, r)
                worst[name] = (max(worst[name][0], a), max(worst[name][1], rr))
    if exact_report and dtype == "bf16":
        REPORT.append(f"{exact_report}: bf16 gradients vs the exact gradient (Delta from the unrounded O): " +
                      ", ".join(f"{n} max abs {a:.3e}, {r:.2f} x bar" for n, (a, r) in worst.items()))
