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


def compare_all(q, k, v, dO, scale, window, softcap, dtype, gpu=None, subset=False):
    """Compare o, lse, dq, dk, dv of the CUDA path against the oracle."""
    if gpu is None:
        gpu = run_gpu(q, k, v, dO, scale, window, softcap)
    o, lse, dq, dk, dv = gpu
    B, Hq, T, D = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    pairs = groups_to_check(B, Hkv) if subset else [(b, h) for b in range(B) for h in range(Hkv)]
    if not subset:
        ro, rl = oracle.attn_fwd(q, k, v, scale, window, softcap)
        rdq, rdk, rdv, _, _ = oracle.attn_bwd(q, k, v, dO, scale, window, softcap, o_round=dtype)
        check_close("o", o, ro, dtype)
        check_close("lse", lse, rl, dtype)
        check_close("dq", dq, rdq, dtype)
        check_close("dk", dk, rdk, dtype)
        check_close("dv", dv, rdv, dtype)
        return
    for b, h in pairs:
        hs = slice(h * G, (h + 1) * G)
        qs, ks, vs, ds = q[b:b + 1, hs], k[b:b + 1, h:h + 1], v[b:b + 1, h:h + 1], dO[b:b + 1, hs]
        ro, rl = oracle.attn_fwd(qs, ks, vs, scale, window, softcap)
        rdq, rdk, rdv, _, _ = oracle.attn_bwd(qs, ks, vs, ds, scale, window, softcap, o_round=dtype)
        tag = f"[b={b},kv={h}]"
        check_close("o" + tag, o[b:b + 1, hs], ro, dtype)
        check_close("lse" + tag, lse[b:b + 1, hs], rl, dtype)
        check_close("dq" + tag, dq[b:b + 1, hs], rdq, dtype)
        check_close("dk" + tag, dk[b:b + 1, h:h + 1], rdk, dtype)
        check_close("dv" + tag, dv[b:b + 1, h:h + 1], rdv, dtype)
