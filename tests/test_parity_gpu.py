"""GPU parity: the CUDA path through the C ABI against the f64 oracle on the same
seeded inputs. Small shapes are compared in full (several tiles and a ragged
tail); at full size the f32 and Forge-default workloads are compared in full and
the long-sequence ones on complete KV groups."""
import math

import pytest
import torch

from causal_flash_attention_attn_b200 import inputs
from parity_util import compare_all, run_gpu

pytestmark = pytest.mark.gpu


def small(B, Hq, Hkv, T, D, dtype, seed, sigma=1.0):
    w = inputs.Workload("small", dtype, B, Hq, Hkv, T, D, seed=seed, sigma_q=sigma, sigma_k=sigma)
    return inputs.make_inputs(w)


# B, Hq, Hkv, T, D, W, C, dtype
SMALL = [
    (1, 2, 2, 1, 64, 0, 0.0, "bf16"),
    (1, 2, 1, 127, 64, 0, 0.0, "bf16"),
    (2, 2, 2, 128, 128, 0, 0.0, "bf16"),
    (1, 4, 2, 129, 128, 0, 0.0, "bf16"),
    (1, 7, 1, 300, 128, 0, 0.0, "bf16"),
    (2, 8, 1, 257, 64, 0, 0.0, "bf16"),
    (1, 2, 1, 1000, 128, 0, 0.0, "bf16"),
    (1, 2, 2, 384, 256, 0, 0.0, "bf16"),
    # few KV groups at head dim 128: the heaviest key tiles run as two work items
    # whose dK, dV are summed (split items)
    (1, 16, 1, 1024, 128, 0, 0.0, "bf16"),
    (1, 6, 1, 777, 128, 0, 0.0, "bf16"),
    (2, 14, 2, 640, 128, 0, 3.0, "bf16"),
    (1, 2, 1, 200, 256, 0, 50.0, "bf16"),
    # windows
    (1, 2, 1, 300, 128, 1, 0.0, "bf16"),
    (1, 2, 1, 300, 128, 17, 0.0, "bf16"),
    (1, 2, 2, 300, 64, 128, 0.0, "bf16"),
    (1, 2, 2, 300, 64, 129, 0.0, "bf16"),
    (1, 2, 1, 300, 128, 299, 0.0, "bf16"),
    (1, 2, 1, 300, 128, 300, 0.0, "bf16"),
    (1, 2, 1, 300, 128, 5000, 0.0, "bf16"),
    (1, 4, 2, 700, 256, 200, 5.0, "bf16"),
    # softcap in the tanh regime
    (1, 2, 1, 256, 128, 0, 5.0, "bf16"),
    (1, 4, 4, 333, 64, 40, 5.0, "bf16"),
    # f32 path
    (1, 2, 2, 128, 64, 0, 0.0, "f32"),
    (1, 4, 2, 200, 128, 33, 0.0, "f32"),
    (1, 2, 1, 150, 256, 0, 5.0, "f32"),
    (2, 2, 1, 1, 64, 0, 0.0, "f32"),
]


@pytest.mark.parametrize("B,Hq,Hkv,T,D,W,C,dtype", SMALL)
def test_small_shapes(B, Hq, Hkv, T, D, W, C, dtype):
    sigma = 2.0 if C else 1.0
    q, k, v, dO = small(B, Hq, Hkv, T, D, dtype, seed=T + D + W, sigma=sigma)
    compare_all(q, k, v, dO, 1.0 / math.sqrt(D), W, C, dtype)


# compared in full (every batch entry and head); the long-sequence workloads on
# their complete first and last KV groups
FULL = ("f32_correctness", "forge_default")


@pytest.mark.parametrize("name", list(inputs.WORKLOADS))
def test_workloads(name):
    w = inputs.WORKLOADS[name]
    q, k, v, dO = inputs.make_inputs(w)
    compare_all(q, k, v, dO, w.sm_scale, w.window, w.softcap, w.dtype, subset=name not in FULL,
                exact_report=name)


def test_window_ge_T_is_full_causal_bitwise():
    q, k, v, dO = small(1, 4, 2, 333, 128, "bf16", seed=3)
    a = run_gpu(q, k, v, dO, 1 / math.sqrt(128), 0, 0.0)
    b = run_gpu(q, k, v, dO, 1 / math.sqrt(128), 333, 0.0)
    c = run_gpu(q, k, v, dO, 1 / math.sqrt(128), 100000, 0.0)
    for x, y, z in zip(a[:2] + a[3:], b[:2] + b[3:], c[:2] + c[3:]):
        assert torch.equal(x, y) and torch.equal(x, z)


def test_dk_dv_deterministic_and_every_output_written():
    q, k, v, dO = small(1, 4, 1, 500, 128, "bf16", seed=4)
    dev = torch.device("cuda:0")
    qd, kd, vd, dOd = (x.to(dev) for x in (q, k, v, dO))
    import causal_flash_attention_attn_b200 as fa
    outs = []
    for _ in range(2):
        o = torch.full_like(qd, float("nan"))
        lse = torch.full((1, 4, 500), float("nan"), device=dev)
        fa.forge_attn_fwd(qd, kd, vd, o, lse, 1, 4, 1, 500, 128, 1 / math.sqrt(128), 0, 0.0, fa.FORGE_DTYPE_BF16)
        dq, dk, dv = (torch.full_like(x, float("nan")) for x in (qd, kd, vd))
        n = fa.forge_attn_bwd_workspace_size(1, 4, 1, 500, 128, fa.FORGE_DTYPE_BF16)
        ws = torch.full((n,), 255, dtype=torch.uint8, device=dev)
        s = fa.forge_attn_bwd(qd, kd, vd, o, lse, dOd, dq, dk, dv, 1, 4, 1, 500, 128, 1 / math.sqrt(128), 0, 0.0,
                              fa.FORGE_DTYPE_BF16, ws, n)
        assert s == fa.FORGE_OK
        torch.cuda.synchronize()
        for x in (o, lse, dq, dk, dv):
            assert torch.isfinite(x.float()).all()
        outs.append((o.clone(), lse.clone(), dk.clone(), dv.clone()))
    for x, y in zip(*outs):
        assert torch.equal(x, y)
