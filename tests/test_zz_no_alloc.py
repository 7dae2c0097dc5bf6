"""forge_attn_bwd_noalloc: the backward for callers that cannot allocate device
memory (hosts that only receive device buffers from another runtime, or processes
whose memory pool owns the whole device). Its scratch is a fixed 32 MiB array in
the library. Checked through the C ABI against forge_attn_bwd (caller workspace)
on two calls in a row, so that what the first call leaves in the shared array
cannot leak into the second. Kept in its own file, collected last."""
import math

import numpy as np
import pytest
import torch

import causal_flash_attention_attn_b200 as fa
from causal_flash_attention_attn_b200 import inputs

pytestmark = pytest.mark.gpu


def _bwd_both(w):
    dev = torch.device("cuda:0")
    q, k, v, dO = (x.to(dev) for x in inputs.make_inputs(w))
    dt = fa.dtype_code(q.dtype)
    sc = 1.0 / math.sqrt(w.D)
    o, lse = fa.attention_fwd(q, k, v, sc, w.window, w.softcap)
    ref = fa.attention_bwd(q, k, v, o, lse, dO, sc, w.window, w.softcap)
    outs = []
    for _ in range(2):
        dq, dk, dv = (torch.full_like(x, float("nan")) for x in (q, k, v))
        s = fa.forge_attn_bwd_noalloc(q, k, v, o, lse, dO, dq, dk, dv, w.B, w.Hq, w.Hkv, w.T, w.D, sc, w.window,
                                      w.softcap, dt)
        assert s == fa.FORGE_OK, fa.forge_attn_status_string(s)
        torch.cuda.synchronize()
        assert fa.forge_attn_check() == fa.FORGE_OK
        outs.append((dq, dk, dv))
    return ref, outs


def _close(a, b, dtype):
    a, b = a.double().cpu().numpy(), b.double().cpu().numpy()
    assert np.all(np.isfinite(a))
    if dtype == "f32":
        assert np.max(np.abs(a - b)) <= 1e-4
    else:
        assert np.all(np.abs(a - b) <= 2e-2 + 1e-2 * np.abs(b))


@pytest.mark.parametrize("w", [
    inputs.Workload("noalloc_bf16", "bf16", 2, 4, 2, 300, 128, window=0, seed=31),
    inputs.Workload("noalloc_bf16_win_cap", "bf16", 1, 4, 1, 257, 64, window=100, softcap=5.0, seed=32,
                    sigma_q=2.0, sigma_k=2.0),
    inputs.Workload("noalloc_f32", "f32", 1, 2, 2, 200, 64, seed=33),
])
def test_noalloc_matches_workspace_backward_twice(w):
    ref, outs = _bwd_both(w)
    for dq, dk, dv in outs:
        for a, b in ((dq, ref[0]), (dk, ref[1]), (dv, ref[2])):
            _close(a, b, w.dtype)


def test_noalloc_rejects_problems_beyond_its_scratch():
    # 2 x 28 x 4096 x 128 needs ~117 MB of scratch: rejected, nothing launched
    A = 0x10000
    s = fa.forge_attn_bwd_noalloc(A, A, A, A, A, A, A, A, A, 2, 28, 4, 4096, 128, 0.088, 0, 0.0,
                                  fa.FORGE_DTYPE_BF16)
    assert s == fa.FORGE_ERR_WORKSPACE
    assert "32 MiB" in fa.forge_attn_last_cuda_error()
