"""Failure detection on the GPU without faulting it: a kernel waits on a barrier
nothing completes, its bounded wait runs out after a short limit, it records
FORGE_ERR_TIMEOUT and returns; the context stays usable."""

import pytest
import torch

import causal_flash_attention_attn_b200 as fa

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives():
    torch.cuda.synchronize()
    assert fa.forge_attn_check() == fa.FORGE_OK
    assert fa.forge_attn_selftest_timeout(20000) == fa.FORGE_OK  # 20 ms limit
    assert fa.forge_attn_check() == fa.FORGE_ERR_TIMEOUT
    assert fa.forge_attn_check() == fa.FORGE_OK  # cleared
    # a normal call still works afterwards
    q = torch.randn(1, 2, 130, 64, device="cuda", dtype=torch.bfloat16)
    o, lse = fa.attention_fwd(q, q[:, :1].contiguous(), q[:, :1].contiguous())
    torch.cuda.synchronize()
    assert torch.isfinite(o.float()).all()
    assert fa.forge_attn_check() == fa.FORGE_OK
