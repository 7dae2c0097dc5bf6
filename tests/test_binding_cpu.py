"""The torch helpers of the binding reject, before any library call, the tensors
the C ABI would misread: strided views, mixed dtypes, shapes that disagree and
host tensors. Runs without a GPU: every case below fails on the host."""
import pytest
import torch

import causal_flash_attention_attn_b200 as fa

BF = torch.bfloat16


def z(*shape, dtype=BF):
    return torch.zeros(*shape, dtype=dtype)


Q, K = z(1, 4, 64, 32), z(1, 2, 64, 32)
LSE = z(1, 4, 64, dtype=torch.float32)


def test_valid_host_tensors_fail_only_on_the_device_check():
    with pytest.raises(ValueError, match="q must be a CUDA tensor"):
        fa.attention_fwd(Q, K, K)
    with pytest.raises(ValueError, match="q must be a CUDA tensor"):
        fa.attention_bwd(Q, K, K, Q, LSE, Q)
    with pytest.raises(ValueError, match="q must be a CUDA tensor"):
        fa.attention_decode(z(1, 4, 32), z(1, 2, 100, 32), z(1, 2, 100, 32),
                            sink=z(4, dtype=torch.float32), seq_lens=z(1, dtype=torch.int32))


def test_strided_views_are_rejected():
    kt = z(1, 2, 32, 64).transpose(2, 3)   # [1, 2, 64, 32] but strided
    with pytest.raises(ValueError, match="k must be contiguous"):
        fa.attention_fwd(Q, kt, K)
    with pytest.raises(ValueError, match="dO must be contiguous"):
        fa.attention_bwd(Q, K, K, Q, LSE, z(1, 4, 32, 64).transpose(2, 3))


def test_mixed_dtypes_are_rejected():
    with pytest.raises(ValueError, match="v has dtype torch.float32"):
        fa.attention_fwd(Q, K, z(1, 2, 64, 32, dtype=torch.float32))
    with pytest.raises(ValueError, match="lse has dtype torch.bfloat16"):
        fa.attention_bwd(Q, K, K, Q, z(1, 4, 64), Q)
    with pytest.raises(ValueError, match="seq_lens has dtype torch.int64"):
        fa.attention_decode(z(1, 4, 32), z(1, 2, 100, 32), z(1, 2, 100, 32), seq_lens=torch.zeros(1, dtype=torch.long))
    with pytest.raises(ValueError, match="sink has dtype torch.bfloat16"):
        fa.attention_decode(z(1, 4, 32), z(1, 2, 100, 32), z(1, 2, 100, 32), sink=z(4))


def test_disagreeing_shapes_are_rejected():
    with pytest.raises(ValueError, match=r"v has shape \(1, 2, 63, 32\)"):
        fa.attention_fwd(Q, K, z(1, 2, 63, 32))
    with pytest.raises(ValueError, match=r"k has shape"):
        fa.attention_fwd(Q, z(1, 2, 65, 32), z(1, 2, 65, 32))
    with pytest.raises(ValueError, match=r"o has shape"):
        fa.attention_bwd(Q, K, K, z(1, 4, 64, 16), LSE, Q)
    with pytest.raises(ValueError, match=r"lse has shape"):
        fa.attention_bwd(Q, K, K, Q, z(1, 4, 63, dtype=torch.float32), Q)
    with pytest.raises(ValueError, match=r"v_cache has shape"):
        fa.attention_decode(z(1, 4, 32), z(1, 2, 100, 32), z(1, 2, 99, 32))
    with pytest.raises(ValueError, match=r"sink has shape"):
        fa.attention_decode(z(1, 4, 32), z(1, 2, 100, 32), z(1, 2, 100, 32), sink=z(2, dtype=torch.float32))


def test_wrong_ranks_are_rejected():
    with pytest.raises(ValueError, match=r"\[B, H, T, D\]"):
        fa.attention_fwd(z(4, 64, 32), z(2, 64, 32), z(2, 64, 32))
    with pytest.raises(ValueError, match=r"\[B, Hq, D\]"):
        fa.attention_decode(z(1, 4, 1, 32), z(1, 2, 64, 32), z(1, 2, 64, 32))


def test_workspace_must_be_contiguous():
    ws = torch.zeros(64, 64, dtype=torch.uint8).t()
    with pytest.raises(ValueError, match="workspace must be contiguous"):
        fa.attention_bwd(Q, K, K, Q, LSE, Q, workspace=ws)


def test_extras_are_checked_like_the_rest():
    with pytest.raises(ValueError, match="sink has dtype torch.bfloat16"):
        fa.attention_fwd(Q, K, K, sink=z(4))
    with pytest.raises(ValueError, match=r"sink has shape \(2,\)"):
        fa.attention_fwd(Q, K, K, sink=z(2, dtype=torch.float32))
    with pytest.raises(ValueError, match=r"sink has shape"):
        fa.attention_bwd(Q, K, K, Q, LSE, Q, sink=z(3, dtype=torch.float32))
    with pytest.raises(ValueError, match="q must be a CUDA tensor"):
        fa.attention_fwd(Q, K, K, sink=z(4, dtype=torch.float32), return_max_logit=True)


def test_dk_ne_dv_shapes_and_restrictions():
    v48 = z(1, 2, 64, 48)          # d_v = 48 against d_k = 32
    o48 = z(1, 4, 64, 48)
    # o and dO take v's head dim
    with pytest.raises(ValueError, match="q must be a CUDA tensor"):
        fa.attention_fwd(Q, K, v48)
    with pytest.raises(ValueError, match="q must be a CUDA tensor"):
        fa.attention_bwd(Q, K, v48, o48, LSE, o48)
    with pytest.raises(ValueError, match=r"o has shape \(1, 4, 64, 32\), expected \(1, 4, 64, 48\)"):
        fa.attention_bwd(Q, K, v48, Q, LSE, o48)
    # the extras are not offered with d_k != d_v
    with pytest.raises(ValueError, match="not offered with d_k != d_v"):
        fa.attention_fwd(Q, K, v48, sink=z(4, dtype=torch.float32))
    with pytest.raises(ValueError, match="not offered with d_k != d_v"):
        fa.attention_fwd(Q, K, v48, return_max_logit=True)
    with pytest.raises(ValueError, match="not offered with d_k != d_v"):
        fa.attention_bwd(Q, K, v48, o48, LSE, o48, sink=z(4, dtype=torch.float32))
