"""The autograd entry point's plumbing on CPU: fa.attention routes its inputs,
options and upstream gradient to attention_fwd / attention_bwd and their results
back to q, k, v and sink. The two helpers are replaced by oracle-backed fakes
(f64 CPU tensors), so what is checked is the wrapper, not the kernels."""
import numpy as np
import pytest
import torch

import oracle
import causal_flash_attention_attn_b200 as fa

calls = []


def fake_fwd(q, k, v, scale=None, window=0, softcap=0.0, stream=None, *, sink=None, return_max_logit=False):
    calls.append(("fwd", scale, window, softcap, sink is not None))
    o, lse, _ = oracle.attn_fwd_ext(q, k, v, scale, window, softcap, sink=sink)
    return torch.from_numpy(o), torch.from_numpy(lse)


def fake_bwd(q, k, v, o, lse, dO, scale=None, window=0, softcap=0.0, workspace=None, stream=None, *, sink=None):
    calls.append(("bwd", scale, window, softcap, sink is not None, dO.is_contiguous()))
    dq, dk, dv, dsink, _, _ = oracle.attn_bwd_ext(q.detach(), k.detach(), v.detach(), dO, scale, window, softcap,
                                                  sink=None if sink is None else sink.detach())
    out = (torch.from_numpy(dq), torch.from_numpy(dk), torch.from_numpy(dv))
    return out + (torch.from_numpy(dsink),) if sink is not None else out


@pytest.fixture(autouse=True)
def fakes(monkeypatch):
    calls.clear()
    monkeypatch.setattr(fa, "attention_fwd", fake_fwd)
    monkeypatch.setattr(fa, "attention_bwd", fake_bwd)


def leaf(shape, seed):
    return torch.from_numpy(np.random.default_rng(seed).standard_normal(shape)).requires_grad_(True)


@pytest.mark.parametrize("with_sink", [False, True])
def test_gradients_reach_q_k_v_and_sink(with_sink):
    B, Hq, Hkv, T, D, W, C = 1, 4, 2, 9, 6, 4, 3.0
    q, k, v = leaf((B, Hq, T, D), 1), leaf((B, Hkv, T, D), 2), leaf((B, Hkv, T, D), 3)
    sink = leaf((Hq,), 4) if with_sink else None
    dO = np.random.default_rng(5).standard_normal((B, Hq, T, D))
    o = fa.attention(q, k, v, window=W, softcap=C, sink=sink)
    (o * torch.from_numpy(dO)).sum().backward()
    scale = 1.0 / np.sqrt(D)
    sk = None if sink is None else sink.detach()
    ro, _, _ = oracle.attn_fwd_ext(q.detach(), k.detach(), v.detach(), scale, W, C, sink=sk)
    rdq, rdk, rdv, rds, _, _ = oracle.attn_bwd_ext(q.detach(), k.detach(), v.detach(), dO, scale, W, C, sink=sk)
    np.testing.assert_array_equal(o.detach().numpy(), ro)
    np.testing.assert_array_equal(q.grad.numpy(), rdq)
    np.testing.assert_array_equal(k.grad.numpy(), rdk)
    np.testing.assert_array_equal(v.grad.numpy(), rdv)
    if with_sink:
        np.testing.assert_array_equal(sink.grad.numpy(), rds)
    # the default scale and the options reach both passes unchanged
    assert calls[0] == ("fwd", scale, W, C, with_sink)
    assert calls[1][:5] == ("bwd", scale, W, C, with_sink)


def test_strided_upstream_gradient_is_made_contiguous():
    q, k, v = leaf((1, 2, 7, 4), 6), leaf((1, 1, 7, 4), 7), leaf((1, 1, 7, 4), 8)
    o = fa.attention(q, k, v, scale=0.7)
    w = torch.from_numpy(np.random.default_rng(9).standard_normal((1, 2, 4, 7)))
    (o.transpose(2, 3) * w).sum().backward()   # o's gradient arrives as a transposed view
    assert calls[-1][0] == "bwd" and calls[-1][5] is True
    assert calls[-1][1] == 0.7
    rdq, _, _, _, _ = oracle.attn_bwd(q.detach(), k.detach(), v.detach(), w.transpose(2, 3).numpy(), 0.7)
    np.testing.assert_array_equal(q.grad.numpy(), rdq)


def test_no_grad_inputs_run_the_forward_only():
    q, k, v = (x.detach() for x in (leaf((1, 2, 5, 4), 10), leaf((1, 2, 5, 4), 11), leaf((1, 2, 5, 4), 12)))
    o = fa.attention(q, k, v)
    assert not o.requires_grad and [c[0] for c in calls] == ["fwd"]
