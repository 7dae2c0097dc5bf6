"""The bench's FLOP accounting on CPU: the allowed-pair count it multiplies by is
the number of (query, key) pairs the oracle's probability matrix leaves nonzero
(and the pages' mask fixtures), and the per-pair factors are those of the
products each pass computes."""
import os

import numpy as np
import pytest

import bench
import oracle
from causal_flash_attention_attn_b200 import inputs


@pytest.mark.parametrize("T,W", [(1, 0), (7, 0), (7, 1), (7, 3), (7, 6), (7, 7), (7, 50), (33, 8), (64, 17)])
def test_allowed_pairs_counts_the_oracles_visible_pairs(T, W):
    rng = np.random.default_rng(T * 100 + W)
    q, k = rng.standard_normal((1, 1, T, 4)), rng.standard_normal((1, 1, T, 4))
    P = oracle.attn_probs(q, k, 0.3, W, 0.0)[0, 0]
    assert inputs.allowed_pairs(T, W) == int(np.count_nonzero(P))


@pytest.mark.parametrize("fname,T,W", [("mask_T6_W3.txt", 6, 3), ("mask_T5_W0.txt", 5, 0)])
def test_allowed_pairs_on_the_page_masks(fname, T, W):
    # the golden fixtures list, per query, the keys the pages' window rule lets it see
    n = 0
    with open(os.path.join(os.path.dirname(__file__), "golden", fname)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                n += len(line.split(":")[1].split())
    assert inputs.allowed_pairs(T, W) == n


def test_flops_per_pair():
    w = inputs.WORKLOADS["gqa_qwen25_4k"]
    fwd, bwd = bench.flops_of(w)
    pairs = w.B * w.Hq * w.T * (w.T + 1) // 2
    # forward: S = QK^T and O += PV, D-deep multiply-adds each (2 flops)
    assert fwd == 2 * 2 * w.D * pairs
    # backward: S recompute, dP = dO V^T, dV += P^T dO, dK += dS^T Q, dQ += dS K
    assert bwd == 5 * 2 * w.D * pairs
    assert round(fwd / 1e9) == 241 and round(bwd / 1e9) == 601
