"""Seeded synthetic workloads shared by the tests, the bench and the oracle checks.

This module holds workload descriptions and random-number draws only: it contains
none of the attention arithmetic, so both the CUDA path and the oracle can take
their inputs from it without sharing any of the method.

Recipe (the same for every workload): a CPU ``torch.Generator`` seeded with the
workload's seed draws standard normals in f32 in the order Q, K, V, dO, each of
shape ``[B, H, T, D]`` (H = Hq for Q and dO, Hkv for K and V); each tensor is then
multiplied by its sigma and cast to the workload dtype. Consumers read the cast
tensor, so the oracle sees exactly the values the GPU sees.

The workloads are the attention shapes of the model families named on the Forge
pages (ARCHITECTURES.md family table; forge-studio RESEARCH.md section 2, config
schema): the Forge default model (d_model 384, 6 heads, context 512), a Qwen2.5-like
GQA layer (28 query heads over 4 KV heads), Mistral/Gemma 3-like sliding-window
layers (window 4096, or 1024 with every 6th layer global), and a Gemma 2-like layer
(head_dim 256, attention softcap 50, local/global alternating).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    dtype: str  # "f32" or "bf16"
    B: int
    Hq: int
    Hkv: int
    T: int
    D: int
    window: int = 0
    softcap: float = 0.0
    scale: float | None = None  # None -> 1/sqrt(D)
    seed: int = 0
    sigma_q: float = 1.0
    sigma_k: float = 1.0
    sigma_v: float = 1.0
    sigma_do: float = 1.0

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def sm_scale(self) -> float:
        return self.scale if self.scale is not None else 1.0 / math.sqrt(self.D)

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


def allowed_pairs(T: int, window: int) -> int:
    """Number of (query, key) pairs a causal (optionally windowed) row set visits,
    per (batch, query head). Counting only; used for FLOP accounting."""
    if window <= 0 or window >= T:
        return T * (T + 1) // 2
    return window * (window + 1) // 2 + (T - window) * window


# The five workloads; 4 and 5 each have several layer types.
WORKLOADS = {
    "f32_correctness": Workload("f32_correctness", "f32", 1, 2, 2, 128, 64, 0, 0.0, 1.0 / 8.0, 0),
    "forge_default": Workload("forge_default", "bf16", 32, 6, 6, 512, 64, 0, 0.0, None, 1),
    "gqa_qwen25_4k": Workload("gqa_qwen25_4k", "bf16", 2, 28, 4, 4096, 128, 0, 0.0, None, 2),
    "swa_w4096_16k": Workload("swa_w4096_16k", "bf16", 1, 32, 8, 16384, 128, 4096, 0.0, None, 3),
    "swa_w1024_16k": Workload("swa_w1024_16k", "bf16", 1, 32, 8, 16384, 128, 1024, 0.0, None, 3),
    "global_16k": Workload("global_16k", "bf16", 1, 32, 8, 16384, 128, 0, 0.0, None, 3),
    "softcap_w4096_8k": Workload("softcap_w4096_8k", "bf16", 1, 8, 4, 8192, 256, 4096, 50.0, None, 4,
                                 2.0, 2.0, 1.0, 1.0),
    "softcap_global_8k": Workload("softcap_global_8k", "bf16", 1, 8, 4, 8192, 256, 0, 50.0, None, 4,
                                  2.0, 2.0, 1.0, 1.0),
}

# The workload the headline throughput is quoted on (the 4K-token GQA layer).
HEADLINE = "gqa_qwen25_4k"


def torch_dtype(name: str) -> torch.dtype:
    return {"f32": torch.float32, "bf16": torch.bfloat16}[name]


def make_inputs(w: Workload, with_grad: bool = True):
    """Return (q, k, v, dO) as CPU tensors in the workload dtype (dO is None when
    ``with_grad`` is false; the draw order is unchanged so q, k, v do not depend on it)."""
    g = torch.Generator(device="cpu")
    g.manual_seed(w.seed)
    dt = torch_dtype(w.dtype)
    q = (torch.randn(w.B, w.Hq, w.T, w.D, generator=g) * w.sigma_q).to(dt)
    k = (torch.randn(w.B, w.Hkv, w.T, w.D, generator=g) * w.sigma_k).to(dt)
    v = (torch.randn(w.B, w.Hkv, w.T, w.D, generator=g) * w.sigma_v).to(dt)
    dO = None
    if with_grad:
        dO = (torch.randn(w.B, w.Hq, w.T, w.D, generator=g) * w.sigma_do).to(dt)
    return q, k, v, dO


def layer_window(layer: int, window: int, global_every: int) -> int:
    """Window a layer passes to the kernels under Forge's ``sliding_window`` /
    ``sliding_global_every`` config pair (forge-studio RESEARCH.md section 2).

    Reading: layers are 0-based and layer l is global (window 0) when
    global_every > 0 and (l + 1) % global_every == 0, so five local layers per
    global one (Gemma 3, ARCHITECTURES.md family table) is global_every = 6 and "alternating"
    (Gemma 2) is global_every = 2. With global_every = 0 every layer uses ``window``.
    """
    if global_every > 0 and (layer + 1) % global_every == 0:
        return 0
    return window
