"""The oracle: plain, slow, f64 CPU causal attention (forward and backward).

TEST INFRASTRUCTURE. Only tests/, the smoke check in __graft_entry__ and the
bench's CPU-baseline leg may import this package. The product library neither
imports it nor links it, and the two share no code.

Parity pins (tests/test_oracle.py): torch SDPA in f64 (causal, band mask, GQA by
repeat_interleave), torch autograd of SDPA, brute-force softmax Jacobian on tiny
shapes, central finite differences, and the invariants and closed forms of the
definition. The sink and max-logit extensions are pinned by: sink = -inf being the
plain softmax bit for bit; a sink being an extra zero-value key at position 0
(checked through the pinned plain oracle, forward, dq/dk/dv and dsink); a one-key
closed form; central differences of dsink; a hand-worked max-logit example. The
decode function is pinned to the last row of the pinned forward (bit for bit, with
window, cap and sink), to per-entry lengths with the cache tail poisoned, and to the
length-1 closed form. The d_k != d_v form of attn_fwd_ext / attn_bwd_ext is pinned to
torch SDPA autograd in f64 (SDPA takes a value head dim of its own) and to the
independence of the value columns. No function here is left unpinned.

Every function takes and returns numpy float64 arrays in [B, H, T, D] layout.
"""
from __future__ import annotations

import ctypes

import numpy as np

from . import build as _build

_lib = None


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        dp = ctypes.POINTER(ctypes.c_double)
        i = ctypes.c_int
        d = ctypes.c_double
        lib.oracle_attn_fwd.argtypes = [dp, dp, dp, dp, dp, i, i, i, i, i, d, i, d]
        lib.oracle_attn_fwd_ext.argtypes = [dp, dp, dp, dp, dp, dp, dp, i, i, i, i, i, i, d, i, d]
        lib.oracle_attn_bwd_ext.argtypes = [dp, dp, dp, dp, dp, dp, dp, dp, dp, dp, dp, i, i, i, i, i, i, d, i, d, i]
        lib.oracle_attn_bwd.argtypes = [dp, dp, dp, dp, dp, dp, dp, dp, dp, i, i, i, i, i, d, i, d, i]
        lib.oracle_attn_decode.argtypes = [dp, dp, dp, dp, ctypes.POINTER(ctypes.c_int), dp, dp, i, i, i, i, i, i, d,
                                           i, d]
        lib.oracle_round.argtypes = [dp, dp, ctypes.c_long, i]
        lib.oracle_attn_probs.argtypes = [dp, dp, dp, i, i, i, i, i, d, i, d]
        lib.oracle_rowdot.argtypes = [dp, dp, dp, ctypes.c_long, i]
        lib.oracle_num_threads.restype = ctypes.c_int
        lib.oracle_set_num_threads.argtypes = [i]
        lib.oracle_set_num_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def _f64(a) -> np.ndarray:
    if hasattr(a, "detach"):  # torch tensor
        a = a.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(a, dtype=np.float64)


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _dims(q, k):
    B, Hq, T, D = q.shape
    Bk, Hkv, Tk, Dk = k.shape
    assert (B, T, D) == (Bk, Tk, Dk) and Hq % Hkv == 0
    return B, Hq, Hkv, T, D


def _dims_kv(q, k, v):
    """(B, Hq, Hkv, T, Dk, Dv): the key head dim of q and k, the value head dim of v."""
    B, Hq, Hkv, T, Dk = _dims(q, k)
    assert v.shape[:3] == (B, Hkv, T)
    return B, Hq, Hkv, T, Dk, v.shape[3]


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def set_num_threads(n: int) -> int:
    """Threads the oracle's parallel loops use from now on; returns the count in
    force. Timing only: the results do not depend on it."""
    return int(_load().oracle_set_num_threads(int(n)))


def attn_fwd(q, k, v, scale: float, window: int = 0, softcap: float = 0.0):
    """Return (o [B,Hq,T,D], lse [B,Hq,T]) in f64."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Hq, Hkv, T, D = _dims(q, k)
    o = np.empty_like(q)
    lse = np.empty((B, Hq, T), dtype=np.float64)
    _load().oracle_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, Hq, Hkv, T, D,
                            float(scale), int(window), float(softcap))
    return o, lse


_ROUND = {None: 0, "f64": 0, "f32": 1, "bf16": 2}


def round_to(x, dtype: str):
    """Round f64 values to a storage type ("f32" or "bf16", nearest even) and back."""
    x = _f64(x)
    y = np.empty_like(x)
    _load().oracle_round(_ptr(x), _ptr(y), x.size, _ROUND[dtype])
    return y


def attn_bwd(q, k, v, dO, scale: float, window: int = 0, softcap: float = 0.0, o_round=None):
    """Return (dq, dk, dv, delta, lse) in f64 for upstream gradient dO.

    o_round=None uses Delta_i = sum_j P_ij dP_ij. o_round="f32"/"bf16" uses
    Delta_i = rowsum(dO * o) with the oracle's own o rounded to that storage type,
    i.e. the O a forward call of that dtype returns to the backward."""
    q, k, v, dO = _f64(q), _f64(k), _f64(v), _f64(dO)
    B, Hq, Hkv, T, D = _dims(q, k)
    dq = np.empty_like(q)
    dk = np.empty_like(k)
    dv = np.empty_like(v)
    delta = np.empty((B, Hq, T), dtype=np.float64)
    lse = np.empty((B, Hq, T), dtype=np.float64)
    _load().oracle_attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(dO), _ptr(dq), _ptr(dk), _ptr(dv),
                            _ptr(delta), _ptr(lse), B, Hq, Hkv, T, D, float(scale), int(window),
                            float(softcap), _ROUND[o_round])
    return dq, dk, dv, delta, lse


def _ptr_or_null(a):
    return None if a is None else _ptr(a)


def attn_fwd_ext(q, k, v, scale: float, window: int = 0, softcap: float = 0.0, sink=None):
    """Forward with an optional per-head sink logit sink [Hq]; v (and o) may have a
    head dim other than q and k (d_k != d_v). Returns (o, lse,
    max_logit [B, Hq]); max_logit is the per-(b, hq) maximum of the scores the
    softmax sees over the allowed pairs (the sink not included)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Hq, Hkv, T, Dk, Dv = _dims_kv(q, k, v)
    sk = None if sink is None else _f64(sink).reshape(Hq)
    o = np.empty((B, Hq, T, Dv), dtype=np.float64)
    lse = np.empty((B, Hq, T), dtype=np.float64)
    ml = np.empty((B, Hq), dtype=np.float64)
    _load().oracle_attn_fwd_ext(_ptr(q), _ptr(k), _ptr(v), _ptr_or_null(sk), _ptr(o), _ptr(lse), _ptr(ml),
                                B, Hq, Hkv, T, Dk, Dv, float(scale), int(window), float(softcap))
    return o, lse, ml


def attn_bwd_ext(q, k, v, dO, scale: float, window: int = 0, softcap: float = 0.0, sink=None, o_round=None):
    """Backward with an optional per-head sink logit sink [Hq]. Returns (dq, dk,
    dv, dsink [Hq] (zeros without a sink), delta, lse)."""
    q, k, v, dO = _f64(q), _f64(k), _f64(v), _f64(dO)
    B, Hq, Hkv, T, Dk, Dv = _dims_kv(q, k, v)
    assert dO.shape == (B, Hq, T, Dv)
    sk = None if sink is None else _f64(sink).reshape(Hq)
    dq = np.empty_like(q)
    dk = np.empty_like(k)
    dv = np.empty_like(v)
    dsink = np.empty((Hq,), dtype=np.float64)
    delta = np.empty((B, Hq, T), dtype=np.float64)
    lse = np.empty((B, Hq, T), dtype=np.float64)
    _load().oracle_attn_bwd_ext(_ptr(q), _ptr(k), _ptr(v), _ptr(dO), _ptr_or_null(sk), _ptr(dq), _ptr(dk),
                                _ptr(dv), _ptr(dsink), _ptr(delta), _ptr(lse), B, Hq, Hkv, T, Dk, Dv, float(scale),
                                int(window), float(softcap), _ROUND[o_round])
    return dq, dk, dv, dsink, delta, lse


def attn_decode(q, k_cache, v_cache, scale: float, T: int, window: int = 0, softcap: float = 0.0, sink=None,
                seq_lens=None):
    """Decode: q [B, Hq, D] (the new token's queries), caches [B, Hkv, Tmax, D]; entry
    b's query sits at position len_b - 1 with len_b = seq_lens[b] (or T). Returns
    (o [B, Hq, D], lse [B, Hq])."""
    q, kc, vc = _f64(q), _f64(k_cache), _f64(v_cache)
    B, Hq, D = q.shape
    Bk, Hkv, Tmax, Dk = kc.shape
    assert (B, D) == (Bk, Dk) and Hq % Hkv == 0 and vc.shape == kc.shape
    sk = None if sink is None else _f64(sink).reshape(Hq)
    sl = None
    if seq_lens is not None:
        sl = np.ascontiguousarray(np.asarray(seq_lens, dtype=np.int32).reshape(B))
        assert np.all((sl >= 1) & (sl <= Tmax))
    else:
        assert 1 <= T <= Tmax
    o = np.empty((B, Hq, D), dtype=np.float64)
    lse = np.empty((B, Hq), dtype=np.float64)
    _load().oracle_attn_decode(_ptr(q), _ptr(kc), _ptr(vc), _ptr_or_null(sk),
                               None if sl is None else sl.ctypes.data_as(ctypes.POINTER(ctypes.c_int)),
                               _ptr(o), _ptr(lse), B, Hq, Hkv, int(T), Tmax, D, float(scale), int(window),
                               float(softcap))
    return o, lse


def attn_probs(q, k, scale: float, window: int = 0, softcap: float = 0.0):
    """Full probability matrix [B,Hq,T,T] (zero where masked). Small shapes only."""
    q, k = _f64(q), _f64(k)
    B, Hq, Hkv, T, D = _dims(q, k)
    P = np.empty((B, Hq, T, T), dtype=np.float64)
    _load().oracle_attn_probs(_ptr(q), _ptr(k), _ptr(P), B, Hq, Hkv, T, D, float(scale),
                              int(window), float(softcap))
    return P


def rowdot(o, dO):
    """Delta = rowsum(dO * O) over the last axis."""
    o, dO = _f64(o), _f64(dO)
    out = np.empty(o.shape[:-1], dtype=np.float64)
    _load().oracle_rowdot(_ptr(o), _ptr(dO), _ptr(out), int(np.prod(o.shape[:-1])), o.shape[-1])
    return out
