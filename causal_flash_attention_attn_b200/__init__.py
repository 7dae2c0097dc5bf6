"""B200 (sm_100a) fused causal attention: Python binding of libforge_attn.so.

The functions named ``forge_attn_*`` mirror the C ABI in include/forge_attn.h one
to one (argument marshalling only: every pointer argument accepts a torch
tensor or an integer device address). ``attention_fwd`` / ``attention_bwd`` /
``attention_decode`` allocate outputs and workspace with torch and call them;
``attention`` wraps the first two in a torch.autograd.Function.

PyTorch is used for device memory and streams only; all arithmetic runs in the
library's CUDA kernels. There is no fallback: if the shared library is missing
or fails to load, every call raises.
"""
from __future__ import annotations

import ctypes
import math
import os

__all__ = [
    "FORGE_OK", "FORGE_ERR_INVALID_ARG", "FORGE_ERR_UNSUPPORTED", "FORGE_ERR_WORKSPACE",
    "FORGE_ERR_CUDA", "FORGE_ERR_TIMEOUT", "FORGE_DTYPE_F32", "FORGE_DTYPE_BF16", "ForgeError",
    "library", "library_path", "forge_attn_fwd", "forge_attn_bwd", "forge_attn_bwd_workspace_size",
    "forge_attn_bwd_noalloc", "forge_attn_fwd_ext", "forge_attn_bwd_ext", "forge_attn_decode",
    "forge_attn_decode_workspace_size", "attention_decode", "forge_attn_fwd_dkv", "forge_attn_bwd_dkv",
    "forge_attn_bwd_workspace_size_dkv",
    "forge_attn_bwd_preprocess", "forge_attn_bwd_main", "forge_attn_bwd_finalize", "forge_attn_check",
    "forge_attn_status_string", "forge_attn_selftest_timeout", "forge_attn_selftest_exp2", "forge_attn_last_cuda_error", "forge_attn_timeout_info", "forge_attn_version",
    "attention_fwd", "attention_bwd", "attention", "dtype_code",
]

FORGE_OK = 0
FORGE_ERR_INVALID_ARG = 1
FORGE_ERR_UNSUPPORTED = 2
FORGE_ERR_WORKSPACE = 3
FORGE_ERR_CUDA = 4
FORGE_ERR_TIMEOUT = 5
FORGE_DTYPE_F32 = 0
FORGE_DTYPE_BF16 = 1

_HERE = os.path.dirname(os.path.abspath(__file__))
library_path = os.path.join(_HERE, "libforge_attn.so")
_lib = None


class ForgeError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        msg = forge_attn_status_string(status)
        if status == FORGE_ERR_CUDA:
            msg += f" ({forge_attn_last_cuda_error()})"
        if status == FORGE_ERR_TIMEOUT:
            try:
                msg += f" (wait info {forge_attn_timeout_info()[1]})"
            except Exception:
                pass
        super().__init__(f"{what}: {msg}" if what else msg)


def library():
    """Load (once) and return the ctypes handle of libforge_attn.so."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(library_path):
        raise RuntimeError(f"{library_path} is missing: run `python -m causal_flash_attention_attn_b200.build`")
    L = ctypes.CDLL(library_path)
    vp, i, f, st, u = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t, ctypes.c_uint
    L.forge_attn_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, i, f, i, vp]
    L.forge_attn_fwd.restype = i
    L.forge_attn_bwd_workspace_size.argtypes = [i, i, i, i, i, i]
    L.forge_attn_bwd_workspace_size.restype = st
    L.forge_attn_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, f, i, f, i, vp, st, vp]
    L.forge_attn_bwd.restype = i
    L.forge_attn_fwd_ext.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, i, f, vp, vp, i, vp]
    L.forge_attn_fwd_ext.restype = i
    L.forge_attn_bwd_ext.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, f, i, f, vp, vp, i, vp, st, vp]
    L.forge_attn_bwd_ext.restype = i
    L.forge_attn_fwd_dkv.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, f, i, f, i, vp]
    L.forge_attn_fwd_dkv.restype = i
    L.forge_attn_bwd_workspace_size_dkv.argtypes = [i, i, i, i, i, i, i]
    L.forge_attn_bwd_workspace_size_dkv.restype = st
    L.forge_attn_bwd_dkv.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, f, i, f, i, vp, st, vp]
    L.forge_attn_bwd_dkv.restype = i
    L.forge_attn_decode_workspace_size.argtypes = [i, i, i, i, i]
    L.forge_attn_decode_workspace_size.restype = st
    L.forge_attn_decode.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, f, i, f, vp, i, vp, st, vp]
    L.forge_attn_decode.restype = i
    L.forge_attn_bwd_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, f, i, f, i, vp]
    L.forge_attn_bwd_noalloc.restype = i
    L.forge_attn_bwd_preprocess.argtypes = [vp, vp, i, i, i, i, i, i, vp, st, vp]
    L.forge_attn_bwd_preprocess.restype = i
    L.forge_attn_bwd_main.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, f, i, f, i, vp, st, vp]
    L.forge_attn_bwd_main.restype = i
    L.forge_attn_bwd_finalize.argtypes = [vp, i, i, i, i, i, i, vp, st, vp]
    L.forge_attn_bwd_finalize.restype = i
    L.forge_attn_check.argtypes = [vp]
    L.forge_attn_check.restype = i
    L.forge_attn_status_string.argtypes = [i]
    L.forge_attn_status_string.restype = ctypes.c_char_p
    L.forge_attn_selftest_timeout.argtypes = [u, vp]
    L.forge_attn_selftest_timeout.restype = i
    L.forge_attn_selftest_exp2.argtypes = [vp, vp, vp, i, vp]
    L.forge_attn_selftest_exp2.restype = i
    L.forge_attn_timeout_info.argtypes = [vp]
    L.forge_attn_timeout_info.restype = i
    L.forge_attn_last_cuda_error.argtypes = []
    L.forge_attn_last_cuda_error.restype = ctypes.c_char_p
    L.forge_attn_version.argtypes = []
    L.forge_attn_version.restype = ctypes.c_char_p
    _lib = L
    return L


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def dtype_code(dtype) -> int:
    import torch
    if dtype == torch.float32:
        return FORGE_DTYPE_F32
    if dtype == torch.bfloat16:
        return FORGE_DTYPE_BF16
    raise ValueError(f"unsupported dtype {dtype}")


# ------------------------------------------------------------------ raw C ABI
def forge_attn_fwd(q, k, v, o, lse, B, Hq, Hkv, T, D, scale, window, softcap, dtype, stream=None) -> int:
    return library().forge_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, Hq, Hkv, T, D,
                                    float(scale), int(window), float(softcap), int(dtype), _stream(stream))


def forge_attn_bwd_workspace_size(B, Hq, Hkv, T, D, dtype) -> int:
    return int(library().forge_attn_bwd_workspace_size(B, Hq, Hkv, T, D, int(dtype)))


def forge_attn_bwd(q, k, v, o, lse, dO, dq, dk, dv, B, Hq, Hkv, T, D, scale, window, softcap, dtype,
                   workspace, workspace_bytes, stream=None) -> int:
    return library().forge_attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dO), _ptr(dq),
                                    _ptr(dk), _ptr(dv), B, Hq, Hkv, T, D, float(scale), int(window),
                                    float(softcap), int(dtype), _ptr(workspace), int(workspace_bytes),
                                    _stream(stream))


def forge_attn_fwd_ext(q, k, v, o, lse, B, Hq, Hkv, T, D, scale, window, softcap, sink, max_logit, dtype,
                       stream=None) -> int:
    return library().forge_attn_fwd_ext(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, Hq, Hkv, T, D,
                                        float(scale), int(window), float(softcap), _ptr(sink), _ptr(max_logit),
                                        int(dtype), _stream(stream))


def forge_attn_bwd_ext(q, k, v, o, lse, dO, dq, dk, dv, B, Hq, Hkv, T, D, scale, window, softcap, sink, dsink,
                       dtype, workspace, workspace_bytes, stream=None) -> int:
    return library().forge_attn_bwd_ext(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dO), _ptr(dq),
                                        _ptr(dk), _ptr(dv), B, Hq, Hkv, T, D, float(scale), int(window),
                                        float(softcap), _ptr(sink), _ptr(dsink), int(dtype), _ptr(workspace),
                                        int(workspace_bytes), _stream(stream))


def forge_attn_fwd_dkv(q, k, v, o, lse, B, Hq, Hkv, T, Dk, Dv, scale, window, softcap, dtype, stream=None) -> int:
    return library().forge_attn_fwd_dkv(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, Hq, Hkv, T, Dk, Dv,
                                        float(scale), int(window), float(softcap), int(dtype), _stream(stream))


def forge_attn_bwd_workspace_size_dkv(B, Hq, Hkv, T, Dk, Dv, dtype) -> int:
    return int(library().forge_attn_bwd_workspace_size_dkv(B, Hq, Hkv, T, Dk, Dv, int(dtype)))


def forge_attn_bwd_dkv(q, k, v, o, lse, dO, dq, dk, dv, B, Hq, Hkv, T, Dk, Dv, scale, window, softcap, dtype,
                       workspace, workspace_bytes, stream=None) -> int:
    return library().forge_attn_bwd_dkv(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dO), _ptr(dq),
                                        _ptr(dk), _ptr(dv), B, Hq, Hkv, T, Dk, Dv, float(scale), int(window),
                                        float(softcap), int(dtype), _ptr(workspace), int(workspace_bytes),
                                        _stream(stream))


def forge_attn_decode_workspace_size(B, Hq, Hkv, T, D) -> int:
    return int(library().forge_attn_decode_workspace_size(B, Hq, Hkv, T, D))


def forge_attn_decode(q, k_cache, v_cache, o, lse, seq_lens, B, Hq, Hkv, T, Tmax, D, scale, window, softcap, sink,
                      dtype, workspace, workspace_bytes, stream=None) -> int:
    return library().forge_attn_decode(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(o), _ptr(lse), _ptr(seq_lens),
                                       B, Hq, Hkv, T, Tmax, D, float(scale), int(window), float(softcap),
                                       _ptr(sink), int(dtype), _ptr(workspace), int(workspace_bytes),
                                       _stream(stream))


def forge_attn_bwd_noalloc(q, k, v, o, lse, dO, dq, dk, dv, B, Hq, Hkv, T, D, scale, window, softcap, dtype,
                           stream=None) -> int:
    """forge_attn_bwd with the library's fixed 32 MiB internal scratch instead of a workspace."""
    return library().forge_attn_bwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dO), _ptr(dq),
                                            _ptr(dk), _ptr(dv), B, Hq, Hkv, T, D, float(scale), int(window),
                                            float(softcap), int(dtype), _stream(stream))


def forge_attn_bwd_preprocess(o, dO, B, Hq, Hkv, T, D, dtype, workspace, workspace_bytes, stream=None) -> int:
    return library().forge_attn_bwd_preprocess(_ptr(o), _ptr(dO), B, Hq, Hkv, T, D, int(dtype),
                                               _ptr(workspace), int(workspace_bytes), _stream(stream))


def forge_attn_bwd_main(q, k, v, lse, dO, dq, dk, dv, B, Hq, Hkv, T, D, scale, window, softcap, dtype,
                        workspace, workspace_bytes, stream=None) -> int:
    return library().forge_attn_bwd_main(_ptr(q), _ptr(k), _ptr(v), _ptr(lse), _ptr(dO), _ptr(dq), _ptr(dk),
                                         _ptr(dv), B, Hq, Hkv, T, D, float(scale), int(window), float(softcap),
                                         int(dtype), _ptr(workspace), int(workspace_bytes), _stream(stream))


def forge_attn_bwd_finalize(dq, B, Hq, Hkv, T, D, dtype, workspace, workspace_bytes, stream=None) -> int:
    return library().forge_attn_bwd_finalize(_ptr(dq), B, Hq, Hkv, T, D, int(dtype), _ptr(workspace),
                                             int(workspace_bytes), _stream(stream))


def forge_attn_check(stream=None) -> int:
    return library().forge_attn_check(_stream(stream))


def forge_attn_status_string(s: int) -> str:
    return library().forge_attn_status_string(int(s)).decode()


def forge_attn_selftest_timeout(limit_us: int, stream=None) -> int:
    return library().forge_attn_selftest_timeout(int(limit_us), _stream(stream))


def forge_attn_selftest_exp2(x, y, y_ref, n, stream=None) -> int:
    return library().forge_attn_selftest_exp2(_ptr(x), _ptr(y), _ptr(y_ref), int(n), _stream(stream))


def forge_attn_timeout_info():
    """(status, [barrier+1, block, thread, (threads << 20) | blocks]) of the first wait that ran out."""
    arr = (ctypes.c_uint * 4)()
    s = library().forge_attn_timeout_info(arr)
    return s, list(arr)


def forge_attn_last_cuda_error() -> str:
    return library().forge_attn_last_cuda_error().decode()


def forge_attn_version() -> str:
    return library().forge_attn_version().decode()


# ---------------------------------------------------------- torch conveniences
# The library reads raw pointers with the documented dense layouts, so these
# helpers reject what it would misread: host tensors, strided views, mixed
# dtypes or devices, and shapes that disagree.
def _check(what, dtype, device, shapes, **tensors):
    import torch
    given = {name: t for name, t in tensors.items() if t is not None}
    for name, t in given.items():
        want = dtype.get(name)
        if not isinstance(t, torch.Tensor):
            raise TypeError(f"{what}: {name} must be a torch tensor")
        if not t.is_contiguous():
            raise ValueError(f"{what}: {name} must be contiguous")
        if want is not None and t.dtype != want:
            raise ValueError(f"{what}: {name} has dtype {t.dtype}, expected {want}")
        if name in shapes and tuple(t.shape) != tuple(shapes[name]):
            raise ValueError(f"{what}: {name} has shape {tuple(t.shape)}, expected {tuple(shapes[name])}")
    for name, t in given.items():
        if not t.is_cuda:
            raise ValueError(f"{what}: {name} must be a CUDA tensor")
        if t.device != device:
            raise ValueError(f"{what}: {name} is on {t.device}, expected {device}")


def _dims(q, k):
    if q.dim() != 4 or k.dim() != 4:
        raise ValueError(f"q and k must be [B, H, T, D], got {tuple(q.shape)} and {tuple(k.shape)}")
    B, Hq, T, D = q.shape
    Hkv = k.shape[1]
    return B, Hq, Hkv, T, D


def _check_bhtd(what, q, k, v, extras=False, **rest):
    """Checks q, k, v and the rest; v (and o, dO) may have a head dim Dv of its own,
    but then without the sink / max-logit extras. Returns (B, Hq, Hkv, T, D, Dv)."""
    import torch
    B, Hq, Hkv, T, D = _dims(q, k)
    if v.dim() != 4:
        raise ValueError(f"{what}: v must be [B, Hkv, T, Dv], got {tuple(v.shape)}")
    Dv = v.shape[3]
    if Dv != D and extras:
        raise ValueError(f"{what}: sinks and the max logit are not offered with d_k != d_v")
    qs, ks, vs, rows = (B, Hq, T, Dv), (B, Hkv, T, D), (B, Hkv, T, Dv), (B, Hq, T)
    shapes = dict(k=ks, v=vs, o=qs, dO=qs, lse=rows, sink=(Hq,))
    f = torch.float32
    dt = dict(k=q.dtype, v=q.dtype, o=q.dtype, dO=q.dtype, lse=f, sink=f)
    _check(what, dt, q.device, shapes, q=q, k=k, v=v, **rest)
    return B, Hq, Hkv, T, D, Dv


def attention_fwd(q, k, v, scale=None, window=0, softcap=0.0, stream=None, *, sink=None, return_max_logit=False):
    """Forward on device tensors q [B,Hq,T,D], k [B,Hkv,T,D], v [B,Hkv,T,Dv] (bf16
    or f32). Returns (o, lse), or (o, lse, max_logit [B,Hq]) with
    return_max_logit. sink: optional f32 [Hq] sink logits. Dv != D runs the
    d_k != d_v entry point (no sink, no max logit there)."""
    import torch
    B, Hq, Hkv, T, D, Dv = _check_bhtd("attention_fwd", q, k, v, extras=sink is not None or return_max_logit,
                                       sink=sink)
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    dt = dtype_code(q.dtype)
    o = torch.empty((B, Hq, T, Dv), dtype=q.dtype, device=q.device)
    lse = torch.empty((B, Hq, T), dtype=torch.float32, device=q.device)
    ml = None
    if Dv != D:
        s, what = forge_attn_fwd_dkv(q, k, v, o, lse, B, Hq, Hkv, T, D, Dv, scale, window, softcap, dt,
                                     stream), "forge_attn_fwd_dkv"
    elif sink is not None or return_max_logit:
        ml = torch.empty((B, Hq), dtype=torch.float32, device=q.device) if return_max_logit else None
        s, what = forge_attn_fwd_ext(q, k, v, o, lse, B, Hq, Hkv, T, D, scale, window, softcap, sink, ml, dt,
                                     stream), "forge_attn_fwd_ext"
    else:
        s, what = forge_attn_fwd(q, k, v, o, lse, B, Hq, Hkv, T, D, scale, window, softcap, dt,
                                 stream), "forge_attn_fwd"
    if s != FORGE_OK:
        raise ForgeError(s, what)
    return (o, lse, ml) if return_max_logit else (o, lse)


def attention_decode(q, k_cache, v_cache, T=None, scale=None, window=0, softcap=0.0, seq_lens=None, sink=None,
                     stream=None):
    """Decode on device tensors: q [B,Hq,D], caches [B,Hkv,Tmax,D]; T defaults to
    Tmax (or the largest of seq_lens, an int32 device tensor [B]). Returns (o, lse)."""
    import torch
    if q.dim() != 3 or k_cache.dim() != 4:
        raise ValueError(f"attention_decode: q must be [B, Hq, D] and the caches [B, Hkv, Tmax, D], got "
                         f"{tuple(q.shape)} and {tuple(k_cache.shape)}")
    B, Hq, D = q.shape
    Hkv, Tmax = k_cache.shape[1], k_cache.shape[2]
    _check("attention_decode", dict(k_cache=q.dtype, v_cache=q.dtype, sink=torch.float32, seq_lens=torch.int32),
           q.device, dict(k_cache=(B, Hkv, Tmax, D), v_cache=(B, Hkv, Tmax, D), sink=(Hq,), seq_lens=(B,)),
           q=q, k_cache=k_cache, v_cache=v_cache, sink=sink, seq_lens=seq_lens)
    if T is None:
        T = int(seq_lens.max().item()) if seq_lens is not None else Tmax
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    ws = torch.empty(forge_attn_decode_workspace_size(B, Hq, Hkv, T, D), dtype=torch.uint8, device=q.device)
    o = torch.empty_like(q)
    lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    s = forge_attn_decode(q, k_cache, v_cache, o, lse, seq_lens, B, Hq, Hkv, T, Tmax, D, scale, window, softcap, sink,
                          dtype_code(q.dtype), ws, ws.numel(), stream)
    if s != FORGE_OK:
        raise ForgeError(s, "forge_attn_decode")
    return o, lse


def attention_bwd(q, k, v, o, lse, dO, scale=None, window=0, softcap=0.0, workspace=None, stream=None, *,
                  sink=None):
    """Backward on device tensors (o and lse from the matching forward). Returns
    (dq, dk, dv), or (dq, dk, dv, dsink [Hq]) when the forward had a sink. Dv != D
    runs the d_k != d_v entry point."""
    import torch
    B, Hq, Hkv, T, D, Dv = _check_bhtd("attention_bwd", q, k, v, extras=sink is not None, o=o, lse=lse, dO=dO,
                                       workspace=workspace, sink=sink)
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    dt = dtype_code(q.dtype)
    if Dv != D:
        nbytes = forge_attn_bwd_workspace_size_dkv(B, Hq, Hkv, T, D, Dv, dt)
        if nbytes == 0:
            raise ForgeError(FORGE_ERR_UNSUPPORTED, "forge_attn_bwd_dkv")
    else:
        nbytes = forge_attn_bwd_workspace_size(B, Hq, Hkv, T, D, dt)
    if workspace is None or workspace.numel() * workspace.element_size() < nbytes:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=q.device)
    wbytes = workspace.numel() * workspace.element_size()
    dq = torch.empty_like(q)
    dk = torch.empty_like(k)
    dv = torch.empty_like(v)
    dsink = None
    if Dv != D:
        s, what = forge_attn_bwd_dkv(q, k, v, o, lse, dO, dq, dk, dv, B, Hq, Hkv, T, D, Dv, scale, window, softcap,
                                     dt, workspace, wbytes, stream), "forge_attn_bwd_dkv"
    elif sink is not None:
        dsink = torch.empty((Hq,), dtype=torch.float32, device=q.device)
        s, what = forge_attn_bwd_ext(q, k, v, o, lse, dO, dq, dk, dv, B, Hq, Hkv, T, D, scale, window, softcap,
                                     sink, dsink, dt, workspace, wbytes, stream), "forge_attn_bwd_ext"
    else:
        s, what = forge_attn_bwd(q, k, v, o, lse, dO, dq, dk, dv, B, Hq, Hkv, T, D, scale, window, softcap, dt,
                                 workspace, wbytes, stream), "forge_attn_bwd"
    if s != FORGE_OK:
        raise ForgeError(s, what)
    return (dq, dk, dv, dsink) if sink is not None else (dq, dk, dv)


# ------------------------------------------------------------------ autograd
_attention_fn = None


def _attention_function():
    """The torch.autograd.Function over attention_fwd / attention_bwd (built on
    first use, so that importing this module does not import torch)."""
    global _attention_fn
    if _attention_fn is None:
        import torch

        class ForgeAttention(torch.autograd.Function):
            @staticmethod
            def forward(ctx, q, k, v, sink, scale, window, softcap):
                o, lse = attention_fwd(q, k, v, scale, window, softcap, sink=sink)
                ctx.save_for_backward(q, k, v, o, lse, sink)
                ctx.args = (scale, window, softcap)
                return o

            @staticmethod
            def backward(ctx, dO):
                q, k, v, o, lse, sink = ctx.saved_tensors
                g = attention_bwd(q, k, v, o, lse, dO.contiguous(), *ctx.args, sink=sink)
                return g[0], g[1], g[2], (g[3] if sink is not None else None), None, None, None

        _attention_fn = ForgeAttention
    return _attention_fn


def attention(q, k, v, scale=None, window=0, softcap=0.0, sink=None):
    """Causal attention with autograd: o = attention(q, k, v), gradients for q, k,
    v (and sink) through the library's backward. Shapes, dtypes and options as
    attention_fwd; scale defaults to 1/sqrt(head dim of q)."""
    scale = 1.0 / math.sqrt(q.shape[-1]) if scale is None else float(scale)
    return _attention_function().apply(q, k, v, sink, scale, int(window), float(softcap))
