"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every function include/forge_attn.h declares, and rejects bad arguments with the
documented status codes before touching the device."""
import ctypes
import os
import re
import subprocess

import pytest

import causal_flash_attention_attn_b200 as fa
from causal_flash_attention_attn_b200 import build as fa_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "forge_attn.h")

A = 0x10000  # a 16-byte (and 256-byte) aligned fake device address: never dereferenced


@pytest.fixture(scope="module", autouse=True)
def built():
    fa_build.build()
    yield


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"\b(forge_attn_\w+)\s*\(", text)))


def test_header_functions_are_exported():
    names = declared_functions()
    assert len(names) >= 10
    lib = ctypes.CDLL(fa.library_path)
    for n in names:
        assert hasattr(lib, n), n
    out = subprocess.run(["nm", "-D", "--defined-only", fa.library_path], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (forge_attn_\w+)", out))
    assert set(names) <= exported, set(names) - exported


def test_status_strings_and_version():
    for code in range(6):
        s = fa.forge_attn_status_string(code)
        assert s.startswith("FORGE_")
    assert fa.forge_attn_status_string(99) == "FORGE_ERR_UNKNOWN"
    assert "sm_100a" in fa.forge_attn_version()


def fwd(**kw):
    a = dict(q=A, k=A, v=A, o=A, lse=A, B=1, Hq=4, Hkv=2, T=128, D=128, scale=0.1, window=0, softcap=0.0,
             dtype=fa.FORGE_DTYPE_BF16, stream=0)
    a.update(kw)
    return fa.forge_attn_fwd(**a)


@pytest.mark.parametrize("kw,code", [
    (dict(Hkv=3), fa.FORGE_ERR_INVALID_ARG),           # Hq % Hkv != 0
    (dict(D=63), fa.FORGE_ERR_INVALID_ARG),            # odd head dim
    (dict(D=96), fa.FORGE_ERR_UNSUPPORTED),            # even but not built
    (dict(D=512), fa.FORGE_ERR_UNSUPPORTED),
    (dict(B=0), fa.FORGE_ERR_INVALID_ARG),
    (dict(T=0), fa.FORGE_ERR_INVALID_ARG),
    (dict(Hq=0), fa.FORGE_ERR_INVALID_ARG),
    (dict(window=-1), fa.FORGE_ERR_INVALID_ARG),
    (dict(softcap=-1.0), fa.FORGE_ERR_INVALID_ARG),
    (dict(softcap=float("inf")), fa.FORGE_ERR_INVALID_ARG),
    (dict(scale=0.0), fa.FORGE_ERR_INVALID_ARG),
    (dict(scale=float("nan")), fa.FORGE_ERR_INVALID_ARG),
    (dict(q=0), fa.FORGE_ERR_INVALID_ARG),             # null
    (dict(o=A + 8), fa.FORGE_ERR_INVALID_ARG),         # misaligned
    (dict(dtype=7), fa.FORGE_ERR_INVALID_ARG),
])
def test_fwd_rejects(kw, code):
    assert fwd(**kw) == code


@pytest.mark.parametrize("kw,code", [
    (dict(B=1 << 12, Hq=1 << 12, Hkv=1 << 12, T=1), fa.FORGE_OK),               # B * Hq = 2^24: allowed
    (dict(B=(1 << 12) + 1, Hq=1 << 12, Hkv=1 << 12, T=1), fa.FORGE_ERR_INVALID_ARG),
    (dict(B=1, Hq=1, Hkv=1, T=1 << 30, D=64), fa.FORGE_OK),                     # 2^36 elements
    (dict(B=1, Hq=1, Hkv=1, T=(1 << 30) + 1, D=64), fa.FORGE_ERR_INVALID_ARG),  # T > 2^30
    (dict(B=1 << 6, Hq=1 << 8, Hkv=1 << 8, T=1 << 20, D=64), fa.FORGE_OK),      # 2^40 elements exactly
    (dict(B=1 << 6, Hq=1 << 8, Hkv=1 << 8, T=1 << 20, D=128), fa.FORGE_ERR_INVALID_ARG),
])
def test_size_limits(kw, code):
    # the index-arithmetic limits the header states; the workspace size is the
    # host-side function that applies them without launching anything
    a = dict(B=1, Hq=4, Hkv=2, T=128, D=128)
    a.update(kw)
    n = fa.forge_attn_bwd_workspace_size(a["B"], a["Hq"], a["Hkv"], a["T"], a["D"], fa.FORGE_DTYPE_BF16)
    assert (n > 0) == (code == fa.FORGE_OK)
    if code != fa.FORGE_OK:
        assert fwd(**kw) == code


def test_workspace_size_and_rejection():
    bf, f32 = fa.FORGE_DTYPE_BF16, fa.FORGE_DTYPE_F32
    n = fa.forge_attn_bwd_workspace_size(2, 28, 4, 4096, 128, bf)
    delta = 2 * 28 * 4096 * 4
    acc = 2 * 28 * 4096 * 128 * 4
    assert n >= delta + acc and n <= delta + acc + 512
    assert fa.forge_attn_bwd_workspace_size(2, 28, 4, 4096, 128, f32) >= delta
    assert fa.forge_attn_bwd_workspace_size(2, 28, 3, 4096, 128, bf) == 0
    # ragged T pads the accumulator to a multiple of 128 rows
    assert fa.forge_attn_bwd_workspace_size(1, 1, 1, 129, 64, bf) >= 256 * 64 * 4
    args = dict(q=A, k=A, v=A, o=A, lse=A, dO=A, dq=A, dk=A, dv=A, B=1, Hq=2, Hkv=1, T=100, D=64, scale=0.1,
                window=0, softcap=0.0, dtype=bf, stream=0)
    need = fa.forge_attn_bwd_workspace_size(1, 2, 1, 100, 64, bf)
    assert fa.forge_attn_bwd(workspace=A, workspace_bytes=need - 1, **args) == fa.FORGE_ERR_WORKSPACE
    assert fa.forge_attn_bwd(workspace=0, workspace_bytes=need, **args) == fa.FORGE_ERR_WORKSPACE
    assert fa.forge_attn_bwd(workspace=A + 16, workspace_bytes=need, **args) == fa.FORGE_ERR_WORKSPACE
    bad = dict(args, Hkv=3)
    assert fa.forge_attn_bwd(workspace=A, workspace_bytes=need, **bad) == fa.FORGE_ERR_INVALID_ARG
    bad = dict(args, dk=A + 4)
    assert fa.forge_attn_bwd(workspace=A, workspace_bytes=need, **bad) == fa.FORGE_ERR_INVALID_ARG


def test_selftest_rejects_bad_limit():
    assert fa.forge_attn_selftest_timeout(0, 0) == fa.FORGE_ERR_INVALID_ARG
    assert fa.forge_attn_selftest_timeout(3000000, 0) == fa.FORGE_ERR_INVALID_ARG


def test_layer_window_pattern():
    from causal_flash_attention_attn_b200.inputs import layer_window
    # Gemma 3-like: five local layers, then one global
    assert [layer_window(l, 1024, 6) for l in range(12)] == [1024] * 5 + [0] + [1024] * 5 + [0]
    # alternating
    assert [layer_window(l, 4096, 2) for l in range(4)] == [4096, 0, 4096, 0]
    assert [layer_window(l, 4096, 0) for l in range(3)] == [4096] * 3


def test_dsink_without_sink_is_rejected_before_any_launch():
    # validation fails before any device access, so fake device addresses are safe
    A = 0x10000
    s = fa.forge_attn_bwd_ext(A, A, A, A, A, A, A, A, A, 1, 2, 2, 128, 64, 0.125, 0, 0.0, None, A,
                              fa.FORGE_DTYPE_BF16, A, 1 << 20, 0)
    assert s == fa.FORGE_ERR_INVALID_ARG


def test_ext_entry_points_reject_misaligned_extras():
    A = 0x10000
    s = fa.forge_attn_fwd_ext(A, A, A, A, A, 1, 2, 2, 128, 64, 0.125, 0, 0.0, A + 2, None, fa.FORGE_DTYPE_BF16, 0)
    assert s == fa.FORGE_ERR_INVALID_ARG
    s = fa.forge_attn_fwd_ext(A, A, A, A, A, 1, 2, 2, 128, 64, 0.125, 0, 0.0, None, A + 1, fa.FORGE_DTYPE_BF16, 0)
    assert s == fa.FORGE_ERR_INVALID_ARG


def test_dkv_entry_points_reject_unsupported_pairs_before_any_launch():
    A = 0x10000
    # only (192, 128) is built; other pairs are refused in both dtypes
    for dt in (fa.FORGE_DTYPE_BF16, fa.FORGE_DTYPE_F32):
        s = fa.forge_attn_bwd_dkv(A, A, A, A, A, A, A, A, A, 1, 2, 2, 128, 128, 64, 0.07, 0, 0.0, dt, A, 1 << 20, 0)
        assert s == fa.FORGE_ERR_UNSUPPORTED
        assert fa.forge_attn_bwd_workspace_size_dkv(1, 2, 2, 128, 256, 128, dt) == 0
    s = fa.forge_attn_fwd_dkv(A, A, A, A, A, 1, 2, 2, 128, 96, 64, 0.1, 0, 0.0, fa.FORGE_DTYPE_F32, 0)
    assert s == fa.FORGE_ERR_UNSUPPORTED
    # the (192, 128) workspace holds Delta only, in both dtypes
    for dt in (fa.FORGE_DTYPE_BF16, fa.FORGE_DTYPE_F32):
        n = fa.forge_attn_bwd_workspace_size_dkv(1, 2, 2, 128, 192, 128, dt)
        assert 2 * 128 * 4 <= n < 4096, n
    # a workspace one byte short is refused before any launch
    n = fa.forge_attn_bwd_workspace_size_dkv(1, 2, 2, 128, 192, 128, fa.FORGE_DTYPE_BF16)
    s = fa.forge_attn_bwd_dkv(A, A, A, A, A, A, A, A, A, 1, 2, 2, 128, 192, 128, 0.07, 0, 0.0, fa.FORGE_DTYPE_BF16,
                              A, n - 1, 0)
    assert s == fa.FORGE_ERR_WORKSPACE


def test_decode_validation_before_any_launch():
    A = 0x10000
    ws = fa.forge_attn_decode_workspace_size(2, 8, 2, 1000, 128)
    assert ws > 0 and ws % 256 == 0
    assert fa.forge_attn_decode_workspace_size(2, 8, 3, 1000, 128) == 0   # Hq % Hkv != 0
    assert fa.forge_attn_decode_workspace_size(2, 8, 2, 1000, 96) == 0    # head dim not built
    assert fa.forge_attn_decode_workspace_size(2, 8, 2, 4000, 128) >= ws  # grows with the cache length

    def call(B=2, Hq=8, Hkv=2, T=1000, Tmax=1024, D=128, seq_lens=None, nbytes=None):
        return fa.forge_attn_decode(A, A, A, A, None, seq_lens, B, Hq, Hkv, T, Tmax, D, 0.088, 0, 0.0, None,
                                    fa.FORGE_DTYPE_BF16, A, ws if nbytes is None else nbytes, 0)

    assert call(Hq=34, Hkv=2) == fa.FORGE_ERR_UNSUPPORTED            # 17 query heads per KV head
    assert call(T=1025) == fa.FORGE_ERR_INVALID_ARG                   # T > Tmax
    assert call(nbytes=ws - 256) == fa.FORGE_ERR_WORKSPACE            # workspace too small
    assert call(seq_lens=A + 2) == fa.FORGE_ERR_INVALID_ARG           # misaligned lengths
    assert call(D=80) == fa.FORGE_ERR_UNSUPPORTED


C_CLIENT = r"""
#include <stdio.h>
#include <string.h>
#include "forge_attn.h"

int main(void) {
    void *fake = (void *)0x10000; /* never dereferenced: every call below fails validation first */
    size_t ws = forge_attn_bwd_workspace_size(2, 28, 4, 4096, 128, FORGE_DTYPE_BF16);
    forge_status bad_group = forge_attn_fwd(fake, fake, fake, fake, (float *)fake, 1, 4, 3, 128, 128,
                                            0.1f, 0, 0.0f, FORGE_DTYPE_BF16, NULL);
    forge_status bad_dim = forge_attn_fwd(fake, fake, fake, fake, (float *)fake, 1, 4, 2, 128, 96,
                                          0.1f, 0, 0.0f, FORGE_DTYPE_BF16, NULL);
    printf("%zu %d %d %s\n%s\n", ws, (int)bad_group, (int)bad_dim,
           strstr(forge_attn_version(), "sm_100a") ? "sm_100a" : "?", forge_attn_status_string(FORGE_ERR_WORKSPACE));
    return 0;
}
"""


def test_header_compiles_as_c99_and_links(tmp_path):
    # the boundary is a C ABI: a plain C99 client, warnings as errors, builds
    # against the header and the shared library and gets the documented answers
    src = tmp_path / "client.c"
    src.write_text(C_CLIENT)
    exe = tmp_path / "client"
    libdir = os.path.dirname(fa.library_path)
    libname = os.path.basename(fa.library_path)[3:-3]
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.dirname(HEADER),
                    str(src), "-o", str(exe), "-L", libdir, "-l" + libname, "-Wl,-rpath," + libdir],
                   check=True, capture_output=True, text=True)
    line1, line2 = subprocess.run([str(exe)], check=True, capture_output=True, text=True,
                                  timeout=60).stdout.splitlines()
    out = line1.split()
    assert int(out[0]) == fa.forge_attn_bwd_workspace_size(2, 28, 4, 4096, 128, fa.FORGE_DTYPE_BF16)
    assert int(out[1]) == fa.FORGE_ERR_INVALID_ARG and int(out[2]) == fa.FORGE_ERR_UNSUPPORTED
    assert out[3] == "sm_100a"
    assert line2 == fa.forge_attn_status_string(fa.FORGE_ERR_WORKSPACE)


def _c_to_ctypes(decl):
    """ctypes type the binding should use for one C parameter or return type."""
    decl = " ".join(decl.replace("const ", "").split())
    if "*" in decl:
        return ctypes.c_char_p if decl.startswith("char") else ctypes.c_void_p
    base = decl.split()[0] if decl.split()[0] != "unsigned" else "unsigned"
    return {"int": ctypes.c_int, "float": ctypes.c_float, "size_t": ctypes.c_size_t, "unsigned": ctypes.c_uint,
            "forge_dtype": ctypes.c_int, "forge_status": ctypes.c_int}[base]


def header_prototypes():
    text = re.sub(r"/\*.*?\*/", " ", open(HEADER).read(), flags=re.S)
    protos = {}
    for ret, name, params in re.findall(r"([\w][\w\s\*]*?)\s*\b(forge_attn_\w+)\s*\(([^)]*)\)\s*;", text):
        params = " ".join(params.split())
        plist = [] if params in ("", "void") else [p.strip() for p in params.split(",")]
        # drop the parameter name, keep its type (pointer stars may sit on the name)
        types = [re.sub(r"\b\w+$", "", p).strip() or p for p in plist]
        protos[name] = (ret.strip(), types)
    return protos


def test_binding_signatures_match_the_header():
    # every prototype's parameter count and kinds (pointer, int, float, size_t,
    # unsigned) and its return kind equal the ctypes declarations the binding uses
    protos = header_prototypes()
    assert set(protos) == set(declared_functions())
    L = fa.library()
    for name, (ret, types) in protos.items():
        fn = getattr(L, name)
        want = [_c_to_ctypes(t) for t in types]
        assert fn.argtypes is not None, name
        assert list(fn.argtypes) == want, (name, fn.argtypes, want)
        want_ret = _c_to_ctypes(ret)
        assert fn.restype == want_ret, (name, fn.restype, want_ret)
