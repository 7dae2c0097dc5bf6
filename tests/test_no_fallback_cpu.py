"""No fallback: without the shared library every call of the binding raises, in a
fresh interpreter whose package points at a library path that does not exist;
nothing computes the result another way."""
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PROBE = r"""
import sys
sys.path.insert(0, ROOT)
import torch
import causal_flash_attention_attn_b200 as fa
fa.library_path = '/nonexistent/libforge_attn.so'
fa._lib = None
failures = 0
calls = [
    lambda: fa.library(),
    lambda: fa.forge_attn_version(),
    lambda: fa.forge_attn_bwd_workspace_size(1, 2, 2, 128, 64, fa.FORGE_DTYPE_BF16),
    lambda: fa.forge_attn_fwd(0x10000, 0x10000, 0x10000, 0x10000, 0x10000, 1, 2, 2, 128, 64, 0.1, 0, 0.0,
                              fa.FORGE_DTYPE_BF16, 0),
]
for c in calls:
    try:
        c()
    except RuntimeError as e:
        assert "missing" in str(e), e
        failures += 1
print(failures, len(calls))
"""


def test_every_call_raises_without_the_library():
    out = subprocess.run([sys.executable, "-c", PROBE.replace("ROOT", repr(ROOT))], capture_output=True, text=True,
                         timeout=300, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    failures, n = map(int, out.stdout.split()[-2:])
    assert failures == n
