"""The debug build (libarl2_debug.so: the kernels compiled with
-DARL2_DEBUG_BOUNDS, checking the indices they take from their parameters and
launch shape) on valid inputs: no check fails, and the results are those the
release build's parity tests demand.

A process loads one of the two libraries, so a child process loads the debug
build first and then runs the parity tests on it: frames of L = 1, 24, 127,
128, 129, 256 and 520 tokens (one token, a ragged tile, tile edges, several
tiles), streams of several frames, batched streams, the fp32 path, the
KV-cache layers, and the token-level passes.  Every one of those tests reads
the handle's error word through arl2_last_error, where a failed check would
show as ARL2_ERR_BOUNDS.  (The file name sorts last, so the release build's
tests have all run before it.)
"""
import os
import subprocess
import sys
import textwrap

import pytest
import torch

from hybrid_linear_attention_arl2_b200 import build

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = textwrap.dedent("""
    import sys
    sys.path.insert(0, {root!r})
    import pytest
    from hybrid_linear_attention_arl2_b200 import arl2
    arl2.load_library({lib!r})
    assert arl2.arl2_debug_bounds_enabled(), "not the debug build"
    sys.exit(pytest.main(["-q", "-x", "-m", "gpu", "-p", "no:cacheprovider", "-k", {select!r}]
                         + [{tests!r} + "/" + f for f in ("test_gpu_parity.py", "test_gpu_token_level.py")]))
""")

# the parity tests that run whole streams (the others check properties that
# do not depend on the build)
SELECT = ("ragged or small_stream or batched or f32 or kv_layer_stream or zero_beta or unit_key "
          "or inter_branch or intra_branch or token")


def test_debug_build_passes_the_parity_tests():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    lib = build.build(debug_bounds=True)
    code = CHILD.format(root=ROOT, lib=lib, select=SELECT, tests=os.path.join(ROOT, "tests"))
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True, timeout=900)
    tail = (r.stdout + r.stderr)[-3000:]
    assert r.returncode == 0, tail
    assert " passed" in r.stdout and " failed" not in r.stdout, tail
