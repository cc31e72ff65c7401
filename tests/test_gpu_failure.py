"""Failure handling on the device: injected allocation failures.

Each case runs in a child process because the injection hook counts device
allocations from the start of the process: ``ARL2_FAIL_ALLOC_AT=n`` makes the
n-th ``cudaMalloc`` of the library fail.  The child first creates and destroys
one handle (so the CUDA runtime's own one-time allocations are done and the
hook's count is known: a bfloat16 handle makes 11 allocations), then asks for
a second handle whose k-th allocation fails, for every k.  It must get
``ARL2_ERR_OUT_OF_MEMORY`` and leave no device memory behind.  The shape
(8 streams, 48 heads) makes the phi copies and the states 1.5 MB and more,
above the 1 MiB slack of the free-memory comparison, so an init that forgot
its earlier buffers on the error path shows; a leak of one of the small
buffers alone (the 256-byte error word, the ready flags) would not.  No GPU fault is involved: the failure is a status code from a fake of
the failing call.
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
ALLOCS_PER_BF16_HANDLE = 11

CHILD = textwrap.dedent("""
    import ctypes, os, sys
    import torch
    sys.path.insert(0, {root!r})
    from hybrid_linear_attention_arl2_b200 import arl2
    lib = arl2.load_library()
    B, H, L = 8, 48, 128
    phi = [torch.zeros((H, 128, 128), dtype=torch.bfloat16, device="cuda") for _ in range(3)]
    cfg = arl2.make_config(B, H, 128, L, arl2.ARL2_BF16)
    h = ctypes.c_void_p()
    rc = lib.arl2_state_init(ctypes.byref(cfg), *(ctypes.c_void_p(p.data_ptr()) for p in phi), None, ctypes.byref(h))
    assert rc == 0, rc
    assert lib.arl2_state_destroy(h) == 0
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    h2 = ctypes.c_void_p()
    rc = lib.arl2_state_init(ctypes.byref(cfg), *(ctypes.c_void_p(p.data_ptr()) for p in phi), None, ctypes.byref(h2))
    torch.cuda.synchronize()
    free1 = torch.cuda.mem_get_info()[0]
    print("RESULT", rc, h2.value or 0, free0 - free1)
""")


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    build.build()


@pytest.mark.parametrize("k", range(1, ALLOCS_PER_BF16_HANDLE + 1))
def test_injected_allocation_failure_returns_out_of_memory_without_leak(k):
    env = dict(os.environ, ARL2_FAIL_ALLOC_AT=str(ALLOCS_PER_BF16_HANDLE + k))
    r = subprocess.run([sys.executable, "-c", CHILD.format(root=ROOT)], env=env, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    line = [x for x in r.stdout.splitlines() if x.startswith("RESULT")][-1]
    _, rc, handle, leaked = line.split()
    assert int(rc) == 3, f"allocation {k}: status {rc}, expected ARL2_ERR_OUT_OF_MEMORY (3)"
    assert int(handle) == 0, "a failed init must not hand out a handle"
    assert int(leaked) <= 1 << 20, f"allocation {k}: {int(leaked)} bytes of device memory not returned"


def test_allocation_count_of_a_bf16_handle():
    """The count the cases above rely on: the 12th allocation is the second
    handle's first, so failing it returns OUT_OF_MEMORY, and failing the 23rd
    (past the second handle's last) lets both handles through."""
    env = dict(os.environ, ARL2_FAIL_ALLOC_AT=str(2 * ALLOCS_PER_BF16_HANDLE + 1))
    r = subprocess.run([sys.executable, "-c", CHILD.format(root=ROOT)], env=env, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    line = [x for x in r.stdout.splitlines() if x.startswith("RESULT")][-1]
    assert int(line.split()[1]) == 0


def test_attention_wait_limit_reports_timeout_and_recovers():
    """The attention kernel's own bounded waits, made to run out on a real
    1560-token layer: with a 1 microsecond limit the first waits of the launch
    (tiles still on their way from memory) give up, the kernel drains its
    asynchronous work and returns, and arl2_last_error reports the timeout.
    With the default limit back, the next frame on the same handle matches the
    oracle: the aborted launch left nothing behind that the next one reads."""
    import numpy as np
    from hybrid_linear_attention_arl2_b200 import arl2
    from hybrid_linear_attention_arl2_b200 import workloads as W
    from oracle import arl2_oracle as o
    from tests.gpu_util import dev, host, make_layer
    from tests.helpers import max_rel

    arl2.load_library()
    cfg = W.CONFIGS[1]
    wl = W.Workload(cfg)
    layer, phi = make_layer(cfg, wl)
    Q, K, V = (dev(x, "bf16") for x in wl.qkv(0, 0, 0))
    arl2.arl2_state_set_wait_limit(layer.handle, 1000)
    layer.query(Q, K, V)
    torch.cuda.synchronize()
    assert layer.last_error() == 5, "expected ARL2_ERR_TIMEOUT from the 1 us wait limit"
    assert layer.last_error() == 0, "the error word is cleared once read"
    arl2.arl2_state_set_wait_limit(layer.handle, 0)
    out = host(layer.query(Q, K, V))
    torch.cuda.synchronize()
    assert layer.last_error() == 0
    rows = np.arange(0, cfg.tokens, 7)
    ref = o.frame_query(np.zeros((cfg.batch, cfg.heads, 128, 128)), wl.qkv(0, 0, 0)[0][:, rows],
                        wl.qkv(0, 0, 0)[1], wl.qkv(0, 0, 0)[2], phi)
    assert max_rel(out[:, rows], ref) <= 2e-2
    layer.close()
