"""The allocation-free state write against the handle's commit.

Some callers cannot allocate device memory while they run a frame (a stream
that is being captured into a CUDA graph, a process with a fixed device-memory
budget, a host runtime that owns the allocator).  ``arl2_state_write_noalloc``
serves them: it computes the same state write as ``arl2_frame_commit`` with
its work space in the library's static scratch array.  This test calls it
through the C ABI for two frames in a row -- the second call reuses the array
the first one left behind -- and checks each new state against the state the
handle's commit wrote from the same inputs.  Both run the same kernels in the
same order on bit-identical inputs, so the states must be equal bit for bit; a
scratch-layout or aliasing mistake that shifts a few values would pass a
tolerance but not this.  The Frobenius-relative error against the bf16 state
tolerance of the parity tests (1e-2) is reported when they differ.

The file name sorts last so that a run which stops at the first failure has
run every other test before this one.
"""
import numpy as np
import pytest
import torch

from hybrid_linear_attention_arl2_b200 import arl2, build
from hybrid_linear_attention_arl2_b200 import workloads as W
from tests.gpu_util import dev, host, make_layer, small_config
from tests.helpers import frob_rel

pytestmark = pytest.mark.gpu

BF16_STATE_TOL = 1e-2


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    build.build()
    arl2.load_library()


@pytest.mark.parametrize("B,H,L,corr", [(1, 2, 300, 1.0), (1, 12, 1560, -1.0)])
def test_noalloc_state_write_matches_commit_twice(B, H, L, corr):
    cfg = small_config(B=B, H=H, L=L, frames=2, queries=0, corr=corr, seed=31)
    wl = W.Workload(cfg)
    layer, phi = make_layer(cfg, wl)
    phi_k, phi_v = dev(phi[1], "bf16"), dev(phi[2], "bf16")
    abi_cfg = arl2.make_config(B, H, 128, L, arl2.ARL2_BF16, corr_scale=corr)
    shape = (B, H, 128, 128)
    S_prev = torch.zeros(shape, dtype=torch.float32, device="cuda")
    S_next = torch.empty(shape, dtype=torch.float32, device="cuda")
    dev_error = torch.full((4,), 7, dtype=torch.int32, device="cuda")
    for n in range(2):
        Q, K, V = (dev(x, "bf16") for x in wl.qkv(0, n, 0))
        alpha = torch.from_numpy(wl.alpha(0, n)).cuda()
        beta = torch.from_numpy(np.ascontiguousarray(wl.beta(0, n))).cuda()
        layer.commit(Q, K, V, alpha, beta)
        S_ref = host(layer.state())
        S_next.fill_(float("nan"))
        arl2.arl2_state_write_noalloc(abi_cfg, K, V, phi_k, phi_v, S_prev, alpha, beta, S_next, dev_error)
        torch.cuda.synchronize()
        assert int(dev_error[0].item()) == 0, f"frame {n}: device error {int(dev_error[0].item())}"
        got = host(S_next)
        assert np.isfinite(got).all(), f"frame {n}: non-finite state"
        assert np.linalg.norm(S_ref) > 0
        if not torch.equal(S_next, layer.state()):
            e = frob_rel(got, S_ref)
            diff = int((S_next != layer.state()).sum().item())
            pytest.fail(f"frame {n}: {diff} state values differ from the commit's (Frobenius-relative "
                        f"{e:.3e}, tolerance of the parity tests {BF16_STATE_TOL})")
        S_prev, S_next = S_next, S_prev
    assert layer.last_error() == 0
    layer.close()
