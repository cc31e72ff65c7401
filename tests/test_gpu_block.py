"""The hybrid attention block (projections and gates around the hybrid layer)
on the GPU through the C ABI, against the oracle's block on the same seeded
inputs and random-init weights."""
import numpy as np
import pytest
import torch

from gpu_util import dev, host, small_config
from helpers import frob_rel, max_rel
from hybrid_linear_attention_arl2_b200 import arl2
from hybrid_linear_attention_arl2_b200 import workloads as W
from oracle import arl2_oracle as o

pytestmark = pytest.mark.gpu

OUT_TOL = 2e-2    # max |y - r| / max |r| over each output (bf16 path)
STATE_TOL = 1e-2  # Frobenius-relative state error


def _run(B, H, L, frames, queries, seed):
    cfg = small_config(B=B, H=H, L=L, frames=frames, queries=queries, seed=seed)
    wl = W.Workload(cfg)
    weights = wl.block_weights(0)
    phi = wl.phi(0)
    blk = arl2.HybridBlock(B, H, L, *(dev(w, "bf16") for w in weights), *(dev(p, "bf16") for p in phi),
                           corr_scale=cfg.corr_scale)
    S = np.zeros((B, H, 128, 128))
    worst_y = worst_s = 0.0
    for n in range(frames):
        for p in range(cfg.passes):
            X = wl.block_input(0, n, p)
            if p < queries:
                Y = blk.query(dev(X, "bf16"))
                ref = o.block_query(S, X, weights, phi)
            else:
                Y = blk.commit(dev(X, "bf16"))
                ref, S = o.block_commit(S, X, weights, phi, cfg.c)
            torch.cuda.synchronize()
            worst_y = max(worst_y, max_rel(host(Y), ref))
        worst_s = max(worst_s, frob_rel(host(blk.state()), S))
    assert blk.last_error() == 0
    blk.close()
    return worst_y, worst_s


def test_block_stream():
    y, s = _run(B=1, H=2, L=200, frames=3, queries=1, seed=93)
    assert y <= OUT_TOL, y
    assert s <= STATE_TOL, s


def test_block_batched_ragged():
    y, s = _run(B=2, H=3, L=130, frames=2, queries=1, seed=94)
    assert y <= OUT_TOL, y
    assert s <= STATE_TOL, s


def test_block_rejects_overlapping_output():
    cfg = small_config(H=2, L=64, seed=95)
    wl = W.Workload(cfg)
    blk = arl2.HybridBlock(1, 2, 64, *(dev(w, "bf16") for w in wl.block_weights(0)),
                           *(dev(p, "bf16") for p in wl.phi(0)))
    x = dev(wl.block_input(0, 0, 0), "bf16")
    with pytest.raises(arl2.Arl2Error) as e:
        arl2.arl2_block_query(blk.handle, x, x)
    assert e.value.status == 1
    blk.close()
