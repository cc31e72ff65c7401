"""Head sharding (hybrid_linear_attention_arl2_b200.sharding) as two gloo ranks
on the CPU: the partition, and the all-gather that assembles O.  Each rank runs
the oracle on its heads, in place of the GPU layer, and the assembled output
must equal the whole layer's.  That also pins the property the sharding rests
on: every head of the layer is independent of the others."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from hybrid_linear_attention_arl2_b200.sharding import head_ranges  # noqa: E402


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_head_ranges_are_balanced_and_contiguous():
    for heads in (1, 5, 12, 13):
        for world in range(1, min(heads, 8) + 1):
            r = head_ranges(heads, world)
            assert r[0][0] == 0 and r[-1][1] == heads
            assert all(a[1] == b[0] for a, b in zip(r, r[1:]))
            sizes = [h1 - h0 for h0, h1 in r]
            assert max(sizes) - min(sizes) <= 1 and min(sizes) >= 1
    assert head_ranges(12, 8) == [(0, 2), (2, 4), (4, 6), (6, 8), (8, 9), (9, 10), (10, 11), (11, 12)]
    with pytest.raises(ValueError):
        head_ranges(3, 4)


def _case(seed=5, B=1, L=9, H=5, d=8):
    rng = np.random.default_rng(seed)
    Q, K, V = (rng.standard_normal((B, L, H, d)) for _ in range(3))
    phi = tuple(np.eye(d)[None] + rng.standard_normal((H, d, d)) / np.sqrt(d) for _ in range(3))
    S = 0.3 * rng.standard_normal((B, H, d, d))
    alpha = rng.uniform(0.5, 1.0, (B, H))
    beta = rng.uniform(0.0, 1.0, (B, H, L))
    return Q, K, V, phi, S, alpha, beta


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        from hybrid_linear_attention_arl2_b200.sharding import gather_heads
        from oracle import arl2_oracle as o
        Q, K, V, phi, S, alpha, beta = _case()
        H = Q.shape[2]
        h0, h1 = head_ranges(H, world)[rank]
        sl = slice(h0, h1)
        O_r, S_r = o.frame_commit(S[:, sl], Q[:, :, sl], K[:, :, sl], V[:, :, sl], tuple(p[sl] for p in phi),
                                  alpha[:, sl], beta[:, sl], 0.5)
        full = gather_heads(torch.from_numpy(O_r), H, dist)
        out[rank] = (full.numpy(), S_r, (h0, h1))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_gathered_shards_equal_the_whole_layer():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank_main, args=(world, _free_port(), out), nprocs=world, start_method="spawn", join=True)
    from oracle import arl2_oracle as o
    Q, K, V, phi, S, alpha, beta = _case()
    O, S_new = o.frame_commit(S, Q, K, V, phi, alpha, beta, 0.5)
    assert [out[r][2] for r in range(world)] == [(0, 3), (3, 5)]  # uneven: the gather pads the smaller shard
    for r in range(world):
        full, S_r, (h0, h1) = out[r]
        np.testing.assert_allclose(full, O, rtol=0, atol=1e-12)
        np.testing.assert_allclose(S_r, S_new[:, h0:h1], rtol=0, atol=1e-12)
