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


@pytest.mark.parametrize("world,ranges", [(2, [(0, 3), (3, 5)]), (3, [(0, 2), (2, 4), (4, 5)])])
def test_gathered_shards_equal_the_whole_layer(world, ranges):
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank_main, args=(world, _free_port(), out), nprocs=world, start_method="spawn", join=True)
    from oracle import arl2_oracle as o
    Q, K, V, phi, S, alpha, beta = _case()
    O, S_new = o.frame_commit(S, Q, K, V, phi, alpha, beta, 0.5)
    assert [out[r][2] for r in range(world)] == ranges  # uneven: the gather pads the smaller shards
    for r in range(world):
        full, S_r, (h0, h1) = out[r]
        np.testing.assert_allclose(full, O, rtol=0, atol=1e-12)
        np.testing.assert_allclose(S_r, S_new[:, h0:h1], rtol=0, atol=1e-12)


def test_sharded_layer_passes_its_head_views_to_the_abi(monkeypatch):
    """What rank 1 of 2 hands the C ABI for a 5-head layer: views that start 3
    heads into each token row with the whole row's pitch, its own gate slices,
    and a handle of 2 heads (the binding's calls are replaced by recorders)."""
    from hybrid_linear_attention_arl2_b200 import arl2, sharding
    made, calls = {}, []

    class FakeLayer:
        def __init__(self, batch, heads, head_dim, tokens, dtype, pq, pk, pv, **kw):
            made.update(batch=batch, heads=heads, phi=(pq, pk, pv))
            self.handle = 7

        def _out(self, like):
            return torch.zeros((like.shape[0], like.shape[1], made["heads"], like.shape[3]))

    monkeypatch.setattr(arl2, "HybridLayer", FakeLayer)
    monkeypatch.setattr(arl2, "arl2_frame_query_strided", lambda *a: calls.append(("q",) + a))
    monkeypatch.setattr(arl2, "arl2_frame_commit_strided", lambda *a: calls.append(("c",) + a))
    B, L, H, d = 1, 4, 5, 128
    phi = [torch.arange(H, dtype=torch.float32)[:, None, None].expand(H, d, d).contiguous() for _ in range(3)]
    layer = sharding.ShardedHybridLayer(1, 2, B, H, L, *phi)
    assert made["heads"] == 2 and torch.equal(made["phi"][0][:, 0, 0], torch.tensor([3.0, 4.0]))
    q, k, v = (torch.zeros((B, L, H, d)) for _ in range(3))
    layer.query(q, k, v)
    alpha = torch.arange(H, dtype=torch.float32)[None]
    beta = torch.arange(H, dtype=torch.float32)[None, :, None].expand(B, H, L).contiguous()
    layer.commit(q, k, v, alpha, beta)
    (_, h, qv, kv, vv, ld, o, _), (_, _, qc, _, _, ldc, a, b, _, _) = calls
    assert h == 7 and ld == ldc == H * d
    for view, full in ((qv, q), (kv, k), (vv, v), (qc, q)):
        assert view.data_ptr() == full.data_ptr() + 3 * d * full.element_size()
        assert view.stride()[1] == H * d
    assert torch.equal(a, torch.tensor([[3.0, 4.0]])) and torch.equal(b[0, :, 0], torch.tensor([3.0, 4.0]))
    assert o.shape == (B, L, 2, d)
