"""Head sharding of a hybrid layer across GPUs, one process per GPU.

Every step of the layer works per head: the intra-frame softmax, the maps,
the read-out and the state write (ARL2 summary, section 2.1).  A frame's heads
can therefore be split across ranks with no exchange inside the layer.  The
one collective is the all-gather that assembles O for the next layer.  Rank r
keeps heads [h0, h1) of the state, reads its heads of Q, K and V in place
through the strided calls (its view starts h0 heads into each token row, and
the row pitch stays H x 128), and contributes its [B, L, h1 - h0, 128] output
to the gather.

This module holds only the partition and the assembly; the compute is the
C ABI's.  The partition and the assembly run on CPU tensors too, which is
how the tests check them with gloo ranks.
"""
from __future__ import annotations

from . import arl2

HEAD_DIM = 128


def head_ranges(heads: int, world: int) -> list[tuple[int, int]]:
    """Contiguous, balanced head ranges, one per rank: the first heads % world
    ranks take one head more."""
    if world < 1 or heads < world:
        raise ValueError(f"{heads} heads cannot be split over {world} ranks")
    base, extra = divmod(heads, world)
    out, h = [], 0
    for r in range(world):
        n = base + (1 if r < extra else 0)
        out.append((h, h + n))
        h += n
    return out


def gather_heads(o_local, heads: int, dist, group=None):
    """All-gather every rank's [B, L, h1 - h0, d] output into [B, L, H, d].
    Shards are padded to the largest one, so that one all-gather moves them
    all; the padding is dropped when the heads are put in place."""
    import torch
    world = dist.get_world_size(group)
    ranges = head_ranges(heads, world)
    n_max = max(h1 - h0 for h0, h1 in ranges)
    B, L, n_local, d = o_local.shape
    send = o_local
    if n_local < n_max:
        send = torch.zeros((B, L, n_max, d), dtype=o_local.dtype, device=o_local.device)
        send[:, :, :n_local] = o_local
    parts = [torch.empty_like(send) for _ in range(world)]
    dist.all_gather(parts, send.contiguous(), group=group)
    out = torch.empty((B, L, heads, d), dtype=o_local.dtype, device=o_local.device)
    for (h0, h1), part in zip(ranges, parts):
        out[:, :, h0:h1] = part[:, :, :h1 - h0]
    return out


class ShardedHybridLayer:
    """Rank `rank`'s heads of one bf16 hybrid layer.  q, k, v, alpha, beta are
    the whole frame's tensors ([B, L, H, 128]; [B, H]; [B, H, L]), identical on
    every rank; query and commit return the whole [B, L, H, 128] output."""

    def __init__(self, rank, world, batch, heads, tokens, phi_q, phi_k, phi_v, *, corr_scale=-1.0,
                 softmax_scale=0.0, dist=None, group=None, stream=None):
        self.heads, self.dist, self.group, self.stream = heads, dist, group, stream
        self.h0, self.h1 = head_ranges(heads, world)[rank]
        sl = slice(self.h0, self.h1)
        self.layer = arl2.HybridLayer(batch, self.h1 - self.h0, HEAD_DIM, tokens, arl2.ARL2_BF16,
                                      phi_q[sl].contiguous(), phi_k[sl].contiguous(), phi_v[sl].contiguous(),
                                      softmax_scale=softmax_scale, corr_scale=corr_scale, stream=stream)

    def _views(self, q, k, v):
        sl = slice(self.h0, self.h1)
        return q[:, :, sl], k[:, :, sl], v[:, :, sl]  # strided views: pitch H x 128, start h0 heads in

    def _gather(self, o_local):
        if self.dist is None or self.dist.get_world_size(self.group) == 1:
            return o_local
        return gather_heads(o_local, self.heads, self.dist, self.group)

    def query(self, q, k, v):
        qv, kv, vv = self._views(q, k, v)
        o = self.layer._out(q)
        arl2.arl2_frame_query_strided(self.layer.handle, qv, kv, vv, self.heads * HEAD_DIM, o, self.stream)
        return self._gather(o)

    def commit(self, q, k, v, alpha, beta):
        qv, kv, vv = self._views(q, k, v)
        a = alpha[:, self.h0:self.h1].contiguous()
        b = beta[:, self.h0:self.h1].contiguous()
        o = self.layer._out(q)
        arl2.arl2_frame_commit_strided(self.layer.handle, qv, kv, vv, self.heads * HEAD_DIM, a, b, o, self.stream)
        return self._gather(o)

    def close(self):
        self.layer.close()
