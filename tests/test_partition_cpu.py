"""Host logic of the attention kernel's work partition (no device needed).

Invariants the kernel relies on: every (slab, block, key tile) unit is covered
exactly once; a split block is finished by the pair holding key tile 0 (that
pair's last segment), whose n_contrib pieces come from the pairs right after
it, each of which holds that block as its first segment (or, on long key
ranges, its last); a pair contributes at most one piece (one scratch slot per
CTA); at most eight pieces per block.
"""
import itertools

import pytest

from hybrid_linear_attention_arl2_b200 import arl2


def check(batch, heads, q_len, kv_len, pairs):
    parts = arl2.arl2_attn_partition(batch, heads, q_len, kv_len, pairs)
    n_blk = ((q_len + 127) // 128 + 1) // 2
    nkv = (kv_len + 127) // 128
    assert 1 <= len(parts) <= pairs
    seen = {}
    for c, segs in enumerate(parts):
        assert segs, "every pair has work"
        contributions = 0
        for i, (slab, blk, j0, j1, nc) in enumerate(segs):
            assert 0 <= slab < batch * heads and 0 <= blk < n_blk and 0 <= j0 < j1 <= nkv
            for j in range(j0, j1):
                assert (slab, blk, j) not in seen
                seen[(slab, blk, j)] = c
            if j0 > 0:  # a continuing piece: the pair's first segment, or its last on long key ranges
                assert i == 0 or (nkv >= 32 and i == len(segs) - 1)
                contributions += 1
            if j0 == 0 and j1 < nkv:  # finishes a split block: the pair's last segment
                assert i == len(segs) - 1
                assert 1 <= nc <= 8
                covered = j1
                for q in range(nc):
                    pieces = [x for x in parts[c + 1 + q] if (x[0], x[1]) == (slab, blk)]
                    assert len(pieces) == 1
                    s2, b2, k0, k1, _ = pieces[0]
                    assert k0 == covered
                    covered = k1
                assert covered == nkv
            else:
                assert nc == 0
        assert contributions <= 1
    assert len(seen) == batch * heads * n_blk * nkv


@pytest.mark.parametrize("batch,heads,q_len,kv_len,pairs", [
    (1, 12, 1560, 1560, 74),    # the 1560-token frame
    (4, 12, 1560, 1560, 74),    # four streams
    (1, 12, 1560, 6240, 74),    # a KV layer over four frames
    (1, 1, 128, 128, 74),       # one tile
    (1, 2, 300, 300, 74),
    (2, 12, 1560, 1560, 1),
    (1, 12, 4096, 4096, 96),
    (8, 16, 1024, 1024, 74),
])
def test_partition_invariants(batch, heads, q_len, kv_len, pairs):
    check(batch, heads, q_len, kv_len, pairs)


def test_partition_sweep():
    for batch, heads, q, kv, pairs in itertools.product([1, 3], [1, 5, 12], [1, 129, 640, 1560], [1, 200, 1560, 3000],
                                                        [1, 7, 37, 74]):
        check(batch, heads, q, kv, pairs)


def test_partition_1560_frame_is_balanced():
    # 84 blocks of 13 key tiles on 74 pairs: no pair walks more than 15 tiles,
    # and every split block merges a single piece (pieces past the first are
    # read with latency-bound loads, which the schedule avoids)
    parts = arl2.arl2_attn_partition(1, 12, 1560, 1560, 74)
    assert len(parts) == 74
    assert max(sum(j1 - j0 for _, _, j0, j1, _ in s) for s in parts) == 15
    assert max(nc for s in parts for *_, nc in s) == 1


def test_partition_takes_whole_blocks_when_they_divide():
    # 148 blocks on 74 pairs: two whole blocks each, nothing split
    parts = arl2.arl2_attn_partition(1, 37, 1024, 1024, 74)
    assert all(len(s) == 2 and all(j0 == 0 and j1 == 8 for _, _, j0, j1, _ in s) for s in parts)


def test_partition_long_key_ranges_start_whole_blocks_together():
    # a KV-cache layer over 21 frames of keys: every pair's first segment is a
    # whole block, and round 0 holds blocks 0 .. 73 (the seven blocks of a head
    # on seven pairs side by side)
    parts = arl2.arl2_attn_partition(1, 12, 1560, 21 * 1560, 74)
    nkv = (21 * 1560 + 127) // 128
    firsts = [s[0] for s in parts]
    assert all(j0 == 0 and j1 == nkv for _, _, j0, j1, _ in firsts)
    assert sorted(slab * 7 + blk for slab, blk, *_ in firsts) == list(range(74))


def test_partition_rejects_bad_arguments():
    with pytest.raises(RuntimeError):
        arl2.arl2_attn_partition(0, 12, 1560, 1560, 74)
    with pytest.raises(RuntimeError):
        arl2.arl2_attn_partition(1, 12, 1560, 1560, 97)
