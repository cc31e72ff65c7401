"""GPU parity at the full workload sizes, in the launch configuration the
benchmark times (persistent grid over all SMs, 1560-token frames, 12 heads).

Outputs are compared on a sample of query rows that covers every query tile
boundary and the ragged last tile, for every pass of the sampled frames; the
state is compared after every frame (the oracle's whole trajectory).
"""
import numpy as np
import pytest
import torch

from hybrid_linear_attention_arl2_b200 import arl2, build
from hybrid_linear_attention_arl2_b200 import workloads as W
from oracle import arl2_oracle as o
from tests.gpu_util import dev, host, run_gpu_stream, run_oracle_stream
from tests.helpers import frob_rel, max_rel

pytestmark = pytest.mark.gpu

OUT_TOL, STATE_TOL = 2e-2, 1e-2


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available()
    build.build()
    arl2.load_library()


def sample_rows(L, n_random=24, seed=0):
    rng = np.random.default_rng(seed)
    edges = [0, 1, 127, 128, 255, 256, 1023, 1024, 1279, 1280, 1407, 1408, 1535, 1536, L - 2, L - 1]
    rows = set(r for r in edges if 0 <= r < L)
    rows.update(int(x) for x in rng.choice(L, n_random, replace=False))
    return np.array(sorted(rows))


def _check(cfg, frames, keep_frames, rows, corr=None):
    if corr is not None:
        cfg = W.Config(cfg.index, cfg.name, cfg.batch, cfg.heads, cfg.head_dim, cfg.tokens, cfg.frames,
                       cfg.queries, cfg.dtype, corr_scale=corr, pool=cfg.pool)
    wl = W.Workload(cfg)
    keep = lambda n, p: n in keep_frames
    g_out, g_S = run_gpu_stream(cfg, wl, frames=frames, keep=keep)
    r_out, r_S = run_oracle_stream(cfg, wl, frames=frames, keep=keep, rows=rows)
    worst_o = max(max_rel(g_out[k][:, rows], r) for k, r in r_out.items())
    worst_s = max(frob_rel(g, r) for g, r in zip(g_S, r_S))
    assert worst_o <= OUT_TOL, worst_o
    assert worst_s <= STATE_TOL, worst_s
    return worst_o, worst_s


def test_single_layer_stream_mean_correction():
    """The single hybrid layer, 21 frames, c = 1/L."""
    cfg = W.CONFIGS[1]
    _check(cfg, cfg.frames, {0, 1, 10, 20}, sample_rows(cfg.tokens))


def test_single_layer_stream_literal_correction():
    """The same layer with the literal c = 1 (the state grows every frame at
    these shapes; fp32 holds it for these frames)."""
    cfg = W.CONFIGS[1]
    _check(cfg, 8, {0, 3, 7}, sample_rows(cfg.tokens, seed=1), corr=1.0)


def test_batched_streams():
    """Four independent streams, 81 frames."""
    cfg = W.CONFIGS[4]
    _check(cfg, cfg.frames, {0, 40, 80}, sample_rows(cfg.tokens, seed=2))


def test_long_stream_flat_time_and_memory():
    """231 frames: parity on the state trajectory and sampled outputs, device
    memory constant, per-frame time flat in the frame index."""
    cfg = W.CONFIGS[2]
    wl = W.Workload(cfg)
    rows = sample_rows(cfg.tokens, seed=3)
    keep = lambda n, p: n in (0, 115, 230) and p == cfg.queries
    g_out, g_S = run_gpu_stream(cfg, wl, keep=keep)
    r_out, r_S = run_oracle_stream(cfg, wl, keep=keep, rows=rows)
    assert max(max_rel(g_out[k][:, rows], r) for k, r in r_out.items()) <= OUT_TOL
    assert max(frob_rel(g, r) for g, r in zip(g_S, r_S)) <= STATE_TOL

    # timing and memory of the same stream, inputs resident
    phi = [dev(x, "bf16") for x in wl.phi(0)]
    layer = arl2.HybridLayer(1, cfg.heads, 128, cfg.tokens, arl2.ARL2_BF16, *phi, corr_scale=cfg.corr_scale)
    pool = [tuple(dev(x[None], "bf16") for x in wl.pool_entry(0, i)) for i in range(cfg.pool)]
    gates = [(torch.from_numpy(wl.alpha(0, n)).cuda(), torch.from_numpy(wl.beta(0, n)).cuda())
             for n in range(cfg.frames)]
    O = torch.empty_like(pool[0][0])
    torch.cuda.synchronize()
    mem0, held = torch.cuda.memory_allocated(), layer.device_bytes()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(cfg.frames + 1)]
    ev[0].record()
    for n in range(cfg.frames):
        for p in range(cfg.passes):
            q, k, v = pool[wl.pool_index(0, n, p)]
            if p < cfg.queries:
                layer.query(q, k, v, O)
            else:
                layer.commit(q, k, v, *gates[n], O)
        ev[n + 1].record()
    torch.cuda.synchronize()
    ms = np.array([ev[i].elapsed_time(ev[i + 1]) for i in range(cfg.frames)])
    assert torch.cuda.memory_allocated() == mem0 and layer.device_bytes() == held
    early, late = np.median(ms[5:40]), np.median(ms[-35:])
    assert late < 1.25 * early, (early, late)
    assert layer.last_error() == 0
    layer.close()


def test_attention_stack_sample():
    """The 30-layer stack (22 hybrid layers, 8 softmax layers with a KV cache)
    over 63 frames.  All layers run; the oracle checks hybrid layers 0 and 21
    (state trajectory, sampled outputs) and softmax layers 22 and 29 (sampled
    outputs of the first, middle and last frames)."""
    cfg = W.CONFIGS[3]
    wl = W.Workload(cfg)
    F = cfg.frames
    rows = sample_rows(cfg.tokens, n_random=8, seed=4)
    check_frames = (0, F // 2, F - 1)
    phis = {l: wl.phi(l) for l in range(cfg.hybrid_layers)}
    hyb = {l: arl2.HybridLayer(1, cfg.heads, 128, cfg.tokens, arl2.ARL2_BF16,
                               *(dev(x, "bf16") for x in phis[l]), corr_scale=cfg.corr_scale)
           for l in range(cfg.hybrid_layers)}
    kvl = {l: arl2.KVLayer(1, cfg.heads, 128, cfg.tokens, arl2.ARL2_BF16, max_frames=F)
           for l in range(cfg.hybrid_layers, cfg.layers)}
    pool = {}

    def trip(l, n, p):
        i = wl.pool_index(l, n, p)
        if i not in pool:
            pool[i] = tuple(dev(x[None], "bf16") for x in wl.pool_entry(0, i))
        return pool[i]

    S_ref = {l: np.zeros((1, cfg.heads, 128, 128)) for l in (0, 21)}
    kv_ctx = {l: [] for l in (22, 29)}  # pool indices of the committed frames
    O = torch.empty_like(trip(0, 0, 0)[0])
    for n in range(F):
        for l in range(cfg.layers):
            for p in range(cfg.passes):
                q, k, v = trip(l, n, p)
                if l in hyb:
                    if p < cfg.queries:
                        hyb[l].query(q, k, v, O)
                    else:
                        hyb[l].commit(q, k, v, torch.from_numpy(wl.alpha(l, n)).cuda(),
                                      torch.from_numpy(wl.beta(l, n)).cuda(), O)
                else:
                    (kvl[l].query if p < cfg.queries else kvl[l].commit)(q, k, v, O)
                if n in check_frames and l in (0, 21, 22, 29):
                    Q, K, V = wl.pool_entry(0, wl.pool_index(l, n, p))
                    Q, K, V = Q[None], K[None], V[None]
                    if l in S_ref:
                        ref = o.frame_query(S_ref[l], Q[:, rows], K, V, phis[l])
                    else:
                        past = [wl.pool_entry(0, i) for i in kv_ctx[l]]
                        Kc = np.concatenate([x[1][None] for x in past] + [K], 1)
                        Vc = np.concatenate([x[2][None] for x in past] + [V], 1)
                        ref = o.kv_attention(Q[:, rows], Kc, Vc)
                    assert max_rel(host(O)[:, rows], ref) <= OUT_TOL, (n, l, p)
            if l in S_ref:
                Q, K, V = wl.pool_entry(0, wl.pool_index(l, n, cfg.queries))
                S_ref[l] = o.state_update(S_ref[l], K[None], V[None], phis[l], wl.alpha(l, n), wl.beta(l, n), cfg.c)
                assert frob_rel(host(hyb[l].state()), S_ref[l]) <= STATE_TOL, (n, l)
            if l in kv_ctx:
                kv_ctx[l].append(wl.pool_index(l, n, cfg.queries))
    for x in list(hyb.values()) + list(kvl.values()):
        assert x.last_error() == 0
        x.close()


@pytest.mark.parametrize("index", [1, 4])
def test_every_query_row_of_a_full_size_pass(index):
    """Every query row (all 1560, every head and stream) of one query pass and
    of the commit pass of the second frame, against the oracle: the rows the
    sampled tests skip include the interior of every query tile and the rows
    of blocks whose key range the launch splits between CTA pairs."""
    cfg = W.CONFIGS[index]
    wl = W.Workload(cfg)
    keep = lambda n, p: n == 1 and p in (0, cfg.queries)
    g_out, g_S = run_gpu_stream(cfg, wl, frames=2, keep=keep)
    r_out, r_S = run_oracle_stream(cfg, wl, frames=2, keep=keep)
    for key, r in r_out.items():
        e = max_rel(g_out[key], r)
        assert e <= OUT_TOL, (key, e)
    assert frob_rel(g_S[-1], r_S[-1]) <= STATE_TOL


def _split_block_rows(cfg, pairs=74):
    """Query rows (of every head) whose 256-row block the pair kernel's stream-K
    partition splits between two or more CTA pairs, for `pairs` resident pairs
    (74 on a 148-SM B200): every block whose key range does not lie inside one
    pair's contiguous range of (block, key tile) units."""
    n_qt = (cfg.tokens + 127) // 128
    n_blk, nkv = (n_qt + 1) // 2, (cfg.tokens + 127) // 128
    units = cfg.batch * cfg.heads * n_blk * nkv
    bounds = [units * c // pairs for c in range(pairs + 1)]
    split = set()
    for c in range(1, pairs):
        u = bounds[c]
        if u % nkv:  # a pair boundary inside a block
            bh, blk = divmod(u // nkv, n_blk)
            split.add((bh, blk))
    return split, n_blk


def test_split_blocks_err_like_whole_blocks():
    """Pieces of split blocks travel between CTA pairs as O / l rounded to bf16
    (one extra rounding step that whole blocks do not take).  Their rows must
    err like the rows of whole blocks: at most twice the largest error of the
    whole blocks' rows, plus one bf16 step of the output scale."""
    cfg = W.CONFIGS[1]
    wl = W.Workload(cfg)
    keep = lambda n, p: n == 1 and p == 0
    g_out, _ = run_gpu_stream(cfg, wl, frames=2, keep=keep)
    r_out, _ = run_oracle_stream(cfg, wl, frames=2, keep=keep)
    g, r = g_out[(1, 0)], r_out[(1, 0)]          # [B, L, H, d]
    scale = np.abs(r).max()
    err = np.abs(g - r).max(axis=3) / scale       # [B, L, H]
    split, n_blk = _split_block_rows(cfg)
    assert split, "the 1560-token frame has split blocks at 74 pairs"
    mask = np.zeros(err.shape, dtype=bool)
    for bh, blk in split:
        b, h = divmod(bh, cfg.heads)
        mask[b, blk * 256:(blk + 1) * 256, h] = True
    e_split, e_whole = err[mask].max(), err[~mask].max()
    assert e_split <= OUT_TOL and e_whole <= OUT_TOL
    assert e_split <= 2 * e_whole + 2.0 ** -8, (e_split, e_whole)
