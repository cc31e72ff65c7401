"""Token-level access on the GPU (arl2_token_query / arl2_token_commit)
against the oracle's token_level_pass on the same seeded inputs: outputs
within 2e-2 (max relative) and states within 1e-2 (Frobenius relative), a
query that leaves the state bit-identical, and frame-level calls that read
the state a token-level commit wrote."""
import numpy as np
import pytest
import torch

from hybrid_linear_attention_arl2_b200 import arl2, build
from hybrid_linear_attention_arl2_b200 import workloads as W
from oracle import arl2_oracle as o
from tests.gpu_util import dev, host, make_layer, small_config
from tests.helpers import frob_rel, max_rel

pytestmark = pytest.mark.gpu

OUT_TOL = 2e-2
STATE_TOL = 1e-2


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    build.build()
    arl2.load_library()


def _gates(wl, n):
    return wl.alpha_tok(0, n), wl.beta(0, n)


def _run(cfg, wl, frames):
    """GPU and oracle side by side: per frame, the query passes then the commit,
    all token-level; returns the worst output and state errors."""
    layer, phi = make_layer(cfg, wl)
    S_ref = np.zeros((cfg.batch, cfg.heads, cfg.head_dim, cfg.head_dim))
    worst_o = worst_s = 0.0
    for n in range(frames):
        a, b = _gates(wl, n)
        a_d, b_d = torch.from_numpy(a).cuda(), torch.from_numpy(b).cuda()
        for p in range(cfg.passes):
            Q, K, V = wl.qkv(0, n, p)
            Qd, Kd, Vd = (dev(x, cfg.dtype) for x in (Q, K, V))
            commit = p == cfg.queries
            O = (layer.token_commit if commit else layer.token_query)(Qd, Kd, Vd, a_d, b_d)
            O_ref, S_new = o.token_level_pass(S_ref, Q, K, V, phi, a, b, cfg.corr_scale)
            e = max_rel(host(O), O_ref)
            assert e <= OUT_TOL, f"frame {n} pass {p}: output {e:.3e}"
            worst_o = max(worst_o, e)
            if commit:
                S_ref = S_new
                e = frob_rel(host(layer.state()), S_ref)
                assert e <= STATE_TOL, f"frame {n}: state {e:.3e}"
                worst_s = max(worst_s, e)
    torch.cuda.synchronize()
    assert layer.last_error() == 0
    assert layer.frame == frames
    layer.close()
    return worst_o, worst_s


@pytest.mark.parametrize("L", [300, 128, 77])
def test_token_level_stream_matches_oracle(L):
    # 300 tokens: two full chunks and a ragged one; 128: one full chunk; 77: one ragged chunk
    cfg = small_config(B=1, H=2, L=L, frames=2, queries=1, corr=1.0, seed=81)
    _run(cfg, W.Workload(cfg, seed=81), frames=2)


def test_token_level_two_streams():
    cfg = small_config(B=2, H=2, L=200, frames=1, queries=1, corr=1.0, seed=82)
    _run(cfg, W.Workload(cfg, seed=82), frames=1)


def test_token_query_leaves_state_bitwise():
    cfg = small_config(B=1, H=2, L=260, frames=1, queries=1, corr=1.0, seed=83)
    wl = W.Workload(cfg, seed=83)
    layer, _ = make_layer(cfg, wl)
    a, b = _gates(wl, 0)
    a_d, b_d = torch.from_numpy(a).cuda(), torch.from_numpy(b).cuda()
    Q, K, V = (dev(x, cfg.dtype) for x in wl.qkv(0, 0, 1))
    layer.token_commit(Q, K, V, a_d, b_d)  # a nonzero state
    before = layer.state().cpu().numpy().tobytes()
    Q, K, V = (dev(x, cfg.dtype) for x in wl.qkv(0, 1, 0))
    layer.token_query(Q, K, V, a_d, b_d)
    after = layer.state().cpu().numpy().tobytes()
    assert before == after
    assert layer.frame == 1
    layer.close()


def test_frame_level_query_reads_token_level_commit():
    cfg = small_config(B=1, H=2, L=260, frames=1, queries=1, corr=1.0, seed=84)
    wl = W.Workload(cfg, seed=84)
    layer, phi = make_layer(cfg, wl)
    a, b = _gates(wl, 0)
    Q, K, V = wl.qkv(0, 0, 1)
    layer.token_commit(*(dev(x, cfg.dtype) for x in (Q, K, V)), torch.from_numpy(a).cuda(), torch.from_numpy(b).cuda())
    S0 = np.zeros((cfg.batch, cfg.heads, cfg.head_dim, cfg.head_dim))
    _, S1 = o.token_level_pass(S0, Q, K, V, phi, a, b, cfg.corr_scale)
    Q, K, V = wl.qkv(0, 1, 0)
    O = layer.query(*(dev(x, cfg.dtype) for x in (Q, K, V)))
    e = max_rel(host(O), o.frame_query(S1, Q, K, V, phi))
    assert e <= OUT_TOL, f"frame-level query after a token-level commit: {e:.3e}"
    layer.close()


def test_token_level_full_size_commit():
    """The single-hybrid-layer shape (B = 1, H = 12, L = 1560: twelve full
    chunks and a 24-token tail), one commit from a nonzero state."""
    cfg = small_config(B=1, H=12, L=1560, frames=2, queries=0, corr=1.0, seed=85)
    wl = W.Workload(cfg, seed=85)
    layer, phi = make_layer(cfg, wl)
    S0 = np.zeros((1, 12, 128, 128))
    for n in range(2):
        a, b = _gates(wl, n)
        Q, K, V = wl.qkv(0, n, 0)
        O = layer.token_commit(*(dev(x, cfg.dtype) for x in (Q, K, V)), torch.from_numpy(a).cuda(),
                               torch.from_numpy(b).cuda())
        O_ref, S0 = o.token_level_pass(S0, Q, K, V, phi, a, b, 1.0)
        assert max_rel(host(O), O_ref) <= OUT_TOL
        assert frob_rel(host(layer.state()), S0) <= STATE_TOL
    assert layer.last_error() == 0
    layer.close()
