"""GPU parity: the C-ABI path against the CPU oracle on the same seeded inputs.

Tolerances (fixed for the method's precisions):
  float32 path: max|x - r| / max|r| <= 1e-5 on outputs and states;
  bf16 path:    outputs max|x - r| / max|r| <= 2e-2,
                states ||S - S_ref||_F / ||S_ref||_F <= 1e-2.
"""
import numpy as np
import pytest
import torch

from hybrid_linear_attention_arl2_b200 import arl2, build
from hybrid_linear_attention_arl2_b200 import workloads as W
from oracle import arl2_oracle as o
from tests.gpu_util import (abi_dtype, dev, host, make_layer, run_gpu_stream, run_oracle_stream,
                            small_config)
from tests.helpers import frob_rel, max_rel

pytestmark = pytest.mark.gpu

F32_TOL = 1e-5
BF16_OUT_TOL = 2e-2
BF16_STATE_TOL = 1e-2


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    build.build()
    arl2.load_library()


def _compare(cfg, gpu, ref, out_tol, state_tol, state_metric):
    g_out, g_S = gpu
    r_out, r_S = ref
    worst = 0.0
    for key, r in r_out.items():
        e = max_rel(g_out[key], r)
        worst = max(worst, e)
        assert e <= out_tol, f"output {key}: {e:.3e} > {out_tol}"
    for n, (gs, rs) in enumerate(zip(g_S, r_S)):
        e = state_metric(gs, rs)
        assert e <= state_tol, f"state after frame {n}: {e:.3e} > {state_tol}"
    return worst


# ------------------------------------------------------------------ float32 path
def test_f32_tiny_stream():
    """The tiny float32 stream: every output of every pass and every state."""
    cfg = W.CONFIGS[0]
    wl = W.Workload(cfg)
    _compare(cfg, run_gpu_stream(cfg, wl), run_oracle_stream(cfg, wl), F32_TOL, F32_TOL, max_rel)


@pytest.mark.parametrize("L,d,H,B", [(1, 32, 1, 1), (37, 64, 3, 2), (130, 128, 2, 1)])
def test_f32_shapes(L, d, H, B):
    cfg = small_config(B=B, H=H, d=d, L=L, frames=3, queries=1, dtype="f32", corr=-1.0, seed=5)
    wl = W.Workload(cfg)
    _compare(cfg, run_gpu_stream(cfg, wl), run_oracle_stream(cfg, wl), F32_TOL, F32_TOL, max_rel)


# ------------------------------------------------------------------ bf16 path
@pytest.mark.parametrize("corr", [-1.0, 1.0])
def test_bf16_small_stream(corr):
    """Several tiles with a ragged tail (L = 300 = 2 x 128 + 44), several frames."""
    cfg = small_config(L=300, frames=3, queries=2, corr=corr)
    wl = W.Workload(cfg)
    _compare(cfg, run_gpu_stream(cfg, wl), run_oracle_stream(cfg, wl), BF16_OUT_TOL, BF16_STATE_TOL, frob_rel)


@pytest.mark.parametrize("L", [1, 24, 127, 128, 129, 256, 520])
def test_bf16_ragged_lengths(L):
    cfg = small_config(L=L, H=3, frames=2, queries=1, seed=L)
    wl = W.Workload(cfg)
    _compare(cfg, run_gpu_stream(cfg, wl), run_oracle_stream(cfg, wl), BF16_OUT_TOL, BF16_STATE_TOL, frob_rel)


def test_bf16_batched_streams():
    cfg = small_config(B=3, H=2, L=200, frames=3, queries=1, seed=9)
    wl = W.Workload(cfg)
    _compare(cfg, run_gpu_stream(cfg, wl), run_oracle_stream(cfg, wl), BF16_OUT_TOL, BF16_STATE_TOL, frob_rel)


def test_bf16_inter_branch_alone():
    """O_inter is exactly zero while S = 0, and matches Q' S after commits."""
    cfg = small_config(L=260, frames=3, queries=1, seed=13)
    wl = W.Workload(cfg)
    g_out, _ = run_gpu_stream(cfg, wl, flags=arl2.ARL2_INTER_ONLY)
    assert np.all(g_out[(0, 0)] == 0.0) and np.all(g_out[(0, 1)] == 0.0)
    phi = wl.phi(0)
    S = np.zeros((cfg.batch, cfg.heads, 128, 128))
    for n in range(cfg.frames):
        for p in range(cfg.passes):
            Q, K, V = wl.qkv(0, n, p)
            Qp, _, _ = o.feature_maps(Q, K, V, *phi)
            ref = o.inter_readout(Qp, S)
            if n > 0:
                assert max_rel(g_out[(n, p)], ref) <= BF16_OUT_TOL
            if p == cfg.queries:
                S = o.state_update(S, K, V, phi, wl.alpha(0, n), wl.beta(0, n), cfg.c)


def test_bf16_intra_branch_alone():
    cfg = small_config(L=333, frames=2, queries=1, seed=17)
    wl = W.Workload(cfg)
    g_out, _ = run_gpu_stream(cfg, wl, flags=arl2.ARL2_INTRA_ONLY)
    for (n, p), g in g_out.items():
        Q, K, V = wl.qkv(0, n, p)
        assert max_rel(g, o.intra_softmax(Q, K, V)) <= BF16_OUT_TOL


# ------------------------------------------------------------------ semantics
def _state_bytes(layer):
    return layer.state().cpu().numpy().tobytes()


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_queries_leave_state_bit_identical(dtype):
    cfg = small_config(L=150, frames=2, queries=1, dtype=dtype, d=128 if dtype == "bf16" else 32)
    wl = W.Workload(cfg)
    layer, _ = make_layer(cfg, wl)
    Q, K, V = (dev(x, dtype) for x in wl.qkv(0, 0, 0))
    a, b = torch.from_numpy(wl.alpha(0, 0)).cuda(), torch.from_numpy(wl.beta(0, 0)).cuda()
    layer.commit(Q, K, V, a, b)
    before = _state_bytes(layer)
    for p in range(4):
        Qp, Kp, Vp = (dev(x, dtype) for x in wl.qkv(0, 1, p))
        layer.query(Qp, Kp, Vp)
    torch.cuda.synchronize()
    assert _state_bytes(layer) == before
    assert layer.frame == 1
    layer.close()


def test_batch_equals_single_streams_bitwise():
    cfg = small_config(B=3, H=2, L=140, frames=2, queries=1, seed=21)
    wl = W.Workload(cfg)
    outs, states = run_gpu_stream(cfg, wl)
    phi = wl.phi(0)
    for b in range(cfg.batch):
        single = arl2.HybridLayer(1, cfg.heads, 128, cfg.tokens, arl2.ARL2_BF16, *(dev(p, "bf16") for p in phi),
                                  corr_scale=cfg.corr_scale)
        for n in range(cfg.frames):
            for p in range(cfg.passes):
                Q, K, V = (dev(x[b:b + 1], "bf16") for x in wl.qkv(0, n, p))
                if p < cfg.queries:
                    O = single.query(Q, K, V)
                else:
                    O = single.commit(Q, K, V, torch.from_numpy(wl.alpha(0, n)[b:b + 1]).cuda(),
                                      torch.from_numpy(np.ascontiguousarray(wl.beta(0, n)[b:b + 1])).cuda())
                assert np.array_equal(host(O)[0], outs[(n, p)][b])
            assert np.array_equal(host(single.state())[0], states[n][b])
        single.close()


def test_runs_are_deterministic():
    cfg = small_config(L=400, frames=3, queries=1, seed=31)
    wl = W.Workload(cfg)
    a = run_gpu_stream(cfg, wl)
    b = run_gpu_stream(cfg, wl)
    for key in a[0]:
        assert np.array_equal(a[0][key], b[0][key])
    for x, y in zip(a[1], b[1]):
        assert np.array_equal(x, y)


def test_save_and_resume_bitwise():
    cfg = small_config(L=200, frames=5, queries=1, seed=41)
    wl = W.Workload(cfg)
    full_out, full_S = run_gpu_stream(cfg, wl)
    layer, _ = make_layer(cfg, wl)
    for n in range(2):  # run two frames, checkpoint
        Q, K, V = (dev(x, "bf16") for x in wl.qkv(0, n, 1))
        layer.commit(Q, K, V, torch.from_numpy(wl.alpha(0, n)).cuda(), torch.from_numpy(wl.beta(0, n)).cuda())
    ckpt = layer.state().clone()
    frame = layer.frame
    layer.close()
    resumed, _ = make_layer(cfg, wl)
    resumed.set_state(ckpt, frame)
    assert resumed.frame == 2
    for n in range(2, cfg.frames):
        for p in range(cfg.passes):
            Q, K, V = (dev(x, "bf16") for x in wl.qkv(0, n, p))
            if p < cfg.queries:
                O = resumed.query(Q, K, V)
            else:
                O = resumed.commit(Q, K, V, torch.from_numpy(wl.alpha(0, n)).cuda(),
                                   torch.from_numpy(wl.beta(0, n)).cuda())
            assert np.array_equal(host(O), full_out[(n, p)])
        assert np.array_equal(host(resumed.state()), full_S[n])
    resumed.close()


def test_device_memory_is_flat_over_frames():
    cfg = small_config(L=256, frames=6, queries=1, seed=51)
    wl = W.Workload(cfg)
    layer, _ = make_layer(cfg, wl)
    Q, K, V = (dev(x, "bf16") for x in wl.qkv(0, 0, 0))
    a, b = torch.from_numpy(wl.alpha(0, 0)).cuda(), torch.from_numpy(wl.beta(0, 0)).cuda()
    O = torch.empty_like(Q)
    held = layer.device_bytes()
    torch.cuda.synchronize()
    alloc0 = torch.cuda.memory_allocated()
    for n in range(cfg.frames):
        layer.query(Q, K, V, O)
        layer.commit(Q, K, V, a, b, O)
        assert layer.device_bytes() == held
    torch.cuda.synchronize()
    assert torch.cuda.memory_allocated() == alloc0
    layer.close()


# ------------------------------------------------------------------ KV-cache softmax layers
@pytest.mark.parametrize("dtype,L,d", [("bf16", 200, 128), ("f32", 24, 32)])
def test_kv_layer_stream(dtype, L, d):
    cfg = small_config(L=L, d=d, H=2, frames=4, queries=2, dtype=dtype, seed=61)
    wl = W.Workload(cfg)
    kv = arl2.KVLayer(cfg.batch, cfg.heads, d, L, abi_dtype(dtype), max_frames=cfg.frames)
    past_k, past_v = [], []
    tol = BF16_OUT_TOL if dtype == "bf16" else F32_TOL
    for n in range(cfg.frames):
        for p in range(cfg.passes):
            Q, K, V = wl.qkv(0, n, p)
            if p < cfg.queries:
                O = kv.query(*(dev(x, dtype) for x in (Q, K, V)))
            else:
                O = kv.commit(*(dev(x, dtype) for x in (Q, K, V)))
            ref = o.kv_attention(Q, np.concatenate(past_k + [K], 1), np.concatenate(past_v + [V], 1))
            assert max_rel(host(O), ref) <= tol, (n, p)
        past_k.append(K)
        past_v.append(V)
        assert kv.frames == n + 1
    assert kv.last_error() == 0
    kv.close()


# ------------------------------------------------------------------ errors
def test_bounded_wait_reports_timeout():
    """A device-side wait on a barrier that nothing completes gives up after
    its limit and reports ARL2_ERR_TIMEOUT; the context stays usable."""
    assert arl2.arl2_selftest_wait_timeout(2_000_000) == 5
    x = torch.ones(4, device="cuda")
    assert float((x * 2).sum()) == 8.0


def test_invalid_device_arguments():
    cfg = small_config(L=128, frames=1, queries=1)
    wl = W.Workload(cfg)
    layer, _ = make_layer(cfg, wl)
    Q, K, V = (dev(x, "bf16") for x in wl.qkv(0, 0, 0))
    with pytest.raises(arl2.Arl2Error) as e:
        arl2.arl2_frame_query(layer.handle, Q, K, V, Q)  # output aliases the input
    assert e.value.status == 1
    flat = torch.empty(Q.numel() + 8, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(arl2.Arl2Error):
        arl2.arl2_frame_query(layer.handle, Q, K, V, flat[1:])  # misaligned output
    h = layer.handle
    layer.close()
    with pytest.raises(arl2.Arl2Error):
        arl2.arl2_frame_query(h, Q, K, V, torch.empty_like(Q))  # use after destroy


def test_fma_pipe_exp2_against_cuda_exp2f():
    """The FMA-pipe exp2 used for part of the softmax stays within its stated
    relative error bound (1e-4) of CUDA's exp2f over the clamped range, and is
    exact at integers."""
    x = torch.cat([torch.linspace(-125.0, 125.0, 1_000_001, device="cuda"),
                   torch.arange(-125, 126, device="cuda", dtype=torch.float32),
                   torch.rand(200_000, device="cuda") * -30.0])
    y = torch.empty_like(x)
    arl2.arl2_selftest_exp2(x, y)
    ref = torch.exp2(x.double())
    rel = ((y.double() - ref).abs() / ref).max().item()
    assert rel <= 1.0e-4, rel
    # at integers f = 0: the result is c0 * 2^n with c0 the polynomial's constant term
    ints = torch.arange(-125, 126, device="cuda", dtype=torch.float32)
    yi = torch.empty_like(ints)
    arl2.arl2_selftest_exp2(ints, yi)
    assert torch.equal(yi / torch.exp2(ints), torch.full_like(ints, yi[125].item()))


def test_strided_views_equal_contiguous_bitwise():
    """Q, K, V read as strided views of [B, L, 3D] rows (a fused QKV
    projection's layout) give the same bits as the contiguous calls."""
    cfg = small_config(B=2, H=2, L=200, frames=1, queries=1, seed=41)
    wl = W.Workload(cfg)
    a_lay, _ = make_layer(cfg, wl)
    b_lay, _ = make_layer(cfg, wl)
    Q, K, V = (dev(x, "bf16") for x in wl.qkv(0, 0, 0))
    B, L, H, d = Q.shape
    D = H * d
    fused = torch.cat([Q.reshape(B, L, D), K.reshape(B, L, D), V.reshape(B, L, D)], dim=2).contiguous()
    alpha = torch.from_numpy(wl.alpha(0, 0)).cuda()
    beta = torch.from_numpy(wl.beta(0, 0)).cuda()
    o1, o2 = torch.empty_like(Q), torch.empty_like(Q)
    for commit in (False, True):
        if commit:
            arl2.arl2_frame_commit(a_lay.handle, Q, K, V, alpha, beta, o1)
            arl2.arl2_frame_commit_strided(b_lay.handle, fused, fused[..., D:], fused[..., 2 * D:], 3 * D, alpha,
                                           beta, o2)
        else:
            arl2.arl2_frame_query(a_lay.handle, Q, K, V, o1)
            arl2.arl2_frame_query_strided(b_lay.handle, fused, fused[..., D:], fused[..., 2 * D:], 3 * D, o2)
        torch.cuda.synchronize()
        assert torch.equal(o1, o2)
    assert torch.equal(a_lay.state(), b_lay.state())
    with pytest.raises(arl2.Arl2Error):  # pitch below a row
        arl2.arl2_frame_query_strided(b_lay.handle, fused, fused[..., D:], fused[..., 2 * D:], D - 8, o2)
    with pytest.raises(arl2.Arl2Error):  # pitch not a multiple of 8 elements
        arl2.arl2_frame_query_strided(b_lay.handle, fused, fused[..., D:], fused[..., 2 * D:], 3 * D + 4, o2)
    a_lay.close()
    b_lay.close()


def test_update_with_zero_beta_is_pure_decay_bitwise():
    """beta = 0: S_N = alpha S_{N-1} exactly (ARL2 summary, section 2.1 state
    update; the fp32 product alpha * S, rounded once)."""
    cfg = small_config(B=2, H=3, L=150, frames=1, queries=1, seed=43)
    wl = W.Workload(cfg)
    lay, _ = make_layer(cfg, wl)
    rng = np.random.default_rng(43)
    S0 = torch.from_numpy(rng.standard_normal((2, 3, 128, 128)).astype(np.float32) * 0.1).cuda()
    lay.set_state(S0, 5)
    Q, K, V = (dev(x, "bf16") for x in wl.qkv(0, 0, 0))
    alpha = torch.from_numpy(wl.alpha(0, 0)).cuda()
    beta = torch.zeros((2, 3, 150), dtype=torch.float32, device="cuda")
    lay.commit(Q, K, V, alpha, beta)
    torch.cuda.synchronize()
    assert torch.equal(lay.state(), alpha[:, :, None, None] * S0)
    lay.close()


def test_update_with_one_unit_key_writes_its_value_bitwise():
    """One token, k = e_i through identity maps, alpha = beta = 1, c = 1, S = 0:
    the update writes V' into row i of S and nothing else, so k^T S_N = v'
    (ARL2 summary, section 2.1: K'^T diag(beta)(V' - K' S_{N-1}))."""
    H, i = 2, 37
    eye = torch.eye(128, dtype=torch.bfloat16, device="cuda").expand(H, 128, 128).contiguous()
    rng = np.random.default_rng(44)
    phi_q = dev(rng.standard_normal((H, 128, 128)).astype(np.float32) * 0.1, "bf16")
    lay = arl2.HybridLayer(1, H, 128, 1, arl2.ARL2_BF16, phi_q, eye, eye, corr_scale=1.0)
    K = torch.zeros((1, 1, H, 128), dtype=torch.bfloat16, device="cuda")
    K[0, 0, :, i] = 1.0
    V = dev(rng.standard_normal((1, 1, H, 128)).astype(np.float32), "bf16")
    Q = dev(rng.standard_normal((1, 1, H, 128)).astype(np.float32), "bf16")
    ones_a = torch.ones((1, H), dtype=torch.float32, device="cuda")
    ones_b = torch.ones((1, H, 1), dtype=torch.float32, device="cuda")
    lay.commit(Q, K, V, ones_a, ones_b)
    torch.cuda.synchronize()
    S = lay.state()
    want = torch.zeros_like(S)
    want[0, :, i, :] = V[0, 0].float()
    assert torch.equal(S, want)
    lay.close()


def test_kv_layer_strided_equals_contiguous_bitwise():
    """The KV-cache layer with Q, K, V as strided views of fused rows gives the
    same bits as with contiguous tensors, over frames that grow the cache."""
    cfg = small_config(B=2, H=2, L=150, frames=3, queries=1, seed=47)
    wl = W.Workload(cfg)
    a = arl2.KVLayer(2, 2, 128, 150, arl2.ARL2_BF16, max_frames=3)
    b = arl2.KVLayer(2, 2, 128, 150, arl2.ARL2_BF16, max_frames=3)
    D = 2 * 128
    for n in range(cfg.frames):
        for p in range(cfg.passes):
            Q, K, V = (dev(x, "bf16") for x in wl.qkv(0, n, p))
            B, L = Q.shape[:2]
            fused = torch.cat([Q.reshape(B, L, D), K.reshape(B, L, D), V.reshape(B, L, D)], dim=2).contiguous()
            o1, o2 = torch.empty_like(Q), torch.empty_like(Q)
            if p < cfg.queries:
                arl2.arl2_kv_query(a.handle, Q, K, V, o1)
                arl2.arl2_kv_query_strided(b.handle, fused, fused[..., D:], fused[..., 2 * D:], 3 * D, o2)
            else:
                arl2.arl2_kv_commit(a.handle, Q, K, V, o1)
                arl2.arl2_kv_commit_strided(b.handle, fused, fused[..., D:], fused[..., 2 * D:], 3 * D, o2)
            torch.cuda.synchronize()
            assert torch.equal(o1, o2), (n, p)
    assert a.frames == b.frames == cfg.frames
    a.close()
    b.close()
