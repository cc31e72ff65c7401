"""Seeded input generators: rounding, determinism, shapes and distributions."""
import numpy as np
import torch

from hybrid_linear_attention_arl2_b200 import workloads as W


def test_round_bf16_matches_torch_rne():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(100000).astype(np.float32) * 10,
                        np.array([1.00390625, 1.01171875, -1.00390625, 0.0, -0.0, 65504.0],
                                 dtype=np.float32)])
    ours = W.round_bf16(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float32).numpy()
    assert np.array_equal(ours.view(np.uint32), ref.view(np.uint32))
    # ties go to even: 1 + 2^-8 lies halfway between 1 and 1 + 2^-7
    assert W.round_bf16(np.float32([1.00390625]))[0] == 1.0
    assert W.round_bf16(np.float32([1.01171875]))[0] == np.float32(1.015625)


def test_bits_round_trip():
    x = W.round_bf16(np.random.default_rng(1).standard_normal(1000).astype(np.float32))
    assert np.array_equal(W.bits_to_f32(W.bf16_bits(x)), x)


def test_deterministic_and_frame_addressable():
    w1, w2 = W.Workload(0), W.Workload(0)
    a = w1.qkv(0, 3, 2)
    b = w2.qkv(0, 3, 2)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)
    c = w1.qkv(0, 3, 1)
    assert not np.array_equal(a[0], c[0])
    assert np.array_equal(w1.alpha(0, 5), w2.alpha(0, 5))
    assert np.array_equal(w1.beta(0, 5), w2.beta(0, 5))


def test_shapes_and_ranges():
    cfg = W.CONFIGS[0]
    w = W.Workload(cfg)
    Q, K, V = w.qkv(0, 0, 0)
    assert Q.shape == (cfg.batch, cfg.tokens, cfg.heads, cfg.head_dim)
    pq, pk, pv = w.phi(0)
    assert pq.shape == (cfg.heads, cfg.head_dim, cfg.head_dim)
    a, b = w.alpha(0, 0), w.beta(0, 0)
    assert a.shape == (cfg.batch, cfg.heads) and b.shape == (cfg.batch, cfg.heads, cfg.tokens)
    assert np.all((a > 0) & (a < 1)) and np.all((b > 0) & (b < 1))


def test_distributions():
    cfg = W.Config(9, "moments", 1, 4, 64, 4096, 1, 0, "bf16", pool=0)
    w = W.Workload(cfg)
    Q, _, _ = w.qkv(0, 0, 0)
    assert abs(Q.mean()) < 0.01 and abs(Q.std() - 1.0) < 0.01
    pq, _, _ = w.phi(0)
    off = pq - np.eye(64)[None]
    assert abs(off.var() - 1.0 / 64) < 1e-3
    # alpha = sigmoid(N(2, 0.5)): median sigmoid(2)
    alphas = np.concatenate([W.Workload(cfg, seed=s).alpha(0, f).ravel()
                             for s in range(20) for f in range(20)])
    assert abs(np.median(alphas) - 1 / (1 + np.exp(-2))) < 0.02
    assert W.bf16_bits(Q).dtype == np.uint16  # bf16 configs store exactly representable values


def test_pool_cycles_without_short_reuse():
    cfg = W.CONFIGS[1]
    w = W.Workload(cfg)
    idx = [w.pool_index(0, f, p) for f in range(4) for p in range(cfg.passes)]
    assert idx == [i % cfg.pool for i in range(len(idx))]
