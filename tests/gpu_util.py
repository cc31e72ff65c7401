"""Helpers of the GPU tests: upload seeded inputs, run a hybrid layer through
the C ABI, and run the oracle on the same inputs."""
from __future__ import annotations

import numpy as np
import torch

from hybrid_linear_attention_arl2_b200 import arl2
from hybrid_linear_attention_arl2_b200 import workloads as W
from oracle import arl2_oracle as o


def dev(x: np.ndarray, dtype: str):
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    t = t.to(torch.bfloat16) if dtype == "bf16" else t
    return t.cuda()


def host(t) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


def abi_dtype(dtype: str) -> int:
    return arl2.ARL2_BF16 if dtype == "bf16" else arl2.ARL2_F32


def small_config(B=1, H=2, d=128, L=300, frames=3, queries=2, dtype="bf16", corr=-1.0, seed=77, layers=1,
                 hybrid_layers=1):
    return W.Config(50 + seed % 50, f"test-B{B}H{H}L{L}", B, H, d, L, frames, queries, dtype,
                    layers=layers, hybrid_layers=hybrid_layers, corr_scale=corr, pool=0)


def make_layer(cfg: W.Config, wl: W.Workload, flags=0, layer=0):
    phi = wl.phi(layer)
    layer_obj = arl2.HybridLayer(cfg.batch, cfg.heads, cfg.head_dim, cfg.tokens, abi_dtype(cfg.dtype),
                                 *(dev(p, cfg.dtype) for p in phi), corr_scale=cfg.corr_scale, flags=flags)
    return layer_obj, phi


def run_gpu_stream(cfg: W.Config, wl: W.Workload, frames=None, flags=0, keep=lambda n, p: True, states=True):
    """Outputs {(frame, pass): np.ndarray} and states [S_1..S_F] from the GPU."""
    layer, _ = make_layer(cfg, wl, flags)
    frames = cfg.frames if frames is None else frames
    outs, S = {}, []
    for n in range(frames):
        for p in range(cfg.passes):
            Q, K, V = (dev(x, cfg.dtype) for x in wl.qkv(0, n, p))
            if p < cfg.queries:
                O = layer.query(Q, K, V)
            else:
                a = torch.from_numpy(wl.alpha(0, n)).cuda()
                b = torch.from_numpy(wl.beta(0, n)).cuda()
                O = layer.commit(Q, K, V, a, b)
            if keep(n, p):
                outs[(n, p)] = host(O)
        if states:
            S.append(host(layer.state()))
    torch.cuda.synchronize()
    err = layer.last_error()
    layer.close()
    assert err == 0, f"device error {arl2.STATUS.get(err, err)}"
    return outs, S


def run_oracle_stream(cfg: W.Config, wl: W.Workload, frames=None, keep=lambda n, p: True, rows=None):
    """The oracle on the same inputs; ``rows`` restricts the outputs to a subset of query tokens."""
    phi = wl.phi(0)
    frames = cfg.frames if frames is None else frames
    S = np.zeros((cfg.batch, cfg.heads, cfg.head_dim, cfg.head_dim))
    outs, states = {}, []
    for n in range(frames):
        for p in range(cfg.passes):
            Q, K, V = wl.qkv(0, n, p)
            if keep(n, p):
                Qs = Q if rows is None else Q[:, rows]
                outs[(n, p)] = o.frame_query(S, Qs, K, V, phi)
            if p == cfg.queries:
                S = o.state_update(S, K, V, phi, wl.alpha(0, n), wl.beta(0, n), cfg.c)
        states.append(S)
    return outs, states

