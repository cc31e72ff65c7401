"""Seeded synthetic inputs for the ARL2 hybrid-attention hot path.

This module draws random numbers and rounds them to the storage precision;
it holds none of the method's arithmetic.  Both the CPU oracle (through the
tests and the benchmark) and the CUDA path read the arrays it produces.

Distributions (stated once, read as N(mean, variance)):

* Q, K, V ~ N(0, 1), per (stream, token, head, channel);
* phi_q, phi_k, phi_v = I + N(0, 1/d), one d x d matrix per head, shared by
  the streams of a layer;
* alpha = sigmoid(N(2, 0.5)), one value per (stream, head, frame);
* beta  = sigmoid(N(0, 1)), one value per (stream, head, token) of a commit;
* S_0 = 0.

bf16 workloads round every draw to bf16 with round-to-nearest-even, written
here as integer bit arithmetic so that the rounding does not depend on any
library's conversion routine.  The arrays stay float32 (each value exactly
representable in bf16); ``bf16_bits`` gives the 16-bit patterns to upload.

Frame inputs are a pure function of (layer, frame, pass), so any frame of any
stream can be regenerated on its own.  Large workloads draw a fixed pool of
(Q, K, V) triples per stream once and cycle through it in a fixed order, so
that consecutive steps touch different memory (the pool is larger than the
126 MB L2 of a B200 at the 1560-token shapes).
"""
from __future__ import annotations

import dataclasses
import numpy as np

__all__ = [
    "CONFIGS", "Config", "round_bf16", "bf16_bits", "bits_to_f32", "Workload",
    "splitmix64",
]

_MASK64 = (1 << 64) - 1


def splitmix64(*words: int) -> int:
    """Counter-based 64-bit mixer (Steele, Lea and Flood's SplitMix64 finaliser),
    folded over the given words; used to derive independent seeds."""
    z = 0x9E3779B97F4A7C15
    for w in words:
        z = (z + (int(w) & _MASK64) + 0x9E3779B97F4A7C15) & _MASK64
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _MASK64
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _MASK64
        z = z ^ (z >> 31)
    return z


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even); returns float32."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    r = (u + np.uint64(0x7FFF) + lsb) & np.uint64(0xFFFF0000)
    return r.astype(np.uint32).view(np.float32).reshape(x.shape)


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """16-bit patterns of float32 values that are already bf16-representable."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32)
    if np.any(u & np.uint32(0xFFFF)):
        raise ValueError("bf16_bits: values are not bf16-representable; call round_bf16 first")
    return (u >> np.uint32(16)).astype(np.uint16).reshape(x.shape)


def bits_to_f32(b: np.ndarray) -> np.ndarray:
    """float32 values of 16-bit bf16 patterns."""
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32).reshape(b.shape)


@dataclasses.dataclass(frozen=True)
class Config:
    """One workload: shapes, precision and stream length."""
    index: int
    name: str
    batch: int             # independent streams B
    heads: int             # H
    head_dim: int          # d
    tokens: int            # L, tokens per frame
    frames: int
    queries: int           # query-only denoising steps per frame
    dtype: str             # "f32" or "bf16"
    layers: int = 1
    hybrid_layers: int = 1  # layers [0, hybrid_layers) are hybrid, the rest softmax + KV cache
    corr_scale: float = 1.0  # coefficient c of the delta correction; < 0 means 1/L
    pool: int = 0           # 0: draw every frame; > 0: cycle through a pool of this many triples

    @property
    def passes(self) -> int:
        return self.queries + 1

    @property
    def c(self) -> float:
        return 1.0 / self.tokens if self.corr_scale < 0 else float(self.corr_scale)

    @property
    def seed(self) -> int:
        return 1000 * self.index


CONFIGS = {
    0: Config(0, "tiny-fp32-stream", 1, 2, 32, 16, 8, 4, "f32", corr_scale=1.0),
    1: Config(1, "single-hybrid-layer-bf16", 1, 12, 128, 1560, 21, 4, "bf16",
              corr_scale=-1.0, pool=20),
    2: Config(2, "long-stream-bf16", 1, 12, 128, 1560, 231, 4, "bf16",
              corr_scale=-1.0, pool=20),
    3: Config(3, "attention-stack-bf16", 1, 12, 128, 1560, 63, 4, "bf16",
              layers=30, hybrid_layers=22, corr_scale=-1.0, pool=20),
    4: Config(4, "batched-streams-bf16", 4, 12, 128, 1560, 81, 4, "bf16",
              corr_scale=-1.0, pool=10),
}


def _rng(*words: int) -> np.random.Generator:
    return np.random.default_rng(splitmix64(*words))


def _sigmoid(x: np.ndarray) -> np.ndarray:
    return (1.0 / (1.0 + np.exp(-x.astype(np.float64)))).astype(np.float32)


class Workload:
    """Seeded inputs of one configuration.

    Every accessor returns float32 arrays whose values are exactly
    representable in the configuration's storage type; layouts follow the
    C ABI: Q/K/V [B, L, H, d] token-major, phi [H, d, d] with
    Q' = Q @ phi, alpha [B, H], beta [B, H, L].
    """

    _PHI, _GATE_A, _GATE_B, _QKV, _POOL, _WBLK, _XBLK, _GATE_T = 1, 2, 3, 4, 5, 6, 7, 8

    def __init__(self, cfg: Config | int, *, seed: int | None = None):
        self.cfg = CONFIGS[cfg] if isinstance(cfg, int) else cfg
        self.seed = self.cfg.seed if seed is None else int(seed)
        self._pool: dict[tuple[int, int], tuple[np.ndarray, ...]] = {}

    # -- storage rounding -------------------------------------------------
    def _store(self, x: np.ndarray) -> np.ndarray:
        x = np.ascontiguousarray(x, dtype=np.float32)
        return round_bf16(x) if self.cfg.dtype == "bf16" else x

    # -- per-layer parameters ---------------------------------------------
    def phi(self, layer: int = 0):
        c = self.cfg
        rng = _rng(self.seed, self._PHI, layer)
        eye = np.eye(c.head_dim, dtype=np.float32)
        out = []
        for _ in range(3):
            w = rng.standard_normal((c.heads, c.head_dim, c.head_dim), dtype=np.float32)
            out.append(self._store(eye[None] + w * np.float32(1.0 / np.sqrt(c.head_dim))))
        return tuple(out)  # phi_q, phi_k, phi_v

    # -- per-frame gates ----------------------------------------------------
    def alpha(self, layer: int, frame: int) -> np.ndarray:
        c = self.cfg
        rows = []
        for b in range(c.batch):
            rng = _rng(self.seed + b, self._GATE_A, layer, frame)
            rows.append(_sigmoid(2.0 + np.sqrt(0.5) * rng.standard_normal(c.heads)))
        return np.stack(rows).astype(np.float32)

    def beta(self, layer: int, frame: int) -> np.ndarray:
        c = self.cfg
        rows = []
        for b in range(c.batch):
            rng = _rng(self.seed + b, self._GATE_B, layer, frame)
            rows.append(_sigmoid(rng.standard_normal((c.heads, c.tokens))))
        return np.stack(rows).astype(np.float32)

    def alpha_tok(self, layer: int, frame: int) -> np.ndarray:
        """Per-token decays [B, H, L] for token-level passes: sigmoid(N(4, 0.5)),
        about 0.98, so that a 128-token chunk keeps a tenth of its entering state."""
        c = self.cfg
        rows = []
        for b in range(c.batch):
            rng = _rng(self.seed + b, self._GATE_T, layer, frame)
            rows.append(_sigmoid(4.0 + np.sqrt(0.5) * rng.standard_normal((c.heads, c.tokens))))
        return np.stack(rows).astype(np.float32)

    # -- per-pass activations -----------------------------------------------
    def pool_index(self, layer: int, frame: int, pas: int) -> int:
        c = self.cfg
        return ((frame * c.layers + layer) * c.passes + pas) % c.pool

    def _draw_triple(self, *words: int):
        c = self.cfg
        rng = _rng(*words)
        shape = (c.tokens, c.heads, c.head_dim)
        return tuple(self._store(rng.standard_normal(shape, dtype=np.float32)) for _ in range(3))

    def pool_entry(self, stream: int, idx: int):
        """(Q, K, V) of one stream, each [L, H, d], from the stream's pool."""
        key = (stream, idx)
        if key not in self._pool:
            self._pool[key] = self._draw_triple(self.seed + stream, self._POOL, idx)
        return self._pool[key]

    def qkv(self, layer: int, frame: int, pas: int):
        """(Q, K, V), each [B, L, H, d], for one pass (pas == queries is the commit)."""
        c = self.cfg
        per_stream = []
        for b in range(c.batch):
            if c.pool:
                per_stream.append(self.pool_entry(b, self.pool_index(layer, frame, pas)))
            else:
                per_stream.append(self._draw_triple(self.seed + b, self._QKV, layer, frame, pas))
        return tuple(np.stack([t[i] for t in per_stream]) for i in range(3))

    # -- hybrid attention block (projections around the layer) ---------------
    def block_weights(self, layer: int = 0):
        """(W_qkv [D, 3D], W_o [D, D], W_gate [D, 2H]) of one block, D = H * d,
        entries N(0, 1/D): unit-variance tokens give unit-variance Q, K, V."""
        c = self.cfg
        D = c.heads * c.head_dim
        rng = _rng(self.seed, self._WBLK, layer)
        s = np.float32(1.0 / np.sqrt(D))
        w_qkv = self._store(rng.standard_normal((D, 3 * D), dtype=np.float32) * s)
        w_o = self._store(rng.standard_normal((D, D), dtype=np.float32) * s)
        w_gate = self._store(rng.standard_normal((D, 2 * c.heads), dtype=np.float32) * s)
        return w_qkv, w_o, w_gate

    def _draw_x(self, *words: int) -> np.ndarray:
        c = self.cfg
        rng = _rng(*words)
        return self._store(rng.standard_normal((c.tokens, c.heads * c.head_dim), dtype=np.float32))

    def block_input(self, layer: int, frame: int, pas: int) -> np.ndarray:
        """X [B, L, D] of one pass of a block: N(0, 1) tokens (pool entries, as
        for Q/K/V, when the configuration has a pool)."""
        c = self.cfg
        rows = []
        for b in range(c.batch):
            if c.pool:
                key = ("x", b, self.pool_index(layer, frame, pas))
                if key not in self._pool:
                    self._pool[key] = self._draw_x(self.seed + b, self._XBLK, key[2])
                rows.append(self._pool[key])
            else:
                rows.append(self._draw_x(self.seed + b, self._XBLK, layer, frame, pas))
        return np.stack(rows)
