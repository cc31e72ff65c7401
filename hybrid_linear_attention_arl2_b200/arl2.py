"""Thin ctypes binding of libarl2.so (C ABI in include/arl2.h).

The functions named ``arl2_*`` mirror the C entry points one to one and only
marshal arguments: torch tensors become device pointers, a torch stream
becomes a ``cudaStream_t``.  ``HybridLayer`` and ``KVLayer`` wrap a handle
for convenience.  Every step of the hot path runs in the library's CUDA
kernels; there is no fallback -- importing works without a GPU, but any call
that needs the library raises if ``libarl2.so`` is missing.
"""
from __future__ import annotations

import ctypes
import os
import re

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libarl2.so")
HEADER = os.path.join(os.path.dirname(_HERE), "include", "arl2.h")

ARL2_F32, ARL2_BF16 = 0, 1
ARL2_INTRA_ONLY, ARL2_INTER_ONLY = 1, 2

STATUS = {
    0: "ARL2_OK", 1: "ARL2_ERR_INVALID_ARGUMENT", 2: "ARL2_ERR_UNSUPPORTED",
    3: "ARL2_ERR_OUT_OF_MEMORY", 4: "ARL2_ERR_CUDA", 5: "ARL2_ERR_TIMEOUT", 6: "ARL2_ERR_NO_DEVICE",
    7: "ARL2_ERR_SCRATCH_LIMIT",
    8: "ARL2_ERR_BOUNDS",
}
ARL2_NOALLOC_SCRATCH_BYTES = 16 << 20


class Arl2Error(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {STATUS.get(status, status)}")


class arl2_config(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int32), ("heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
        ("tokens_per_frame", ctypes.c_int32), ("dtype", ctypes.c_int32),
        ("softmax_scale", ctypes.c_float), ("corr_scale", ctypes.c_float), ("flags", ctypes.c_uint32),
    ]


_VP, _I32, _I64, _U64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_uint64
_SIGS = {
    "arl2_state_init": (_I32, [ctypes.POINTER(arl2_config), _VP, _VP, _VP, _VP, ctypes.POINTER(_VP)]),
    "arl2_frame_query": (_I32, [_VP, _VP, _VP, _VP, _VP, _VP]),
    "arl2_frame_commit": (_I32, [_VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP]),
    "arl2_frame_query_strided": (_I32, [_VP, _VP, _VP, _VP, _I64, _VP, _VP]),
    "arl2_frame_commit_strided": (_I32, [_VP, _VP, _VP, _VP, _I64, _VP, _VP, _VP, _VP]),
    "arl2_token_query": (_I32, [_VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP]),
    "arl2_token_commit": (_I32, [_VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP]),
    "arl2_state_get": (_I32, [_VP, _VP, ctypes.POINTER(_I64), _VP]),
    "arl2_state_set": (_I32, [_VP, _VP, _I64, _VP]),
    "arl2_last_error": (_I32, [_VP]),
    "arl2_state_device_bytes": (_I64, [_VP]),
    "arl2_state_set_wait_limit": (_I32, [_VP, _U64]),
    "arl2_state_destroy": (_I32, [_VP]),
    "arl2_kv_init": (_I32, [ctypes.POINTER(arl2_config), _I32, _VP, ctypes.POINTER(_VP)]),
    "arl2_kv_query": (_I32, [_VP, _VP, _VP, _VP, _VP, _VP]),
    "arl2_kv_commit": (_I32, [_VP, _VP, _VP, _VP, _VP, _VP]),
    "arl2_kv_query_strided": (_I32, [_VP, _VP, _VP, _VP, _I64, _VP, _VP]),
    "arl2_kv_commit_strided": (_I32, [_VP, _VP, _VP, _VP, _I64, _VP, _VP]),
    "arl2_kv_frames": (_I64, [_VP]),
    "arl2_kv_device_bytes": (_I64, [_VP]),
    "arl2_kv_last_error": (_I32, [_VP]),
    "arl2_kv_destroy": (_I32, [_VP]),
    "arl2_block_init": (_I32, [ctypes.POINTER(arl2_config), _VP, _VP, _VP, _VP, _VP, _VP, _VP, ctypes.POINTER(_VP)]),
    "arl2_block_query": (_I32, [_VP, _VP, _VP, _VP]),
    "arl2_block_commit": (_I32, [_VP, _VP, _VP, _VP]),
    "arl2_block_layer": (_VP, [_VP]),
    "arl2_block_destroy": (_I32, [_VP]),
    "arl2_state_write_noalloc": (_I32, [ctypes.POINTER(arl2_config), _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP,
                                        _VP]),
    "arl2_selftest_wait_timeout": (_I32, [_U64, _VP]),
    "arl2_selftest_exp2": (_I32, [_VP, _VP, _I64, _VP]),
    "arl2_gemm_bf16": (_I32, [_VP, _I64, _VP, _I64, _VP, _I64, _I64, _I64, _I64, _VP]),
    "arl2_attn_partition": (_I32, [_I32, _I32, _I32, _I32, _I32, _VP, _I32, _VP, _VP, _VP]),
    "arl2_status_string": (ctypes.c_char_p, [_I32]),
    "arl2_abi_version": (_I32, []),
    "arl2_debug_bounds_enabled": (_I32, []),
}

_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libarl2.so; raise if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"libarl2.so not built at {path}; run python -m hybrid_linear_attention_arl2_b200.build")
    lib = ctypes.CDLL(path)
    for name, (res, args) in _SIGS.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def declared_symbols(header: str = HEADER) -> list[str]:
    """Entry points declared in include/arl2.h."""
    text = open(header).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(arl2_[a-z0-9_]+)\s*\(", text)))


# ---------------------------------------------------------------- marshalling
def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(status: int, what: str) -> None:
    if status != 0:
        raise Arl2Error(status, what)


def make_config(batch, heads, head_dim, tokens, dtype, softmax_scale=0.0, corr_scale=-1.0, flags=0):
    return arl2_config(batch, heads, head_dim, tokens, dtype, softmax_scale, corr_scale, flags)


# ---------------------------------------------------------------- C entry points
def arl2_state_init(cfg: arl2_config, phi_q, phi_k, phi_v, stream=None) -> int:
    h = _VP()
    _check(load_library().arl2_state_init(ctypes.byref(cfg), _ptr(phi_q), _ptr(phi_k), _ptr(phi_v),
                                          _stream(stream), ctypes.byref(h)), "arl2_state_init")
    return h.value


def arl2_frame_query(h, q, k, v, o, stream=None) -> None:
    _check(load_library().arl2_frame_query(h, _ptr(q), _ptr(k), _ptr(v), _ptr(o), _stream(stream)),
           "arl2_frame_query")


def arl2_frame_commit(h, q, k, v, alpha, beta, o, stream=None) -> None:
    _check(load_library().arl2_frame_commit(h, _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), _ptr(o),
                                            _stream(stream)), "arl2_frame_commit")


def arl2_frame_query_strided(h, q, k, v, ld, o, stream=None) -> None:
    _check(load_library().arl2_frame_query_strided(h, _ptr(q), _ptr(k), _ptr(v), int(ld), _ptr(o), _stream(stream)),
           "arl2_frame_query_strided")


def arl2_frame_commit_strided(h, q, k, v, ld, alpha, beta, o, stream=None) -> None:
    _check(load_library().arl2_frame_commit_strided(h, _ptr(q), _ptr(k), _ptr(v), int(ld), _ptr(alpha), _ptr(beta),
                                                    _ptr(o), _stream(stream)), "arl2_frame_commit_strided")


def arl2_token_query(h, q, k, v, alpha_tok, beta, o, stream=None) -> None:
    _check(load_library().arl2_token_query(h, _ptr(q), _ptr(k), _ptr(v), _ptr(alpha_tok), _ptr(beta), _ptr(o),
                                           _stream(stream)), "arl2_token_query")


def arl2_token_commit(h, q, k, v, alpha_tok, beta, o, stream=None) -> None:
    _check(load_library().arl2_token_commit(h, _ptr(q), _ptr(k), _ptr(v), _ptr(alpha_tok), _ptr(beta), _ptr(o),
                                            _stream(stream)), "arl2_token_commit")


def arl2_state_get(h, dst, stream=None) -> int:
    frame = _I64()
    _check(load_library().arl2_state_get(h, _ptr(dst), ctypes.byref(frame), _stream(stream)), "arl2_state_get")
    return frame.value


def arl2_state_set(h, src, frame: int, stream=None) -> None:
    _check(load_library().arl2_state_set(h, _ptr(src), frame, _stream(stream)), "arl2_state_set")


def arl2_last_error(h) -> int:
    return load_library().arl2_last_error(h)


def arl2_state_device_bytes(h) -> int:
    return load_library().arl2_state_device_bytes(h)


def arl2_state_set_wait_limit(h, limit_ns: int) -> None:
    _check(load_library().arl2_state_set_wait_limit(h, limit_ns), "arl2_state_set_wait_limit")


def arl2_state_destroy(h) -> None:
    _check(load_library().arl2_state_destroy(h), "arl2_state_destroy")


def arl2_kv_init(cfg: arl2_config, max_frames: int, stream=None) -> int:
    h = _VP()
    _check(load_library().arl2_kv_init(ctypes.byref(cfg), max_frames, _stream(stream), ctypes.byref(h)),
           "arl2_kv_init")
    return h.value


def arl2_kv_query(h, q, k, v, o, stream=None) -> None:
    _check(load_library().arl2_kv_query(h, _ptr(q), _ptr(k), _ptr(v), _ptr(o), _stream(stream)), "arl2_kv_query")


def arl2_kv_commit(h, q, k, v, o, stream=None) -> None:
    _check(load_library().arl2_kv_commit(h, _ptr(q), _ptr(k), _ptr(v), _ptr(o), _stream(stream)), "arl2_kv_commit")


def arl2_kv_frames(h) -> int:
    return load_library().arl2_kv_frames(h)


def arl2_kv_device_bytes(h) -> int:
    return load_library().arl2_kv_device_bytes(h)


def arl2_kv_last_error(h) -> int:
    return load_library().arl2_kv_last_error(h)


def arl2_kv_query_strided(h, q, k, v, ld, o, stream=None) -> None:
    _check(load_library().arl2_kv_query_strided(h, _ptr(q), _ptr(k), _ptr(v), int(ld), _ptr(o), _stream(stream)),
           "arl2_kv_query_strided")


def arl2_kv_commit_strided(h, q, k, v, ld, o, stream=None) -> None:
    _check(load_library().arl2_kv_commit_strided(h, _ptr(q), _ptr(k), _ptr(v), int(ld), _ptr(o), _stream(stream)),
           "arl2_kv_commit_strided")


def arl2_kv_destroy(h) -> None:
    _check(load_library().arl2_kv_destroy(h), "arl2_kv_destroy")


def arl2_block_init(cfg: arl2_config, w_qkv, w_o, w_gate, phi_q, phi_k, phi_v, stream=None) -> int:
    h = _VP()
    _check(load_library().arl2_block_init(ctypes.byref(cfg), _ptr(w_qkv), _ptr(w_o), _ptr(w_gate), _ptr(phi_q),
                                          _ptr(phi_k), _ptr(phi_v), _stream(stream), ctypes.byref(h)),
           "arl2_block_init")
    return h.value


def arl2_block_query(h, x, y, stream=None) -> None:
    _check(load_library().arl2_block_query(h, _ptr(x), _ptr(y), _stream(stream)), "arl2_block_query")


def arl2_block_commit(h, x, y, stream=None) -> None:
    _check(load_library().arl2_block_commit(h, _ptr(x), _ptr(y), _stream(stream)), "arl2_block_commit")


def arl2_block_layer(h) -> int | None:
    return load_library().arl2_block_layer(h)


def arl2_block_destroy(h) -> None:
    _check(load_library().arl2_block_destroy(h), "arl2_block_destroy")


def arl2_state_write_noalloc(cfg: arl2_config, k, v, phi_k, phi_v, S_prev, alpha, beta, S_next, dev_error,
                             stream=None) -> None:
    """One frame's state write with no handle and no device allocation (its
    work space is the library's static scratch array); ``dev_error`` is a
    device uint32 that a kernel's timed-out wait sets."""
    _check(load_library().arl2_state_write_noalloc(ctypes.byref(cfg), _ptr(k), _ptr(v), _ptr(phi_k), _ptr(phi_v),
                                                   _ptr(S_prev), _ptr(alpha), _ptr(beta), _ptr(S_next),
                                                   _ptr(dev_error), _stream(stream)), "arl2_state_write_noalloc")


def arl2_selftest_wait_timeout(limit_ns: int, stream=None) -> int:
    return load_library().arl2_selftest_wait_timeout(limit_ns, _stream(stream))


def arl2_gemm_bf16(a, b, c, m, n, k, lda=None, ldb=None, ldc=None, stream=None) -> None:
    """C[m, n] = A[m, k] B[k, n] on bf16 device tensors (row-major; leading
    dimensions default to k, n and n)."""
    _check(load_library().arl2_gemm_bf16(_ptr(a), lda or k, _ptr(b), ldb or n, _ptr(c), ldc or n, m, n, k,
                                         _stream(stream)), "arl2_gemm_bf16")


def arl2_attn_partition(batch, heads, q_len, kv_len, pairs, max_segs=1024):
    """The attention kernel's work partition (host only): a list per pair of
    segments (slab, block, j0, j1, n_contrib)."""
    segs = (ctypes.c_int32 * (5 * max_segs))()
    first = (ctypes.c_int32 * 97)()
    n_segs, n_pairs = ctypes.c_int(0), ctypes.c_int(0)
    _check(load_library().arl2_attn_partition(batch, heads, q_len, kv_len, pairs, ctypes.cast(segs, ctypes.c_void_p).value,
                                              max_segs, ctypes.cast(first, ctypes.c_void_p).value,
                                              ctypes.addressof(n_segs), ctypes.addressof(n_pairs)), "arl2_attn_partition")
    out = []
    for c in range(n_pairs.value):
        out.append([tuple(segs[5 * i:5 * i + 5]) for i in range(first[c], first[c + 1])])
    return out


def arl2_selftest_exp2(x, y, stream=None) -> None:
    _check(load_library().arl2_selftest_exp2(_ptr(x), _ptr(y), x.numel(), _stream(stream)), "arl2_selftest_exp2")


def arl2_status_string(status: int) -> str:
    return load_library().arl2_status_string(status).decode()


def arl2_abi_version() -> int:
    return load_library().arl2_abi_version()


def arl2_debug_bounds_enabled() -> bool:
    """Whether the loaded library is the debug build (index checks in its kernels)."""
    return bool(load_library().arl2_debug_bounds_enabled())


# ---------------------------------------------------------------- convenience wrappers
def _torch_dtype(dtype: int):
    import torch
    return torch.float32 if dtype == ARL2_F32 else torch.bfloat16


class HybridLayer:
    """One ARL2 hybrid attention layer over B streams (a handle of the C ABI)."""

    def __init__(self, batch, heads, head_dim, tokens, dtype, phi_q, phi_k, phi_v, *,
                 softmax_scale=0.0, corr_scale=-1.0, flags=0, stream=None):
        self.cfg = make_config(batch, heads, head_dim, tokens, dtype, softmax_scale, corr_scale, flags)
        self.handle = arl2_state_init(self.cfg, phi_q, phi_k, phi_v, stream)

    @property
    def out_shape(self):
        c = self.cfg
        return (c.batch, c.tokens_per_frame, c.heads, c.head_dim)

    def _out(self, like):
        import torch
        return torch.empty(self.out_shape, dtype=_torch_dtype(self.cfg.dtype), device=like.device)

    def query(self, q, k, v, o=None, stream=None):
        o = self._out(q) if o is None else o
        arl2_frame_query(self.handle, q, k, v, o, stream)
        return o

    def commit(self, q, k, v, alpha, beta, o=None, stream=None):
        o = self._out(q) if o is None else o
        arl2_frame_commit(self.handle, q, k, v, alpha, beta, o, stream)
        return o

    def token_query(self, q, k, v, alpha_tok, beta, o=None, stream=None):
        """Token-level access: token t reads the state the earlier tokens of
        this pass left; the handle's state is not written."""
        o = self._out(q) if o is None else o
        arl2_token_query(self.handle, q, k, v, alpha_tok, beta, o, stream)
        return o

    def token_commit(self, q, k, v, alpha_tok, beta, o=None, stream=None):
        """Token-level access on the clean pass: the state after the frame's
        last token becomes the handle's state."""
        o = self._out(q) if o is None else o
        arl2_token_commit(self.handle, q, k, v, alpha_tok, beta, o, stream)
        return o

    def state(self, stream=None):
        import torch
        c = self.cfg
        dst = torch.empty((c.batch, c.heads, c.head_dim, c.head_dim), dtype=torch.float32, device="cuda")
        arl2_state_get(self.handle, dst, stream)
        return dst

    @property
    def frame(self) -> int:
        return arl2_state_get(self.handle, None)

    def set_state(self, S, frame: int, stream=None):
        arl2_state_set(self.handle, S, frame, stream)

    def last_error(self) -> int:
        return arl2_last_error(self.handle)

    def device_bytes(self) -> int:
        return arl2_state_device_bytes(self.handle)

    def close(self):
        if self.handle:
            arl2_state_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class KVLayer:
    """A softmax layer with a growing per-frame KV cache (a handle of the C ABI)."""

    def __init__(self, batch, heads, head_dim, tokens, dtype, max_frames, *, softmax_scale=0.0, stream=None):
        self.cfg = make_config(batch, heads, head_dim, tokens, dtype, softmax_scale, -1.0, 0)
        self.handle = arl2_kv_init(self.cfg, max_frames, stream)

    def _out(self, like):
        import torch
        c = self.cfg
        return torch.empty((c.batch, c.tokens_per_frame, c.heads, c.head_dim), dtype=_torch_dtype(c.dtype),
                           device=like.device)

    def query(self, q, k, v, o=None, stream=None):
        o = self._out(q) if o is None else o
        arl2_kv_query(self.handle, q, k, v, o, stream)
        return o

    def commit(self, q, k, v, o=None, stream=None):
        o = self._out(q) if o is None else o
        arl2_kv_commit(self.handle, q, k, v, o, stream)
        return o

    @property
    def frames(self) -> int:
        return arl2_kv_frames(self.handle)

    def last_error(self) -> int:
        return arl2_kv_last_error(self.handle)

    def device_bytes(self) -> int:
        return arl2_kv_device_bytes(self.handle)

    def close(self):
        if self.handle:
            arl2_kv_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class HybridBlock:
    """A hybrid attention block: X W_qkv -> hybrid layer -> O W_o, with the
    commit's gates from X W_gate (a handle of the C ABI; bf16, head_dim 128)."""

    def __init__(self, batch, heads, tokens, w_qkv, w_o, w_gate, phi_q, phi_k, phi_v, *, softmax_scale=0.0,
                 corr_scale=-1.0, stream=None):
        self.cfg = make_config(batch, heads, 128, tokens, ARL2_BF16, softmax_scale, corr_scale, 0)
        self.handle = arl2_block_init(self.cfg, w_qkv, w_o, w_gate, phi_q, phi_k, phi_v, stream)

    def _out(self, like):
        import torch
        return torch.empty_like(like)

    def query(self, x, y=None, stream=None):
        y = self._out(x) if y is None else y
        arl2_block_query(self.handle, x, y, stream)
        return y

    def commit(self, x, y=None, stream=None):
        y = self._out(x) if y is None else y
        arl2_block_commit(self.handle, x, y, stream)
        return y

    def state(self, stream=None):
        import torch
        c = self.cfg
        dst = torch.empty((c.batch, c.heads, c.head_dim, c.head_dim), dtype=torch.float32, device="cuda")
        arl2_state_get(arl2_block_layer(self.handle), dst, stream)
        return dst

    def last_error(self) -> int:
        return arl2_last_error(arl2_block_layer(self.handle))

    def close(self):
        if self.handle:
            arl2_block_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
