"""The C-ABI library without a GPU: it loads, exports every entry point that
include/arl2.h declares, and rejects bad arguments on the host before any
CUDA call."""
import ctypes

import pytest

from hybrid_linear_attention_arl2_b200 import arl2, build


@pytest.fixture(scope="module")
def lib():
    build.build()
    return arl2.load_library()


def test_exports_every_declared_symbol(lib):
    names = arl2.declared_symbols()
    assert len(names) >= 19
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, missing
    assert set(names) == set(arl2._SIGS), "binding and header disagree"


def test_status_strings_and_version(lib):
    assert arl2.arl2_abi_version() == 1
    for s, name in arl2.STATUS.items():
        assert arl2.arl2_status_string(s)
    assert arl2.arl2_status_string(99) == "unknown status"


def _init(cfg, phis=(16, 16, 16)):
    h = ctypes.c_void_p()
    return arl2.load_library().arl2_state_init(ctypes.byref(cfg) if cfg is not None else None,
                                               *phis, None, ctypes.byref(h))


def test_host_validation_of_config(lib):
    ok = arl2.make_config(1, 2, 128, 64, arl2.ARL2_BF16)
    assert _init(None) == 1
    assert arl2.load_library().arl2_state_init(ctypes.byref(ok), 16, 16, 16, None, None) == 1  # null out
    assert _init(arl2.make_config(0, 2, 128, 64, arl2.ARL2_BF16)) == 1
    assert _init(arl2.make_config(1, 2, 128, 0, arl2.ARL2_BF16)) == 1
    assert _init(arl2.make_config(1, 2, 64, 64, arl2.ARL2_BF16)) == 2       # bf16 needs d = 128
    assert _init(arl2.make_config(1, 2, 256, 64, arl2.ARL2_F32)) == 2       # f32 d <= 128
    assert _init(arl2.make_config(1, 2, 32, 5000, arl2.ARL2_F32)) == 2      # f32 L <= 4096
    assert _init(arl2.make_config(1, 2, 128, 64, 7)) == 2                   # unknown dtype
    assert _init(arl2.make_config(1, 2, 128, 64, arl2.ARL2_BF16, flags=3)) == 1
    assert _init(arl2.make_config(1, 2, 128, 64, arl2.ARL2_BF16, softmax_scale=-1.0)) == 1
    assert _init(ok, phis=(None, 16, 16)) == 1                              # null phi
    assert _init(ok, phis=(17, 16, 16)) == 1                                # misaligned phi


def test_foreign_handles_rejected(lib):
    L = arl2.load_library()
    bogus = ctypes.c_void_p(0x1000)
    assert L.arl2_frame_query(bogus, 16, 16, 16, 16, None) == 1
    assert L.arl2_frame_commit(None, 16, 16, 16, 16, 16, 16, None) == 1
    assert L.arl2_state_destroy(bogus) == 1
    assert L.arl2_state_device_bytes(bogus) == -1
    assert L.arl2_kv_query(bogus, 16, 16, 16, 16, None) == 1
    assert L.arl2_kv_frames(bogus) == -1
    assert L.arl2_selftest_wait_timeout(0, None) == 1


def test_kv_validation(lib):
    L = arl2.load_library()
    h = ctypes.c_void_p()
    cfg = arl2.make_config(1, 2, 128, 64, arl2.ARL2_BF16)
    assert L.arl2_kv_init(ctypes.byref(cfg), 0, None, ctypes.byref(h)) == 1
    assert L.arl2_kv_init(None, 4, None, ctypes.byref(h)) == 1


def test_noalloc_state_write_host_checks(lib):
    """The allocation-free state write rejects, before any CUDA call, what it
    cannot run: a float32 config, null or misaligned pointers, an output
    (S_next or the error word) that shares a byte with an input or with the
    other output, and sizes whose work space exceeds its fixed static array."""
    L = arl2.load_library()
    G = 1 << 30  # fake, never dereferenced addresses 1 GiB apart
    # k, v, phi_k, phi_v, S_prev, alpha, beta, S_next, dev_error
    ptrs = [1 * G, 2 * G, 3 * G, 4 * G, 5 * G, 6 * G, 7 * G, 8 * G, 9 * G]
    call = lambda cfg, p=ptrs: L.arl2_state_write_noalloc(ctypes.byref(cfg), *p, None)
    assert call(arl2.make_config(1, 2, 32, 16, arl2.ARL2_F32)) == 2
    assert call(arl2.make_config(1, 2, 64, 16, arl2.ARL2_BF16)) == 2
    bad = list(ptrs)
    bad[0] = None
    assert call(arl2.make_config(1, 2, 128, 16, arl2.ARL2_BF16), bad) == 1
    bad[0] = 17
    assert call(arl2.make_config(1, 2, 128, 16, arl2.ARL2_BF16), bad) == 1
    small = arl2.make_config(1, 2, 128, 16, arl2.ARL2_BF16)  # k, v: 8 KiB; states 128 KiB; beta 128 B
    for out, target, offset in [(7, 4, 0),            # S_next over S_prev
                                (7, 0, 8192 - 16),    # S_next starts inside the last 16 bytes of k
                                (7, 1, -128 * 1024 + 16),  # S_next ends inside v
                                (7, 5, 0), (7, 6, 64),     # over alpha, over beta
                                (7, 2, 4096),              # over phi_k
                                (8, 0, 4096), (8, 6, 0),   # the error word inside k, inside beta
                                (8, 7, 1024)]:             # the error word inside S_next
        bad = list(ptrs)
        bad[out] = ptrs[target] + offset
        assert call(small, bad) == 1, (out, target, offset)
    assert call(arl2.make_config(4, 12, 128, 1560, arl2.ARL2_BF16)) == 7    # 4 streams x 1560 tokens
    assert arl2.arl2_status_string(7).startswith("sizes exceed")


def test_block_host_validation(lib):
    """The block's argument checks run before any CUDA call."""
    ok = arl2.make_config(1, 2, 128, 64, arl2.ARL2_BF16)
    h = ctypes.c_void_p()
    w = 16  # any 16-byte-aligned non-null address: rejected before use
    assert lib.arl2_block_init(ctypes.byref(ok), w, w, w, w, w, w, None, None) == 1      # no out pointer
    assert lib.arl2_block_init(ctypes.byref(ok), None, w, w, w, w, w, None, ctypes.byref(h)) == 1
    assert lib.arl2_block_init(ctypes.byref(ok), 17, w, w, w, w, w, None, ctypes.byref(h)) == 1  # misaligned
    f32 = arl2.make_config(1, 2, 128, 64, arl2.ARL2_F32)
    assert lib.arl2_block_init(ctypes.byref(f32), w, w, w, w, w, w, None, ctypes.byref(h)) == 2
    d64 = arl2.make_config(1, 2, 64, 64, arl2.ARL2_BF16)
    assert lib.arl2_block_init(ctypes.byref(d64), w, w, w, w, w, w, None, ctypes.byref(h)) == 2
    assert lib.arl2_block_query(None, w, w, None) == 1
    assert lib.arl2_block_commit(12345, w, w, None) == 1
    assert lib.arl2_block_destroy(None) == 1
    assert lib.arl2_block_layer(None) is None


def test_strided_calls_host_validation(lib):
    assert lib.arl2_frame_query_strided(None, 16, 16, 16, 0, 32, None) == 1
    assert lib.arl2_frame_commit_strided(None, 16, 16, 16, 384, 16, 16, 32, None) == 1
    assert lib.arl2_frame_query_strided(12345, 16, 16, 16, -8, 32, None) == 1


def test_kv_strided_calls_host_validation(lib):
    assert lib.arl2_kv_query_strided(None, 16, 16, 16, 0, 32, None) == 1
    assert lib.arl2_kv_commit_strided(12345, 16, 16, 16, 768, 32, None) == 1


def test_token_level_calls_host_validation(lib):
    # a null or unknown handle is rejected before any CUDA call
    assert lib.arl2_token_query(None, 16, 16, 16, 16, 16, 32, None) == 1
    assert lib.arl2_token_commit(None, 16, 16, 16, 16, 16, 32, None) == 1
    assert lib.arl2_token_commit(12345, 16, 16, 16, 16, 16, 32, None) == 1


def test_gemm_host_validation(lib):
    """The projection GEMM rejects bad pointers, sizes and leading dimensions
    before any CUDA call; an empty product returns at once."""
    a, b, c = 1 << 20, 2 << 20, 3 << 20   # 16-byte-aligned, disjoint fake addresses, never dereferenced
    g = lib.arl2_gemm_bf16
    assert g(None, 64, b, 64, c, 64, 32, 64, 64, None) == 1
    assert g(a, 64, b, 64, None, 64, 32, 64, 64, None) == 1
    assert g(a + 8, 64, b, 64, c, 64, 32, 64, 64, None) == 1          # misaligned A
    assert g(a, 64, b, 64, c, 64, -1, 64, 64, None) == 1              # negative size
    assert g(a, 32, b, 64, c, 64, 32, 64, 64, None) == 1              # lda < k
    assert g(a, 64, b, 32, c, 64, 32, 64, 64, None) == 1              # ldb < n
    assert g(a, 64, b, 64, c, 60, 32, 64, 64, None) == 1              # ldc < n
    assert g(a, 68, b, 64, c, 64, 32, 64, 64, None) == 1              # lda not a multiple of 8
    assert g(a, 64, b, 64, a + 64, 64, 32, 64, 64, None) == 1         # C overlaps A
    assert g(a, 64, b, 64, c, 64, 0, 64, 64, None) == 0               # empty: nothing to do
    assert g(a, 64, b, 64, c, 64, 32, 0, 64, None) == 0


def test_debug_build_is_flagged_and_complete(lib):
    """libarl2_debug.so (kernels compiled with -DARL2_DEBUG_BOUNDS) reports
    itself as the debug build, exports every declared entry point, and the
    release library reports that it is not."""
    from hybrid_linear_attention_arl2_b200 import build as _b
    dbg = ctypes.CDLL(_b.build(debug_bounds=True))
    assert dbg.arl2_debug_bounds_enabled() == 1
    assert lib.arl2_debug_bounds_enabled() == 0
    missing = [n for n in arl2.declared_symbols() if not hasattr(dbg, n)]
    assert not missing, missing
    assert arl2.arl2_status_string(8) == "a kernel index check failed (debug build)"
