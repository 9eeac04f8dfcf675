"""The C-ABI library on the CPU: it builds, loads, exports every declared symbol,
draws the same sketch as the oracle and rejects bad arguments before touching
the GPU. No compute call runs here."""

import ctypes
import os
import re

import numpy as np
import pytest

import oracle as O
from decode_attention_qjl_b200 import build as build_mod
from decode_attention_qjl_b200 import qjl as Q

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build_mod.build()
    return Q.load_library()


def _declared_symbols():
    text = open(os.path.join(ROOT, "include", "qjl.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(qjl_[a-z_0-9]+)\s*\(", text)))


def test_exports_every_declared_symbol(lib):
    declared = _declared_symbols()
    assert declared == sorted(Q.EXPORTED)
    for name in declared:
        assert hasattr(lib, name), name


def test_library_is_sm100a_only():
    # the fatbin is built for sm_100a alone; the build flags say so
    assert build_mod.ARCH_FLAGS == ["-gencode", "arch=compute_100a,code=sm_100a"]


@pytest.mark.parametrize("seed,m,m_out", [(0, 256, 64), (12345, 128, 32), (2 ** 63 + 7, 512, 64)])
def test_host_sketch_matches_oracle(lib, seed, m, m_out):
    S_bits, So_bits = Q.qjl_sketch_host(seed, 128, m, m_out)
    S, So = O.sketch_pair(seed, 128, m, m_out)
    to_bits = lambda a: (a.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    assert np.array_equal(S_bits, to_bits(S))
    assert np.array_equal(So_bits, to_bits(So))


def test_argument_errors_without_gpu(lib):
    ctx = ctypes.c_void_p()
    assert lib.qjl_init(0, 64, 256, 64, 8, ctypes.byref(ctx)) == 3  # d != 128: unsupported
    assert ctx.value is None
    assert b"d = 128" in lib.qjl_last_error()
    assert lib.qjl_init(0, 128, 48, 64, 8, ctypes.byref(ctx)) == 1  # m not a multiple of 32
    assert lib.qjl_init(0, 128, 256, 0, 4, ctypes.byref(ctx)) == 1  # outliers without an outlier sketch
    assert lib.qjl_init(0, 128, 256, 64, 33, ctypes.byref(ctx)) == 1
    assert lib.qjl_init(0, 128, 256, 64, 8, None) == 1
    cache = Q.qjl_cache()
    assert lib.qjl_quantize_keys(None, ctypes.byref(cache), None, 0, 1, 128, 128, 128, None, 0, None, 0, None) == 1
    assert lib.qjl_quantize_values(None, ctypes.byref(cache), None, 0, 1, 128, 128, 128, None, None) == 1
    assert lib.qjl_decode_attention(None, ctypes.byref(cache), None, 0, 1, 1, None, 0.0, None, None, None, 0,
                                    None) == 1
    assert lib.qjl_decode_step(None, ctypes.byref(cache), None, None, 0, 0, None, 0, 0, 0, 1, 1, None, 0.0, None,
                               None, None, 0, None) == 1
    assert lib.qjl_set_wait_limit(None, 1000) == 1
    assert lib.qjl_decode_attention_partial(None, ctypes.byref(cache), None, 0, 1, 1, None, 0.0, None, None, None,
                                            None, 0, None) == 1
    buf = (ctypes.c_float * 1024)()
    assert lib.qjl_merge_partials(buf, 512, buf, 4, 0, 2, buf, None) == 1        # R < 1
    assert lib.qjl_merge_partials(buf, 128, buf, 4, 2, 2, buf, None) == 1        # rank stride < rows * d
    assert lib.qjl_merge_partials(None, 256, None, 4, 1, 2, None, None) == 1     # null buffers
    assert lib.qjl_merge_partials(None, 0, None, 0, 1, 0, None, None) == 0       # nothing to merge
    assert lib.qjl_fp8_quantize(None, 0, 12, 1.0, None, None) == 1              # n not a multiple of 8
    assert lib.qjl_fp8_quantize(None, 0, 8, 0.0, None, None) == 1               # scale <= 0
    assert lib.qjl_exact_decode_workspace_bytes(2, 8, 300) == 2 * 8 * 130 * 4 * 2  # two 256-token blocks
    assert lib.qjl_minmax_quantize(None, 0, 4, 3, None, None) == 1             # bits must be 2 or 4
    assert lib.qjl_minmax_quantize(None, 0, 0, 2, None, None) == 0             # nothing to do
    assert lib.qjl_exact_decode(0, None, None, 1.0, 1.0, 1, 3, 2, 64, 64, None, 0, None, 0.0, None, None, 0,
                                None) == 1                                      # Hq not a multiple of Hkv
    assert lib.qjl_exact_decode(0, None, None, 1.0, 1.0, 1, 6, 2, 64, 64, None, 0, None, 0.0, None, None, 0,
                                None) == 3                                      # g = 3 unsupported
    assert lib.qjl_decode_workspace_status(None, None, 1, 1, 1, None) == 1
    assert lib.qjl_decode_workspace_bytes(None, 1, 1, 1, 1) == 0
    assert lib.qjl_sketch_host(0, 128, 256, 64, None, None) == 1
    with pytest.raises(Q.QJLError, match="QJL_ERR_UNSUPPORTED"):
        Q.qjl_init(0, 256, 256, 64, 8)


@pytest.mark.parametrize("m,m_out", [(256, 64), (128, 0), (512, 256), (32, 32)])
def test_cache_tile_bytes(lib, m, m_out):
    # per token: m/8 + m_out/8 sign bytes, two fp16 norms, 64 code bytes, 4 x (scale, zero) fp16
    want = 64 * (m // 8 + m_out // 8 + 4 + 64 + 16)
    assert lib.qjl_cache_tile_bytes(128, m, m_out) == want == Q.tile_bytes(m, m_out)
    # 2-bit value codes: d/4 lines of 64 token bytes plus 4 bytes of padding instead of 64 x d/2 bytes
    want2 = want - 64 * 64 + 32 * 68
    assert lib.qjl_cache_tile_bytes_ex(128, m, m_out, 2) == want2 == Q.tile_bytes(m, m_out, value_bits=2)
    assert lib.qjl_cache_tile_bytes_ex(128, m, m_out, 4) == want
    assert lib.qjl_cache_tile_bytes_ex(128, m, m_out, 3) == 0
    assert want % 16 == 0  # whole tiles are moved with 16-byte-granular bulk copies


def test_cache_tile_bytes_rejects_bad_sizes(lib):
    assert lib.qjl_cache_tile_bytes(64, 256, 64) == 0
    assert lib.qjl_cache_tile_bytes(128, 48, 64) == 0
    assert lib.qjl_cache_tile_bytes(128, 256, 288) == 0
