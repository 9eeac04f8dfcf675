"""QJL 1-bit key cache and decode attention for NVIDIA B200 (sm_100a).

The compute path is libqjl.so (C ABI in include/qjl.h, CUDA kernels in csrc/);
this package holds its thin ctypes binding (qjl.py), the in-tree build script
(build.py) and the seeded synthetic input generator (inputs.py).
"""

from .qjl import (  # noqa: F401
    EXPORTED,
    HEAD_DIM,
    LIB_PATH,
    QJL_APPEND,
    QJL_BF16,
    QJL_FP32,
    QJL_PREFILL,
    QJLCache,
    QJLContext,
    QJLError,
    load_library,
    qjl_ctx_guard,
    qjl_ctx_sketch,
    qjl_decode_attention,
    qjl_decode_attention_static,
    qjl_decode_workspace_bytes,
    qjl_free,
    qjl_init,
    qjl_last_error,
    qjl_quantize_keys,
    qjl_quantize_keys_workspace_bytes,
    qjl_quantize_values,
    qjl_sketch_host,
)
