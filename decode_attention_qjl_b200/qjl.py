"""Thin ctypes binding of libqjl.so (declared in include/qjl.h).

Every function here only marshals arguments: it turns torch tensors into device
pointers, picks the current CUDA stream, calls the C entry point of the same
name and raises QJLError on a non-zero status. All arithmetic runs in the CUDA
kernels of libqjl.so; if the library is not built, loading fails loudly.
"""

from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import numpy as np

_PKG_DIR = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG_DIR, "libqjl.so")

QJL_OK = 0
QJL_BF16, QJL_FP32 = 0, 1
QJL_PREFILL, QJL_APPEND = 0, 1
HEAD_DIM = 128

STATUS_NAMES = {0: "QJL_OK", 1: "QJL_ERR_ARG", 2: "QJL_ERR_CUDA", 3: "QJL_ERR_UNSUPPORTED", 4: "QJL_ERR_OOM",
                5: "QJL_ERR_WORKSPACE", 6: "QJL_ERR_TIMEOUT"}
QJL_ERR_TIMEOUT = 6

# Every symbol include/qjl.h declares.
EXPORTED = [
    "qjl_init", "qjl_init_ex", "qjl_cache_tile_bytes_ex", "qjl_free", "qjl_last_error", "qjl_sketch_host", "qjl_ctx_sketch", "qjl_ctx_guard",
    "qjl_cache_tile_bytes",
    "qjl_quantize_keys_workspace_bytes", "qjl_quantize_keys", "qjl_quantize_values",
    "qjl_decode_workspace_bytes", "qjl_decode_attention", "qjl_decode_step", "qjl_set_wait_limit",
    "qjl_decode_workspace_status", "qjl_decode_attention_static", "qjl_decode_attention_partial",
    "qjl_merge_partials", "qjl_fp8_quantize", "qjl_exact_decode_workspace_bytes", "qjl_exact_decode",
    "qjl_minmax_quantize",
]
QJL_KV_BF16, QJL_KV_FP8_E4M3, QJL_KV_MINMAX2, QJL_KV_MINMAX4 = 0, 1, 2, 3
_ROW_FORMAT = {128: QJL_KV_FP8_E4M3, 48: QJL_KV_MINMAX2, 80: QJL_KV_MINMAX4}  # uint8 row bytes -> format

STATIC_SCRATCH_BYTES = 8 * 1024 * 1024  # QJL_STATIC_SCRATCH_BYTES in include/qjl.h
CAP_ALIGN = 64  # the cache capacity must be a multiple of this (one tile)
TILE_TOKENS = 64


class QJLError(RuntimeError):
    def __init__(self, fn: str, status: int, message: str):
        super().__init__(f"{fn} failed with {STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


class qjl_cache(ctypes.Structure):
    _fields_ = [
        ("outlier_idx", ctypes.c_void_p),
        ("tiles", ctypes.c_void_p),
        ("B", ctypes.c_int),
        ("Hkv", ctypes.c_int),
        ("cap", ctypes.c_int),
    ]


_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libqjl.so and declare its C signatures. Raises if it is not built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"libqjl.so not found at {path}: build it with "
                           "`python -m decode_attention_qjl_b200.build` (there is no fallback path)")
    L = ctypes.CDLL(path)
    vp, i32, i64, u64, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_uint64, ctypes.c_size_t
    cachep = ctypes.POINTER(qjl_cache)
    sig = {
        "qjl_init": (i32, [u64, i32, i32, i32, i32, ctypes.POINTER(vp)]),
        "qjl_init_ex": (i32, [u64, i32, i32, i32, i32, i32, ctypes.POINTER(vp)]),
        "qjl_cache_tile_bytes_ex": (sz, [i32, i32, i32, i32]),
        "qjl_free": (None, [vp]),
        "qjl_last_error": (ctypes.c_char_p, []),
        "qjl_sketch_host": (i32, [u64, i32, i32, i32, vp, vp]),
        "qjl_ctx_sketch": (i32, [vp, vp, vp]),
        "qjl_ctx_guard": (ctypes.c_float, [vp]),
        "qjl_cache_tile_bytes": (sz, [i32, i32, i32]),
        "qjl_quantize_keys_workspace_bytes": (sz, [vp, i32, i32, i32]),
        "qjl_quantize_keys": (i32, [vp, cachep, vp, i32, i32, i64, i64, i64, vp, i32, vp, sz, vp]),
        "qjl_quantize_values": (i32, [vp, cachep, vp, i32, i32, i64, i64, i64, vp, vp]),
        "qjl_decode_workspace_bytes": (sz, [vp, i32, i32, i32, i32]),
        "qjl_decode_attention": (i32, [vp, cachep, vp, i32, i32, i32, vp, ctypes.c_float, vp, vp, vp, sz, vp]),
        "qjl_decode_step": (i32, [vp, cachep, vp, vp, i64, i64, vp, i64, i64, i32, i32, i32, vp, ctypes.c_float,
                                  vp, vp, vp, sz, vp]),
        "qjl_set_wait_limit": (i32, [vp, u64]),
        "qjl_decode_workspace_status": (i32, [vp, vp, i32, i32, i32, vp]),
        "qjl_decode_attention_static": (i32, [vp, cachep, vp, i32, i32, i32, vp, ctypes.c_float, vp, vp, vp]),
        "qjl_decode_attention_partial": (i32, [vp, cachep, vp, i32, i32, i32, vp, ctypes.c_float, vp, vp, vp, vp,
                                               sz, vp]),
        "qjl_merge_partials": (i32, [vp, i64, vp, i64, i32, i64, vp, vp]),
        "qjl_fp8_quantize": (i32, [vp, i32, i64, ctypes.c_float, vp, vp]),
        "qjl_exact_decode_workspace_bytes": (sz, [i32, i32, i32]),
        "qjl_minmax_quantize": (i32, [vp, i32, i64, i32, vp, vp]),
        "qjl_exact_decode": (i32, [i32, vp, vp, ctypes.c_float, ctypes.c_float, i32, i32, i32, i32, i32, vp, i32, vp,
                                   ctypes.c_float, vp, vp, sz, vp]),
    }
    for name, (res, args) in sig.items():
        f = getattr(L, name)
        f.restype = res
        f.argtypes = args
    _lib = L
    return L


def _check(fn: str, status: int) -> None:
    if status != QJL_OK:
        msg = load_library().qjl_last_error()
        raise QJLError(fn, status, msg.decode() if msg else "")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    import torch

    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dtype_code(t) -> int:
    import torch

    if t.dtype == torch.bfloat16:
        return QJL_BF16
    if t.dtype == torch.float32:
        return QJL_FP32
    raise TypeError(f"unsupported dtype {t.dtype}: use bfloat16 or float32")


# ----------------------------------------------------------------- context

def qjl_init(seed: int, d: int, m: int, m_out: int, n_outlier: int, value_bits: int = 4) -> ctypes.c_void_p:
    ctx = ctypes.c_void_p()
    _check("qjl_init_ex", load_library().qjl_init_ex(seed, d, m, m_out, n_outlier, value_bits, ctypes.byref(ctx)))
    return ctx


def qjl_free(ctx) -> None:
    load_library().qjl_free(ctx)


def qjl_last_error() -> str:
    return load_library().qjl_last_error().decode()


def qjl_sketch_host(seed: int, d: int, m: int, m_out: int):
    """Host copies of S and S_out (bf16 bit patterns as uint16 arrays); needs no GPU."""
    S = np.zeros((m, d), np.uint16)
    So = np.zeros((m_out, d), np.uint16)
    _check("qjl_sketch_host", load_library().qjl_sketch_host(seed, d, m, m_out, S.ctypes.data_as(ctypes.c_void_p),
                                                             So.ctypes.data_as(ctypes.c_void_p) if m_out else None))
    return S, So


def qjl_ctx_sketch(ctx, m: int, m_out: int, d: int = HEAD_DIM):
    S = np.zeros((m, d), np.uint16)
    So = np.zeros((m_out, d), np.uint16)
    _check("qjl_ctx_sketch", load_library().qjl_ctx_sketch(ctx, S.ctypes.data_as(ctypes.c_void_p),
                                                           So.ctypes.data_as(ctypes.c_void_p) if m_out else None))
    return S, So


def qjl_ctx_guard(ctx) -> float:
    return float(load_library().qjl_ctx_guard(ctx))


# ----------------------------------------------------------------- cache

def qjl_cache_tile_bytes(d: int, m: int, m_out: int) -> int:
    return int(load_library().qjl_cache_tile_bytes(d, m, m_out))


V2_LINE_BYTES = TILE_TOKENS + 4  # a 2-bit code line: one byte per token, 4 bytes of padding


def tile_sections(m: int, m_out: int, d: int = HEAD_DIM, value_bits: int = 4):
    """(name, byte offset, bytes per token, section bytes) of the sections of a 64-token tile, in order."""
    vc = (d // 4, (d // 4) * V2_LINE_BYTES) if value_bits == 2 else (d // 2, TILE_TOKENS * d // 2)
    per_tok = [("kbits", m // 8, None), ("kbits_out", m_out // 8, None), ("knorm", 4, None), ("vcode",) + vc,
               ("vsz", d // 8, None)]
    out, off = [], 0
    for name, nb, sec in per_tok:
        sec = TILE_TOKENS * nb if sec is None else sec
        out.append((name, off, nb, sec))
        off += sec
    return out


def tile_bytes(m: int, m_out: int, d: int = HEAD_DIM, value_bits: int = 4) -> int:
    return sum(sec for _, _, _, sec in tile_sections(m, m_out, d, value_bits))


@dataclass
class QJLCache:
    """Device tensors of a QJL cache (layout in include/qjl.h), owned by torch.

    `tiles` is uint8 [B, Hkv, cap / 64, tile_bytes]; `section(name)` gives a
    view of one part with its tokens in order, e.g. kbits as int32
    [B, Hkv, cap, m / 32]."""

    outlier_idx: "object"
    tiles: "object"
    B: int
    Hkv: int
    cap: int
    m: int
    m_out: int
    value_bits: int = 4

    @staticmethod
    def allocate(B: int, Hkv: int, cap: int, m: int, m_out: int, n_outlier: int, device="cuda", d: int = HEAD_DIM,
                 value_bits: int = 4):
        """Zero-filled cache for at least `cap` tokens (rounded up to a multiple of CAP_ALIGN)."""
        import torch

        cap = -(-max(cap, 1) // CAP_ALIGN) * CAP_ALIGN
        tb = tile_bytes(m, m_out, d, value_bits)
        return QJLCache(
            outlier_idx=torch.zeros(B, Hkv, max(n_outlier, 1), dtype=torch.int32, device=device),
            tiles=torch.zeros(B, Hkv, cap // TILE_TOKENS, tb, dtype=torch.uint8, device=device),
            B=B, Hkv=Hkv, cap=cap, m=m, m_out=m_out, value_bits=value_bits,
        )

    def struct(self) -> qjl_cache:
        return qjl_cache(self.outlier_idx.data_ptr(), self.tiles.data_ptr(), self.B, self.Hkv, self.cap)

    def nbytes(self) -> int:
        return sum(t.numel() * t.element_size() for t in (self.outlier_idx, self.tiles))

    def section(self, name: str):
        """View of one tile section over all tokens: kbits / kbits_out int32 [B, Hkv, cap, words],
        knorm fp16 [B, Hkv, cap, 2], vcode uint8 [B, Hkv, cap, d/2] (4-bit: dim 2i in the low nibble of
        byte i) or [B, Hkv, cap, d/4] (2-bit: dim 4i + k in bits 2k, 2k+1 of byte i), vsz fp16
        [B, Hkv, cap, d/32, 2]."""
        import torch

        for nm, off, nb, sec in tile_sections(self.m, self.m_out, value_bits=self.value_bits):
            if nm == name:
                break
        else:
            raise KeyError(name)
        nt = self.cap // TILE_TOKENS
        if nb == 0:  # no outlier sketch
            return torch.zeros(self.B, self.Hkv, self.cap, 0, dtype=torch.int32, device=self.tiles.device)
        if name == "vcode" and self.value_bits == 2:  # lines (group, quad) of 64 token bytes + padding
            lines = self.tiles[..., off:off + sec].reshape(self.B, self.Hkv, nt, nb, V2_LINE_BYTES)[..., :TILE_TOKENS]
            return lines.transpose(-1, -2).reshape(self.B, self.Hkv, self.cap, nb).contiguous()
        raw = self.tiles[..., off:off + TILE_TOKENS * nb].reshape(self.B, self.Hkv, nt, TILE_TOKENS, nb)
        raw = raw.reshape(self.B, self.Hkv, self.cap, nb)
        if name in ("kbits", "kbits_out"):
            return raw.contiguous().view(torch.int32)
        if name == "knorm":
            return raw.contiguous().view(torch.float16)
        if name == "vsz":
            return raw.contiguous().view(torch.float16).reshape(self.B, self.Hkv, self.cap, nb // 4, 2)
        # vcode: group g of token j is stored at 16-byte chunk g ^ ((j >> 1) & 3)
        j = torch.arange(TILE_TOKENS, device=raw.device)
        chunk = torch.arange(nb // 16, device=raw.device)[None, :] ^ ((j[:, None] >> 1) & 3)  # [64, groups]
        phys = self.tiles[..., off:off + TILE_TOKENS * nb].reshape(self.B, self.Hkv, nt, TILE_TOKENS, nb // 16, 16)
        idx = chunk[None, None, None, :, :, None].expand(self.B, self.Hkv, nt, TILE_TOKENS, nb // 16, 16)
        return torch.gather(phys, 4, idx).reshape(self.B, self.Hkv, self.cap, nb)


# ----------------------------------------------------------------- entry points

def qjl_quantize_keys_workspace_bytes(ctx, B: int, Hkv: int, mode: int = QJL_PREFILL) -> int:
    return int(load_library().qjl_quantize_keys_workspace_bytes(ctx, B, Hkv, mode))


def qjl_quantize_keys(ctx, cache: QJLCache, K, mode: int = QJL_PREFILL, t_start=None, workspace=None, stream=None):
    """K: device tensor [B, Hkv, T, d] (bf16 or fp32) with a contiguous last dim."""
    T = K.shape[2]
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = load_library().qjl_quantize_keys(ctx, ctypes.byref(cache.struct()), _ptr(K), _dtype_code(K), T,
                                          K.stride(0), K.stride(1), K.stride(2), _ptr(t_start), mode,
                                          _ptr(workspace), ws_bytes, _stream(stream))
    _check("qjl_quantize_keys", st)


def qjl_quantize_values(ctx, cache: QJLCache, V, t_start=None, stream=None):
    """V: device tensor [B, Hkv, T, d] (bf16 or fp32) with a contiguous last dim."""
    T = V.shape[2]
    st = load_library().qjl_quantize_values(ctx, ctypes.byref(cache.struct()), _ptr(V), _dtype_code(V), T,
                                            V.stride(0), V.stride(1), V.stride(2), _ptr(t_start), _stream(stream))
    _check("qjl_quantize_values", st)


def qjl_decode_workspace_bytes(ctx, B: int, Hq: int, Hkv: int, T: int) -> int:
    return int(load_library().qjl_decode_workspace_bytes(ctx, B, Hq, Hkv, T))


def qjl_decode_attention(ctx, cache: QJLCache, Q, T: int, O, seqlens=None, sm_scale: float = 0.0, scores=None,
                         workspace=None, stream=None):
    """Q: device [B, Hq, d] (bf16 or fp32, contiguous); O: device fp32 [B, Hq, d], written."""
    Hq = Q.shape[1]
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = load_library().qjl_decode_attention(ctx, ctypes.byref(cache.struct()), _ptr(Q), _dtype_code(Q), Hq, T,
                                             _ptr(seqlens), sm_scale, _ptr(O), _ptr(scores), _ptr(workspace),
                                             ws_bytes, _stream(stream))
    _check("qjl_decode_attention", st)
    return O


def qjl_decode_step(ctx, cache: QJLCache, Q, K_new, V_new, T: int, O, seqlens=None, sm_scale: float = 0.0,
                    scores=None, workspace=None, stream=None):
    """One decode step in one launch: append K_new / V_new (device [B, Hkv, d], or [B, Hkv, 1, d]) at each
    sequence's length, then attend over T + 1 (or seqlens[b] + 1) tokens. Q: device [B, Hq, d]; O: fp32 [B, Hq, d]."""
    Hq = Q.shape[1]
    if K_new.dim() == 4:
        K_new, V_new = K_new[:, :, 0], V_new[:, :, 0]
    if K_new.dtype != Q.dtype or V_new.dtype != Q.dtype:
        raise TypeError("Q, K_new and V_new must share one dtype")
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = load_library().qjl_decode_step(ctx, ctypes.byref(cache.struct()), _ptr(Q), _ptr(K_new), K_new.stride(0),
                                        K_new.stride(1), _ptr(V_new), V_new.stride(0), V_new.stride(1),
                                        _dtype_code(Q), Hq, T, _ptr(seqlens), sm_scale, _ptr(O), _ptr(scores),
                                        _ptr(workspace), ws_bytes, _stream(stream))
    _check("qjl_decode_step", st)
    return O


def qjl_decode_attention_partial(ctx, cache: QJLCache, Q, T: int, O_part, ML_part, seqlens=None,
                                 sm_scale: float = 0.0, scores=None, workspace=None, stream=None):
    """This rank's shard of a context-parallel decode. O_part: device fp32 [B, Hq, d] (unnormalised);
    ML_part: device fp32 [B, Hq, 2] (maximum logit in log2 units, sum of 2^(x - max)); both written."""
    Hq = Q.shape[1]
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = load_library().qjl_decode_attention_partial(ctx, ctypes.byref(cache.struct()), _ptr(Q), _dtype_code(Q), Hq,
                                                     T, _ptr(seqlens), sm_scale, _ptr(O_part), _ptr(ML_part),
                                                     _ptr(scores), _ptr(workspace), ws_bytes, _stream(stream))
    _check("qjl_decode_attention_partial", st)
    return O_part, ML_part


def qjl_merge_partials(O_parts, ML_parts, O, stream=None):
    """Merge R ranks' parts into O (device fp32 [B, Hq, d]). O_parts: fp32 [R, B, Hq, d] and ML_parts:
    fp32 [R, B, Hq, 2], or views into one packed buffer per rank (dim 0 = rank, rows contiguous)."""
    R = O_parts.shape[0]
    rows = O.numel() // O.shape[-1]
    if O_parts[0].numel() != O.numel() or ML_parts[0].numel() != rows * 2 or ML_parts.shape[0] != R:
        raise ValueError("O_parts / ML_parts do not match O")
    for t in (O_parts[0], ML_parts[0], O):
        if t.dtype.itemsize != 4 or not t.is_contiguous():
            raise ValueError("qjl_merge_partials takes fp32 parts with contiguous rows")
    st = load_library().qjl_merge_partials(_ptr(O_parts), O_parts.stride(0), _ptr(ML_parts), ML_parts.stride(0), R,
                                           rows, _ptr(O), _stream(stream))
    _check("qjl_merge_partials", st)
    return O


def qjl_fp8_quantize(X, scale: float, out=None, stream=None):
    """E4M3 codes (torch.uint8, same shape) of X / scale; X: device bf16 or fp32, contiguous, numel % 8 == 0."""
    import torch

    if out is None:
        out = torch.empty(X.shape, dtype=torch.uint8, device=X.device)
    st = load_library().qjl_fp8_quantize(_ptr(X), _dtype_code(X), X.numel(), float(scale), _ptr(out), _stream(stream))
    _check("qjl_fp8_quantize", st)
    return out


def qjl_minmax_quantize(X, bits: int, out=None, stream=None):
    """Min-max b-bit rows (torch.uint8 [..., 128 * bits / 8 + 16]) of X (device [..., 128], bf16 or fp32)."""
    import torch

    n = X.numel() // X.shape[-1]
    if out is None:
        out = torch.empty(*X.shape[:-1], X.shape[-1] * bits // 8 + 16, dtype=torch.uint8, device=X.device)
    st = load_library().qjl_minmax_quantize(_ptr(X), _dtype_code(X), n, int(bits), _ptr(out), _stream(stream))
    _check("qjl_minmax_quantize", st)
    return out


def qjl_exact_decode(K, V, Q, O, T: int | None = None, seqlens=None, sm_scale: float = 0.0, k_scale: float = 1.0,
                     v_scale: float = 1.0, workspace=None, stream=None):
    """Decode over a comparison cache. K, V: device [B, Hkv, cap, row]: bf16 rows of d (exact), or uint8 rows of
    E4M3 codes (d bytes, with k_scale / v_scale) or of min-max codes (qjl_minmax_quantize: 48 or 80 bytes);
    Q: device [B, Hq, d] bf16 or fp32; O: device fp32 [B, Hq, d], written."""
    import torch

    B, Hkv, cap, row = K.shape
    Hq = Q.shape[1]
    T = cap if T is None else T
    if K.dtype == torch.bfloat16:
        fmt = QJL_KV_BF16
    elif K.dtype == torch.uint8 and row in _ROW_FORMAT:
        fmt = _ROW_FORMAT[row]
    else:
        raise TypeError("K, V must be bfloat16 rows or uint8 rows of E4M3 or min-max codes")
    if workspace is None:
        n = int(load_library().qjl_exact_decode_workspace_bytes(B, Hq, T))
        workspace = torch.empty(max(n, 16), dtype=torch.uint8, device=K.device)
    ws_bytes = workspace.numel() * workspace.element_size()
    st = load_library().qjl_exact_decode(fmt, _ptr(K), _ptr(V), float(k_scale), float(v_scale), B, Hq, Hkv, cap, T,
                                         _ptr(Q), _dtype_code(Q), _ptr(seqlens), sm_scale, _ptr(O), _ptr(workspace),
                                         ws_bytes, _stream(stream))
    _check("qjl_exact_decode", st)
    return O


def qjl_set_wait_limit(ctx, ns: int) -> None:
    _check("qjl_set_wait_limit", load_library().qjl_set_wait_limit(ctx, int(ns)))


def qjl_decode_workspace_status(ctx, workspace, B: int, Hq: int, Hkv: int, stream=None) -> None:
    """Synchronise and raise QJLError (QJL_ERR_TIMEOUT) if a wait inside a decode kernel that used
    this workspace ran out; the workspace counters are then cleared for the next call."""
    _check("qjl_decode_workspace_status",
           load_library().qjl_decode_workspace_status(ctx, _ptr(workspace), B, Hq, Hkv, _stream(stream)))


def qjl_decode_attention_static(ctx, cache: QJLCache, Q, T: int, O, seqlens=None, sm_scale: float = 0.0,
                                scores=None, stream=None):
    """qjl_decode_attention with the library's fixed scratch array instead of a workspace.

    For callers that cannot allocate device memory. Calls that overlap on the
    GPU share the array and race; the first call on a device does a one-time
    set-up and should come before any stream capture."""
    Hq = Q.shape[1]
    st = load_library().qjl_decode_attention_static(ctx, ctypes.byref(cache.struct()), _ptr(Q), _dtype_code(Q), Hq,
                                                    T, _ptr(seqlens), sm_scale, _ptr(O), _ptr(scores),
                                                    _stream(stream))
    _check("qjl_decode_attention_static", st)
    return O


class QJLContext:
    """Owns a qjl_ctx handle (S and S_out on the device) for its lifetime."""

    def __init__(self, seed: int = 0, d: int = HEAD_DIM, m: int = 256, m_out: int = 64, n_outlier: int = 8,
                 value_bits: int = 4):
        self.seed, self.d, self.m, self.m_out, self.n_outlier = seed, d, m, m_out, n_outlier
        self.value_bits = value_bits
        self.handle = qjl_init(seed, d, m, m_out, n_outlier, value_bits)

    def close(self):
        if self.handle is not None and self.handle.value:
            qjl_free(self.handle)
        self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def allocate_cache(self, B: int, Hkv: int, cap: int, device="cuda") -> QJLCache:
        return QJLCache.allocate(B, Hkv, cap, self.m, self.m_out, self.n_outlier, device, self.d, self.value_bits)

    def decode_workspace(self, B: int, Hq: int, Hkv: int, T: int, device="cuda"):
        import torch

        n = qjl_decode_workspace_bytes(self.handle, B, Hq, Hkv, T)
        return torch.zeros(max(n, 16), dtype=torch.uint8, device=device)

    def keys_workspace(self, B: int, Hkv: int, device="cuda"):
        import torch

        n = qjl_quantize_keys_workspace_bytes(self.handle, B, Hkv, QJL_PREFILL)
        return torch.zeros(max(n, 16), dtype=torch.uint8, device=device)
