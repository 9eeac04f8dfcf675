"""Helpers shared by the GPU parity tests: run the CUDA path, convert its cache
to numpy, and compare with the oracle under the stated tolerances."""

from __future__ import annotations

import math

import numpy as np
import torch

import oracle as O
from decode_attention_qjl_b200 import qjl as Q

# Tolerances (stated for floating point; integer and byte outputs are bit-exact).
SCORE_RTOL = 1e-3      # relative error of a score ...
SCORE_FLOOR = 1e-3     # ... measured against max(|s|, SCORE_FLOOR * rms of the row's scores)
OUT_ATOL = 2e-3        # max absolute error of the attention output
SIGN_BAND = 1e-6       # signs with |S k| < SIGN_BAND * |k_part| are excluded (counted)


def to64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def sketch64(w):
    return O.sketch_pair(0, 128, w.m, w.m_out)


def quantize_on_gpu(ctx: Q.QJLContext, K: torch.Tensor, V: torch.Tensor, cap: int | None = None) -> Q.QJLCache:
    B, Hkv, T, _ = K.shape
    cache = ctx.allocate_cache(B, Hkv, cap or T)
    ws = ctx.keys_workspace(B, Hkv)
    Q.qjl_quantize_keys(ctx.handle, cache, K, Q.QJL_PREFILL, workspace=ws)
    Q.qjl_quantize_values(ctx.handle, cache, V)
    torch.cuda.synchronize()
    cache.filled = T  # tokens written (the capacity is rounded up to a multiple of 64)
    return cache


def cache_to_numpy(cache: Q.QJLCache, m_out: int, n_out: int, T: int | None = None, b=None, h=None) -> dict:
    """Host copy of the cache in the oracle's format; b / h select one sequence / kv head (kept as a size-1 dim)."""
    T = getattr(cache, "filled", cache.cap) if T is None else T
    bs = slice(None) if b is None else slice(b, b + 1)
    hs = slice(None) if h is None else slice(h, h + 1)
    return {
        "idx": cache.outlier_idx[bs, hs, :n_out].cpu().numpy().astype(np.int64),
        "bits_in": cache.section("kbits")[bs, hs, :T].cpu().numpy().view(np.uint32),
        "bits_out": cache.section("kbits_out")[bs, hs, :T].cpu().numpy().view(np.uint32),
        "norms": cache.section("knorm")[bs, hs, :T].cpu().numpy(),
        "codes": unpack_value_codes(cache.section("vcode")[bs, hs, :T].cpu().numpy(), getattr(cache, "value_bits", 4)),
        "scale": cache.section("vsz")[bs, hs, :T, :, 0].cpu().numpy(),
        "zero": cache.section("vsz")[bs, hs, :T, :, 1].cpu().numpy(),
    }


def unpack_value_codes(raw: np.ndarray, bits: int) -> np.ndarray:
    """Per-dim codes from the cache's packed bytes: 4-bit (dim 2i in the low nibble of byte i) through the
    oracle's unpack_codes; 2-bit: dim 4i + k in bits 2k, 2k+1 of byte i."""
    if bits == 4:
        return O.unpack_codes(raw)
    return np.stack([(raw >> (2 * k)) & 3 for k in range(4)], -1).reshape(*raw.shape[:-1], raw.shape[-1] * 4)


def unpack_bits(words: np.ndarray, n: int) -> np.ndarray:
    return O.unpack_signs(words, n) > 0


def compare_keys(g: dict, K64: np.ndarray, S, So, n_out: int, pairs, planted=None, idx_given=None) -> dict:
    """Bit-exact comparison of outlier channels, sign bits and fp16 norms for (b, h) pairs.

    Returns counts: excluded sign entries (|S k| within SIGN_BAND |k| of zero) and
    mismatches outside the band (must be 0)."""
    m, m_out = S.shape[0], So.shape[0]
    stats = {"entries": 0, "excluded": 0, "mismatch": 0, "norm_mismatch": 0}
    for b, h in pairs:
        if idx_given is None:
            idx = O.select_outliers(K64[b, h], n_out)
            assert np.array_equal(g["idx"][b, h], idx), (b, h, g["idx"][b, h], idx)
            if planted is not None:
                assert np.array_equal(idx, planted[b, h]), (b, h)
        else:
            idx = idx_given[b, h]
        ks = O.sketch_keys(K64[b, h], S, So, idx)
        for part, y, nrm, mm in (("bits_in", ks["y_in"], ks["norm_in"], m), ("bits_out", ks["y_out"], ks["norm_out"], m_out)):
            if mm == 0:
                continue
            excl = np.abs(y) < SIGN_BAND * nrm[:, None]
            want = y >= 0
            got = unpack_bits(g[part][b, h], mm)
            stats["entries"] += want.size
            stats["excluded"] += int(excl.sum())
            stats["mismatch"] += int(((got != want) & ~excl).sum())
        stats["norm_mismatch"] += int(np.sum(g["norms"][b, h].view(np.uint16) != ks["norms"].view(np.uint16)))
    return stats


def compare_values(g: dict, V64: np.ndarray, pairs, bits: int = 4) -> int:
    bad = 0
    for b, h in pairs:
        c, s, z = O.quantize_values(V64[b, h], bits, 32)
        bad += int(np.sum(g["codes"][b, h] != c))
        bad += int(np.sum(g["scale"][b, h].view(np.uint16) != s.view(np.uint16)))
        bad += int(np.sum(g["zero"][b, h].view(np.uint16) != z.view(np.uint16)))
    return bad


def run_decode(ctx: Q.QJLContext, cache: Q.QJLCache, Qt: torch.Tensor, T: int, seqlens=None, sm_scale=0.0,
               want_scores=True):
    B, Hq, d = Qt.shape
    O_ = torch.empty(B, Hq, d, dtype=torch.float32, device="cuda")
    scores = torch.full((B, Hq, max(T, 1)), float("nan"), dtype=torch.float32, device="cuda") if want_scores else None
    ws = ctx.decode_workspace(B, Hq, cache.Hkv, T)
    sl = None if seqlens is None else torch.as_tensor(seqlens, dtype=torch.int32, device="cuda")
    Q.qjl_decode_attention(ctx.handle, cache, Qt, T, O_, seqlens=sl, sm_scale=sm_scale, scores=scores, workspace=ws)
    Q.qjl_decode_workspace_status(ctx.handle, ws, B, Hq, cache.Hkv)  # raises if a wait inside ran out
    return O_.cpu().numpy().astype(np.float64), (None if scores is None else scores.cpu().numpy().astype(np.float64))


def compare_decode(g: dict, Q64, S, So, O_gpu, sc_gpu, pairs, seqlens=None, sm_scale=None) -> dict:
    """Scores (relative 1e-3 with a floor) and outputs (absolute 2e-3) against the oracle
    evaluated on the same (GPU-produced, already checked) cache."""
    Oo, so = O.decode_batch(Q64, S, So, g["idx"], g["bits_in"], g["bits_out"], g["norms"], g["codes"], g["scale"],
                            g["zero"], seqlens=seqlens, sm_scale=sm_scale, pairs=pairs)
    worst_s, worst_o = 0.0, 0.0
    for b, h in pairs:
        s_or = so[(b, h)]
        n = len(s_or)
        if n:
            s_g = sc_gpu[b, h, :n]
            floor = SCORE_FLOOR * math.sqrt(float(np.mean(s_or ** 2)))
            rel = np.abs(s_g - s_or) / np.maximum(np.abs(s_or), floor)
            worst_s = max(worst_s, float(rel.max()))
        worst_o = max(worst_o, float(np.max(np.abs(O_gpu[b, h] - Oo[b, h]))))
    assert worst_s <= SCORE_RTOL, worst_s
    assert worst_o <= OUT_ATOL, worst_o
    return {"score_rel": worst_s, "out_abs": worst_o, "O_oracle": Oo}
