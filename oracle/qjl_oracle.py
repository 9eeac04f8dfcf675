"""fp64 CPU oracle of QJL: key sketch, value quantizer, estimator and decode attention.

TEST INFRASTRUCTURE ONLY (see the package docstring): the CUDA library never
calls this module, and this module never calls the library.

All arithmetic is fp64 unless a stored format fixes a rounding (bf16 sketch
entries, fp16 norms, fp16 scale/zero), or a quantisation decision must be taken
in the same precision on both sides (the value codes, decided in IEEE fp32).
Arrays are numpy; a matmul serves as a step where the definition is a matrix
product. There is no blocking, fusion or reordering beyond the definitions.

Readings of the pages that this oracle fixes (the pages are silent on them):
  * S (m x d) and S_out (m_out x d) are i.i.d. N(0,1), drawn by SplitMix64
    (Steele, Lea & Flood, "Fast splittable pseudorandom number generators",
    OOPSLA 2014) -> uniform in (0,1) -> Box-Muller cosine branch, then rounded
    to the nearest bf16 (ties to even). Both come from the stream ``seed``:
    S from counters 1, 2, ..., S_out from counters 2^62 + 1, 2^62 + 2, ...
    One pair serves every batch entry and every head.
  * Outlier channels of a (sequence, kv head): the n_outlier channels with the
    largest sum over the prefill tokens of k_c^2; exact ties go to the lower
    channel index; stored in ascending channel order.
  * The inlier sketch uses k with the outlier coordinates zeroed; the outlier
    sketch (its own quantiser copy: QJL summary, Approach) uses only the
    outlier coordinates, with its own matrix S_out and its own norm.
  * Sign bit = 1 when the projection is >= 0 (so +0 and -0 give 1). Packed
    LSB-first: bit j of 32-bit word w holds sketch row 32*w + j.
  * Norms are fp64, stored as fp16 (round to nearest even).
  * Values: token-wise asymmetric min-max quantisation in groups. zero = fp16(min),
    scale = fp16((max - min) / (2^bits - 1)), code = clamp(rint((v - zero)/scale)),
    every step an IEEE fp32 operation with round-to-nearest-even; scale == 0
    gives code 0. Codes are packed two per byte, the even dimension in the low
    nibble.
  * Score of a cached token (the asymmetric estimator of the QJL summary,
    Approach): sqrt(pi/2)/m * |k_in| * <S q_in, sign(S k_in)> plus the same term
    for the outlier sketch with m_out, |k_out|, S_out, q_out.
  * Attention logits are score * sm_scale with sm_scale = 1/sqrt(d) by default;
    output = softmax(logits) @ dequantised values.
"""

from __future__ import annotations

import math

import numpy as np

__all__ = [
    "splitmix64",
    "uniform01",
    "bf16_round",
    "sketch_matrix",
    "sketch_pair",
    "SKETCH_OUT_OFFSET",
    "select_outliers",
    "pack_bits",
    "unpack_signs",
    "sketch_keys",
    "quantize_values",
    "pack_codes",
    "unpack_codes",
    "dequantize_values",
    "project_query",
    "estimate_scores",
    "softmax",
    "decode_attention",
    "exact_attention",
    "quantize_cache",
    "decode_batch",
    "exact_batch",
    "decode_partial",
    "merge_partials",
    "fp8_e4m3_round",
    "fp8_quantize",
    "fp8_decode_attention",
    "PIN_STATUS",
]

_GAMMA = np.uint64(0x9E3779B97F4A7C15)
_MIX1 = np.uint64(0xBF58476D1CE4E5B9)
_MIX2 = np.uint64(0x94D049BB133111EB)
_TWO_PI = 6.283185307179586  # the fp64 value nearest to 2*pi
_MASK64 = (1 << 64) - 1


# --------------------------------------------------------------------------
# Random sketch matrices
# --------------------------------------------------------------------------

def splitmix64(seed: int, n: np.ndarray) -> np.ndarray:
    """The n-th output (n >= 1) of a SplitMix64 stream whose state starts at ``seed``.

    SplitMix64 (Steele, Lea & Flood 2014): the state advances by the golden
    gamma 0x9E3779B97F4A7C15 before each output, and the output is the state
    passed through the 'mix64' finaliser (xor-shift 30, multiply, xor-shift 27,
    multiply, xor-shift 31). The n-th output therefore depends on seed + n*gamma
    only, which makes the stream counter-based.
    """
    n = np.asarray(n, dtype=np.uint64)
    z = np.uint64(seed & _MASK64) + n * _GAMMA
    z = (z ^ (z >> np.uint64(30))) * _MIX1
    z = (z ^ (z >> np.uint64(27))) * _MIX2
    return z ^ (z >> np.uint64(31))


def uniform01(x: np.ndarray) -> np.ndarray:
    """Map 64 random bits to a double in the open interval (0, 1): ((x >> 12) + 1/2) * 2^-52.

    The top 52 bits give 2^52 equally spaced cell centres, each exactly
    representable, from 2^-53 to 1 - 2^-53.
    """
    top = (np.asarray(x, dtype=np.uint64) >> np.uint64(12)).astype(np.float64)
    return (top + 0.5) * 2.0 ** -52


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round fp64 values to the nearest bfloat16 value (ties to even); result as fp64.

    bfloat16 keeps 7 fraction bits, so the 45 low fraction bits of the double are
    rounded away. Only values in bf16's normal range (or zero) are accepted.
    """
    x = np.ascontiguousarray(x, dtype=np.float64)
    ax = np.abs(x)
    if np.any((ax != 0) & (ax < 2.0 ** -126)) or np.any(~np.isfinite(x)):
        raise ValueError("bf16_round: value outside the normal bf16 range")
    b = x.view(np.uint64)
    lsb = (b >> np.uint64(45)) & np.uint64(1)
    b = (b + np.uint64((1 << 44) - 1) + lsb) & ~np.uint64((1 << 45) - 1)
    return b.view(np.float64)


SKETCH_OUT_OFFSET = 1 << 62  # counter offset of S_out within the stream


def sketch_matrix(seed: int, rows: int, d: int, offset: int = 0) -> np.ndarray:
    """A rows x d matrix of i.i.d. standard normal entries from SplitMix64 stream ``seed``.

    Element e = i*d + c (row-major) takes outputs offset+2e+1 and offset+2e+2 of
    the stream as uniforms u1, u2 and uses the cosine branch of the Box-Muller
    transform, sqrt(-2 ln u1) * cos(2 pi u2); the result is rounded to bf16.
    """
    e = np.arange(rows * d, dtype=np.uint64) * np.uint64(2) + np.uint64(offset)
    u1 = uniform01(splitmix64(seed, e + np.uint64(1)))
    u2 = uniform01(splitmix64(seed, e + np.uint64(2)))
    g = np.sqrt(-2.0 * np.log(u1)) * np.cos(_TWO_PI * u2)
    return bf16_round(g).reshape(rows, d)


def sketch_pair(seed: int, d: int, m: int, m_out: int):
    """The inlier JL matrix S (m x d) and the outlier matrix S_out (m_out x d) of stream ``seed``.

    QJL summary, Approach: the JL matrix is random Gaussian, and the outlier
    channels are sketched apart from the rest, here with a matrix of their own. S_out starts at counter
    2^62 of the same stream, so it never overlaps S of this or a nearby seed.
    """
    S = sketch_matrix(seed, m, d)
    S_out = sketch_matrix(seed, m_out, d, SKETCH_OUT_OFFSET) if m_out > 0 else np.zeros((0, d))
    return S, S_out


# --------------------------------------------------------------------------
# Keys: outlier channels, sign sketch, norms
# --------------------------------------------------------------------------

def select_outliers(K: np.ndarray, n_outlier: int) -> np.ndarray:
    """Channels with the largest energy sum_t K[t, c]^2 over the prefill tokens.

    Outlier channels are the few channels of much larger magnitude ("2 numbers
    out of 128", section "The Real Problem: Outlier Channels"; QJL summary,
    Approach). Exact ties go to the lower channel index. Returned ascending.
    """
    K = np.asarray(K, dtype=np.float64)
    d = K.shape[-1]
    if n_outlier == 0:
        return np.zeros(0, dtype=np.int64)
    energy = np.sum(K * K, axis=0)
    order = np.lexsort((np.arange(d), -energy))  # primary key: -energy, then index
    return np.sort(order[:n_outlier]).astype(np.int64)


def pack_bits(b: np.ndarray) -> np.ndarray:
    """Pack a [..., n] boolean array (n a multiple of 32) into uint32 words, LSB-first."""
    b = np.asarray(b, dtype=bool)
    n = b.shape[-1]
    assert n % 32 == 0
    w = b.reshape(*b.shape[:-1], n // 32, 32).astype(np.uint64)
    weights = np.uint64(1) << np.arange(32, dtype=np.uint64)
    return np.sum(w * weights, axis=-1).astype(np.uint32)


def unpack_signs(words: np.ndarray, n: int) -> np.ndarray:
    """Inverse of pack_bits as signs: bit 1 -> +1.0, bit 0 -> -1.0 (shape [..., n])."""
    words = np.asarray(words, dtype=np.uint64)
    bits = (words[..., None] >> np.arange(32, dtype=np.uint64)) & np.uint64(1)
    bits = bits.reshape(*words.shape[:-1], words.shape[-1] * 32)[..., :n]
    return np.where(bits == 1, 1.0, -1.0)


def _split_channels(K: np.ndarray, idx: np.ndarray):
    out_mask = np.zeros(K.shape[-1], dtype=bool)
    out_mask[np.asarray(idx, dtype=np.int64)] = True
    K_in = np.where(out_mask, 0.0, K)
    K_out = np.where(out_mask, K, 0.0)
    return K_in, K_out


def sketch_keys(K: np.ndarray, S: np.ndarray, S_out: np.ndarray, idx: np.ndarray) -> dict:
    """QJL key quantisation of one head's keys K [T, d].

    QJL summary, Approach: apply the Gaussian JL transform and keep only the sign
    bits plus the key norm; outlier channels get a separate copy. Returns
      bits_in  [T, m/32] uint32   sign(S k_in), packed
      bits_out [T, m_out/32] uint32   sign(S_out k_out), packed
      norms    [T, 2] float16     (|k_in|, |k_out|)
      y_in, y_out                 the fp64 projections (for the exclusion band)
    """
    K = np.asarray(K, dtype=np.float64)
    K_in, K_out = _split_channels(K, idx)
    y_in = K_in @ S.T
    y_out = K_out @ S_out.T
    norm_in = np.sqrt(np.sum(K_in * K_in, axis=-1))
    norm_out = np.sqrt(np.sum(K_out * K_out, axis=-1))
    norms = np.stack([norm_in, norm_out], axis=-1).astype(np.float16)
    return {
        "bits_in": pack_bits(y_in >= 0),
        "bits_out": pack_bits(y_out >= 0) if S_out.shape[0] else np.zeros((K.shape[0], 0), np.uint32),
        "norms": norms,
        "y_in": y_in,
        "y_out": y_out,
        "norm_in": norm_in,
        "norm_out": norm_out,
    }


# --------------------------------------------------------------------------
# Values: token-wise asymmetric min-max quantisation
# --------------------------------------------------------------------------

def quantize_values(V: np.ndarray, bits: int = 4, group: int = 32):
    """Token-wise asymmetric min-max quantisation of V [T, d] in groups of ``group`` dims.

    QJL summary, Limitations: values use standard token-wise quantisation.
    "2 numbers out of 128", "The Obvious Fix": find the range [min, max], divide
    it into 2^bits equally spaced levels and round each number to the nearest.
    Levels are zero + c*scale, c = 0 .. 2^bits-1, with zero = min and
    scale = (max-min)/(2^bits-1), both stored as fp16. Each step below is one
    IEEE fp32 operation rounded to nearest even, so that the code decision is
    taken in one stated precision.
    Returns (codes [T, d] uint8, scale [T, d/group] fp16, zero [T, d/group] fp16).
    """
    V32 = np.asarray(V, dtype=np.float32)
    if not np.array_equal(V32.astype(np.float64), np.asarray(V, dtype=np.float64)):
        raise ValueError("quantize_values: inputs must be fp32-representable")
    T, d = V32.shape
    assert d % group == 0
    levels = np.float32(2 ** bits - 1)
    Vg = V32.reshape(T, d // group, group)
    lo = Vg.min(axis=-1)
    hi = Vg.max(axis=-1)
    zero_h = lo.astype(np.float16)
    scale_h = ((hi - lo) / levels).astype(np.float16)
    diff = Vg - zero_h.astype(np.float32)[..., None]
    with np.errstate(divide="ignore", invalid="ignore"):
        x = diff / scale_h.astype(np.float32)[..., None]
    code = np.clip(np.rint(x), 0, levels)
    code = np.where((scale_h == 0)[..., None], 0, code)
    return code.reshape(T, d).astype(np.uint8), scale_h, zero_h


def pack_codes(codes: np.ndarray) -> np.ndarray:
    """Two 4-bit codes per byte: dimension 2i in the low nibble, 2i+1 in the high nibble."""
    c = np.asarray(codes, dtype=np.uint8)
    return (c[..., 0::2] | (c[..., 1::2] << 4)).astype(np.uint8)


def unpack_codes(packed: np.ndarray) -> np.ndarray:
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty(p.shape[:-1] + (p.shape[-1] * 2,), dtype=np.uint8)
    out[..., 0::2] = p & 0x0F
    out[..., 1::2] = p >> 4
    return out


def dequantize_values(codes: np.ndarray, scale: np.ndarray, zero: np.ndarray) -> np.ndarray:
    """v_hat = zero + code * scale in fp64, with the group's fp16 scale and zero."""
    codes = np.asarray(codes, dtype=np.float64)
    T, d = codes.shape
    G = scale.shape[-1]
    g = d // G
    s = np.repeat(np.asarray(scale, dtype=np.float64), g, axis=-1)
    z = np.repeat(np.asarray(zero, dtype=np.float64), g, axis=-1)
    return z + codes * s


# --------------------------------------------------------------------------
# Decode: query projection, estimator, softmax, value accumulation
# --------------------------------------------------------------------------

def project_query(q: np.ndarray, S: np.ndarray, S_out: np.ndarray, idx: np.ndarray):
    """S q_in and S_out q_out in fp64: the query is JL-projected without quantisation.

    QJL summary, Approach. q_in is q with the outlier coordinates zeroed and
    q_out keeps only them, matching the split of the keys.
    """
    q = np.asarray(q, dtype=np.float64)
    q_in, q_out = _split_channels(q[None, :], idx)
    return S @ q_in[0], S_out @ q_out[0]


def estimate_scores(sq_in, sq_out, bits_in, bits_out, norms, m: int, m_out: int) -> np.ndarray:
    """Unbiased asymmetric estimates of <q, k_t> for every cached token t.

    QJL summary, Approach and Surprising findings: with the query projected
    unquantised and the key reduced to sign(S k) and |k|, the estimator
    sqrt(pi/2)/m * |k| * <S q, sign(S k)> is unbiased for <q, k>. The outlier
    sketch adds the same term with its own matrix, size and norm.
    """
    norms = np.asarray(norms, dtype=np.float64)
    sgn_in = unpack_signs(bits_in, m)
    score = math.sqrt(math.pi / 2.0) / m * norms[:, 0] * (sgn_in @ np.asarray(sq_in, np.float64))
    if m_out > 0:
        sgn_out = unpack_signs(bits_out, m_out)
        score = score + math.sqrt(math.pi / 2.0) / m_out * norms[:, 1] * (sgn_out @ np.asarray(sq_out, np.float64))
    return score


def softmax(x: np.ndarray) -> np.ndarray:
    """exp(x - max x) / sum exp(x - max x) ("Your Brain Already Runs on 1-Bit Keys", "Why Truncation Kills")."""
    x = np.asarray(x, dtype=np.float64)
    if x.size == 0:
        return x.copy()
    e = np.exp(x - np.max(x))
    return e / np.sum(e)


def decode_attention(q, S, S_out, idx, bits_in, bits_out, norms, codes, scale, zero, sm_scale=None):
    """Attention output of one query head over one cached sequence, using the QJL cache.

    score_t = QJL estimate of <q, k_t>; p = softmax(sm_scale * score);
    out = sum_t p_t * dequantised v_t. Returns (out [d], score [T]). An empty
    cache (T = 0) gives a zero output.
    """
    q = np.asarray(q, dtype=np.float64)
    d = q.shape[0]
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(d)
    m, m_out = S.shape[0], S_out.shape[0]
    sq_in, sq_out = project_query(q, S, S_out, idx)
    score = estimate_scores(sq_in, sq_out, bits_in, bits_out, norms, m, m_out)
    if score.size == 0:
        return np.zeros(d), score
    p = softmax(sm_scale * score)
    out = p @ dequantize_values(codes, scale, zero)
    return out, score


def exact_attention(q, K, V, sm_scale=None) -> np.ndarray:
    """softmax(sm_scale * K q) @ V in fp64 on the original, unquantised cache."""
    q = np.asarray(q, dtype=np.float64)
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(q.shape[0])
    K = np.asarray(K, dtype=np.float64)
    if K.shape[0] == 0:
        return np.zeros(q.shape[0])
    return softmax(sm_scale * (K @ q)) @ np.asarray(V, dtype=np.float64)


# --------------------------------------------------------------------------
# Batched helpers: plain loops over (batch, head)
# --------------------------------------------------------------------------

def quantize_cache(K, V, S, S_out, n_outlier, bits=4, group=32, idx=None) -> dict:
    """Quantise a whole cache K, V [B, Hkv, T, d]: outliers, signs, norms, value codes.

    ``idx`` [B, Hkv, n_outlier] may be given (append mode: the channels chosen at
    prefill); otherwise the channels are selected from K itself (prefill mode).
    """
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    B, H, T, d = K.shape
    m, m_out = S.shape[0], S_out.shape[0]
    out = {
        "idx": np.zeros((B, H, n_outlier), np.int64),
        "bits_in": np.zeros((B, H, T, m // 32), np.uint32),
        "bits_out": np.zeros((B, H, T, m_out // 32), np.uint32),
        "norms": np.zeros((B, H, T, 2), np.float16),
        "y_in": np.zeros((B, H, T, m)),
        "y_out": np.zeros((B, H, T, m_out)),
        "norm_in": np.zeros((B, H, T)),
        "norm_out": np.zeros((B, H, T)),
        "codes": np.zeros((B, H, T, d), np.uint8),
        "scale": np.zeros((B, H, T, d // group), np.float16),
        "zero": np.zeros((B, H, T, d // group), np.float16),
    }
    for b in range(B):
        for h in range(H):
            ix = select_outliers(K[b, h], n_outlier) if idx is None else np.asarray(idx[b, h], np.int64)
            out["idx"][b, h] = ix
            ks = sketch_keys(K[b, h], S, S_out, ix)
            for key in ("bits_in", "bits_out", "norms", "y_in", "y_out", "norm_in", "norm_out"):
                out[key][b, h] = ks[key]
            c, s, z = quantize_values(V[b, h], bits, group)
            out["codes"][b, h], out["scale"][b, h], out["zero"][b, h] = c, s, z
    return out


def decode_batch(Q, S, S_out, idx, bits_in, bits_out, norms, codes, scale, zero,
                 seqlens=None, sm_scale=None, pairs=None):
    """Decode attention for Q [B, Hq, d] over a quantised cache [B, Hkv, T, ...].

    Query head h reads kv head h // (Hq // Hkv) (grouped-query attention with
    contiguous groups). ``seqlens`` [B] limits the cached tokens per sequence.
    ``pairs`` optionally restricts the work to a list of (b, hq) pairs; other
    outputs stay zero. Returns (O [B, Hq, d], scores list-of-lists).
    """
    Q = np.asarray(Q, dtype=np.float64)
    B, Hq, d = Q.shape
    Hkv = bits_in.shape[1]
    g = Hq // Hkv
    T = bits_in.shape[2]
    O = np.zeros((B, Hq, d))
    scores = {}
    todo = pairs if pairs is not None else [(b, h) for b in range(B) for h in range(Hq)]
    for b, h in todo:
        hk = h // g
        n = T if seqlens is None else int(seqlens[b])
        o, s = decode_attention(Q[b, h], S, S_out, idx[b, hk], bits_in[b, hk, :n], bits_out[b, hk, :n],
                                norms[b, hk, :n], codes[b, hk, :n], scale[b, hk, :n], zero[b, hk, :n], sm_scale)
        O[b, h] = o
        scores[(b, h)] = s
    return O, scores


def exact_batch(Q, K, V, seqlens=None, sm_scale=None, pairs=None) -> np.ndarray:
    """fp64 exact attention for Q [B, Hq, d] over K, V [B, Hkv, T, d] (same GQA mapping)."""
    Q = np.asarray(Q, dtype=np.float64)
    B, Hq, d = Q.shape
    Hkv, T = K.shape[1], K.shape[2]
    g = Hq // Hkv
    O = np.zeros((B, Hq, d))
    todo = pairs if pairs is not None else [(b, h) for b in range(B) for h in range(Hq)]
    for b, h in todo:
        n = T if seqlens is None else int(seqlens[b])
        O[b, h] = exact_attention(Q[b, h], K[b, h // g, :n], V[b, h // g, :n], sm_scale)
    return O


# --------------------------------------------------------------------------
# Context-parallel decode: one shard of the cached tokens per rank
# --------------------------------------------------------------------------
# A long context can be split over ranks by token position ("2 numbers out of
# 128 destroy the entire KV cache" (Towards AI), "The Memory Math": the cache
# grows linearly with the context and outgrows one device). softmax(x) is
# exp(x - M) / sum exp(x - M) for any M >= max x ("Your Brain Already Runs on
# 1-Bit Keys", "Why Truncation Kills"), so each shard can report its logits'
# maximum, the sum of exponentials below it and the unnormalised output, and
# the shards' reports combine exactly.

def decode_partial(q, S, S_out, idx, bits_in, bits_out, norms, codes, scale, zero, sm_scale=None):
    """One shard's part of decode attention for one query head.

    With logits x_t = sm_scale * score_t over the shard's tokens: mx = max_t x_t,
    l = sum_t exp(x_t - mx), o = sum_t exp(x_t - mx) * dequantised v_t. An empty
    shard gives (zeros, -inf, 0), the neutral element of merge_partials.
    Returns (o [d], mx, l).
    """
    q = np.asarray(q, dtype=np.float64)
    d = q.shape[0]
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(d)
    m, m_out = S.shape[0], S_out.shape[0]
    sq_in, sq_out = project_query(q, S, S_out, idx)
    x = sm_scale * estimate_scores(sq_in, sq_out, bits_in, bits_out, norms, m, m_out)
    if x.size == 0:
        return np.zeros(d), -math.inf, 0.0
    mx = float(np.max(x))
    w = np.exp(x - mx)
    return w @ dequantize_values(codes, scale, zero), mx, float(np.sum(w))


def merge_partials(parts) -> np.ndarray:
    """Attention output from the shards' (o, mx, l): with M = max_r mx_r,
    out = sum_r o_r exp(mx_r - M) / sum_r l_r exp(mx_r - M); zero when every
    shard is empty."""
    parts = list(parts)
    d = len(parts[0][0])
    M = max(p[1] for p in parts)
    if M == -math.inf:
        return np.zeros(d)
    num = np.zeros(d)
    den = 0.0
    for o, mx, l in parts:
        if mx == -math.inf:
            continue
        f = math.exp(mx - M)
        num += f * np.asarray(o, dtype=np.float64)
        den += f * l
    return num / den


# --------------------------------------------------------------------------
# Comparison point: an FP8 KV cache (TurboQuant slides, section 05: storing
# the cache in FP8 halves it at no algorithmic cost on hardware with FP8
# support). The slides name no variant or scaling: E4M3 (OCP "FN": 1 sign,
# 4 exponent bits with bias 7, 3 mantissa bits, largest finite 448) with one
# scale for K and one for V is taken here.
# --------------------------------------------------------------------------

def fp8_e4m3_round(x: np.ndarray) -> np.ndarray:
    """Round to the nearest E4M3 value, ties to even, saturating at +-448; result as fp64.

    Normal values: 2^e (1 + k/8), e in [-6, 8]; subnormals: k 2^-9, k < 8."""
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.clip(e, -6, 8)                      # below 2^-6 the spacing stays 2^-9
    quantum = np.exp2(e - 3)
    r = np.round(a / quantum) * quantum        # np.round: half to even; a / quantum is exact (power of 2)
    r = np.minimum(r, 448.0)
    return np.where(x < 0, -r, r)


def fp8_quantize(x: np.ndarray, scale: float) -> np.ndarray:
    """E4M3 code values of x / scale, the quotient taken as one IEEE fp32 division."""
    q = np.asarray(x, dtype=np.float32) / np.float32(scale)
    return fp8_e4m3_round(q.astype(np.float64))


def fp8_decode_attention(q, K8, V8, k_scale: float, v_scale: float, sm_scale=None) -> np.ndarray:
    """Exact softmax attention over the dequantised FP8 cache: K = K8 k_scale, V = V8 v_scale (fp64)."""
    return exact_attention(q, np.asarray(K8, dtype=np.float64) * float(np.float32(k_scale)),
                           np.asarray(V8, dtype=np.float64) * float(np.float32(v_scale)), sm_scale)


# Which -m "not gpu" test pins each function (none is left unpinned).
PIN_STATUS = {
    "splitmix64": "tests/test_oracle_pins.py::test_splitmix64_published_outputs",
    "sketch_matrix": "tests/test_oracle_pins.py::test_sketch_moments (moments of N(0,1), bf16 grid)",
    "select_outliers": "tests/test_oracle_pins.py::test_select_outliers_planted_and_ties",
    "sketch_keys": "tests/test_oracle_pins.py::test_estimator_bruteforce_tiny, test_sign_invariants",
    "quantize_values": "tests/test_oracle_pins.py::test_minmax_* (page worked examples), test_value_code_properties",
    "estimate_scores": "tests/test_oracle_pins.py::test_unbiased_over_seeds, test_variance_closed_form",
    "softmax": "tests/test_oracle_pins.py::test_softmax_page_examples",
    "decode_attention": "tests/test_oracle_pins.py::test_decode_closed_forms",
    "exact_attention": "tests/test_oracle_pins.py::test_exact_dot_page_examples, test_decode_closed_forms",
    "decode_partial": "tests/test_oracle_pins.py::test_partials_merge_to_the_whole_decode (split invariance)",
    "merge_partials": "tests/test_oracle_pins.py::test_partials_merge_to_the_whole_decode, test_merge_neutral_and_order",
    "fp8_e4m3_round": "tests/test_oracle_pins.py::test_fp8_grid_and_ties (the format's 256 codes), test_fp8_matches_torch",
    "fp8_quantize": "tests/test_oracle_pins.py::test_fp8_matches_torch (fp32 quotient then torch's float8_e4m3fn)",
    "fp8_decode_attention": "tests/test_oracle_pins.py::test_fp8_decode_is_exact_attention_on_the_grid",
}
