"""Pins of the fp64 oracle against what the pages and the mathematics fix (CPU only).

Each test checks the oracle against something other than itself: numbers the
pages print for their worked examples (tests/golden/page_examples.json), the
published SplitMix64 outputs, closed forms (mean and variance of the QJL
estimator), invariants, library routines for special cases, and brute force in
plain Python loops on tiny inputs.
"""

import math

import numpy as np
import pytest

import oracle as O


# ---------------------------------------------------------------- generator

def test_splitmix64_published_outputs():
    # SplitMix64 started from state 0 gives these first outputs (Steele, Lea &
    # Flood 2014; the same values appear in the reference implementation's
    # published test output).
    out = O.splitmix64(0, np.arange(1, 4, dtype=np.uint64))
    assert [int(x) for x in out] == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]


def test_uniform01_open_interval():
    u = O.uniform01(np.array([0, (1 << 64) - 1], dtype=np.uint64))
    assert u[0] == 2.0 ** -53 and 0 < u[0]
    assert u[1] == 1.0 - 2.0 ** -53 and u[1] < 1


def test_bf16_round_matches_library_on_fp32_inputs():
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(7)
    x = (rng.standard_normal(200000) * np.exp(rng.uniform(-20, 20, 200000))).astype(np.float32)
    # ties: fp32 values exactly half-way between bf16 neighbours
    ties = ((np.arange(0x3E00, 0x4200, dtype=np.uint32) << 16) | 0x8000).view(np.float32)
    x = np.concatenate([x, ties, -ties]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    got = O.bf16_round(x.astype(np.float64))
    assert np.array_equal(got, ref)


def test_sketch_moments():
    S = O.sketch_matrix(1, 1024, 1024).ravel()
    n = S.size
    assert np.all((S.astype(np.float32).view(np.uint32) & 0xFFFF) == 0)  # on the bf16 grid
    assert abs(S.mean()) < 5 / math.sqrt(n)
    var = S.var()
    assert abs(var - 1.0) < 5 * math.sqrt(2.0 / n) + 2e-5  # bf16 rounding adds ~1e-5 variance
    kurt = np.mean(S ** 4) / var ** 2
    assert abs(kurt - 3.0) < 5 * math.sqrt(24.0 / n)
    frac1 = np.mean(np.abs(S) < 1.0)
    assert abs(frac1 - 0.682689492) < 5 * math.sqrt(0.6827 * 0.3173 / n)
    assert abs(np.mean(S > 0) - 0.5) < 5 * math.sqrt(0.25 / n)


def test_sketch_pair_streams_distinct_and_deterministic():
    S, So = O.sketch_pair(3, 64, 64, 32)
    S2, So2 = O.sketch_pair(3, 64, 64, 32)
    assert np.array_equal(S, S2) and np.array_equal(So, So2)
    S4, So4 = O.sketch_pair(4, 64, 64, 32)
    assert not np.array_equal(S[:32], So) and not np.array_equal(S4[:32], So)
    assert not np.array_equal(S, S4)
    # rows of S do not depend on m: S(m=64) is the first 64 rows of S(m=128)
    S128, _ = O.sketch_pair(3, 64, 128, 0)
    assert np.array_equal(S128[:64], S)


# ---------------------------------------------------------------- bits

def test_pack_bits_layout():
    b = np.zeros((1, 64), bool)
    b[0, 0] = True
    b[0, 33] = True
    b[0, 63] = True
    w = O.pack_bits(b)
    assert w.dtype == np.uint32 and w.tolist() == [[1, (1 << 1) | (1 << 31)]]
    s = O.unpack_signs(w, 64)
    assert s[0, 0] == 1 and s[0, 1] == -1 and s[0, 33] == 1 and s[0, 63] == 1 and s.sum() == -58


# ---------------------------------------------------------------- estimator

def _brute_score(q, k, S, So, idx, m, m_out):
    """The estimator written out with plain loops and +/-1 signs."""
    d = len(q)
    outs = set(int(i) for i in idx)
    kin = [0.0 if c in outs else float(k[c]) for c in range(d)]
    kout = [float(k[c]) if c in outs else 0.0 for c in range(d)]
    qin = [0.0 if c in outs else float(q[c]) for c in range(d)]
    qout = [float(q[c]) if c in outs else 0.0 for c in range(d)]

    def part(M, rows, kv, qv):
        if rows == 0:
            return 0.0
        nrm = float(np.float16(math.sqrt(sum(x * x for x in kv))))
        acc = 0.0
        for i in range(rows):
            y = sum(float(M[i][c]) * kv[c] for c in range(d))
            sgn = 1.0 if y >= 0 else -1.0
            acc += sgn * sum(float(M[i][c]) * qv[c] for c in range(d))
        return math.sqrt(math.pi / 2) / rows * nrm * acc

    return part(S, m, kin, qin) + part(So, m_out, kout, qout)


def _oracle_scores(Q, K, S, So, idx):
    ks = O.sketch_keys(K, S, So, idx)
    sq_in, sq_out = O.project_query(Q, S, So, idx)
    return O.estimate_scores(sq_in, sq_out, ks["bits_in"], ks["bits_out"], ks["norms"], S.shape[0], So.shape[0])


@pytest.mark.parametrize("n_o,m_out", [(0, 0), (2, 32), (0, 32)])
def test_estimator_bruteforce_tiny(n_o, m_out):
    rng = np.random.default_rng(11)
    d, m, T = 8, 32, 5
    S, So = O.sketch_pair(5, d, m, m_out)
    K = rng.standard_normal((T, d))
    K[:, [1, 6]] *= 20.0
    q = rng.standard_normal(d)
    idx = O.select_outliers(K, n_o)
    got = _oracle_scores(q, K, S, So, idx)
    ref = [_brute_score(q, K[t], S, So, idx, m, m_out) for t in range(T)]
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)
    if n_o == 0 and m_out > 0:
        # no outlier channels: the outlier norm is 0 and the score is plain QJL
        got0 = _oracle_scores(q, K, S, So[:0], idx)
        np.testing.assert_allclose(got, got0, rtol=1e-13, atol=1e-13)


def _est_over_seeds(q, k, seeds, m, m_out=0, n_o=0):
    d = len(q)
    idx = np.argsort(-np.abs(k))[:n_o] if n_o else np.zeros(0, np.int64)
    idx = np.sort(idx)
    vals = []
    for s in seeds:
        S, So = O.sketch_pair(int(s), d, m, m_out)
        vals.append(_oracle_scores(q, k[None, :], S, So, idx)[0])
    return np.array(vals)


def _pairs():
    rng = np.random.default_rng(3)
    d = 16
    q1, k1 = rng.standard_normal(d), rng.standard_normal(d)
    k2 = 0.8 * q1 + 0.2 * rng.standard_normal(d)  # strongly aligned pair
    k3 = rng.standard_normal(d)
    k3[[2, 9]] *= 20.0  # outlier channels
    return [(q1, k1, 0, 0), (q1, k2, 0, 0), (q1, k3, 32, 2)]


@pytest.mark.parametrize("case", range(3))
def test_unbiased_over_seeds(case):
    # QJL summary, Approach and Surprising findings: quantising only the key side
    # to signs gives an UNBIASED estimate of <q, k>.
    q, k, m_out, n_o = _pairs()[case]
    N = 2000
    for m, base in ((64, 10_000), (256, 20_000)):
        seeds = base + 2 * np.arange(N)  # distinct seeds, an independent range per m
        e = _est_over_seeds(q, k, seeds, m, m_out, n_o)
        z = (e.mean() - q @ k) / (e.std(ddof=1) / math.sqrt(N))
        assert abs(z) < 3.0, (m, z)


def test_variance_closed_form():
    # For Gaussian S the terms sqrt(pi/2)|k|(s.q)sign(s.k) are i.i.d. with mean
    # q.k and second moment (pi/2)|q|^2|k|^2, so Var = ((pi/2)|q|^2|k|^2 - (q.k)^2)/m.
    rng = np.random.default_rng(5)
    d = 16
    q, k = rng.standard_normal(d), rng.standard_normal(d)
    closed = lambda m: ((math.pi / 2) * (q @ q) * (k @ k) - (q @ k) ** 2) / m
    ms, vs = [32, 128, 512], []
    for j, m in enumerate(ms):
        e = _est_over_seeds(q, k, 40_000 + 5000 * j + np.arange(2000), m)
        v = e.var(ddof=1)
        vs.append(v)
        assert 0.85 < v / closed(m) < 1.15, (m, v / closed(m))
    slope = np.polyfit(np.log(ms), np.log(vs), 1)[0]
    assert -1.1 < slope < -0.9
    # for contrast: the unquantised JL estimator has variance (|q|^2|k|^2 + (q.k)^2)/m,
    # which is not the one the sign estimator shows
    jl = ((q @ q) * (k @ k) + (q @ k) ** 2) / 128
    assert abs(vs[1] / jl - 1) > 0.15


def test_large_m_converges():
    rng = np.random.default_rng(9)
    d = 16
    q, k = rng.standard_normal(d), rng.standard_normal(d)
    m = 16384
    e = _est_over_seeds(q, k, [777], m)[0]
    sigma = math.sqrt(((math.pi / 2) * (q @ q) * (k @ k) - (q @ k) ** 2) / m)
    assert abs(e - q @ k) < 4 * sigma
    assert sigma < 0.05 * math.sqrt((q @ q) * (k @ k))


def test_sign_invariants():
    rng = np.random.default_rng(13)
    d, m, m_out, T = 32, 64, 32, 50
    S, So = O.sketch_pair(21, d, m, m_out)
    K = rng.standard_normal((T, d))
    idx = np.array([4, 17])
    a = O.sketch_keys(K, S, So, idx)
    b = O.sketch_keys(-K, S, So, idx)
    nz = (a["y_in"] != 0).reshape(T, m // 32, 32).all(-1)
    assert np.all(np.where(nz, a["bits_in"] ^ b["bits_in"], 0xFFFFFFFF) == 0xFFFFFFFF)
    c = O.sketch_keys(4.0 * K, S, So, idx)  # power-of-two scale: exact
    assert np.array_equal(c["bits_in"], a["bits_in"]) and np.array_equal(c["bits_out"], a["bits_out"])
    np.testing.assert_array_equal(c["norms"].astype(np.float64), 4.0 * a["norms"].astype(np.float64))
    # linear in q (bits fixed)
    q1, q2 = rng.standard_normal(d), rng.standard_normal(d)
    sc = lambda q: O.estimate_scores(*O.project_query(q, S, So, idx), a["bits_in"], a["bits_out"], a["norms"], m, m_out)
    np.testing.assert_allclose(sc(2.5 * q1 - 0.75 * q2), 2.5 * sc(q1) - 0.75 * sc(q2), rtol=1e-10, atol=1e-10)


def test_select_outliers_planted_and_ties():
    rng = np.random.default_rng(17)
    K = rng.standard_normal((300, 128))
    planted = np.sort(rng.choice(128, 8, replace=False))
    K[:, planted] *= rng.uniform(10, 50, 8)
    assert np.array_equal(O.select_outliers(K, 8), planted)
    # exact tie between channels 5 and 2: the lower index wins
    K2 = np.ones((4, 8))
    K2[:, 5] = 3.0
    K2[:, 2] = -3.0
    assert O.select_outliers(K2, 1).tolist() == [2]
    assert O.select_outliers(K2, 2).tolist() == [2, 5]
    assert O.select_outliers(K2, 0).size == 0


# ---------------------------------------------------------------- values

def test_minmax_2bit_page_example(golden):
    ex = golden["towardsai_2bit"]
    V = np.array([ex["key"]])
    codes, scale, zero = O.quantize_values(V.astype(np.float32).astype(np.float64), bits=ex["bits"], group=3)
    assert codes[0].tolist() == ex["bucket_printed"]
    deq = O.dequantize_values(codes, scale, zero)[0]
    np.testing.assert_allclose(deq, ex["compressed_printed"], atol=0.005)
    q = np.array(ex["query"])
    assert abs(q @ deq - ex["compressed_dot_printed"]) < 0.005
    assert abs(q @ np.array(ex["key"]) - ex["dot_printed"]) < 0.005


def test_minmax_3bit_outlier_page_example(golden):
    ex = golden["towardsai_3bit_outlier"]
    V = np.array([ex["key"]], dtype=np.float32).astype(np.float64)
    codes, scale, zero = O.quantize_values(V, bits=ex["bits"], group=8)
    levels = zero[0, 0].astype(np.float64) + np.arange(8) * scale[0, 0].astype(np.float64)
    np.testing.assert_allclose(levels, ex["levels_printed"], atol=0.06)
    assert abs(float(scale[0, 0]) - ex["step_printed"]) < 0.01
    deq = O.dequantize_values(codes, scale, zero)[0]
    np.testing.assert_allclose(deq, ex["compressed_printed"], atol=0.06)
    assert codes[0].tolist() == [4, 4, 7, 4, 0, 4, 4, 4]
    q = np.array(ex["query"], dtype=np.float64)
    assert abs(q @ V[0] - ex["dot_printed"]) < 1e-5
    assert abs(q @ deq - ex["compressed_dot_printed"]) < 0.1  # page rounds levels to 0.1


def test_value_code_properties():
    rng = np.random.default_rng(19)
    V = rng.standard_normal((400, 128)).astype(np.float32)
    V[:, 7] *= 30
    V = V.astype(np.float64)
    codes, scale, zero = O.quantize_values(V, 4, 32)
    assert codes.max() <= 15
    Vg = V.reshape(400, 4, 32)
    cg = codes.reshape(400, 4, 32)
    rows, grp = np.arange(400)[:, None], np.arange(4)[None, :]
    assert np.all(cg[rows, grp, Vg.argmin(-1)] == 0)
    assert np.all(cg[rows, grp, Vg.argmax(-1)] == 15)
    s = scale.astype(np.float64)[..., None]
    z = zero.astype(np.float64)[..., None]
    deq = z + cg * s
    rng_ = (Vg.max(-1) - Vg.min(-1))[..., None]
    bound = s / 2 + 16 * 2.0 ** -11 * rng_ + 2.0 ** -11 * np.abs(z)
    assert np.all(np.abs(deq - Vg) <= bound)
    # brute force: the code is the nearest level (ties within fp32 rounding excepted)
    lv = z[..., None] + np.arange(16)[None, None, None, :] * s[..., None]
    dist = np.abs(Vg[..., None] - lv)
    best = dist.argmin(-1)
    second = np.sort(dist, -1)[..., 1]
    clear = (second - dist.min(-1)) > 1e-6 * s
    assert np.array_equal(np.where(clear, cg, 0), np.where(clear, best, 0))
    # constant group -> scale 0 -> code 0, dequantises exactly when fp16-representable
    c0, s0, z0 = O.quantize_values(np.full((1, 32), 0.5), 4, 32)
    assert s0[0, 0] == 0 and np.all(c0 == 0) and O.dequantize_values(c0, s0, z0)[0, 0] == 0.5
    packed = O.pack_codes(codes)
    assert packed.shape == (400, 64) and np.array_equal(O.unpack_codes(packed), codes)
    assert packed[0, 0] == (codes[0, 0] | (codes[0, 1] << 4))


# ---------------------------------------------------------------- softmax / attention

def test_softmax_page_examples(golden):
    b = golden["onebit_blog_dot"]
    np.testing.assert_allclose(O.softmax(np.array(b["softmax_in"])), b["softmax_printed"], atol=0.005)
    np.testing.assert_allclose(O.softmax(np.array(b["softmax_truncated_in"])), b["softmax_truncated_printed"], atol=0.005)
    t = golden["towardsai_2bit"]
    np.testing.assert_allclose(O.softmax(np.array(t["scores_printed"])), t["weights_printed"], atol=0.005)
    np.testing.assert_allclose(O.softmax(np.array(t["compressed_scores_printed"])), t["compressed_weights_printed"], atol=0.011)


def test_exact_dot_page_examples(golden):
    # exact_attention with a one-hot value matrix returns softmax(K q * scale):
    # with K holding the page's keys, the weights follow the page's dot products.
    t = golden["turboquant_8dim"]
    k, q = np.array(t["k"]), np.array(t["q"])
    assert abs(q @ k - t["dot_printed"]) < 5e-5
    b = golden["onebit_blog_dot"]
    qo, kc = np.array(b["query_on"]), np.array(b["key_cat"])
    assert abs(qo @ kc - 16.2021) < 1e-9 and abs(qo @ kc - b["dot_printed"]) < 0.002
    K = np.stack([kc, np.zeros(8)])
    w = O.exact_attention(qo, K, np.eye(2), sm_scale=1.0)
    np.testing.assert_allclose(w, [1 / (1 + math.exp(-16.2021)), 1 / (1 + math.exp(16.2021))], rtol=1e-9)
    # the 1-bit key printed on the blog page is the sign pattern of the key
    assert np.array_equal(np.where(kc >= 0, 1, -1), b["sign_key_printed"])
    # the quantised dot printed on the slides does not follow from its printed centroids
    assert abs(q @ np.array(t["printed_centroids"]) - (-0.9025)) < 1e-9
    assert abs(q @ np.array(t["printed_centroids"]) - t["quantized_dot_printed"]) > 0.25


def test_decode_closed_forms():
    rng = np.random.default_rng(23)
    d, m, m_out, T = 32, 64, 32, 40
    S, So = O.sketch_pair(2, d, m, m_out)
    idx = np.array([3, 30])
    V = rng.standard_normal((T, d))
    codes, scale, zero = O.quantize_values(V.astype(np.float32).astype(np.float64), 4, 32)
    deq = O.dequantize_values(codes, scale, zero)
    q = rng.standard_normal(d)
    # identical keys: uniform weights, output = mean of the dequantised values
    K = np.tile(rng.standard_normal(d), (T, 1))
    ks = O.sketch_keys(K, S, So, idx)
    out, sc = O.decode_attention(q, S, So, idx, ks["bits_in"], ks["bits_out"], ks["norms"], codes, scale, zero)
    np.testing.assert_allclose(out, deq.mean(0), rtol=1e-12, atol=1e-12)
    # one key far larger along q than the others: its value wins
    K = rng.standard_normal((T, d))
    K[17] = 200.0 * q / np.linalg.norm(q)
    ks = O.sketch_keys(K, S, So, idx)
    out, sc = O.decode_attention(q, S, So, idx, ks["bits_in"], ks["bits_out"], ks["norms"], codes, scale, zero)
    assert np.argmax(sc) == 17
    np.testing.assert_allclose(out, deq[17], atol=1e-6)
    # sm_scale = 0: uniform
    out0, _ = O.decode_attention(q, S, So, idx, ks["bits_in"], ks["bits_out"], ks["norms"], codes, scale, zero, sm_scale=0.0)
    np.testing.assert_allclose(out0, deq.mean(0), rtol=1e-12, atol=1e-12)
    # empty cache
    oute, sce = O.decode_attention(q, S, So, idx, ks["bits_in"][:0], ks["bits_out"][:0], ks["norms"][:0],
                                   codes[:0], scale[:0], zero[:0])
    assert sce.size == 0 and np.all(oute == 0)
    # brute force: weights from the loop estimator, plain weighted sum
    Kt = rng.standard_normal((6, d))
    ks = O.sketch_keys(Kt, S, So, idx)
    out, _ = O.decode_attention(q, S, So, idx, ks["bits_in"], ks["bits_out"], ks["norms"], codes[:6], scale[:6], zero[:6])
    s_bf = [_brute_score(q, Kt[t], S, So, idx, m, m_out) / math.sqrt(d) for t in range(6)]
    mx = max(s_bf)
    w = [math.exp(x - mx) for x in s_bf]
    w = [x / sum(w) for x in w]
    ref = [sum(w[t] * deq[t, c] for t in range(6)) for c in range(d)]
    np.testing.assert_allclose(out, ref, rtol=1e-11, atol=1e-12)
    # exact attention against loops
    e = O.exact_attention(q, Kt, V[:6])
    lg = [sum(q[c] * Kt[t, c] for c in range(d)) / math.sqrt(d) for t in range(6)]
    mx = max(lg)
    w = [math.exp(x - mx) for x in lg]
    w = [x / sum(w) for x in w]
    np.testing.assert_allclose(e, [sum(w[t] * V[t, c] for t in range(6)) for c in range(d)], rtol=1e-11, atol=1e-12)


def test_batch_gqa_mapping():
    rng = np.random.default_rng(29)
    B, Hq, Hkv, T, d = 2, 4, 2, 33, 32
    S, So = O.sketch_pair(8, d, 32, 32)
    K = rng.standard_normal((B, Hkv, T, d))
    V = rng.standard_normal((B, Hkv, T, d)).astype(np.float32).astype(np.float64)
    Q = rng.standard_normal((B, Hq, d))
    c = O.quantize_cache(K, V, S, So, 2)
    seqlens = np.array([33, 5])
    Ob, sc = O.decode_batch(Q, S, So, c["idx"], c["bits_in"], c["bits_out"], c["norms"], c["codes"],
                            c["scale"], c["zero"], seqlens=seqlens)
    for b in range(B):
        for h in range(Hq):
            hk = h // 2
            n = seqlens[b]
            o, _ = O.decode_attention(Q[b, h], S, So, c["idx"][b, hk], c["bits_in"][b, hk, :n], c["bits_out"][b, hk, :n],
                                      c["norms"][b, hk, :n], c["codes"][b, hk, :n], c["scale"][b, hk, :n], c["zero"][b, hk, :n])
            np.testing.assert_array_equal(Ob[b, h], o)
            assert len(sc[(b, h)]) == n
    # with a long sketch the estimator-based output approaches exact attention
    S2, So2 = O.sketch_pair(8, d, 8192, 1024)
    c2 = O.quantize_cache(K, V, S2, So2, 2)
    Ob2, _ = O.decode_batch(Q, S2, So2, c2["idx"], c2["bits_in"], c2["bits_out"], c2["norms"], c2["codes"],
                            c2["scale"], c2["zero"], seqlens=seqlens)
    Ex = O.exact_batch(Q, K, V, seqlens=seqlens)
    err_long = np.max(np.abs(Ex - Ob2))
    assert err_long < 0.15 and err_long < np.max(np.abs(Ex - Ob))


# ----------------------------------------------------------------------------- value codes against exact arithmetic

def _round_f32(x):
    """The fp32 value nearest to the rational x (ties to even), exactly, for |x| in the normal range."""
    from fractions import Fraction

    if x == 0:
        return Fraction(0)
    sign = 1 if x > 0 else -1
    a = abs(Fraction(x))
    e = a.numerator.bit_length() - a.denominator.bit_length()  # 2^e <= a < 2^(e+2)
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    ulp = Fraction(2) ** (e - 23)
    q = a / ulp
    n = q.numerator // q.denominator
    r = q - n
    if r > Fraction(1, 2) or (r == Fraction(1, 2) and n % 2 == 1):
        n += 1
    return sign * n * ulp


def _exact_code(v, zero, scale):
    """The value code the pages' min-max rule gives when each step is one IEEE fp32
    operation, evaluated in exact rational arithmetic: t = fp32(v - zero),
    x = fp32(t / scale), code = round-half-even(x) clamped to [0, 15]."""
    from fractions import Fraction

    if scale == 0:
        return 0
    t = _round_f32(Fraction(v) - Fraction(zero))
    x = _round_f32(t / Fraction(scale))
    n = x.numerator // x.denominator
    r = x - n
    if r > Fraction(1, 2) or (r == Fraction(1, 2) and n % 2 == 1):
        n += 1
    return int(min(max(n, 0), 15))


def test_value_codes_near_ties_match_exact_rationals():
    """Pins the oracle's code decision (taken in IEEE fp32) against exact rational
    arithmetic on values built to sit exactly on, and one fp32 step beside, the
    half-way points between two levels, where a division done another way (or a
    rounding to a different precision) would pick the other code."""
    rng = np.random.default_rng(23)
    rows = []
    for _ in range(24):
        row = []
        for _g in range(4):
            s = np.float32(np.float16(rng.uniform(0.01, 0.5)))  # an fp16 scale, exact in fp32
            z = np.float32(np.float16(rng.uniform(-2, 2)))
            g = [z, np.float32(z + np.float32(15) * s)]  # min and max fix zero = z, scale = s
            for _ in range(10):
                k = int(rng.integers(0, 15))
                h = np.float32(z + np.float32(k + 0.5) * s)  # on (or next to) a half-way point
                g += [h, np.nextafter(h, np.float32(np.inf)), np.nextafter(h, np.float32(-np.inf))]
            row += g
        rows.append(np.array(row, dtype=np.float32))
    V = np.stack(rows).astype(np.float64)
    codes, scale, zero = O.quantize_values(V, 4, 32)
    from fractions import Fraction

    T = V.shape[0]
    ties = 0
    for t in range(T):
        for g in range(4):
            s, z = float(scale[t, g]), float(zero[t, g])
            for c in range(32):
                v = float(V[t, 32 * g + c])
                want = _exact_code(v, z, s)
                assert codes[t, 32 * g + c] == want, (t, g, c)
                x = _round_f32(_round_f32(Fraction(v) - Fraction(z)) / Fraction(s))
                ties += (x - x.numerator // x.denominator) == Fraction(1, 2)
    assert ties >= 100  # the construction really lands on exact half-way points


def _cp_cache(T=50, d=32, m=64, m_out=32, seed=31):
    rng = np.random.default_rng(seed)
    S, So = O.sketch_pair(4, d, m, m_out)
    idx = np.array([5, 20])
    K = rng.standard_normal((T, d))
    V = rng.standard_normal((T, d)).astype(np.float32).astype(np.float64)
    q = rng.standard_normal(d)
    ks = O.sketch_keys(K, S, So, idx)
    codes, scale, zero = O.quantize_values(V, 4, 32)
    return q, S, So, idx, ks, codes, scale, zero, K


def _shard(args, a, b, sm_scale=None):
    q, S, So, idx, ks, codes, scale, zero, _ = args
    return O.decode_partial(q, S, So, idx, ks["bits_in"][a:b], ks["bits_out"][a:b], ks["norms"][a:b],
                            codes[a:b], scale[a:b], zero[a:b], sm_scale)


def test_partials_merge_to_the_whole_decode():
    """Split invariance: the shards' (o, max, sum) merge to the decode of the whole cache."""
    args = _cp_cache()
    q, S, So, idx, ks, codes, scale, zero, K = args
    T = codes.shape[0]
    for sm in (None, 3.0):  # sm_scale = 3 spreads the shards' maxima far apart
        whole, _ = O.decode_attention(q, S, So, idx, ks["bits_in"], ks["bits_out"], ks["norms"], codes, scale,
                                      zero, sm)
        rng = np.random.default_rng(7)
        splits = [[0, T], [0, 17, 17, 50], [0, 1, T], [0, 49, T]]
        splits += [[0] + sorted(rng.integers(0, T, 3).tolist()) + [T] for _ in range(6)]
        for cuts in splits:
            parts = [_shard(args, a, b, sm) for a, b in zip(cuts[:-1], cuts[1:])]
            np.testing.assert_allclose(O.merge_partials(parts), whole, rtol=1e-12, atol=1e-13)
    # a shard's own report: max and sum of its logits, output = its softmax-weighted values times the sum
    o, mx, l = _shard(args, 10, 20)
    _, sc = O.decode_attention(q, S, So, idx, ks["bits_in"][10:20], ks["bits_out"][10:20], ks["norms"][10:20],
                               codes[10:20], scale[10:20], zero[10:20])
    x = sc / math.sqrt(q.shape[0])
    assert mx == pytest.approx(max(x), abs=0.0)
    assert l == pytest.approx(sum(math.exp(v - mx) for v in x), rel=1e-14)
    part_out, _ = O.decode_attention(q, S, So, idx, ks["bits_in"][10:20], ks["bits_out"][10:20],
                                     ks["norms"][10:20], codes[10:20], scale[10:20], zero[10:20])
    np.testing.assert_allclose(o / l, part_out, rtol=1e-12, atol=1e-13)


def test_merge_neutral_and_order():
    args = _cp_cache(T=24, seed=5)
    d = args[0].shape[0]
    empty = _shard(args, 3, 3)
    assert empty[1] == -math.inf and empty[2] == 0.0 and np.all(empty[0] == 0)
    assert np.all(O.merge_partials([empty, empty]) == 0)
    parts = [_shard(args, 0, 9), _shard(args, 9, 10), _shard(args, 10, 24)]
    ref = O.merge_partials(parts)
    for perm in ([2, 0, 1], [1, 2, 0]):
        np.testing.assert_allclose(O.merge_partials([parts[i] for i in perm]), ref, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(O.merge_partials(parts + [empty]), ref, rtol=0, atol=0)
    assert O.merge_partials([empty]).shape == (d,)


def _e4m3_values():
    """Every finite E4M3FN value, from its bit fields (sign, exponent 4 bits bias 7, mantissa 3 bits)."""
    vals = []
    for code in range(256):
        sgn, ex, man = code >> 7, (code >> 3) & 15, code & 7
        if ex == 15 and man == 7:
            continue  # NaN
        v = man * 2.0 ** -9 if ex == 0 else (1 + man / 8) * 2.0 ** (ex - 7)
        vals.append(-v if sgn else v)
    return np.array(sorted(set(vals)))


def test_fp8_grid_and_ties():
    grid = _e4m3_values()
    assert grid.max() == 448.0 and grid.min() == -448.0 and len(grid) == 253  # +-0 merged
    np.testing.assert_array_equal(O.fp8_e4m3_round(grid), grid)  # every value is its own rounding
    pos = grid[grid >= 0]
    mids = (pos[:-1] + pos[1:]) / 2
    got = O.fp8_e4m3_round(mids)
    # a midpoint goes to the neighbour with the even mantissa (the even code)
    for mid, lo, hi, g in zip(mids, pos[:-1], pos[1:], got):
        even = lo if (np.where(pos == lo)[0][0] % 2 == 0) else hi
        assert g == even, (mid, lo, hi, g)
    # just off the midpoints: the nearer neighbour
    np.testing.assert_array_equal(O.fp8_e4m3_round(np.nextafter(mids, 0)), pos[:-1])
    np.testing.assert_array_equal(O.fp8_e4m3_round(np.nextafter(mids, np.inf)), pos[1:])
    # saturation and signs
    np.testing.assert_array_equal(O.fp8_e4m3_round(np.array([460.0, 1e6, -1e6, -449.0])), [448, 448, -448, -448])
    assert O.fp8_e4m3_round(np.array([2.0 ** -11]))[0] == 0.0          # below half the smallest subnormal
    assert O.fp8_e4m3_round(np.array([3 * 2.0 ** -10]))[0] == 2.0 ** -8  # 1.5 quanta: tie to even (2 quanta)


def test_fp8_matches_torch():
    """Inside the finite range the rounding is torch's float8_e4m3fn conversion (round to nearest even)."""
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(41)
    x = np.concatenate([rng.standard_normal(20000) * s for s in (1e-3, 0.1, 1.0, 30.0, 150.0)])
    x = x[np.abs(x) < 440]
    x32 = x.astype(np.float32)
    ref = torch.from_numpy(x32).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    np.testing.assert_array_equal(O.fp8_e4m3_round(x32.astype(np.float64)), ref)
    scale = 0.37
    q32 = (x32 / np.float32(scale)).astype(np.float32)
    q32 = q32[np.abs(q32) < 440]
    ref_q = torch.from_numpy(q32).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    keep = np.abs(x32 / np.float32(scale)) < 440
    np.testing.assert_array_equal(O.fp8_quantize(x[keep], scale), ref_q)


def test_fp8_decode_is_exact_attention_on_the_grid():
    rng = np.random.default_rng(43)
    d, T = 128, 50
    q = rng.standard_normal(d)
    K = rng.standard_normal((T, d))
    V = rng.standard_normal((T, d))
    ks, vs = 0.05, 0.02
    K8, V8 = O.fp8_quantize(K, ks), O.fp8_quantize(V, vs)
    # values on the grid times the scale come back unchanged through quantisation
    np.testing.assert_array_equal(O.fp8_quantize(K8 * np.float32(ks), ks), K8)
    out = O.fp8_decode_attention(q, K8, V8, ks, vs)
    logits = (K8 * float(np.float32(ks))) @ q / math.sqrt(d)
    w = np.exp(logits - logits.max())
    ref = (w / w.sum()) @ (V8 * float(np.float32(vs)))
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-14)
    # coarse but close: the FP8 error of the output against the unquantised attention is small
    assert np.max(np.abs(out - O.exact_attention(q, K, V))) < 0.05
