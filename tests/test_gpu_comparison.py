"""Comparison kernels on the GPU: the FP8 quantiser bit-exact against the
oracle's E4M3 rounding, and decode over a bf16 or FP8 cache against the
oracle's exact attention on the same (dequantised) cache."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle as O  # noqa: E402
from decode_attention_qjl_b200 import inputs as I  # noqa: E402
from decode_attention_qjl_b200 import qjl as Q  # noqa: E402

pytestmark = pytest.mark.gpu
OUT_ATOL = 1e-4  # fp32 logits and sums over at most a few thousand tokens


def _e4m3_to_f64(codes: np.ndarray) -> np.ndarray:
    """Decode E4M3 bytes from their bit fields."""
    c = codes.astype(np.int64)
    sgn, ex, man = c >> 7, (c >> 3) & 15, c & 7
    v = np.where(ex == 0, man * 2.0 ** -9, (1 + man / 8) * 2.0 ** (ex - 7))
    return np.where(sgn == 1, -v, v)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_fp8_quantize_bit_exact(dtype):
    g = torch.Generator().manual_seed(11)
    x = torch.cat([torch.randn(40000, generator=g) * s for s in (1e-3, 0.3, 3.0, 60.0)])
    x = torch.cat([x, torch.tensor([500.0, -1e4, 0.0, -0.0, 2.0 ** -12, 448.0 * 0.37, 464.0 * 0.37, 1e-30])])
    x = x[: (x.numel() // 8) * 8].to(dtype)
    scale = 0.37
    codes = Q.qjl_fp8_quantize(x.cuda(), scale).cpu().numpy()
    got = _e4m3_to_f64(codes)
    want = O.fp8_quantize(x.float().numpy().astype(np.float64), scale)
    assert np.array_equal(got, want), int(np.sum(got != want))
    assert not np.any((codes & 0x7F) == 0x7F)  # saturating: no NaN codes


@pytest.mark.parametrize("case", [
    # name, B, T, Hkv, seqlens, overrides
    ("llama2_7b_mha", 2, 700, 2, None, {}),
    ("llama3_8b_gqa", 2, 1000, 2, [1000, 37], {}),   # g = 4, a ragged batch
    ("llama3_8b_gqa", 1, 300, 1, [0], {"Hq": 64}),    # g = 8, an empty sequence
    ("single_head_fp32", 1, 1024, None, None, {"Hq": 2}),
])
@pytest.mark.parametrize("fmt", ["bf16", "fp8"])
def test_exact_and_fp8_decode_match_the_oracle(case, fmt):
    name, B, T, Hkv, seqlens, over = case
    w = I.WORKLOADS[name]
    if over:
        w = I.Workload(**{**w.__dict__, **over})
    inp = I.make_inputs(w, seed=77, device="cpu", B=B, T=T, Hkv=Hkv)
    K = inp["K"].to(torch.bfloat16)
    V = inp["V"].to(torch.bfloat16)
    Qt = inp["Q"]
    Bq, Hq, d = Qt.shape
    g = Hq // K.shape[1]
    cap = ((T + 63) // 64) * 64 + 64  # a capacity larger than T
    Kc = torch.zeros(B, K.shape[1], cap, d, dtype=torch.bfloat16)
    Vc = torch.zeros_like(Kc)
    Kc[:, :, :T], Vc[:, :, :T] = K, V
    ks, vs = 0.25, 0.02
    if fmt == "fp8":
        Kd = Q.qjl_fp8_quantize(Kc.cuda(), ks)
        Vd = Q.qjl_fp8_quantize(Vc.cuda(), vs)
        K64 = _e4m3_to_f64(Kd.cpu().numpy())
        V64 = _e4m3_to_f64(Vd.cpu().numpy())
        assert np.array_equal(K64[:, :, :T], O.fp8_quantize(K.float().numpy().astype(np.float64), ks))
    else:
        Kd, Vd = Kc.cuda(), Vc.cuda()
        K64 = Kc.double().numpy()
        V64 = Vc.double().numpy()
    Out = torch.full((B, Hq, d), float("nan"), dtype=torch.float32, device="cuda")
    sl = None if seqlens is None else torch.tensor(seqlens, dtype=torch.int32, device="cuda")
    Q.qjl_exact_decode(Kd, Vd, Qt.cuda(), Out, T=T, seqlens=sl, k_scale=ks, v_scale=vs)
    got = Out.cpu().numpy().astype(np.float64)
    Q64 = Qt.float().numpy().astype(np.float64)
    worst = 0.0
    for b in range(B):
        n = T if seqlens is None else seqlens[b]
        for h in range(Hq):
            if fmt == "fp8":
                ref = O.fp8_decode_attention(Q64[b, h], K64[b, h // g, :n], V64[b, h // g, :n], ks, vs)
            else:
                ref = O.exact_attention(Q64[b, h], K64[b, h // g, :n], V64[b, h // g, :n])
            worst = max(worst, float(np.max(np.abs(got[b, h] - ref))))
    print(f"{name} {fmt}: out abs {worst:.2e}")
    assert worst <= OUT_ATOL


def _minmax_unpack(rows: np.ndarray, bits: int):
    """codes [.., 128], scale, zero [.., 4] from min-max rows (codes, then four fp16 (scale, zero) pairs)."""
    nb = 128 * bits // 8
    raw = rows[..., :nb]
    per = 8 // bits
    codes = np.stack([(raw >> (bits * k)) & ((1 << bits) - 1) for k in range(per)], -1).reshape(*rows.shape[:-1], 128)
    sz = rows[..., nb:nb + 16].copy().view(np.float16).reshape(*rows.shape[:-1], 4, 2)
    return codes.astype(np.uint8), sz[..., 0], sz[..., 1]


@pytest.mark.parametrize("bits", [2, 4])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_minmax_quantize_bit_exact(bits, dtype):
    g = torch.Generator().manual_seed(13)
    X = torch.randn(3000, 128, generator=g) * torch.exp(torch.randn(3000, 1, generator=g))
    X[5] = 0.0                     # a constant row: scale 0, codes 0
    X[6, :32] = 1.5                # a constant group
    X[7, 64:96] *= 1e4             # a wide group
    X = X.to(dtype)
    rows = Q.qjl_minmax_quantize(X.cuda(), bits).cpu().numpy()
    codes, scale, zero = _minmax_unpack(rows, bits)
    c, s, z = O.quantize_values(X.float().numpy().astype(np.float64), bits, 32)
    assert np.array_equal(codes, c), int(np.sum(codes != c))
    assert np.array_equal(scale.view(np.uint16), s.view(np.uint16))
    assert np.array_equal(zero.view(np.uint16), z.view(np.uint16))


@pytest.mark.parametrize("bits", [2, 4])
@pytest.mark.parametrize("case", [
    ("llama3_8b_gqa", 2, 1000, 2, [1000, 37], {}),
    ("llama2_7b_mha", 2, 700, 2, None, {}),
])
def test_minmax_decode_matches_the_oracle(case, bits):
    name, B, T, Hkv, seqlens, over = case
    w = I.WORKLOADS[name]
    inp = I.make_inputs(w, seed=79, device="cpu", B=B, T=T, Hkv=Hkv)
    K, V, Qt = inp["K"], inp["V"], inp["Q"]
    Hq, d = Qt.shape[1], Qt.shape[2]
    g = Hq // K.shape[1]
    Kr = Q.qjl_minmax_quantize(K.cuda(), bits)
    Vr = Q.qjl_minmax_quantize(V.cuda(), bits)
    kc, ks, kz = _minmax_unpack(Kr.cpu().numpy(), bits)
    vc, vs, vz = _minmax_unpack(Vr.cpu().numpy(), bits)
    Out = torch.full((B, Hq, d), float("nan"), dtype=torch.float32, device="cuda")
    sl = None if seqlens is None else torch.tensor(seqlens, dtype=torch.int32, device="cuda")
    Q.qjl_exact_decode(Kr, Vr, Qt.cuda(), Out, T=T, seqlens=sl)
    got = Out.cpu().numpy().astype(np.float64)
    Q64 = Qt.float().numpy().astype(np.float64)
    worst = 0.0
    for b in range(B):
        n = T if seqlens is None else seqlens[b]
        for h in range(Hq):
            hk = h // g
            Kh = O.dequantize_values(kc[b, hk, :n], ks[b, hk, :n], kz[b, hk, :n])
            Vh = O.dequantize_values(vc[b, hk, :n], vs[b, hk, :n], vz[b, hk, :n])
            worst = max(worst, float(np.max(np.abs(got[b, h] - O.exact_attention(Q64[b, h], Kh, Vh)))))
    print(f"{name} minmax{bits}: out abs {worst:.2e}")
    assert worst <= OUT_ATOL
