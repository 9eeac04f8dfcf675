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
