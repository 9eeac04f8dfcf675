"""qjl_decode_attention_static: decode attention for callers that cannot allocate.

Some callers cannot call cudaMalloc: a plugin inside a host runtime that owns
all device memory and forbids its plugins to allocate, or a latency-critical
caller that cannot accept cudaMalloc's implicit synchronisation. For them the
library keeps a fixed scratch array and this entry point uses it instead of a
caller workspace. This test calls it through the C ABI, twice in a row, and
checks it against qjl_decode_attention with a caller workspace. The file is
named so that pytest collects it last.
"""

import numpy as np
import pytest

torch = pytest.importorskip("torch")

from decode_attention_qjl_b200 import build as build_mod  # noqa: E402
from decode_attention_qjl_b200 import inputs as I  # noqa: E402
from decode_attention_qjl_b200 import qjl as Q  # noqa: E402

pytestmark = pytest.mark.gpu

OUT_ATOL = 2e-3  # the output tolerance used by the other parity tests


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build_mod.build()
    Q.load_library()


def _setup(name, B, T, Hkv):
    inp = I.make_inputs(I.WORKLOADS[name], device="cuda", B=B, T=T, Hkv=Hkv)
    w = inp["workload"]
    ctx = Q.QJLContext(0, 128, w.m, w.m_out, w.n_outlier)
    cache = ctx.allocate_cache(w.B, w.Hkv, T)
    Q.qjl_quantize_keys(ctx.handle, cache, inp["K"], Q.QJL_PREFILL, workspace=ctx.keys_workspace(w.B, w.Hkv))
    Q.qjl_quantize_values(ctx.handle, cache, inp["V"])
    torch.cuda.synchronize()
    return w, ctx, cache, inp["Q"]


@pytest.mark.parametrize("name,B,T,Hkv,seqlens", [
    ("llama2_7b_mha", 2, 3000, 4, [3000, 1234]),   # several splits per head, ragged tail
    ("llama3_8b_gqa", 2, 2500, 2, None),           # grouped-query heads
])
def test_static_scratch_matches_workspace_entry_point(name, B, T, Hkv, seqlens):
    w, ctx, cache, Qt = _setup(name, B, T, Hkv)
    assert 0 < Q.qjl_decode_workspace_bytes(ctx.handle, w.B, w.Hq, w.Hkv, T) <= Q.STATIC_SCRATCH_BYTES
    sl = None if seqlens is None else torch.tensor(seqlens, dtype=torch.int32, device="cuda")
    ref = torch.empty(w.B, w.Hq, 128, device="cuda")
    ref_s = torch.zeros(w.B, w.Hq, T, device="cuda")
    Q.qjl_decode_attention(ctx.handle, cache, Qt, T, ref, seqlens=sl, scores=ref_s,
                           workspace=ctx.decode_workspace(w.B, w.Hq, w.Hkv, T))
    outs = []
    for _ in range(2):  # two calls in a row share the same scratch array
        o = torch.empty(w.B, w.Hq, 128, device="cuda")
        s = torch.zeros(w.B, w.Hq, T, device="cuda")
        Q.qjl_decode_attention_static(ctx.handle, cache, Qt, T, o, seqlens=sl, scores=s)
        outs.append((o, s))
    torch.cuda.synchronize()
    for o, s in outs:
        assert torch.isfinite(o).all()
        assert float((o - ref).abs().max()) <= OUT_ATOL
        np.testing.assert_allclose(s.cpu().numpy(), ref_s.cpu().numpy(), rtol=1e-6, atol=1e-6)
    ctx.close()


def test_static_scratch_rejects_oversized_calls():
    # 128 sequences x 32 kv heads: the decode's workspace holds the prepared
    # query sketches of 4096 (sequence, kv head) pairs (about 2.6 KB each),
    # about 10.6 MB, more than the fixed array holds.
    B, Hkv, Hq, T = 128, 32, 32, 64
    ctx = Q.QJLContext(0, 128, 256, 64, 8)
    need = Q.qjl_decode_workspace_bytes(ctx.handle, B, Hq, Hkv, T)
    assert need > Q.STATIC_SCRATCH_BYTES
    cache = ctx.allocate_cache(B, Hkv, T)
    Qt = torch.zeros(B, Hq, 128, dtype=torch.bfloat16, device="cuda")
    out = torch.zeros(B, Hq, 128, device="cuda")
    with pytest.raises(Q.QJLError, match="WORKSPACE") as ei:
        Q.qjl_decode_attention_static(ctx.handle, cache, Qt, T, out)
    assert "QJL_STATIC_SCRATCH_BYTES" in str(ei.value)
    torch.cuda.synchronize()
    assert int(out.count_nonzero()) == 0  # nothing was launched
    ctx.close()


def test_static_scratch_fits_every_configured_workload():
    """Every workload shape the tests and the bench use fits the fixed array (its decode workspace is
    at most QJL_STATIC_SCRATCH_BYTES), as the header and the design notes state."""
    for name, w in I.WORKLOADS.items():
        ctx = Q.QJLContext(0, 128, w.m, w.m_out, w.n_outlier)
        need = Q.qjl_decode_workspace_bytes(ctx.handle, w.B, w.Hq, w.Hkv, w.T + 1)
        assert 0 < need <= Q.STATIC_SCRATCH_BYTES, (name, need)
        ctx.close()
