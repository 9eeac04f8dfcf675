"""Context-parallel decode on one GPU: shards as separate caches, the partial
decode kernel per shard, then the merge kernel; against the oracle's
decode_partial / merge_partials on the same (bit-exact, checked elsewhere)
caches, and against the single-call decode."""
import math

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle as O  # noqa: E402
from decode_attention_qjl_b200 import context_parallel as CP  # noqa: E402
from decode_attention_qjl_b200 import inputs as I  # noqa: E402
from decode_attention_qjl_b200 import qjl as Q  # noqa: E402
from tests import gpu_common as C  # noqa: E402

pytestmark = pytest.mark.gpu
LOG2E = 1.0 / math.log(2.0)


def _inputs(name, B, T, Hkv, over):
    w = I.WORKLOADS[name]
    if over:
        w = I.Workload(**{**w.__dict__, **over})
    return I.make_inputs(w, seed=1234, device="cpu", B=B, T=T, Hkv=Hkv)


@pytest.mark.parametrize("case", [
    # name, B, T, Hkv, shards, seqlens, overrides
    ("llama2_7b_mha", 2, 700, 2, 3, None, {}),
    ("llama3_8b_gqa", 2, 1000, 2, 4, [1000, 37], {}),   # g = 4; sequence 1 lives in shard 0 only
    ("single_head_fp32", 1, 1024, None, 2, None, {"Hq": 2}),  # fp32 queries
    ("llama2_7b_mha", 1, 300, 1, 2, None, {"n_outlier": 0, "m_out": 0}),
])
def test_partials_and_merge_match_the_oracle(case):
    name, B, T, Hkv, R, seqlens, over = case
    inp = _inputs(name, B, T, Hkv, over)
    w = inp["workload"]
    ctx = Q.QJLContext(0, 128, w.m, w.m_out, w.n_outlier)
    Qd = inp["Q"].cuda()
    Hq, d = Qd.shape[1], Qd.shape[2]
    g = Hq // w.Hkv
    S, So = C.sketch64(w)
    Q64 = C.to64(inp["Q"])
    O_parts = torch.zeros(R, B, Hq, d, dtype=torch.float32, device="cuda")
    ML_parts = torch.zeros(R, B, Hq, 2, dtype=torch.float32, device="cuda")
    ref_parts = {}
    worst = {"out": 0.0, "max": 0.0, "sum": 0.0}
    for r in range(R):
        a, b = CP.shard_bounds(T, R, r)
        cache = C.quantize_on_gpu(ctx, inp["K"][:, :, a:b].contiguous().cuda(), inp["V"][:, :, a:b].contiguous().cuda())
        lens = [b - a] * B if seqlens is None else CP.local_seqlens(seqlens, T, R, r)
        sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
        ws = ctx.decode_workspace(B, Hq, w.Hkv, b - a)
        Q.qjl_decode_attention_partial(ctx.handle, cache, Qd, b - a, O_parts[r], ML_parts[r], seqlens=sl, workspace=ws)
        Q.qjl_decode_workspace_status(ctx.handle, ws, B, Hq, w.Hkv)
        gc = C.cache_to_numpy(cache, w.m_out, w.n_outlier)
        o_g, ml_g = O_parts[r].cpu().numpy().astype(np.float64), ML_parts[r].cpu().numpy().astype(np.float64)
        for bb in range(B):
            n = lens[bb]
            for h in range(Hq):
                hk = h // g
                o, mx, l = O.decode_partial(Q64[bb, h], S, So, gc["idx"][bb, hk], gc["bits_in"][bb, hk, :n],
                                            gc["bits_out"][bb, hk, :n], gc["norms"][bb, hk, :n], gc["codes"][bb, hk, :n],
                                            gc["scale"][bb, hk, :n], gc["zero"][bb, hk, :n])
                ref_parts[(r, bb, h)] = (o, mx, l)
                if n == 0:
                    assert ml_g[bb, h, 0] == -np.inf and ml_g[bb, h, 1] == 0 and np.all(o_g[bb, h] == 0)
                    continue
                # the shard's softmax output, its maximum logit and its sum (rescaled to the oracle's maximum)
                worst["out"] = max(worst["out"], float(np.max(np.abs(o_g[bb, h] / ml_g[bb, h, 1] - o / l))))
                worst["max"] = max(worst["max"], abs(ml_g[bb, h, 0] / LOG2E - mx) / max(1.0, abs(mx)))
                worst["sum"] = max(worst["sum"], abs(ml_g[bb, h, 1] * 2.0 ** (ml_g[bb, h, 0] - mx * LOG2E) / l - 1.0))
    Out = torch.empty(B, Hq, d, dtype=torch.float32, device="cuda")
    Q.qjl_merge_partials(O_parts, ML_parts, Out)
    got = Out.cpu().numpy().astype(np.float64)
    ref = np.zeros_like(got)
    for bb in range(B):
        for h in range(Hq):
            ref[bb, h] = O.merge_partials([ref_parts[(r, bb, h)] for r in range(R)])
    err = float(np.max(np.abs(got - ref)))
    print(f"{name} R={R}: merged out abs {err:.2e}; part out {worst['out']:.2e}, max rel {worst['max']:.2e}, "
          f"sum rel {worst['sum']:.2e}")
    assert err <= C.OUT_ATOL
    assert worst["out"] <= C.OUT_ATOL
    # a maximum logit is one score times sm_scale: the score tolerance applies
    assert worst["max"] <= C.SCORE_RTOL and worst["sum"] <= 2e-2
    ctx.close()


def test_one_shard_is_the_single_call_decode():
    """R = 1: the partial then the merge give qjl_decode_attention's output bit for bit."""
    inp = _inputs("llama3_8b_gqa", 2, 777, 2, {})
    w = inp["workload"]
    ctx = Q.QJLContext(0, 128, w.m, w.m_out, w.n_outlier)
    Qd = inp["Q"].cuda()
    B, Hq, d = Qd.shape
    cache = C.quantize_on_gpu(ctx, inp["K"].cuda(), inp["V"].cuda())
    sl = torch.tensor([777, 300], dtype=torch.int32, device="cuda")
    ws = ctx.decode_workspace(B, Hq, w.Hkv, 777)
    want = torch.empty(B, Hq, d, dtype=torch.float32, device="cuda")
    Q.qjl_decode_attention(ctx.handle, cache, Qd, 777, want, seqlens=sl, workspace=ws)
    o = torch.empty(1, B, Hq, d, dtype=torch.float32, device="cuda")
    ml = torch.empty(1, B, Hq, 2, dtype=torch.float32, device="cuda")
    Q.qjl_decode_attention_partial(ctx.handle, cache, Qd, 777, o[0], ml[0], seqlens=sl, workspace=ws)
    got = torch.empty_like(want)
    Q.qjl_merge_partials(o, ml, got)
    torch.cuda.synchronize()
    assert torch.equal(got, want)
    ctx.close()


def test_merge_reads_packed_rank_buffers():
    """The layout ContextParallelDecode gathers (one packed buffer per rank) merges like two plain arrays."""
    R, B, Hq, d = 3, 2, 5, 128  # rows = 10: the per-rank (max, sum) block is padded to 16 bytes
    g = torch.Generator().manual_seed(9)
    o = torch.randn(R, B, Hq, d, generator=g)
    mx = torch.randn(R, B, Hq, generator=g) * 4
    mx[1, 0, 2] = -math.inf  # an empty shard of one row
    ml = torch.stack([mx, torch.rand(R, B, Hq, generator=g) + 0.5], -1)
    o[1, 0, 2] = 0.0
    ml[1, 0, 2, 1] = 0.0
    rows = B * Hq
    part = rows * d + ((2 * rows + 3) // 4) * 4
    packed = torch.zeros(R, part)
    packed[:, :rows * d] = o.reshape(R, -1)
    packed[:, rows * d:rows * d + 2 * rows] = ml.reshape(R, -1)
    packed = packed.cuda()
    a = torch.empty(B, Hq, d, device="cuda")
    Q.qjl_merge_partials(packed[:, :rows * d], packed[:, rows * d:rows * d + 2 * rows], a)
    b = torch.empty(B, Hq, d, device="cuda")
    Q.qjl_merge_partials(o.cuda(), ml.cuda(), b)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    # against the oracle's merge
    for bb in range(B):
        for h in range(Hq):
            parts = [(o[r, bb, h].double().numpy(), float(ml[r, bb, h, 0]) / LOG2E, float(ml[r, bb, h, 1]))
                     for r in range(R)]
            np.testing.assert_allclose(b[bb, h].cpu().double().numpy(), O.merge_partials(parts), rtol=1e-5, atol=1e-6)
