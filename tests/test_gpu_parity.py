"""GPU parity: the CUDA path through the C ABI against the fp64 oracle.

Bit-exact: outlier channels, sign bits (outside the 1e-6 |k| band, counted),
fp16 norms, 4-bit codes and fp16 scale/zero. Floating point: scores within
relative 1e-3 (floor 1e-3 of the row's rms score), outputs within 2e-3 absolute.
"""

import math

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle as O  # noqa: E402
from decode_attention_qjl_b200 import build as build_mod  # noqa: E402
from decode_attention_qjl_b200 import inputs as I  # noqa: E402
from decode_attention_qjl_b200 import qjl as Q  # noqa: E402

from tests import gpu_common as C  # noqa: E402

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build_mod.build()
    Q.load_library()


def _ctx(w, value_bits=4):
    return Q.QJLContext(0, 128, w.m, w.m_out, w.n_outlier, value_bits=value_bits)


def _small(name, B, T, Hkv=None, device="cpu", seed=1234, **over):
    """Inputs of a workload recipe at a smaller size; `value_bits` in `over` is the context's, not the recipe's."""
    over = {k: v for k, v in over.items() if k != "value_bits"}
    w = I.WORKLOADS[name]
    if over:
        w = I.Workload(**{**w.__dict__, **over})
    return I.make_inputs(w, seed=seed, device=device, B=B, T=T, Hkv=Hkv)


def test_ctx_sketch_matches_oracle():
    for m, m_out in ((256, 64), (128, 32), (512, 64)):
        ctx = Q.QJLContext(0, 128, m, m_out, 8)
        S_bits, So_bits = Q.qjl_ctx_sketch(ctx.handle, m, m_out)
        S, So = O.sketch_pair(0, 128, m, m_out)
        bits = lambda a: (a.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
        assert np.array_equal(S_bits, bits(S)) and np.array_equal(So_bits, bits(So))
        ctx.close()


@pytest.mark.parametrize("case", [
    ("single_head_fp32", 1, 1024, None, {}),
    ("llama2_7b_mha", 2, 333, 3, {}),
    ("long_context", 1, 2000, 2, {}),
    ("llama3_8b_gqa", 2, 257, 2, {}),
    ("llama3_8b_gqa", 1, 300, 2, {"m": 128}),
    ("llama3_8b_gqa", 1, 300, 2, {"m": 512}),
    ("llama2_7b_mha", 1, 100, 2, {"n_outlier": 0, "m_out": 0}),
    ("llama2_7b_mha", 1, 100, 2, {"n_outlier": 0, "m_out": 64}),
    ("llama2_7b_mha", 1, 64, 1, {"n_outlier": 32, "m_out": 256}),
    # 128 tokens or more per (sequence, kv head): the tensor-core sketch
    ("llama2_7b_mha", 1, 300, 2, {"n_outlier": 0, "m_out": 0}),
    ("llama2_7b_mha", 1, 200, 1, {"n_outlier": 32, "m_out": 256}),
    ("llama2_7b_mha", 1, 130, 1, {"m": 96, "m_out": 32}),
    ("llama3_8b_gqa", 3, 1000, 3, {}),
    # more 128-token blocks than SMs: every persistent CTA of the tensor-core
    # sketch takes several blocks, reuses its A buffers and accumulators, and
    # reloads the masked image where its range crosses into the next pair
    ("llama3_8b_gqa", 2, 20000, 4, {}),
    ("llama3_8b_gqa", 1, 40000, 2, {"m": 512}),  # five accumulator passes per block, two A buffers
    ("llama2_7b_mha", 1, 30000, 2, {"n_outlier": 32, "m_out": 256}),
    # 2-bit value codes (levels 0..3), in their line layout
    ("llama2_7b_mha", 2, 333, 3, {"value_bits": 2}),
    ("single_head_fp32", 1, 1024, None, {"value_bits": 2}),
    ("llama3_8b_gqa", 2, 20000, 4, {"value_bits": 2}),
])
def test_quantize_bit_exact(case):
    name, B, T, Hkv, over = case
    vb = over.get("value_bits", 4)
    inp = _small(name, B, T, Hkv, **over)
    w = inp["workload"]
    ctx = _ctx(w, vb)
    cache = C.quantize_on_gpu(ctx, inp["K"].cuda(), inp["V"].cuda())
    g = C.cache_to_numpy(cache, w.m_out, w.n_outlier)
    K64, V64 = C.to64(inp["K"]), C.to64(inp["V"])
    S, So = C.sketch64(w)
    pairs = [(b, h) for b in range(w.B) for h in range(w.Hkv)]
    planted = inp["outlier_channels"].numpy() if w.n_outlier else None
    st = C.compare_keys(g, K64, S, So, w.n_outlier, pairs, planted=planted)
    assert st["mismatch"] == 0 and st["norm_mismatch"] == 0, st
    assert st["excluded"] <= 1e-4 * st["entries"], st
    assert C.compare_values(g, V64, pairs, vb) == 0
    ctx.close()


@pytest.mark.parametrize("case", [
    ("single_head_fp32", 1, 1024, None, None, {}),
    ("llama2_7b_mha", 2, 1000, 3, [1000, 613], {}),
    ("long_context", 1, 3000, 2, None, {}),
    ("llama3_8b_gqa", 3, 777, 2, [777, 1, 0], {}),
    ("llama3_8b_gqa", 2, 600, 2, None, {"m": 512}),
    ("llama3_8b_gqa", 2, 600, 1, None, {"m": 128, "Hq": 64}),  # g = 8
    # g = 8 with m = 512: S and S_out do not fit the cache ring, so the query
    # projection reads them from global memory
    ("llama3_8b_gqa", 1, 300, 1, None, {"m": 512, "Hq": 64}),
    # fp32 query with g = 4: the projection's bf16 hi/lo split on several heads
    ("single_head_fp32", 1, 700, 2, None, {"Hq": 4}),
    # a large outlier sketch (m_out = 256, 32 outlier channels)
    ("llama2_7b_mha", 1, 400, 2, None, {"n_outlier": 32, "m_out": 256}),
    ("llama3_8b_gqa", 2, 300, 2, None, {"Hq": 16}),            # g = 2
    ("llama2_7b_mha", 1, 500, 2, None, {"n_outlier": 0, "m_out": 0}),
    # 2-bit value codes: expanded to the 4-bit MMA operands from their lines
    ("llama2_7b_mha", 2, 1000, 3, [1000, 613], {"value_bits": 2}),
    ("llama3_8b_gqa", 3, 777, 2, [777, 1, 0], {"value_bits": 2}),
    ("single_head_fp32", 1, 700, 2, None, {"Hq": 4, "value_bits": 2}),
    ("llama3_8b_gqa", 1, 300, 1, None, {"m": 512, "Hq": 64, "value_bits": 2}),
])
def test_decode_parity(case):
    name, B, T, Hkv, seqlens, over = case
    inp = _small(name, B, T, Hkv, **over)
    w = inp["workload"]
    ctx = _ctx(w, over.get("value_bits", 4))
    cache = C.quantize_on_gpu(ctx, inp["K"].cuda(), inp["V"].cuda())
    g = C.cache_to_numpy(cache, w.m_out, w.n_outlier)
    S, So = C.sketch64(w)
    O_gpu, sc_gpu = C.run_decode(ctx, cache, inp["Q"].cuda(), T, seqlens=seqlens)
    pairs = [(b, h) for b in range(w.B) for h in range(w.Hq)]
    r = C.compare_decode(g, C.to64(inp["Q"]), S, So, O_gpu, sc_gpu, pairs, seqlens=seqlens)
    # error against exact attention on the original K, V (reported, not gated)
    Ex = O.exact_batch(C.to64(inp["Q"]), C.to64(inp["K"]), C.to64(inp["V"]), seqlens=seqlens)
    print(f"{name} {over}: score rel {r['score_rel']:.2e}, out abs {r['out_abs']:.2e}, "
          f"vs exact attention max abs {np.max(np.abs(Ex - O_gpu)):.3f}")
    ctx.close()


def test_decode_sm_scale_and_fp32_queries():
    inp = _small("llama3_8b_gqa", 1, 400, 2)
    w = inp["workload"]
    ctx = _ctx(w)
    cache = C.quantize_on_gpu(ctx, inp["K"].cuda(), inp["V"].cuda())
    g = C.cache_to_numpy(cache, w.m_out, w.n_outlier)
    S, So = C.sketch64(w)
    Qf = inp["Q"].float()
    O_gpu, sc_gpu = C.run_decode(ctx, cache, Qf.cuda(), 400, sm_scale=0.05)
    C.compare_decode(g, C.to64(Qf), S, So, O_gpu, sc_gpu, [(0, h) for h in range(w.Hq)], sm_scale=0.05)
    ctx.close()


def test_append_mode_matches_prefill_channels():
    """Prefill T0 tokens (selects the outlier channels), then append tokens at
    ragged positions with QJL_APPEND: they use the stored channels."""
    inp = _small("llama2_7b_mha", 2, 200, 2)
    w = inp["workload"]
    ctx = _ctx(w)
    K, V = inp["K"].cuda(), inp["V"].cuda()
    cap = 256
    cache = C.quantize_on_gpu(ctx, K[:, :, :150].contiguous(), V[:, :, :150].contiguous(), cap=cap)
    g0 = C.cache_to_numpy(cache, w.m_out, w.n_outlier, T=150)
    # append 3 tokens per sequence at positions 150 (b=0) and 180 (b=1)
    t_start = torch.tensor([150, 180], dtype=torch.int32, device="cuda")
    Kn, Vn = K[:, :, 150:153], V[:, :, 150:153]
    Q.qjl_quantize_keys(ctx.handle, cache, Kn, Q.QJL_APPEND, t_start=t_start)
    Q.qjl_quantize_values(ctx.handle, cache, Vn, t_start=t_start)
    torch.cuda.synchronize()
    g = C.cache_to_numpy(cache, w.m_out, w.n_outlier, T=cap)
    S, So = C.sketch64(w)
    K64, V64 = C.to64(inp["K"]), C.to64(inp["V"])
    for b, pos in ((0, 150), (1, 180)):
        for h in range(w.Hkv):
            ks = O.sketch_keys(K64[b, h, 150:153], S, So, g0["idx"][b, h])
            assert np.array_equal(g["bits_in"][b, h, pos:pos + 3], ks["bits_in"])
            assert np.array_equal(g["bits_out"][b, h, pos:pos + 3], ks["bits_out"])
            assert np.array_equal(g["norms"][b, h, pos:pos + 3].view(np.uint16), ks["norms"].view(np.uint16))
            c, s, z = O.quantize_values(V64[b, h, 150:153])
            assert np.array_equal(g["codes"][b, h, pos:pos + 3], c)
    assert np.array_equal(g["idx"], g0["idx"])
    ctx.close()


def test_decode_edge_cases():
    inp = _small("llama2_7b_mha", 3, 70, 1)
    w = inp["workload"]
    ctx = _ctx(w)
    cache = C.quantize_on_gpu(ctx, inp["K"].cuda(), inp["V"].cuda())
    g = C.cache_to_numpy(cache, w.m_out, w.n_outlier)
    S, So = C.sketch64(w)
    Qt = inp["Q"].cuda()
    # ragged lengths with an empty and a one-token sequence
    O_gpu, sc = C.run_decode(ctx, cache, Qt, 70, seqlens=[0, 1, 70])
    assert np.all(O_gpu[0] == 0)
    C.compare_decode(g, C.to64(inp["Q"]), S, So, O_gpu, sc, [(b, h) for b in range(3) for h in range(w.Hq)],
                     seqlens=[0, 1, 70])
    # T = 0 for everyone
    O0, _ = C.run_decode(ctx, cache, Qt, 0, want_scores=False)
    assert np.all(O0 == 0)
    # scores pointer omitted
    O1, _ = C.run_decode(ctx, cache, Qt, 70, want_scores=False)
    O2, _ = C.run_decode(ctx, cache, Qt, 70)
    assert np.array_equal(O1, O2)
    # one workspace reused by consecutive calls (the split counters reset themselves)
    B, Hq = Qt.shape[:2]
    ws = ctx.decode_workspace(B, Hq, w.Hkv, 70)
    outs = []
    for _ in range(3):
        o = torch.empty(B, Hq, 128, device="cuda")
        Q.qjl_decode_attention(ctx.handle, cache, Qt, 70, o, workspace=ws)
        outs.append(o)
    torch.cuda.synchronize()
    assert torch.equal(outs[0], outs[1]) and torch.equal(outs[1], outs[2])
    assert np.array_equal(outs[0].cpu().numpy(), O1)
    # too-small workspace is rejected before launch
    need = Q.qjl_decode_workspace_bytes(ctx.handle, B, Hq, w.Hkv, 70)
    if need > 0:
        small = torch.zeros(need - 16, dtype=torch.uint8, device="cuda")
        out = torch.empty(B, Hq, 128, device="cuda")
        with pytest.raises(Q.QJLError, match="WORKSPACE"):
            Q.qjl_decode_attention(ctx.handle, cache, Qt, 70, out, workspace=small)
    ctx.close()


def _full_size(name, n_pairs=6, n_key_pairs=3):
    """The full workload in the launch configuration the bench times; the oracle
    checks sampled (sequence, head) pairs, and the planted outlier channels of
    every head."""
    w = I.WORKLOADS[name]
    inp = I.make_inputs(w, device="cuda")
    ctx = _ctx(w)
    cache = C.quantize_on_gpu(ctx, inp["K"], inp["V"])
    S, So = C.sketch64(w)
    rng = np.random.default_rng(0)
    assert torch.equal(cache.outlier_idx[..., : w.n_outlier].long(), inp["outlier_channels"])
    for _ in range(n_key_pairs):
        b, h = int(rng.integers(w.B)), int(rng.integers(w.Hkv))
        g1 = C.cache_to_numpy(cache, w.m_out, w.n_outlier, b=b, h=h)
        st = C.compare_keys(g1, C.to64(inp["K"][b:b + 1, h:h + 1]), S, So, w.n_outlier, [(0, 0)])
        assert st["mismatch"] == 0 and st["norm_mismatch"] == 0, st
        assert C.compare_values(g1, C.to64(inp["V"][b:b + 1, h:h + 1]), [(0, 0)]) == 0
    O_gpu, sc = C.run_decode(ctx, cache, inp["Q"], w.T)
    for _ in range(n_pairs):
        b, hq = int(rng.integers(w.B)), int(rng.integers(w.Hq))
        hk = hq // w.g
        g1 = C.cache_to_numpy(cache, w.m_out, w.n_outlier, b=b, h=hk)
        q1 = C.to64(inp["Q"][b:b + 1, hq:hq + 1])
        r = C.compare_decode(g1, q1, S, So, O_gpu[b:b + 1, hq:hq + 1], sc[b:b + 1, hq:hq + 1], [(0, 0)])
        print(f"{name} full size b={b} h={hq}: score rel {r['score_rel']:.2e}, out abs {r['out_abs']:.2e}")
    ctx.close()


@pytest.mark.parametrize("name", ["llama2_7b_mha", "long_context", "llama3_8b_gqa"])
def test_full_size_sampled(name):
    _full_size(name)


@pytest.mark.parametrize("name", [n for n in I.WORKLOADS if n.startswith("sweep_")])
def test_sweep_sampled(name):
    _full_size(name, n_pairs=3, n_key_pairs=1)


# ----------------------------------------------------------------------------- decode step (append + decode)

@pytest.mark.parametrize("case", [
    # name, B, T0 (tokens before the step), Hkv, seqlens before the step, overrides
    ("llama2_7b_mha", 3, 300, 2, [300, 0, 129], {}),
    ("llama3_8b_gqa", 2, 191, 2, None, {}),                           # g = 4, the new token opens a tile
    ("single_head_fp32", 1, 700, 2, None, {"Hq": 4}),                 # fp32 q, k, v
    ("llama3_8b_gqa", 1, 300, 1, None, {"m": 512, "Hq": 64}),        # g = 8, m = 512
    ("llama2_7b_mha", 2, 130, 2, None, {"n_outlier": 0, "m_out": 0}),  # plain QJL
    ("llama2_7b_mha", 1, 200, 1, [63], {"n_outlier": 32, "m_out": 256}),
    ("llama3_8b_gqa", 2, 191, 2, [191, 64], {"value_bits": 2}),        # 2-bit values, a token opens a tile
])
def test_decode_step_parity(case):
    """qjl_decode_step writes each sequence's new token (bit-exact against the
    oracle's key sketch and value quantiser, with the outlier channels chosen at
    prefill) and attends over it in the same launch."""
    name, B, T0, Hkv, seqlens, over = case
    vb = over.get("value_bits", 4)
    inp = _small(name, B, T0 + 1, Hkv, **over)
    w = inp["workload"]
    ctx = _ctx(w, vb)
    K, V = inp["K"].cuda(), inp["V"].cuda()
    lens = seqlens if seqlens is not None else [T0] * B
    cap = T0 + 1
    cache = C.quantize_on_gpu(ctx, K[:, :, :T0].contiguous(), V[:, :, :T0].contiguous(), cap=cap)
    # the new token of sequence b is token lens[b] of its input rows
    kn = torch.stack([K[b, :, lens[b]] for b in range(B)]).contiguous()
    vn = torch.stack([V[b, :, lens[b]] for b in range(B)]).contiguous()
    Qt = inp["Q"].cuda()
    out = torch.empty(B, w.Hq, 128, device="cuda")
    sc = torch.full((B, w.Hq, T0 + 1), float("nan"), device="cuda")
    sl = None if seqlens is None else torch.tensor(seqlens, dtype=torch.int32, device="cuda")
    ws = ctx.decode_workspace(B, w.Hq, w.Hkv, T0 + 1)
    Q.qjl_decode_step(ctx.handle, cache, Qt, kn, vn, T0, out, seqlens=sl, scores=sc, workspace=ws)
    torch.cuda.synchronize()
    Q.qjl_decode_workspace_status(ctx.handle, ws, B, w.Hq, w.Hkv)
    g = C.cache_to_numpy(cache, w.m_out, w.n_outlier, T=cache.cap)
    S, So = C.sketch64(w)
    K64, V64 = C.to64(inp["K"]), C.to64(inp["V"])
    guard_excl = 0
    for b in range(B):
        for h in range(w.Hkv):
            pos = lens[b]
            ks = O.sketch_keys(K64[b, h, pos:pos + 1], S, So, g["idx"][b, h])
            for part, mm in (("in", w.m), ("out", w.m_out)):
                if mm == 0:
                    continue
                want = ks[f"y_{part}"][0] >= 0
                excl = np.abs(ks[f"y_{part}"][0]) < C.SIGN_BAND * ks[f"norm_{part}"][0]
                got = C.unpack_bits(g[f"bits_{part}"][b, h, pos:pos + 1], mm)[0]
                assert not np.any((got != want) & ~excl), (b, h, part)
                guard_excl += int(excl.sum())
            assert np.array_equal(g["norms"][b, h, pos].view(np.uint16), ks["norms"][0].view(np.uint16))
            c, s_, z = O.quantize_values(V64[b, h, pos:pos + 1], vb)
            assert np.array_equal(g["codes"][b, h, pos], c[0])
            assert np.array_equal(g["scale"][b, h, pos].view(np.uint16), s_[0].view(np.uint16))
            assert np.array_equal(g["zero"][b, h, pos].view(np.uint16), z[0].view(np.uint16))
    assert guard_excl == 0
    new_lens = [l + 1 for l in lens]
    pairs = [(b, hq) for b in range(B) for hq in range(w.Hq)]
    C.compare_decode(g, C.to64(inp["Q"]), S, So, out.cpu().numpy().astype(np.float64),
                     sc.cpu().numpy().astype(np.float64), pairs, seqlens=new_lens)
    ctx.close()


@pytest.mark.parametrize("case", [
    ("long_context", 1, 3000, 2),    # 94 tiles over 94 blocks: each pair is merged from 47 parts
    ("llama3_8b_gqa", 64, 100, 4),   # 512 tiles, 148 blocks: several pairs per block
    ("llama2_7b_mha", 5, 1, 3),      # one token per sequence
])
def test_decode_stream_k_partition(case):
    """Tile ranges that cut pairs at arbitrary tiles, with merges of many parts."""
    name, B, T, Hkv = case
    inp = _small(name, B, T, Hkv)
    w = inp["workload"]
    ctx = _ctx(w)
    cache = C.quantize_on_gpu(ctx, inp["K"].cuda(), inp["V"].cuda())
    g = C.cache_to_numpy(cache, w.m_out, w.n_outlier)
    S, So = C.sketch64(w)
    O_gpu, sc_gpu = C.run_decode(ctx, cache, inp["Q"].cuda(), T)
    rng = np.random.default_rng(1)
    pairs = sorted({(int(rng.integers(w.B)), int(rng.integers(w.Hq))) for _ in range(12)})
    C.compare_decode(g, C.to64(inp["Q"]), S, So, O_gpu, sc_gpu, pairs)
    ctx.close()


def test_decode_wait_limit_reports_timeout():
    """A wait limit shorter than the work makes waits run out: the kernel
    returns with NaN in the outputs it owns and an error bit in the workspace
    header, the host reads QJL_ERR_TIMEOUT (and the status call clears the
    header), and the next call with the normal limit on the same workspace is
    correct again. Nothing faults or hangs: every wait is bounded."""
    # one sequence of 65536 tokens over 8 kv heads: about 55 tiles per block,
    # more than the shared-memory ring holds, so consumers wait for refills
    T = 65536
    inp = I.make_inputs(I.WORKLOADS["llama3_8b_gqa"], device="cuda", B=1, T=T, Hkv=8)
    w = inp["workload"]
    ctx = _ctx(w)
    cache = C.quantize_on_gpu(ctx, inp["K"], inp["V"])
    Qt = inp["Q"]
    ws = ctx.decode_workspace(w.B, w.Hq, w.Hkv, T)
    good, _ = C.run_decode(ctx, cache, Qt, T, want_scores=False)
    Q.qjl_set_wait_limit(ctx.handle, 1)  # 1 ns: any wait that is not over at once runs out
    timed_out = 0
    for _ in range(5):
        bad = torch.zeros(w.B, w.Hq, 128, device="cuda")
        Q.qjl_decode_attention(ctx.handle, cache, Qt, T, bad, workspace=ws)
        try:
            Q.qjl_decode_workspace_status(ctx.handle, ws, w.B, w.Hq, w.Hkv)
            assert np.array_equal(bad.cpu().numpy(), good.astype(np.float32))  # nothing ran out this time
        except Q.QJLError as e:
            assert "QJL_ERR_TIMEOUT" in str(e)
            assert torch.isnan(bad).any()
            timed_out += 1
    assert timed_out > 0
    Q.qjl_set_wait_limit(ctx.handle, 2_000_000_000)
    ref = torch.empty(w.B, w.Hq, 128, device="cuda")
    Q.qjl_decode_attention(ctx.handle, cache, Qt, T, ref, workspace=ws)
    Q.qjl_decode_workspace_status(ctx.handle, ws, w.B, w.Hq, w.Hkv)
    assert np.array_equal(ref.cpu().numpy(), good.astype(np.float32))
    ctx.close()


def _near_tie_values(rows, seed=29, top=15):
    """fp32 value rows [rows, 128] whose groups fix zero and scale (a min and a
    max) and whose other entries sit on, or one fp32 step beside, the half-way
    points between two of the top + 1 levels (the inputs where only the exact
    fp32 code decision gives the oracle's code)."""
    rng = np.random.default_rng(seed)
    out = np.empty((rows, 128), np.float32)
    for t in range(rows):
        for g in range(4):
            s = np.float32(np.float16(rng.uniform(0.01, 0.5)))
            z = np.float32(np.float16(rng.uniform(-2, 2)))
            vals = [z, np.float32(z + np.float32(top) * s)]
            while len(vals) < 32:
                h = np.float32(z + np.float32(int(rng.integers(0, top)) + 0.5) * s)
                vals += [h, np.nextafter(h, np.float32(np.inf)), np.nextafter(h, np.float32(-np.inf))]
            out[t, 32 * g:32 * g + 32] = np.array(vals[:32], np.float32)[rng.permutation(32)]
    return out


def test_two_bit_value_codes_near_ties_bit_exact():
    """2-bit codes (levels 0..3) on inputs built on their own half-way points:
    the oracle's code, scale and zero bit for bit."""
    V = torch.from_numpy(_near_tie_values(200, seed=31, top=3)).reshape(1, 2, 100, 128)
    K = torch.randn(1, 2, 100, 128, generator=torch.Generator().manual_seed(5))
    ctx = Q.QJLContext(0, 128, 256, 64, 8, value_bits=2)
    cache = C.quantize_on_gpu(ctx, K.cuda(), V.cuda())
    g = C.cache_to_numpy(cache, 64, 8)
    assert C.compare_values(g, V.double().numpy(), [(0, 0), (0, 1)], bits=2) == 0
    ctx.close()


def test_value_codes_near_ties_bit_exact():
    """The value quantiser (prefill kernel and the decode step's append) takes the
    oracle's IEEE fp32 code decision on inputs built on the half-way points."""
    V = torch.from_numpy(_near_tie_values(200)).reshape(1, 2, 100, 128)
    K = torch.randn(1, 2, 100, 128, generator=torch.Generator().manual_seed(3))
    ctx = Q.QJLContext(0, 128, 256, 64, 8)
    cache = C.quantize_on_gpu(ctx, K.cuda(), V.cuda())
    g = C.cache_to_numpy(cache, 64, 8)
    assert C.compare_values(g, V.double().numpy(), [(0, 0), (0, 1)]) == 0
    # the decode step's append of one such token per (sequence, kv head)
    cache2 = C.quantize_on_gpu(ctx, K[:, :, :99].cuda().contiguous(), V[:, :, :99].cuda().contiguous(), cap=128)
    Qt = torch.randn(1, 8, 128, device="cuda")
    out = torch.empty(1, 8, 128, device="cuda")
    ws = ctx.decode_workspace(1, 8, 2, 100)
    Q.qjl_decode_step(ctx.handle, cache2, Qt, K[:, :, 99].cuda().contiguous(), V[:, :, 99].cuda().contiguous(),
                      99, out, workspace=ws)
    torch.cuda.synchronize()
    g2 = C.cache_to_numpy(cache2, 64, 8, T=100)
    for h in range(2):
        c, s_, z = O.quantize_values(V[0, h, 99:100].double().numpy())
        assert np.array_equal(g2["codes"][0, h, 99], c[0])
        assert np.array_equal(g2["scale"][0, h, 99].view(np.uint16), s_[0].view(np.uint16))
    ctx.close()
