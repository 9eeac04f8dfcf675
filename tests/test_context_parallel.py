"""Context-parallel decode, host side, on two gloo ranks (no GPU).

decode_attention_qjl_b200.context_parallel shards each sequence's tokens over
the ranks, lays out the packed per-rank parts, all-gathers them and hands them
to the merge. Here the two compute steps are the oracle's (injected), so the
test runs the module's own sharding, buffer layout and collective on the CPU
and checks the result against the oracle's merge of the same shards and
against the oracle's decode of the whole context. The CUDA steps are covered
by tests/test_gpu_context_parallel.py.
"""
import math
import os
import socket

import numpy as np
import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402

import oracle as O  # noqa: E402
from decode_attention_qjl_b200 import context_parallel as CP  # noqa: E402

LOG2E = 1.0 / math.log(2.0)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _problem(B=2, Hkv=2, g=2, T=37, d=128, m=64, m_out=32, seed=3):
    """A small cache with planted outlier channels (so every shard selects the same ones)."""
    rng = np.random.default_rng(seed)
    K = rng.standard_normal((B, Hkv, T, d))
    planted = np.array([[rng.choice(d, 4, replace=False) for _ in range(Hkv)] for _ in range(B)])
    for b in range(B):
        for h in range(Hkv):
            K[b, h][:, np.sort(planted[b, h])] *= 20.0
    V = rng.standard_normal((B, Hkv, T, d)).astype(np.float32).astype(np.float64)
    Qv = rng.standard_normal((B, Hkv * g, d))
    S, So = O.sketch_pair(0, d, m, m_out)
    return K, V, Qv, S, So


def _oracle_cache(K, V, S, So, a, b):
    return O.quantize_cache(K[:, :, a:b], V[:, :, a:b], S, So, 4)


def _oracle_decode_partial(S, So, g):
    def run(ctx, cache, Qt, T_local, o, ml, seqlens=None, sm_scale=0.0, workspace=None):
        B, Hq, _ = Qt.shape
        for b in range(B):
            n = T_local if seqlens is None else int(seqlens[b])
            for h in range(Hq):
                hk = h // g
                ob, mx, l = O.decode_partial(Qt[b, h].numpy(), S, So, cache["idx"][b, hk], cache["bits_in"][b, hk, :n],
                                             cache["bits_out"][b, hk, :n], cache["norms"][b, hk, :n],
                                             cache["codes"][b, hk, :n], cache["scale"][b, hk, :n],
                                             cache["zero"][b, hk, :n], sm_scale or None)
                o[b, h] = torch.from_numpy(ob)
                ml[b, h, 0] = mx * LOG2E  # the library keeps logits in log2 units
                ml[b, h, 1] = l
        return o, ml
    return run


def _oracle_merge(O_parts, ML_parts, Out):
    R = O_parts.shape[0]
    B, Hq, d = Out.shape
    op = O_parts.reshape(R, B * Hq, d).numpy()
    mlp = ML_parts.reshape(R, B * Hq, 2).numpy()
    for row in range(B * Hq):
        parts = [(op[r, row], mlp[r, row, 0] / LOG2E, mlp[r, row, 1]) for r in range(R)]
        Out.view(B * Hq, d)[row] = torch.from_numpy(O.merge_partials(parts))
    return Out


def _worker(rank, world, port, seqlens, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        K, V, Qv, S, So = _problem()
        B, Hkv, T, d = K.shape
        g = Qv.shape[1] // Hkv
        a, b = CP.shard_bounds(T, world, rank)
        cache = _oracle_cache(K, V, S, So, a, b)
        sl = None if seqlens is None else CP.local_seqlens(seqlens, T, world, rank)
        dec = CP.ContextParallelDecode(B, Qv.shape[1], d, device="cpu", decode_partial=_oracle_decode_partial(S, So, g),
                                       merge=_oracle_merge)
        Out = torch.zeros(B, Qv.shape[1], d, dtype=torch.float32)
        dec(None, cache, torch.from_numpy(Qv), b - a, Out, seqlens_local=sl)
        out[rank] = Out.numpy().astype(np.float64)
    finally:
        dist.destroy_process_group()


def _reference(seqlens, world):
    """The oracle, by hand: every shard's partial over its own cache, merged; and the whole-context decode."""
    K, V, Qv, S, So = _problem()
    B, Hkv, T, d = K.shape
    g = Qv.shape[1] // Hkv
    whole = _oracle_cache(K, V, S, So, 0, T)
    merged = np.zeros((B, Qv.shape[1], d))
    for r_b in range(B):
        n_all = T if seqlens is None else seqlens[r_b]
        parts_by_rank = []
        for r in range(world):
            a, b = CP.shard_bounds(T, world, r)
            parts_by_rank.append((_oracle_cache(K, V, S, So, a, b), max(0, min(n_all, b) - a)))
        for h in range(Qv.shape[1]):
            hk = h // g
            parts = []
            for c, n in parts_by_rank:
                parts.append(O.decode_partial(Qv[r_b, h], S, So, c["idx"][r_b, hk], c["bits_in"][r_b, hk, :n],
                                              c["bits_out"][r_b, hk, :n], c["norms"][r_b, hk, :n],
                                              c["codes"][r_b, hk, :n], c["scale"][r_b, hk, :n], c["zero"][r_b, hk, :n]))
            merged[r_b, h] = O.merge_partials(parts)
    full, _ = O.decode_batch(Qv, S, So, whole["idx"], whole["bits_in"], whole["bits_out"], whole["norms"],
                             whole["codes"], whole["scale"], whole["zero"], seqlens=seqlens)
    return merged, full


def test_shard_bounds_and_local_lengths():
    for T in (0, 1, 5, 37, 64):
        for world in (1, 2, 3, 8):
            bounds = [CP.shard_bounds(T, world, r) for r in range(world)]
            assert bounds[0][0] == 0 and bounds[-1][1] == T
            assert all(bounds[r][1] == bounds[r + 1][0] for r in range(world - 1))
            sizes = [b - a for a, b in bounds]
            assert max(sizes) - min(sizes) <= 1
            lens = [0, min(1, T), T // 2, T]
            per_rank = [CP.local_seqlens(lens, T, world, r) for r in range(world)]
            assert [sum(x[i] for x in per_rank) for i in range(len(lens))] == lens
    with pytest.raises(ValueError):
        CP.shard_bounds(5, 2, 2)


@pytest.mark.timeout(300)
@pytest.mark.parametrize("seqlens", [None, [37, 11]])  # sequence 1 lies in rank 0's shard only
def test_two_gloo_ranks_merge_their_shards(seqlens):
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        mp.start_processes(_worker, args=(world, port, seqlens, out), nprocs=world, join=True, start_method="spawn")
        res = dict(out)
    merged, full = _reference(seqlens, world)
    for rank in range(world):
        # every rank ends with the same merged output: the oracle's merge of the same shards (fp32 buffers)
        np.testing.assert_allclose(res[rank], merged, rtol=1e-5, atol=1e-6)
        # the planted outliers make every shard pick the whole context's channels: the merge is the full decode
        np.testing.assert_allclose(res[rank], full, rtol=1e-5, atol=1e-6)
