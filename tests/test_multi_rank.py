"""The multi-rank host path of bench.py on CPU: two gloo ranks.

With N GPUs every rank decodes its own batch (seeded DATA_SEED + rank), with
no collective in the data path; the only exchange is the step time, the
maximum over the ranks, and the whole-job value counts the tokens of all
ranks. These tests run that exchange and the per-rank input recipe on two
processes over gloo, without a GPU.
"""
import os
import socket

import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402

import bench  # noqa: E402
from decode_attention_qjl_b200 import inputs as I  # noqa: E402


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # each rank's own (step, decode) times; the job takes the slowest of each
        mine = [10.0 + rank, 5.0 - rank]
        bench.barrier(world)
        got = bench.max_over_ranks(world, mine, device="cpu")
        # the per-rank input recipe: a small case of the bench workload
        w = I.WORKLOADS["llama2_7b_mha"]
        inp = I.make_inputs(w, seed=I.DATA_SEED + rank, device="cpu", B=1, T=64, Hkv=1)
        q = inp["Q"].float()
        sums = [torch.zeros_like(q) for _ in range(world)]
        dist.all_gather(sums, q)
        out[rank] = {"max": got, "distinct": not torch.equal(sums[0], sums[1])}
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(300)
def test_two_gloo_ranks_take_the_slowest_time_and_draw_their_own_inputs():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        mp.start_processes(_worker, args=(world, port, out), nprocs=world, join=True, start_method="spawn")
        res = dict(out)
    for rank in range(world):
        assert res[rank]["max"] == [11.0, 5.0]  # step: rank 1's 11 ms; decode: rank 0's 5 ms
        assert res[rank]["distinct"]            # DATA_SEED + rank gives each rank its own batch


def test_whole_job_value_counts_every_rank():
    # 2 ranks x 8 sequences x 4097 tokens in 0.1 ms
    assert bench.cached_tokens_per_s(2, 8, 4097, 0.1) == pytest.approx(2 * 8 * 4097 / 1e-4)
    assert bench.cached_tokens_per_s(1, 8, 4097, 0.1) * 2 == pytest.approx(bench.cached_tokens_per_s(2, 8, 4097, 0.1))
