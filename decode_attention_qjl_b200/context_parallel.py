"""Context-parallel decode: a long context split over the ranks of a process group.

"2 numbers out of 128 destroy the entire KV cache" (Towards AI), "The Memory
Math": the KV cache grows linearly with the context and outgrows one device.
Here every rank holds a contiguous shard of each sequence's cached tokens (its
own QJL cache, quantised from its own tokens), and a decode step is

  1. qjl_decode_attention_partial on the local shard: per (sequence, query
     head) the unnormalised output, the maximum logit and the sum of
     exponentials, written into one packed fp32 buffer;
  2. one all-gather of that buffer over the group (NCCL between GPUs): the
     only exchange, B * Hq * (d + 2) floats per rank;
  3. qjl_merge_partials on every rank: softmax is exp(x - M) / sum exp(x - M)
     for any M >= max x ("Your Brain Already Runs on 1-Bit Keys", "Why
     Truncation Kills"), so the shards' parts combine exactly.

Steps 1 and 3 are the library's kernels; this module only lays out the buffers
and issues the collective. The outlier channels of a shard are the ones its
own prefill keys select (qjl_quantize_keys in prefill mode on the shard).
"""

from __future__ import annotations

import torch
import torch.distributed as dist

from . import qjl as Q

__all__ = ["shard_bounds", "local_seqlens", "ContextParallelDecode"]


def shard_bounds(T: int, world: int, rank: int) -> tuple[int, int]:
    """Token positions [start, stop) of rank `rank` in a context of T tokens:
    contiguous shards, the first T % world ranks one token longer."""
    if world < 1 or not 0 <= rank < world or T < 0:
        raise ValueError("need world >= 1, 0 <= rank < world and T >= 0")
    base, extra = divmod(T, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def local_seqlens(seqlens, T: int, world: int, rank: int) -> list[int]:
    """The number of each sequence's first seqlens[b] tokens that fall in this rank's shard."""
    start, stop = shard_bounds(T, world, rank)
    return [max(0, min(int(n), stop) - start) for n in seqlens]


class ContextParallelDecode:
    """One decode step over a context sharded across a process group.

    ``decode_partial`` and ``merge`` default to the library's
    qjl_decode_attention_partial and qjl_merge_partials (CUDA); the buffers
    live on ``device``. Every rank must call with the same B, Hq and d.
    """

    def __init__(self, B: int, Hq: int, d: int = 128, group=None, device=None, decode_partial=None, merge=None):
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.B, self.Hq, self.d = B, Hq, d
        self.rows = B * Hq
        # one rank's packed parts: O [rows, d], then (max, sum) [rows, 2], padded to 16 bytes
        self.o_floats = self.rows * d
        self.ml_floats = 2 * self.rows
        self.part_floats = self.o_floats + ((self.ml_floats + 3) // 4) * 4
        dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
        self.part = torch.zeros(self.part_floats, dtype=torch.float32, device=dev)
        self.gathered = torch.zeros(self.world * self.part_floats, dtype=torch.float32, device=dev)
        self.decode_partial = decode_partial or Q.qjl_decode_attention_partial
        self.merge = merge or Q.qjl_merge_partials

    def local_parts(self):
        """Views of this rank's packed buffer: O_part [B, Hq, d] and ML_part [B, Hq, 2]."""
        o = self.part[:self.o_floats].view(self.B, self.Hq, self.d)
        ml = self.part[self.o_floats:self.o_floats + self.ml_floats].view(self.B, self.Hq, 2)
        return o, ml

    def gathered_parts(self):
        """Every rank's parts after the exchange: [world, rows * d] and [world, rows * 2] views
        (rank stride part_floats)."""
        g = self.gathered.view(self.world, self.part_floats)
        return g[:, :self.o_floats], g[:, self.o_floats:self.o_floats + self.ml_floats]

    def __call__(self, ctx, cache, Qt, T_local: int, O, seqlens_local=None, sm_scale: float = 0.0, workspace=None):
        """Decode Qt [B, Hq, d] over this rank's shard (T_local tokens, or seqlens_local [B] on the
        device) and all other ranks' shards; O [B, Hq, d] fp32 receives the merged output."""
        o, ml = self.local_parts()
        self.decode_partial(ctx, cache, Qt, T_local, o, ml, seqlens=seqlens_local, sm_scale=sm_scale,
                            workspace=workspace)
        dist.all_gather_into_tensor(self.gathered, self.part, group=self.group)
        O_parts, ML_parts = self.gathered_parts()
        self.merge(O_parts, ML_parts, O)
        return O
