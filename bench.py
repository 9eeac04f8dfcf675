#!/usr/bin/env python
"""Benchmark of the QJL decode step on B200: cached tokens/s and HBM GB/s.

One step is one decode step of an attention layer for a batch of sequences:
  1. qjl_quantize_keys (QJL_APPEND) and qjl_quantize_values write the new
     token of every sequence into the cache (sign sketch, norms, 4-bit codes);
  2. qjl_decode_attention scores all T+1 cached tokens with the QJL estimator,
     runs the online softmax and accumulates the 4-bit values.
The prefill quantisation of the whole context (outlier-channel selection,
sign sketch, value codes) is timed separately and reported under "prefill".

Timing: CUDA events on the launching stream after warm-up, with a device
synchronise on both sides; the cache rotates over several copies whose total
size exceeds the 126 MB L2, so every step reads its cache from HBM. With
torchrun (N > 1) every rank runs its own batch (weak scaling, no collective in
the data path); the step time is the max over ranks.

`--impl reference` times the fp64 CPU oracle on the host cores instead (a
bounded sample of the same workload per step).
"""

from __future__ import annotations

import argparse
import ctypes
import datetime
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "QJL decode attention cached tokens/s and HBM GB/s (% of B200 roofline)"
UNIT = "cached tokens/s"
DEFAULT_WORKLOAD = "llama2_7b_mha"
L2_BYTES = 126 * 1024 * 1024


def parse_args():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", default="qjl", choices=["qjl", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--copies", type=int, default=0, help="rotating cache copies (0 = enough to exceed 3x L2)")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="bounded oracle sample for cpu_baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-prefill", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--decode-only", action="store_true",
                    help="profiling aid: prefill the cache once, then run only decode launches (no JSON line)")
    return ap.parse_args()


# ----------------------------------------------------------------------------- helpers

def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def recorded_traffic(kernel: str, workload: str):
    """dram bytes per launch from a committed ncu summary, if it matches the current kernel source."""
    import hashlib

    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f).get(f"{kernel}:{workload}")
    if not rec:
        return None
    src = os.path.join(ROOT, "decode_attention_qjl_b200", "csrc", rec["source"])
    sha = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16] if os.path.exists(src) else None
    return rec["dram_bytes_per_launch"] if sha == rec["source_sha"] else None


class ClockSampler:
    """Samples the SM clock and clock-event reasons of one GPU via NVML (read-only) in a thread."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x2: "applications_clocks_setting", 0x1: "gpu_idle"}

    def __init__(self, device_index: int, period_s: float = 0.01):
        self.samples, self.reasons, self.max_mhz, self.ok = [], set(), None, False
        self.period = period_s
        self._stop = threading.Event()
        try:
            import pynvml
            import torch

            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            try:
                self.h = pynvml.nvmlDeviceGetHandleByUUID(("GPU-" + uuid).encode() if not uuid.startswith("GPU-") else uuid.encode())
            except Exception:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.nvml = pynvml
            self.ok = True
        except Exception as e:  # pragma: no cover - depends on the box
            self.err = repr(e)

    def _run(self):
        nv = self.nvml
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                getr = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or nv.nvmlDeviceGetCurrentClocksThrottleReasons
                r = getr(self.h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0, "note": "NVML unavailable"}
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None, "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons - {"gpu_idle"}), "samples": len(self.samples)}


class FastCalls:
    """Pre-marshalled C-ABI calls for one decode step on one cache copy (argument
    marshalling done once, so the host enqueues a step in a few microseconds)."""

    def __init__(self, lib, ctx, cache, k_new, v_new, q, T_total, t_start, out, ws, stream_handle):
        from decode_attention_qjl_b200 import qjl as Q

        self.lib = lib
        self.cs = cache.struct()
        cp = ctypes.byref(self.cs)
        vp = ctypes.c_void_p
        s = vp(stream_handle)
        self.keys_args = (ctx, cp, vp(k_new.data_ptr()), Q.QJL_BF16 if k_new.dtype.itemsize == 2 else Q.QJL_FP32, 1,
                          k_new.stride(0), k_new.stride(1), k_new.stride(2), vp(t_start.data_ptr()), Q.QJL_APPEND,
                          None, 0, s)
        self.vals_args = (ctx, cp, vp(v_new.data_ptr()), Q.QJL_BF16 if v_new.dtype.itemsize == 2 else Q.QJL_FP32, 1,
                          v_new.stride(0), v_new.stride(1), v_new.stride(2), vp(t_start.data_ptr()), s)
        ws_bytes = ws.numel()
        self.dec_args = (ctx, cp, vp(q.data_ptr()), Q.QJL_BF16 if q.dtype.itemsize == 2 else Q.QJL_FP32, q.shape[1],
                         T_total, None, 0.0, vp(out.data_ptr()), None, vp(ws.data_ptr()), ws_bytes, s)

    def append(self):
        assert self.lib.qjl_quantize_keys(*self.keys_args) == 0
        assert self.lib.qjl_quantize_values(*self.vals_args) == 0

    def decode(self):
        assert self.lib.qjl_decode_attention(*self.dec_args) == 0


def dist_setup(args):
    import torch

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180), device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def max_over_ranks(world, values, device="cuda"):
    """Element-wise maximum over the ranks (the slowest rank sets each time);
    `device` is where the collective's tensor lives (cuda for NCCL, cpu for gloo)."""
    import torch

    t = torch.tensor(values, dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist

        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def cached_tokens_per_s(world, B, T_total, step_ms):
    """Whole-job throughput: every rank reads its own B sequences of T_total
    cached tokens per step (weak scaling); the step time is the max over ranks."""
    return world * B * T_total / (step_ms / 1e3)


# ----------------------------------------------------------------------------- oracle timing

def oracle_decode_sample(w, cache_np_fn, Q_host, seconds: float, max_pairs: int = 10_000):
    """Time the oracle's decode over (b, hq) pairs of the workload until `seconds` pass.

    Returns (token-heads per second, pairs done). The oracle runs with one BLAS thread."""
    import numpy as np
    from threadpoolctl import threadpool_limits

    import oracle as O

    S, So = O.sketch_pair(0, 128, w.m, w.m_out)
    rng = np.random.default_rng(0)
    done, tok_heads, elapsed = 0, 0, 0.0
    with threadpool_limits(limits=1):
        while elapsed < seconds and done < max_pairs:
            b, hq = int(rng.integers(w.B)), int(rng.integers(w.Hq))
            g = cache_np_fn(b, hq // w.g)
            q = Q_host[b:b + 1, hq:hq + 1]
            t0 = time.perf_counter()
            O.decode_batch(q, S, So, g["idx"], g["bits_in"], g["bits_out"], g["norms"], g["codes"], g["scale"],
                           g["zero"], pairs=[(0, 0)])
            elapsed += time.perf_counter() - t0
            done += 1
            tok_heads += g["bits_in"].shape[2]
    return tok_heads / elapsed, done, elapsed


# ----------------------------------------------------------------------------- reference arm

def run_reference(args):
    """The oracle as it stands, on the host cores: each step decodes one sampled
    (sequence, query head) pair of the workload over its full context (the oracle
    quantises that head's cache first, outside the timed step)."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import numpy as np
    import torch
    from threadpoolctl import threadpool_limits

    import oracle as O
    from decode_attention_qjl_b200 import inputs as I

    w = I.WORKLOADS[args.workload]
    S, So = O.sketch_pair(0, 128, w.m, w.m_out)
    rng = np.random.default_rng(0)
    n_heads = 4
    heads = []
    for _ in range(n_heads):
        b, hk = int(rng.integers(w.B)), int(rng.integers(w.Hkv))
        inp = I.make_inputs(w, seed=I.DATA_SEED + 7919 * b + hk, device="cpu", B=1, Hkv=1)
        K64 = inp["K"].float().numpy().astype(np.float64)
        V64 = inp["V"].float().numpy().astype(np.float64)
        c = O.quantize_cache(K64, V64, S, So, w.n_outlier)
        heads.append((c, inp["Q"].float().numpy().astype(np.float64)))
    times = []
    with threadpool_limits(limits=1):
        for i in range(args.warmup + args.steps):
            c, q = heads[i % n_heads]
            t0 = time.perf_counter()
            O.decode_batch(q[:, :1], S, So, c["idx"], c["bits_in"], c["bits_out"], c["norms"], c["codes"],
                           c["scale"], c["zero"], pairs=[(0, 0)])
            dt = time.perf_counter() - t0
            if i >= args.warmup:
                times.append(dt)
    step_s = sum(times) / len(times)
    # one step = T tokens of one query head; the metric counts a cached token over all Hq heads
    value = w.T / w.Hq / step_s
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": step_s * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "T": w.T, "m": w.m, "m_out": w.m_out,
                   "n_outlier": w.n_outlier, "step": "oracle decode of one sampled (sequence, query head) over T tokens"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle",
                         "sample": f"one (sequence, query head) pair of {w.T} tokens per step, {n_heads} heads rotated"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- GPU arm

def run_qjl(args):
    import numpy as np
    import torch

    from decode_attention_qjl_b200 import build as build_mod
    from decode_attention_qjl_b200 import inputs as I
    from decode_attention_qjl_b200 import qjl as Q

    world, rank, local = dist_setup(args)
    if rank == 0:
        build_mod.build()
    barrier(world)
    lib = Q.load_library()
    w = I.WORKLOADS[args.workload]
    dev = torch.device("cuda", torch.cuda.current_device())
    B, Hq, Hkv, T = w.B, w.Hq, w.Hkv, w.T
    Ttot = T + 1  # the decode step attends the T cached tokens plus the appended one
    peaks = measured_peaks()

    ctx = Q.QJLContext(0, 128, w.m, w.m_out, w.n_outlier)
    inp = I.make_inputs(w, seed=I.DATA_SEED + rank, device=dev)
    K, V, Qt = inp["K"], inp["V"], inp["Q"]
    cache_bytes = B * Hkv * Ttot * w.bytes_per_token_head()
    copies = args.copies or max(2, math.ceil(3 * L2_BYTES / cache_bytes))
    caches = [ctx.allocate_cache(B, Hkv, Ttot) for _ in range(copies)]
    kws = ctx.keys_workspace(B, Hkv)
    stream = torch.cuda.current_stream()

    # ---------------- prefill leg: outlier selection + sign sketch + value codes over T tokens
    prefill = None
    if args.decode_only:
        args.no_prefill = True
    pre_steps = 1 if args.no_prefill else max(3, min(10, args.steps))
    ev = lambda: torch.cuda.Event(enable_timing=True)
    keys_ms, vals_ms = [], []
    for i in range(copies + (0 if args.no_prefill else 2 + pre_steps)):
        c = caches[i % copies]
        a, b_, e_ = ev(), ev(), ev()
        a.record()
        Q.qjl_quantize_keys(ctx.handle, c, K, Q.QJL_PREFILL, workspace=kws)
        b_.record()
        Q.qjl_quantize_values(ctx.handle, c, V)
        e_.record()
        if i >= copies + 2:
            keys_ms.append((a, b_))
            vals_ms.append((b_, e_))
    torch.cuda.synchronize()
    if keys_ms:
        km = statistics.mean(x.elapsed_time(y) for x, y in keys_ms)
        vm = statistics.mean(x.elapsed_time(y) for x, y in vals_ms)
        ntok = B * Hkv * T
        k_bytes = ntok * (2 * 128) * 2 + ntok * (w.m // 8 + w.m_out // 8 + 4)  # K read twice (select, sketch) + out
        v_bytes = ntok * 2 * 128 + ntok * (64 + 16)
        flops = 2.0 * ntok * 128 * w.m  # the inlier projection K_in S^T on the tensor cores
        prefill = {
            "tokens": ntok, "quantize_keys_ms": km, "quantize_values_ms": vm,
            "token_heads_per_s": ntok / ((km + vm) / 1e3),
            "keys": {"bound": "tensor", "achieved_tflops": flops / (km / 1e3) / 1e12, "peak_tflops": peaks["bf16_tflops"],
                     "frac": flops / (km / 1e3) / 1e12 / peaks["bf16_tflops"], "hbm_gbs": k_bytes / (km / 1e3) / 1e9,
                     "note": "channel energy + outlier selection + tcgen05 inlier projection (bf16, fp32 accumulation "
                             "in tensor memory) with CUDA-core outlier sketch, norms and sign packing in one launch"},
            "values": {"bound": "hbm", "achieved": v_bytes / (vm / 1e3) / 1e9, "peak": peaks["hbm_gbs"],
                       "unit": "GB/s", "frac": v_bytes / (vm / 1e3) / 1e9 / peaks["hbm_gbs"]},
        }

    # ---------------- decode step inputs
    app = I.append_inputs(w, B, Hq, Hkv, seed=I.DATA_SEED + 100 + rank, device=dev,
                          outlier_ch=inp["outlier_channels"])
    t_start = torch.full((B,), T, dtype=torch.int32, device=dev)
    out = torch.empty(B, Hq, 128, dtype=torch.float32, device=dev)
    dws = ctx.decode_workspace(B, Hq, Hkv, Ttot)
    calls = [FastCalls(lib, ctx.handle, c, app["k"], app["v"], app["q"], Ttot, t_start, out, dws, stream.cuda_stream)
             for c in caches]
    del K, V
    torch.cuda.synchronize()

    if args.decode_only:
        for i in range(args.warmup + args.steps):
            calls[i % copies].decode()
        torch.cuda.synchronize()
        ctx.close()
        return
    for i in range(args.warmup):
        calls[i % copies].append()
        calls[i % copies].decode()
    torch.cuda.synchronize()
    barrier(world)

    K_steps = args.steps
    e0, e1 = ev(), ev()
    d_ev = [(ev(), ev()) for _ in range(K_steps)]
    sampler = ClockSampler(torch.cuda.current_device())
    with sampler:
        torch.cuda.synchronize()
        e0.record()
        for i in range(K_steps):
            c = calls[i % copies]
            c.append()
            d_ev[i][0].record()
            c.decode()
            d_ev[i][1].record()
        e1.record()
        torch.cuda.synchronize()
    barrier(world)
    step_ms = e0.elapsed_time(e1) / K_steps
    dec_ms = statistics.mean(a.elapsed_time(b) for a, b in d_ev)
    step_ms, dec_ms = max_over_ranks(world, [step_ms, dec_ms])

    dec_bytes = B * Hkv * Ttot * w.bytes_per_token_head() + B * Hq * 128 * (2 + 4) + B * Hkv * w.n_outlier * 4
    app_bytes = B * Hkv * (2 * 128 * 2 + w.bytes_per_token_head())
    value = cached_tokens_per_s(world, B, Ttot, step_ms)
    achieved = dec_bytes / (dec_ms / 1e3) / 1e9

    # ---------------- end to end through the public API with pinned host buffers
    e2e = None
    if not args.no_e2e:
        kh = app["k"].cpu().pin_memory()
        vh = app["v"].cpu().pin_memory()
        qh = app["q"].cpu().pin_memory()
        oh = torch.empty(B, Hq, 128, dtype=torch.float32).pin_memory()
        kd, vd, qd = torch.empty_like(app["k"]), torch.empty_like(app["v"]), torch.empty_like(app["q"])
        n_e2e = max(3, min(K_steps, 1000))

        def e2e_step(c):
            kd.copy_(kh, non_blocking=True)
            vd.copy_(vh, non_blocking=True)
            qd.copy_(qh, non_blocking=True)
            Q.qjl_quantize_keys(ctx.handle, c, kd, Q.QJL_APPEND, t_start=t_start)
            Q.qjl_quantize_values(ctx.handle, c, vd, t_start=t_start)
            Q.qjl_decode_attention(ctx.handle, c, qd, Ttot, out, workspace=dws)
            oh.copy_(out, non_blocking=True)

        for i in range(3):
            e2e_step(caches[i % copies])
        torch.cuda.synchronize()
        barrier(world)
        a, b_ = ev(), ev()
        a.record()
        for i in range(n_e2e):
            e2e_step(caches[i % copies])
        b_.record()
        torch.cuda.synchronize()
        (e2e_ms,) = max_over_ranks(world, [a.elapsed_time(b_) / n_e2e])
        e2e = {"value": cached_tokens_per_s(world, B, Ttot, e2e_ms), "unit": UNIT,
               "h2d_bytes_per_step": int(kh.numel() * kh.element_size() + vh.numel() * vh.element_size()
                                         + qh.numel() * qh.element_size()),
               "d2h_bytes_per_step": int(oh.numel() * oh.element_size()), "ms_per_step": e2e_ms, "steps": n_e2e}

    # ---------------- CPU oracle baseline (rank 0, N = 1 only)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        from tests.gpu_common import cache_to_numpy  # noqa: F401  (host copy of a cache slice)

        c0 = caches[0]
        Q_host = app["q"].float().cpu().numpy().astype(np.float64)
        fn = lambda b, hk: cache_to_numpy(c0, w.m_out, w.n_outlier, b=b, h=hk)
        th_per_s, pairs, secs = oracle_decode_sample(w, fn, Q_host, args.cpu_seconds)
        cpu = {"value": th_per_s / Hq, "unit": UNIT, "cores": 1, "kind": "oracle",
               "sample": f"{pairs} random (sequence, query head) pairs over {Ttot} tokens each ({secs:.1f} s of CPU), "
                         f"scaled to cached tokens/s by 1/Hq"}

    clocks = sampler.summary()
    traffic = recorded_traffic("decode", w.name)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K_steps, "warmup": args.warmup,
        "ms_per_step": step_ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic: K,V,Q ~ N(0,1) bf16 with planted outlier key channels; seed 1234 + rank",
        "config": {"workload": w.name, "B": B, "Hq": Hq, "Hkv": Hkv, "T": Ttot, "d": 128, "m": w.m, "m_out": w.m_out,
                   "n_outlier": w.n_outlier, "value_bits": 4, "value_group": 32,
                   "l2": f"{copies} rotating cache copies, {copies * cache_bytes / 1e6:.0f} MB > 126 MB L2",
                   "parallelism": f"dp{world}: independent batches per GPU, no collective",
                   "step": "append-quantize 1 token/sequence + decode over T+1 tokens"},
        "hbm_gbs": (dec_bytes + app_bytes) / (step_ms / 1e3) / 1e9,
        "decode_ms": dec_ms,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved / peaks["hbm_gbs"], "traffic": traffic,
                     "kernel": "qjl_decode_attention", "algorithmic_bytes_per_launch": dec_bytes,
                     "peak_source": peaks["source"], "frac_of_8TBs": achieved / 8000.0},
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": 3 * K_steps,
        "clocks": clocks,
        "prefill": prefill,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    ctx.close()
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()


def main():
    args = parse_args()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_qjl(args)


if __name__ == "__main__":
    main()
