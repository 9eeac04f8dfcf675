#!/usr/bin/env python
"""Benchmark of the QJL decode step on B200: cached tokens/s and HBM GB/s.

One step is one decode step of an attention layer for a batch of sequences,
one launch of qjl_decode_step: every sequence's new token is appended to the
cache (key sign sketch, norms, 4-bit value codes) and then all T+1 cached
tokens are scored with the QJL estimator, softmaxed and their 4-bit values
accumulated.

The headline line is the large-context GQA workload (4 sequences x 131072
tokens, 8 kv heads, 32 query heads); `per_workload` in the same line carries
the step time and roofline of the other decode workloads (Llama-2-7B MHA,
long context, Llama-3-8B GQA, the batch-64 sweep point). The prefill
quantisation of the whole context (outlier-channel selection, sign sketch,
value codes) is timed separately and reported under "prefill". The same
step with 2-bit value codes, and decode over the same tokens kept as bf16, FP8
and min-max caches (the library's comparison kernels), are reported under
"comparison". `--bits-table` prints the bits-per-number table instead.

Timing: CUDA events on the launching stream after warm-up, with a device
synchronise on both sides; the cache rotates over enough copies that their
total exceeds 3x the 126 MB L2 (one copy when a single cache already does),
so every step reads its cache from HBM. With torchrun (N > 1) every rank runs
its own batch (weak scaling, no collective in the data path); the step time
is the max over ranks.

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
HEADLINE = "sweep_m256_b4_t128k"
OTHER_WORKLOADS = ["long_context", "sweep_m256_b64_t16k", "llama3_8b_gqa", "llama2_7b_mha"]
PREFILL_WORKLOAD = "long_context"  # 32768 tokens x 32 heads
L2_BYTES = 126 * 1024 * 1024


def parse_args():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="qjl", choices=["qjl", "reference"])
    ap.add_argument("--workload", default=HEADLINE)
    ap.add_argument("--only", action="store_true", help="time the --workload alone (no per-workload table)")
    ap.add_argument("--cpu-seconds", type=float, default=6.0, help="bounded oracle sample per cpu_baseline leg")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-prefill", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-comparison", action="store_true", help="skip the bf16 / FP8 cache decode comparison")
    ap.add_argument("--bits-table", action="store_true",
                    help="print the bits-per-FPN vs estimator-error table (m, outlier channels) and exit")
    ap.add_argument("--decode-only", action="store_true",
                    help="profiling aid: prefill the cache once, then run only decode-step launches (no JSON line)")
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

    def __init__(self, device_index: int, period_s: float = 0.002):
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

    def _sample(self):
        nv = self.nvml
        try:
            self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
            getr = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or nv.nvmlDeviceGetCurrentClocksThrottleReasons
            r = getr(self.h)
            for bit, name in self.REASONS.items():
                if r & bit:
                    self.reasons.add(name)
        except Exception:
            pass

    def _run(self):
        while not self._stop.is_set():
            self._sample()
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self._sample()
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


class StepCall:
    """A pre-marshalled qjl_decode_step call on one cache copy (argument
    marshalling done once, so the host enqueues a step in a few microseconds)."""

    def __init__(self, lib, ctx, cache, q, k_new, v_new, T, out, ws, stream_handle):
        from decode_attention_qjl_b200 import qjl as Q

        self.lib = lib
        self.cs = cache.struct()
        vp = ctypes.c_void_p
        dt = Q.QJL_BF16 if q.dtype.itemsize == 2 else Q.QJL_FP32
        self.args = (ctx, ctypes.byref(self.cs), vp(q.data_ptr()), vp(k_new.data_ptr()), k_new.stride(0),
                     k_new.stride(1), vp(v_new.data_ptr()), v_new.stride(0), v_new.stride(1), dt, q.shape[1], T, None,
                     0.0, vp(out.data_ptr()), None, vp(ws.data_ptr()), ws.numel(), vp(stream_handle))

    def __call__(self):
        assert self.lib.qjl_decode_step(*self.args) == 0


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


def step_bytes(w, T_total):
    """Algorithmic HBM bytes of one decode step: the cache of T_total tokens per
    (sequence, kv head), the queries, the outputs, the outlier channels, the new
    token's key and value rows and the slot they are written to."""
    bh = w.B * w.Hkv
    return (bh * T_total * w.bytes_per_token_head() + w.B * w.Hq * 128 * (2 + 4) + bh * w.n_outlier * 4
            + bh * 2 * 128 * 2 + bh * w.bytes_per_token_head())


def pair_to_host(cache, b, hk, T, m_out):
    """Host copies (numpy) of one (sequence, kv head) slab of a cache, in the
    cache's own stored formats: sign words, fp16 norms, packed codes, fp16
    scale / zero (the binding's section views; no arithmetic)."""
    import numpy as np

    sec = lambda name: cache.section(name)[b:b + 1, hk:hk + 1, :T].cpu().numpy()
    return {
        "idx": cache.outlier_idx[b:b + 1, hk:hk + 1].cpu().numpy().astype(np.int64),
        "bits_in": sec("kbits").view(np.uint32),
        "bits_out": sec("kbits_out").view(np.uint32) if m_out else np.zeros((1, 1, T, 0), np.uint32),
        "norms": sec("knorm"),
        "vcode": sec("vcode"),
        "vsz": cache.section("vsz")[b:b + 1, hk:hk + 1, :T].cpu().numpy(),
    }


# ----------------------------------------------------------------------------- oracle timing

def _oracle_decode_loop(payload):
    """Worker: decode one (sequence, query head) pair with the oracle for `seconds`;
    returns (pairs decoded, tokens per pair, seconds). One BLAS thread."""
    import numpy as np
    from threadpoolctl import threadpool_limits

    import oracle as O

    (S_seed, m, m_out, q, host, seconds) = payload
    S, So = O.sketch_pair(S_seed, 128, m, m_out)
    codes = O.unpack_codes(host["vcode"])
    scale, zero = host["vsz"][..., 0], host["vsz"][..., 1]
    n, t_total = 0, 0.0
    with threadpool_limits(limits=1):
        t0 = time.perf_counter()
        while time.perf_counter() - t0 < seconds:
            O.decode_batch(q, S, So, host["idx"], host["bits_in"], host["bits_out"], host["norms"], codes, scale, zero,
                           pairs=[(0, 0)])
            n += 1
        t_total = time.perf_counter() - t0
    return n, host["bits_in"].shape[2], t_total


def cpu_baseline(w, host, q, seconds, T_total, max_procs=64):
    """The oracle as it stands on this machine's host cores: one thread, and one
    spawned process per core (at most max_procs), each decoding the same
    (sequence, query head) pair over its first tokens for `seconds`. Scaled to
    cached tokens/s over all query heads by 1/Hq."""
    import multiprocessing as mp

    payload = (0, w.m, w.m_out, q, host, seconds)
    n1, tok, s1 = _oracle_decode_loop(payload)
    one = n1 * tok / s1 / w.Hq
    cores = os.cpu_count() or 1
    procs = min(cores, max_procs)
    ctx = mp.get_context("spawn")
    t0 = time.perf_counter()
    with ctx.Pool(procs) as pool:
        res = pool.map(_oracle_decode_loop, [payload] * procs)
    wall = time.perf_counter() - t0
    nN = sum(r[0] for r in res)
    allc = nN * tok / max(r[2] for r in res) / w.Hq
    sample = (f"one (sequence, query head) pair, its first {tok} of {T_total} cached tokens, decoded repeatedly by "
              f"the fp64 oracle for {seconds:.0f} s per process; scaled to cached tokens/s by 1/Hq")
    return ({"value": one, "unit": UNIT, "cores": 1, "kind": "oracle", "sample": sample + f" ({n1} decodes)"},
            {"value": allc, "unit": UNIT, "cores": procs, "host_cpu_count": cores, "kind": "oracle",
             "sample": sample + f" ({nN} decodes in {procs} processes, {wall:.1f} s wall)"})


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
    from threadpoolctl import threadpool_limits

    import oracle as O
    from decode_attention_qjl_b200 import inputs as I

    w = I.WORKLOADS[args.workload]
    T = w.T + 1  # the GPU arm's step attends the T cached tokens and the appended one
    S, So = O.sketch_pair(0, 128, w.m, w.m_out)
    rng = np.random.default_rng(0)
    n_heads = 2
    heads = []
    for _ in range(n_heads):
        b, hk = int(rng.integers(w.B)), int(rng.integers(w.Hkv))
        inp = I.make_inputs(w, seed=I.DATA_SEED + 7919 * b + hk, device="cpu", B=1, Hkv=1, T=T)
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
    value = T / w.Hq / step_s
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": step_s * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "T": T, "d": 128, "m": w.m,
                   "m_out": w.m_out, "n_outlier": w.n_outlier, "value_bits": 4, "value_group": 32,
                   "step": "oracle decode of one sampled (sequence, query head) over T tokens"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle",
                         "sample": f"one (sequence, query head) pair of {T} tokens per step, {n_heads} heads rotated"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- GPU arm

class Setup:
    """One workload on the device: the context, rotating prefilled caches, the
    step inputs and pre-marshalled step calls."""

    def __init__(self, w, rank, lib, dev, prefill_steps=0):
        import torch

        from decode_attention_qjl_b200 import inputs as I
        from decode_attention_qjl_b200 import qjl as Q

        self.w = w
        self.T = w.T
        self.Ttot = w.T + 1  # the step attends the T cached tokens plus the appended one
        self.ctx = Q.QJLContext(0, 128, w.m, w.m_out, w.n_outlier)
        inp = I.make_inputs(w, seed=I.DATA_SEED + rank, device=dev)
        self.K, self.V = inp["K"], inp["V"]
        cache_bytes = w.B * w.Hkv * self.Ttot * w.bytes_per_token_head()
        self.copies = max(1, math.ceil(3 * L2_BYTES / cache_bytes))
        self.cache_bytes = cache_bytes
        self.caches = [self.ctx.allocate_cache(w.B, w.Hkv, self.Ttot) for _ in range(self.copies)]
        kws = self.ctx.keys_workspace(w.B, w.Hkv)
        ev = lambda: torch.cuda.Event(enable_timing=True)
        keys_ms, vals_ms = [], []
        for i in range(self.copies + (2 + prefill_steps if prefill_steps else 0)):
            c = self.caches[i % self.copies]
            a, b_, e_ = ev(), ev(), ev()
            a.record()
            Q.qjl_quantize_keys(self.ctx.handle, c, self.K, Q.QJL_PREFILL, workspace=kws)
            b_.record()
            Q.qjl_quantize_values(self.ctx.handle, c, self.V)
            e_.record()
            if i >= self.copies + 2:
                keys_ms.append((a, b_))
                vals_ms.append((b_, e_))
        torch.cuda.synchronize()
        self.prefill = None
        if keys_ms:
            self.prefill = (statistics.mean(x.elapsed_time(y) for x, y in keys_ms),
                            statistics.mean(x.elapsed_time(y) for x, y in vals_ms))
        self.app = I.append_inputs(w, w.B, w.Hq, w.Hkv, seed=I.DATA_SEED + 100 + rank, device=dev,
                                   outlier_ch=inp["outlier_channels"])
        self.k_new = self.app["k"][:, :, 0].contiguous()
        self.v_new = self.app["v"][:, :, 0].contiguous()
        self.q = self.app["q"]
        self.out = torch.empty(w.B, w.Hq, 128, dtype=torch.float32, device=dev)
        self.ws = self.ctx.decode_workspace(w.B, w.Hq, w.Hkv, self.Ttot)
        stream = torch.cuda.current_stream()
        self.calls = [StepCall(lib, self.ctx.handle, c, self.q, self.k_new, self.v_new, self.T, self.out, self.ws,
                               stream.cuda_stream) for c in self.caches]

    def time_steps(self, K_steps, warmup, world, sampler=None):
        """(step ms, mean launch ms), K_steps timed steps after `warmup`, max over ranks."""
        import torch

        ev = lambda: torch.cuda.Event(enable_timing=True)
        for i in range(warmup):
            self.calls[i % self.copies]()
        torch.cuda.synchronize()
        barrier(world)
        e0, e1 = ev(), ev()
        d_ev = [(ev(), ev()) for _ in range(K_steps)]
        ctxm = sampler if sampler is not None else _Null()
        with ctxm:
            torch.cuda.synchronize()
            e0.record()
            for i in range(K_steps):
                d_ev[i][0].record()
                self.calls[i % self.copies]()
                d_ev[i][1].record()
            e1.record()
            torch.cuda.synchronize()
        barrier(world)
        step_ms = e0.elapsed_time(e1) / K_steps
        launch_ms = statistics.mean(a.elapsed_time(b) for a, b in d_ev)
        return max_over_ranks(world, [step_ms, launch_ms])

    def exact_error(self, n_pairs=4):
        """Error of the last step's output against exact softmax attention on the
        original K, V (plus the appended token), fp64, on sampled (sequence,
        query head) pairs: max / mean absolute error and the lowest cosine."""
        import torch

        w = self.w
        gen = torch.Generator().manual_seed(5)
        errs, cos = [], []
        for _ in range(n_pairs):
            b = int(torch.randint(w.B, (1,), generator=gen))
            hq = int(torch.randint(w.Hq, (1,), generator=gen))
            hk = hq // w.g
            k = torch.cat([self.K[b, hk, :self.T], self.k_new[b, hk][None]]).double()
            v = torch.cat([self.V[b, hk, :self.T], self.v_new[b, hk][None]]).double()
            q = self.q[b, hq].double()
            p = torch.softmax(k @ q / math.sqrt(128), dim=0)
            ref = p @ v
            got = self.out[b, hq].double()
            errs.append((got - ref).abs())
            cos.append(float(torch.dot(got, ref) / (got.norm() * ref.norm())))
        e = torch.cat(errs)
        return {"max_abs": float(e.max()), "mean_abs": float(e.mean()), "min_cosine": min(cos), "pairs": n_pairs,
                "reference": "softmax(q K^T / sqrt(d)) V in fp64 on the original bf16 K, V"}

    def close(self):
        self.ctx.close()


class _Null:
    def __enter__(self):
        return self

    def __exit__(self, *a):
        return False


def roofline(w, Ttot, launch_ms, peaks, traffic=None):
    nbytes = step_bytes(w, Ttot)
    achieved = nbytes / (launch_ms / 1e3) / 1e9
    return {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": achieved / peaks["hbm_gbs"], "traffic": traffic, "kernel": "qjl_decode_step (decode_kernel)",
            "algorithmic_bytes_per_launch": nbytes, "peak_source": peaks["source"],
            "frac_of_8TBs": achieved / 8000.0}


def run_qjl(args):
    import torch

    from decode_attention_qjl_b200 import build as build_mod
    from decode_attention_qjl_b200 import inputs as I
    from decode_attention_qjl_b200 import qjl as Q

    world, rank, local = dist_setup(args)
    if rank == 0:
        build_mod.build()
    barrier(world)
    lib = Q.load_library()
    dev = torch.device("cuda", torch.cuda.current_device())
    peaks = measured_peaks()
    K_steps, W = args.steps, max(3, args.warmup)

    w = I.WORKLOADS[args.workload]
    s = Setup(w, rank, lib, dev, prefill_steps=0 if args.no_prefill or args.decode_only else 5)
    if args.decode_only:
        for i in range(W + K_steps):
            s.calls[i % s.copies]()
        torch.cuda.synchronize()
        s.close()
        return

    sampler = ClockSampler(torch.cuda.current_device())
    step_ms, launch_ms = s.time_steps(K_steps, W, world, sampler)
    Q.qjl_decode_workspace_status(s.ctx.handle, s.ws, w.B, w.Hq, w.Hkv)  # raises if a wait inside ran out
    value = cached_tokens_per_s(world, w.B, s.Ttot, step_ms)
    exact_err = s.exact_error() if rank == 0 else None

    # ---------------- prefill leg: outlier selection + sign sketch + value codes
    prefill = None
    if not args.no_prefill:
        prefill = {}
        for name, ps in ((w.name, s), (PREFILL_WORKLOAD, None)):
            if name in prefill:
                continue
            own = ps is None
            if own:
                ps = Setup(I.WORKLOADS[name], rank, lib, dev, prefill_steps=5)
            km, vm = ps.prefill
            pw = ps.w
            ntok = pw.B * pw.Hkv * pw.T
            k_bytes = ntok * (2 * 128) * 2 + ntok * (pw.m // 8 + pw.m_out // 8 + 4)  # K read twice (select, sketch)
            v_bytes = ntok * 2 * 128 + ntok * (64 + 16)
            flops = 2.0 * ntok * 128 * pw.m  # the inlier projection K_in S^T on the tensor cores
            prefill[name] = {
                "tokens": ntok, "quantize_keys_ms": km, "quantize_values_ms": vm,
                "token_heads_per_s": ntok / ((km + vm) / 1e3),
                "keys": {"bound": "tensor", "achieved_tflops": flops / (km / 1e3) / 1e12,
                         "peak_tflops": peaks["bf16_tflops"], "frac": flops / (km / 1e3) / 1e12 / peaks["bf16_tflops"],
                         "hbm_gbs": k_bytes / (km / 1e3) / 1e9,
                         "note": "channel energy + outlier selection + tcgen05 inlier projection"},
                "values": {"bound": "hbm", "achieved": v_bytes / (vm / 1e3) / 1e9, "peak": peaks["hbm_gbs"],
                           "unit": "GB/s", "frac": v_bytes / (vm / 1e3) / 1e9 / peaks["hbm_gbs"]},
            }
            if own:
                ps.close()
                del ps
                torch.cuda.empty_cache()

    # ---------------- end to end through the public API with pinned host buffers
    e2e = None
    if not args.no_e2e:
        # the step's q, k and v staged in one pinned host buffer and copied in
        # one transfer (views of one device buffer, each 256-byte aligned)
        parts = [s.q, s.k_new, s.v_new]
        assert all(t.dtype == s.q.dtype for t in parts)
        esz = s.q.element_size()
        offs, n = [], 0
        for t in parts:
            offs.append(n)
            n += -(-t.numel() * esz // 256) * 256 // esz
        hbuf = torch.zeros(n, dtype=s.q.dtype).pin_memory()
        for t, o in zip(parts, offs):
            hbuf[o:o + t.numel()] = t.reshape(-1).cpu()
        dbuf = torch.empty_like(hbuf, device=s.q.device)
        qd, kd, vd = (dbuf[o:o + t.numel()].view_as(t) for t, o in zip(parts, offs))
        oh = torch.empty(w.B, w.Hq, 128, dtype=torch.float32).pin_memory()
        n_e2e = max(3, min(K_steps, 300))

        def e2e_step(c):
            dbuf.copy_(hbuf, non_blocking=True)
            Q.qjl_decode_step(s.ctx.handle, c, qd, kd, vd, s.T, s.out, workspace=s.ws)
            oh.copy_(s.out, non_blocking=True)

        for i in range(3):
            e2e_step(s.caches[i % s.copies])
        torch.cuda.synchronize()
        barrier(world)
        a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for i in range(n_e2e):
            e2e_step(s.caches[i % s.copies])
        b_.record()
        torch.cuda.synchronize()
        (e2e_ms,) = max_over_ranks(world, [a.elapsed_time(b_) / n_e2e])
        e2e = {"value": cached_tokens_per_s(world, w.B, s.Ttot, e2e_ms), "unit": UNIT,
               "h2d_bytes_per_step": int(hbuf.numel() * hbuf.element_size()),
               "d2h_bytes_per_step": int(oh.numel() * oh.element_size()), "ms_per_step": e2e_ms, "steps": n_e2e}

    # ---------------- the other decode workloads (step time and roofline each)
    per_workload = {}
    if not args.only:
        for name in OTHER_WORKLOADS:
            if name == w.name:
                continue
            o = Setup(I.WORKLOADS[name], rank, lib, dev)
            o_step, o_launch = o.time_steps(K_steps, W, world)
            Q.qjl_decode_workspace_status(o.ctx.handle, o.ws, o.w.B, o.w.Hq, o.w.Hkv)
            rf = roofline(o.w, o.Ttot, o_launch, peaks, recorded_traffic("decode", name))
            per_workload[name] = {"ms_per_step": o_step, "launch_ms": o_launch,
                                  "value": cached_tokens_per_s(world, o.w.B, o.Ttot, o_step), "unit": UNIT,
                                  "B": o.w.B, "Hq": o.w.Hq, "Hkv": o.w.Hkv, "T": o.Ttot, "m": o.w.m,
                                  "roofline": {k: rf[k] for k in ("achieved", "frac", "frac_of_8TBs", "traffic")},
                                  "exact_err": o.exact_error() if rank == 0 else None}
            o.close()
            del o
            torch.cuda.empty_cache()

    # ---------------- the same step over a plain bf16 cache and an FP8 cache
    comparison = None
    if not args.no_comparison:
        comparison = compare_plain_caches(s, world, K_steps, W, peaks)
        comparison["qjl_2bit_values"] = qjl_two_bit_values(s, world, K_steps, W, peaks)

    # ---------------- CPU oracle baseline (rank 0, N = 1 only)
    cpu, cpu_all = None, None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        host = pair_to_host(s.caches[0], 0, 0, min(s.Ttot, 16384), w.m_out)
        q = s.q[0:1, 0:1].float().cpu().numpy().astype("float64")
        cpu, cpu_all = cpu_baseline(w, host, q, args.cpu_seconds, s.Ttot)

    clocks = sampler.summary()
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K_steps, "warmup": W,
        "ms_per_step": step_ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic: K,V,Q ~ N(0,1) bf16 with planted outlier key channels; seed 1234 + rank",
        "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "T": s.Ttot, "d": 128, "m": w.m,
                   "m_out": w.m_out, "n_outlier": w.n_outlier, "value_bits": 4, "value_group": 32,
                   "l2": (f"{s.copies} rotating cache copies, {s.copies * s.cache_bytes / 1e6:.0f} MB > 126 MB L2"),
                   "parallelism": f"dp{world}: independent batches per GPU, no collective",
                   "step": "one qjl_decode_step launch: append 1 token per sequence + decode over T+1 tokens"},
        "hbm_gbs": step_bytes(w, s.Ttot) / (step_ms / 1e3) / 1e9,
        "launch_ms": launch_ms,
        "roofline": roofline(w, s.Ttot, launch_ms, peaks, recorded_traffic("decode", w.name)),
        "exact_err": exact_err,
        "cpu_baseline": cpu,
        "cpu_baseline_all_cores": cpu_all,
        "e2e": e2e,
        "gpu_launches": 2 * K_steps,  # per step: the prep kernel and the decode kernel of qjl_decode_step
        "clocks": clocks,
        "prefill": prefill,
        "per_workload": per_workload,
        "comparison": comparison,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    s.close()
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()


def qjl_two_bit_values(s, world, K_steps, W, peaks):
    """The same decode step with 2-bit value codes (qjl_init_ex, value_bits = 2):
    m/8 + m_out/8 + 4 + 32 + 16 bytes per token-head instead of 124 at m = 256."""
    import torch

    from decode_attention_qjl_b200 import qjl as Q

    w = s.w
    ctx = Q.QJLContext(0, 128, w.m, w.m_out, w.n_outlier, value_bits=2)
    cache = ctx.allocate_cache(w.B, w.Hkv, s.Ttot)
    Q.qjl_quantize_keys(ctx.handle, cache, s.K, Q.QJL_PREFILL, workspace=ctx.keys_workspace(w.B, w.Hkv))
    Q.qjl_quantize_values(ctx.handle, cache, s.V)
    out = torch.empty(w.B, w.Hq, 128, dtype=torch.float32, device=s.K.device)
    ws = ctx.decode_workspace(w.B, w.Hq, w.Hkv, s.Ttot)
    step = lambda: Q.qjl_decode_step(ctx.handle, cache, s.q, s.k_new, s.v_new, s.T, out, workspace=ws)
    for _ in range(W):
        step()
    torch.cuda.synchronize()
    barrier(world)
    a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n = max(3, min(K_steps, 100))
    a.record()
    for _ in range(n):
        step()
    b_.record()
    torch.cuda.synchronize()
    (ms,) = max_over_ranks(world, [a.elapsed_time(b_) / n])
    Q.qjl_decode_workspace_status(ctx.handle, ws, w.B, w.Hq, w.Hkv)
    per_tok = w.m // 8 + w.m_out // 8 + 4 + 32 + 16
    nbytes = w.B * w.Hkv * s.Ttot * per_tok + w.B * w.Hq * 128 * (2 + 4) + w.B * w.Hkv * w.n_outlier * 4
    gbs = nbytes / (ms / 1e3) / 1e9
    # error against exact attention, the pairs exact_error samples
    saved = s.out.clone()
    s.out.copy_(out)
    err = s.exact_error() if (not torch.distributed.is_initialized() or torch.distributed.get_rank() == 0) else None
    s.out.copy_(saved)
    ctx.close()
    return {"ms_per_step": ms, "value": cached_tokens_per_s(world, w.B, s.Ttot, ms), "unit": UNIT,
            "bytes_per_token_head": per_tok, "hbm_gbs": gbs, "frac": gbs / peaks["hbm_gbs"], "exact_err": err,
            "note": "qjl_decode_step with 2-bit value codes (levels 0..3, groups of 32): "
                    "(m + m_out + 32) / 128 + 2 + 1 bits per key and value FPN on average"}


def compare_plain_caches(s, world, K_steps, W, peaks):
    """Decode over the step's T+1 tokens kept as a plain bf16 cache, an FP8 E4M3
    cache (amax scales, one for K and one for V) and 4- and 2-bit min-max
    caches, with the library's comparison kernels: time per call, HBM bytes
    read per call and each quantised output's error against exact attention
    on the bf16 cache."""
    import torch

    from decode_attention_qjl_b200 import qjl as Q

    w = s.w
    K = torch.cat([s.K, s.k_new[:, :, None]], 2).contiguous()
    V = torch.cat([s.V, s.v_new[:, :, None]], 2).contiguous()
    ks = float(K.float().abs().max()) / 448.0
    vs = float(V.float().abs().max()) / 448.0
    K8, V8 = Q.qjl_fp8_quantize(K, ks), Q.qjl_fp8_quantize(V, vs)
    K2, V2 = Q.qjl_minmax_quantize(K, 2), Q.qjl_minmax_quantize(V, 2)
    K4, V4 = Q.qjl_minmax_quantize(K, 4), Q.qjl_minmax_quantize(V, 4)
    out = {}
    ref = torch.empty(w.B, w.Hq, 128, dtype=torch.float32, device=K.device)
    for name, (Kc, Vc, per_tok) in (("bf16", (K, V, 2 * 128 * 2)), ("fp8_e4m3", (K8, V8, 2 * 128)),
                                    ("minmax4", (K4, V4, 2 * 80)), ("minmax2", (K2, V2, 2 * 48))):
        O_ = torch.empty(w.B, w.Hq, 128, dtype=torch.float32, device=K.device)
        ws = torch.empty(max(16, int(Q.load_library().qjl_exact_decode_workspace_bytes(w.B, w.Hq, s.Ttot))),
                         dtype=torch.uint8, device=K.device)
        call = lambda: Q.qjl_exact_decode(Kc, Vc, s.q, O_, T=s.Ttot, k_scale=ks, v_scale=vs, workspace=ws)
        for _ in range(W):
            call()
        torch.cuda.synchronize()
        barrier(world)
        a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n = max(3, min(K_steps, 50))
        a.record()
        for _ in range(n):
            call()
        b_.record()
        torch.cuda.synchronize()
        (ms,) = max_over_ranks(world, [a.elapsed_time(b_) / n])
        nbytes = w.B * w.Hkv * s.Ttot * per_tok + w.B * w.Hq * 128 * (2 + 4)
        gbs = nbytes / (ms / 1e3) / 1e9
        out[name] = {"ms_per_call": ms, "value": cached_tokens_per_s(world, w.B, s.Ttot, ms), "unit": UNIT,
                     "bytes_per_call": nbytes, "hbm_gbs": gbs, "frac": gbs / peaks["hbm_gbs"], "launches_per_call": 2}
        if name == "bf16":
            ref.copy_(O_)
        else:  # FP8 and min-max outputs against the exact one
            e = (O_.double() - ref.double()).abs()
            cos = torch.nn.functional.cosine_similarity(O_.double(), ref.double(), dim=-1)
            out[name]["err_vs_bf16_exact"] = {"max_abs": float(e.max()), "min_cosine": float(cos.min())}
    out["note"] = ("qjl_exact_decode on the step's T+1 tokens; bf16 = the unquantised cache (exact attention), "
                   f"fp8_e4m3 = E4M3 codes with k_scale {ks:.3g}, v_scale {vs:.3g}; minmax4 / minmax2 = the "
                   "token-wise min-max quantiser on K and V (groups of 32, fp16 scale and zero); every cache "
                   "exceeds L2")
    del K, V, K8, V8, K2, V2, K4, V4
    torch.cuda.empty_cache()
    return out


def bits_table():
    """Storage (bits per floating-point number) against error, on one GPU.

    For m in {128, 256, 512, 1024} sketch rows and n_o in {0, 8} outlier
    channels (m_out = 64 or 256 when n_o = 8), on the same synthetic keys (8 planted
    outlier channels x20 per kv head, the Llama-3-8B GQA recipe): the RMS of
    the score error (QJL estimate minus the exact <q, k> of the bf16 inputs)
    measured through qjl_decode_attention, next to the RMS the closed-form
    variance predicts, var = ((pi/2) |q_p|^2 |k_p|^2 - <q_p, k_p>^2) / m_p
    summed over the parts p (inlier with m rows, outlier with m_out rows; QJL
    summary, Approach: the estimator is unbiased and its variance shrinks as
    1/m), and the attention output against exact softmax attention. m = 1024
    is beyond the kernels (m <= 512): only its prediction is shown.
    Key bits per FPN = (m + m_out + 32) / 128 (sign bits and two fp16 norms per
    token and head); value bits per FPN = 4 + 32 / 32 (codes, fp16 scale and
    zero per 32 dims; 2 + 1 with 2-bit codes, the rows marked value bits 2)."""
    import torch

    from decode_attention_qjl_b200 import inputs as I
    from decode_attention_qjl_b200 import qjl as Q

    torch.cuda.set_device(0)
    base = I.Workload("bits_table", 2, 32, 8, 8192, 256, 64, 8, "bf16", "x20", "")
    inp = I.make_inputs(base, device="cuda")
    K, V, Qt = inp["K"], inp["V"], inp["Q"]
    B, Hkv, T, d = K.shape
    Hq = Qt.shape[1]
    g = Hq // Hkv
    Kd, Vd, Qd = K.double(), V.double(), Qt.double()
    Kq = Kd.repeat_interleave(g, dim=1)                      # [B, Hq, T, d]
    exact = torch.einsum("bhtd,bhd->bht", Kq, Qd)            # <q, k_t>
    p = torch.softmax(exact / math.sqrt(d), dim=-1)
    out_ref = torch.einsum("bht,bhtd->bhd", p, Vd.repeat_interleave(g, dim=1))
    rows = []
    configs = [(m, n_o, m_out, 4) for m in (128, 256, 512, 1024) for n_o, m_out in ((0, 0), (8, 64), (8, 256))]
    configs += [(m, 8, m_out, 2) for m, m_out in ((128, 64), (256, 64), (512, 64), (256, 256))]
    for m, n_o, m_out, vb in configs:
        if True:
            key_bits = (m + m_out + 32) / 128
            row = {"m": m, "m_out": m_out, "n_o": n_o, "value_bits": vb, "key_bits": key_bits,
                   "kv_bits": (key_bits + vb + 1.0) / 2}
            # the parts: the GPU's chosen outlier channels (the planted ones, checked below)
            mask = torch.zeros(B, Hq, d, dtype=torch.bool, device="cuda")
            if n_o:
                ch = inp["outlier_channels"].repeat_interleave(g, dim=1)
                mask.scatter_(2, ch, True)
            var = torch.zeros(B, Hq, T, dtype=torch.float64, device="cuda")
            for part, rows_p in ((~mask, m), (mask, m_out)):
                if rows_p == 0:
                    continue
                qp = Qd * part
                kp = Kq * part[:, :, None, :]
                qk = torch.einsum("bhtd,bhd->bht", kp, qp)
                var += ((math.pi / 2) * (qp * qp).sum(-1)[..., None] * (kp * kp).sum(-1) - qk * qk) / rows_p
            row["pred_rms"] = float(var.mean().sqrt())
            row["exact_rms"] = float(exact.pow(2).mean().sqrt())
            if m <= 512:
                ctx = Q.QJLContext(0, 128, m, m_out, n_o, value_bits=vb)
                cache = ctx.allocate_cache(B, Hkv, T)
                Q.qjl_quantize_keys(ctx.handle, cache, K, Q.QJL_PREFILL, workspace=ctx.keys_workspace(B, Hkv))
                Q.qjl_quantize_values(ctx.handle, cache, V)
                if n_o:
                    got_ch = cache.outlier_idx[:, :, :n_o].long()
                    assert torch.equal(got_ch, inp["outlier_channels"].sort(-1).values.to(got_ch.device))
                out = torch.empty(B, Hq, d, dtype=torch.float32, device="cuda")
                sc = torch.empty(B, Hq, T, dtype=torch.float32, device="cuda")
                ws = ctx.decode_workspace(B, Hq, Hkv, T)
                Q.qjl_decode_attention(ctx.handle, cache, Qt, T, out, scores=sc, workspace=ws)
                Q.qjl_decode_workspace_status(ctx.handle, ws, B, Hq, Hkv)
                err = sc.double() - exact
                row["meas_rms"] = float(err.pow(2).mean().sqrt())
                row["mean_err"] = float(err.mean())
                o = out.double()
                row["out_max_abs"] = float((o - out_ref).abs().max())
                row["out_min_cos"] = float(torch.nn.functional.cosine_similarity(o, out_ref, dim=-1).min())
                ctx.close()
            rows.append(row)
    hdr = ("| m | m_out | n_o | value bits | key bits/FPN | K+V bits/FPN | score RMS err (measured) "
           "| score RMS err (closed form) | mean err | RMS of exact q.k | output max abs err | output min cosine |")
    print(hdr)
    print("|" + "---|" * 12)
    for r in rows:
        meas = f"{r['meas_rms']:.3f}" if "meas_rms" in r else "m > 512: not run"
        print(f"| {r['m']} | {r['m_out']} | {r['n_o']} | {r['value_bits']} | {r['key_bits']:.3f} | {r['kv_bits']:.3f} | {meas} | "
              f"{r['pred_rms']:.3f} | {r.get('mean_err', float('nan')):+.4f} | {r['exact_rms']:.2f} | "
              f"{r.get('out_max_abs', float('nan')):.2e} | {r.get('out_min_cos', float('nan')):.5f} |")
    print(json.dumps({"bits_table": rows, "workload": "B=2, Hq=32, Hkv=8, T=8192, bf16, 8 planted channels x20"}))


def main():
    args = parse_args()
    if args.bits_table:
        bits_table()
        return
    if args.impl == "reference":
        run_reference(args)
    else:
        run_qjl(args)


if __name__ == "__main__":
    main()
