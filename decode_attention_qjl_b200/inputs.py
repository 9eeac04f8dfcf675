"""Seeded synthetic inputs shaped like the decode workloads (no QJL arithmetic here).

The pages measure QJL on Llama-2-7B, Llama-3-8B and longchat-7b-v1.5-32k
(LongBench, LM-eval; QJL summary, Key results). Neither the models nor the
datasets are used: keys, values and queries are drawn i.i.d. N(0,1) with the
shapes of those models' attention layers, and a few outlier channels per kv
head are scaled up, the phenomenon described in "2 numbers out of 128 destroy
the entire KV cache" (section "The Real Problem: Outlier Channels") and in the
TurboQuant slides (section 05, "The Third Problem: Magnitude Outliers").
Outliers are applied to the keys only; values and queries are plain N(0,1).

Both the CUDA path and the oracle receive the tensors made here.
"""

from __future__ import annotations

from dataclasses import dataclass, field

import torch

HEAD_DIM = 128
DATA_SEED = 1234
SKETCH_SEED = 0


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    T: int
    m: int = 256
    m_out: int = 64
    n_outlier: int = 8
    dtype: str = "bf16"        # key/value/query storage type: "bf16" or "fp32"
    outliers: str = "x20"      # "fixed4_x20", "u10_50", "t3_x20", "x20"
    note: str = ""

    @property
    def g(self) -> int:
        return self.Hq // self.Hkv

    def bytes_per_token_head(self) -> int:
        """Algorithmic bytes of one cached token of one kv head read by decode."""
        return self.m // 8 + self.m_out // 8 + 4 + HEAD_DIM // 2 + (HEAD_DIM // 32) * 4


WORKLOADS = {
    "single_head_fp32": Workload("single_head_fp32", 1, 1, 1, 1024, 256, 64, 4, "fp32", "fixed4_x20",
                                 "1 head, 1024 tokens, fp32, 4 fixed outlier channels x20"),
    "llama2_7b_mha": Workload("llama2_7b_mha", 8, 32, 32, 4096, 256, 64, 8, "bf16", "u10_50",
                              "Llama-2-7B-shaped layer: batch 8, 32 MHA heads, context 4096"),
    "long_context": Workload("long_context", 1, 32, 32, 32768, 256, 64, 8, "bf16", "t3_x20",
                             "batch 1, 32 heads, context 32768, Student-t(3) x20 outliers"),
    "llama3_8b_gqa": Workload("llama3_8b_gqa", 16, 32, 8, 8192, 256, 64, 8, "bf16", "x20",
                              "Llama-3-8B-shaped GQA layer: batch 16, 32 q heads / 8 kv heads, context 8192"),
}
for _m in (128, 256, 512):
    WORKLOADS[f"sweep_m{_m}_b64_t16k"] = Workload(f"sweep_m{_m}_b64_t16k", 64, 32, 8, 16384, _m, 64, 8, "bf16", "x20",
                                                  "HBM sweep: 8 kv heads (GQA 4:1), batch 64 x 16384")
    WORKLOADS[f"sweep_m{_m}_b4_t128k"] = Workload(f"sweep_m{_m}_b4_t128k", 4, 32, 8, 131072, _m, 64, 8, "bf16", "x20",
                                                  "HBM sweep: 8 kv heads (GQA 4:1), batch 4 x 131072")

FIXED_OUTLIER_CHANNELS = (10, 37, 64, 101)


def _dtype(name: str):
    return {"bf16": torch.bfloat16, "fp32": torch.float32}[name]


def outlier_channels(w: Workload, gen: torch.Generator, device) -> torch.Tensor:
    """Distinct outlier channels per (b, kv head): [B, Hkv, n_outlier] int64, ascending."""
    if w.outliers == "fixed4_x20":
        ch = torch.tensor(FIXED_OUTLIER_CHANNELS[: w.n_outlier], device=device)
        return ch.expand(w.B, w.Hkv, -1).clone()
    keys = torch.rand(w.B, w.Hkv, HEAD_DIM, generator=gen, device=device)
    return torch.sort(torch.argsort(keys, dim=-1)[..., : w.n_outlier], dim=-1).values


def make_inputs(w: Workload, seed: int = DATA_SEED, device="cpu", B: int | None = None, T: int | None = None,
                Hkv: int | None = None) -> dict:
    """K, V [B, Hkv, T, d], Q [B, Hq, d] in the workload's dtype, plus the planted outlier channels.

    B, T and Hkv may be overridden to draw a smaller case with the same recipe.
    """
    B = w.B if B is None else B
    T = w.T if T is None else T
    Hkv = w.Hkv if Hkv is None else Hkv
    Hq = Hkv * w.g
    w2 = Workload(w.name, B, Hq, Hkv, T, w.m, w.m_out, w.n_outlier, w.dtype, w.outliers, w.note)
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    K = torch.randn(B, Hkv, T, HEAD_DIM, generator=gen, device=device)
    ch = outlier_channels(w2, gen, device) if w.n_outlier > 0 else torch.zeros(B, Hkv, 0, dtype=torch.long, device=device)
    if w.n_outlier > 0:
        idx = ch[:, :, None, :].expand(B, Hkv, T, w.n_outlier)
        if w.outliers in ("fixed4_x20", "x20"):
            vals = torch.gather(K, 3, idx) * 20.0
        elif w.outliers == "u10_50":
            f = 10.0 + 40.0 * torch.rand(B, Hkv, 1, w.n_outlier, generator=gen, device=device)
            vals = torch.gather(K, 3, idx) * f
        elif w.outliers == "t3_x20":
            z = torch.randn(B, Hkv, T, w.n_outlier, generator=gen, device=device)
            chi2 = torch.randn(3, B, Hkv, T, w.n_outlier, generator=gen, device=device).pow(2).sum(0)
            vals = 20.0 * z / torch.sqrt(chi2 / 3.0)
        else:
            raise ValueError(w.outliers)
        K.scatter_(3, idx, vals)
    V = torch.randn(B, Hkv, T, HEAD_DIM, generator=gen, device=device)
    Q = torch.randn(B, Hq, HEAD_DIM, generator=gen, device=device)
    dt = _dtype(w.dtype)
    return {"K": K.to(dt), "V": V.to(dt), "Q": Q.to(dt), "outlier_channels": ch, "workload": w2}


def append_inputs(w: Workload, B: int, Hq: int, Hkv: int, seed: int, device="cpu", outlier_ch=None) -> dict:
    """One new token per sequence (k, v [B, Hkv, 1, d]) and its query (q [B, Hq, d]) for a decode step."""
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    k = torch.randn(B, Hkv, 1, HEAD_DIM, generator=gen, device=device)
    if outlier_ch is not None and outlier_ch.shape[-1] > 0:
        idx = outlier_ch[:, :, None, :].to(device)
        k.scatter_(3, idx, torch.gather(k, 3, idx) * 20.0)
    v = torch.randn(B, Hkv, 1, HEAD_DIM, generator=gen, device=device)
    q = torch.randn(B, Hq, HEAD_DIM, generator=gen, device=device)
    dt = _dtype(w.dtype)
    return {"k": k.to(dt), "v": v.to(dt), "q": q.to(dt)}
