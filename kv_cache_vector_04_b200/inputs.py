"""Seeded synthetic inputs and the workload shapes they are drawn for.

This module holds no arithmetic of the method: it only draws K/V and query
tensors with torch's generators. Tests, the bench and the oracle side of the
parity tests all take their inputs from here.

The workloads mirror the shapes the pages discuss (a single head at d=128, 3
bits, 8192 keys and 64 queries as in the GB10 speed test of "[Benchmark]
TurboQuant 實測：KV Cache 3-bit 壓縮，真的零損失？" §"GB10 速度"; a
Qwen2.5-3B-shaped 8K decode with 36 layers x 2 kv heads as in its
§"壓縮率與精度"; Llama-3.3-70B- and Qwen2.5-32B-shaped long-context decodes;
a sweep over d, bits and context length). No model weights or datasets are
involved: every tensor is random with the stated distribution.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    d: int
    bits: int
    layers: int
    B: int
    Hq: int
    Hkv: int
    N: int
    kv_dist: str          # "lognormal_norm" | "outlier_channels" | "spiky_tokens"
    q_dtype: torch.dtype
    seed: int
    decode_steps: int = 1
    notes: str = ""
    fmt: tuple | None = None   # (B_K, B_V, qjl); None: TurboQuant at `bits`, (bits-1, bits, 1)


WORKLOADS = {
    "single_head_d128_b3": Workload(
        "single_head_d128_b3", d=128, bits=3, layers=1, B=1, Hq=64, Hkv=1, N=8192,
        kv_dist="lognormal_norm", q_dtype=torch.float16, seed=1001,
        notes="8192 keys/values, 64 fp16 queries on one kv head"),
    "qwen2.5-3b_decode_8k": Workload(
        "qwen2.5-3b_decode_8k", d=128, bits=3, layers=36, B=1, Hq=16, Hkv=2, N=8192,
        kv_dist="outlier_channels", q_dtype=torch.bfloat16, seed=1002),
    "llama3.3-70b_decode_32k": Workload(
        "llama3.3-70b_decode_32k", d=128, bits=4, layers=80, B=16, Hq=64, Hkv=8, N=32768,
        kv_dist="lognormal_norm", q_dtype=torch.bfloat16, seed=1003),
    "qwen2.5-32b_prefill_decode_128k": Workload(
        "qwen2.5-32b_prefill_decode_128k", d=128, bits=3, layers=64, B=1, Hq=40, Hkv=8,
        N=131072, kv_dist="spiky_tokens", q_dtype=torch.bfloat16, seed=1004, decode_steps=32),
}


def sweep_workloads():
    """d x bits x context sweep: 8 kv heads, 32 query heads, batch 8, one layer."""
    out = []
    for d in (64, 128, 256):
        for bits in (2, 3, 4):
            for N in (4096, 16384, 65536):
                out.append(Workload("sweep_d%d_b%d_n%d" % (d, bits, N), d=d, bits=bits, layers=1,
                                    B=8, Hq=32, Hkv=8, N=N, kv_dist="lognormal_norm",
                                    q_dtype=torch.bfloat16, seed=1005))
    return out


# Every built cache format: TurboQuant at 2, 3, 4 bits, k8v4, and the MSE-only keys.
FORMATS = {"tq2": (1, 2, 1), "tq3": (2, 3, 1), "tq4": (3, 4, 1), "k8v4": (7, 4, 1),
           "nc2": (2, 2, 0), "nc3": (3, 3, 0), "nc4": (4, 4, 0), "k3v4nc": (3, 4, 0)}


def format_workloads():
    """One decode layer per built format: d = 128, 8 kv heads, 32 query heads,
    batch 8, 32K context."""
    return [Workload("format_%s_d128_n32768" % name, d=128, bits=f[1], layers=1, B=8, Hq=32, Hkv=8,
                     N=32768, kv_dist="lognormal_norm", q_dtype=torch.bfloat16, seed=1007, fmt=f)
            for name, f in FORMATS.items()]


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def kv_tensor(shape, dist: str, seed: int, device="cpu", dtype=torch.float16) -> torch.Tensor:
    """Draw one K or V tensor of shape [B, Hkv, T, d].

    lognormal_norm:   direction ~ N(0, I) normalised, norm ~ LogNormal(0, 0.5)
    outlier_channels: N(0, 1) with 4 channels per kv head (a seeded choice, the
                      same for every token and layer) scaled x15
    spiky_tokens:     N(0, 1) with 2% of token positions (Bernoulli, shared by
                      all heads) scaled x10
    """
    B, H, T, d = shape
    g = _gen(seed, device)
    x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if dist == "lognormal_norm":
        x = x / x.norm(dim=-1, keepdim=True).clamp_min(1e-30)
        nrm = torch.exp(0.5 * torch.randn((B, H, T, 1), generator=g, device=device))
        x = x * nrm
    elif dist == "outlier_channels":
        gc = _gen(seed + 7919, "cpu")
        scale = torch.ones((H, d))
        for h in range(H):
            scale[h, torch.randperm(d, generator=gc)[:4]] = 15.0
        x = x * scale.to(device)[None, :, None, :]
    elif dist == "spiky_tokens":
        spike = torch.rand((B, 1, T, 1), generator=g, device=device) < 0.02
        x = torch.where(spike, x * 10.0, x)
    else:
        raise ValueError(dist)
    return x.to(dtype)


def kv_pair(w: Workload, T: int, layer: int = 0, device="cpu", B: int | None = None,
            Hkv: int | None = None):
    B = w.B if B is None else B
    Hkv = w.Hkv if Hkv is None else Hkv
    base = w.seed * 1_000_003 + layer * 7_919
    k = kv_tensor((B, Hkv, T, w.d), w.kv_dist, base + 1, device)
    v = kv_tensor((B, Hkv, T, w.d), "lognormal_norm" if w.kv_dist == "lognormal_norm" else
                  w.kv_dist, base + 2, device)
    return k, v


def queries(w: Workload, layer: int = 0, step: int = 0, device="cpu", B: int | None = None,
            Hq: int | None = None) -> torch.Tensor:
    B = w.B if B is None else B
    Hq = w.Hq if Hq is None else Hq
    g = _gen(w.seed * 1_000_003 + layer * 7_919 + 104_729 * (step + 1), device)
    return torch.randn((B, Hq, w.d), generator=g, device=device).to(w.q_dtype)

