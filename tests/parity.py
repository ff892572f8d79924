"""Helpers shared by the GPU parity tests: run the CUDA path and the oracle on
the same seeded inputs and compare them element by element.

Quantize criterion: codes and QJL sign bits are bit-exact, except where the
oracle's rotated coordinate lies within 1e-5 of a cell boundary (or |S r| <
1e-5 for a sign); such boundary cases are counted and must stay below a 1e-6
fraction of all coordinates compared. A key whose cell index legitimately
differs has a different residual, so its signs and |r| are not compared.
Norms agree within one fp16 ulp. Attention: max |o - o_ref| / |o_ref|_inf
<= 2e-3 per (batch, query head).
"""
from __future__ import annotations

import numpy as np
import torch

import kv_cache_vector_04_b200 as tq
from oracle import oracle as O

BAND = 1e-5
FRACTION = 1e-6
ATTN_TOL = 2e-3


def fp16_ulps(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    """Distance in units in the last place between fp16 bit patterns (finite)."""
    def ordered(x):
        x = x.astype(np.int32)
        return np.where(x & 0x8000, 0x8000 - (x & 0x7FFF), 0x8000 + x)
    return np.abs(ordered(a) - ordered(b))


def stream_bytes(cache_host: np.ndarray, tile_bytes: int, cap: int, Hkv: int, b: int, h: int,
                 ntok: int) -> np.ndarray:
    per_stream = (cap // 16) * tile_bytes
    s0 = (b * Hkv + h) * per_stream
    return cache_host[s0: s0 + ((ntok + 15) // 16) * tile_bytes]


class QuantStats:
    def __init__(self):
        self.total = 0
        self.band = 0

    def check(self):
        assert self.band <= FRACTION * self.total, (self.band, self.total)


def compare_stream(tab: O.Tables, gpu: dict, ora: dict, N: int, stats: QuantStats):
    """Compare decoded GPU codes with the oracle's for tokens [0, N)."""
    d = tab.d
    kmis = gpu["kidx"][:N] != ora["kidx"][:N]
    assert np.all(ora["kydist"][:N][kmis] < BAND), "key code differs away from a boundary"
    vmis = gpu["vidx"][:N] != ora["vidx"][:N]
    assert np.all(ora["vydist"][:N][vmis] < BAND), "value code differs away from a boundary"
    clean = ~kmis.any(axis=1)
    smis = (gpu["ksign"][:N] != ora["ksign"][:N]) & clean[:, None]
    assert np.all(ora["zabs"][:N][smis] < BAND), "QJL sign differs away from z = 0"
    stats.band += int(kmis.sum() + vmis.sum() + smis.sum())
    stats.total += int(N * d * 3)
    assert fp16_ulps(gpu["knorm"][:N], ora["knorm"][:N]).max(initial=0) <= 1
    assert fp16_ulps(gpu["vnorm"][:N], ora["vnorm"][:N]).max(initial=0) <= 1
    if clean.any():
        assert fp16_ulps(gpu["rnorm"][:N][clean], ora["rnorm"][:N][clean]).max(initial=0) <= 1


def quantize_on_gpu(ctx, k: torch.Tensor, v: torch.Tensor, capacity: int, start=None,
                    cache=None):
    B, Hkv, T, d = k.shape
    if cache is None:
        cache = tq.new_cache(ctx, B, Hkv, capacity)
    sp = torch.zeros(B, dtype=torch.int32) if start is None else torch.as_tensor(start, dtype=torch.int32)
    tq.tq_quantize(ctx, k.cuda(), v.cuda(), sp.cuda(), cache)
    torch.cuda.synchronize()
    return cache


def oracle_codes(tab: O.Tables, k: torch.Tensor, v: torch.Tensor):
    """Per (b, h) oracle codes for fp16 K/V [B, Hkv, T, d]."""
    B, Hkv, T, d = k.shape
    kn = k.cpu().numpy()
    vn = v.cpu().numpy()
    return [[O.quantize(tab, np.ascontiguousarray(kn[b, h]), np.ascontiguousarray(vn[b, h]))
             for h in range(Hkv)] for b in range(B)]


def stack_codes(codes, cap: int):
    """[B][Hkv] list of per-stream code dicts -> arrays [B, Hkv, cap, ...]."""
    B, Hkv = len(codes), len(codes[0])
    out = {}
    for key in ("kidx", "ksign", "knorm", "rnorm", "vidx", "vnorm"):
        ref = codes[0][0][key]
        arr = np.zeros((B, Hkv, cap) + ref.shape[1:], ref.dtype)
        for b in range(B):
            for h in range(Hkv):
                n = codes[b][h][key].shape[0]
                arr[b, h, :n] = codes[b][h][key]
        out[key] = arr
    return out


def pack_cache(tab: O.Tables, codes, cap: int, d: int, bits: int) -> torch.Tensor:
    """Oracle-packed cache bytes for [B][Hkv] code streams, as a CUDA tensor."""
    B, Hkv = len(codes), len(codes[0])
    tb = O.tile_bytes(d, tab)   # the context's format (tab.fmt)
    host = np.zeros(B * Hkv * (cap // 16) * tb, np.uint8)
    for b in range(B):
        for h in range(Hkv):
            s = O.pack_stream(d, tab, codes[b][h])
            s0 = (b * Hkv + h) * (cap // 16) * tb
            host[s0: s0 + s.size] = s
    return torch.from_numpy(host).cuda()


def q_bits(q: torch.Tensor) -> np.ndarray:
    return q.cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def attn_error(out_gpu: np.ndarray, out_ref: np.ndarray) -> np.ndarray:
    """max |delta| / |o_ref|_inf per (b, h)."""
    num = np.abs(out_gpu - out_ref).max(axis=-1)
    den = np.abs(out_ref).max(axis=-1)
    return np.where(den > 0, num / np.maximum(den, 1e-300), num)
