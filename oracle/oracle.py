"""TurboQuant KV-cache oracle: ctypes front end of ``tq_oracle.c``.

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module. It is a plain, slow
fp64 CPU statement of the method and shares no code with the CUDA library
(``kv_cache_vector_04_b200``); the two meet only at seeded input tensors.

Sources are cited in ``tq_oracle.c`` (page title, section). Every function
here is a thin numpy wrapper around the C function of the same name.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "tq_oracle.c")
_LIB = os.path.join(_HERE, "libtq_oracle.so")
_lock = threading.Lock()
_lib = None

TILE = 16


def build(force: bool = False) -> str:
    """Compile the oracle (gcc, fp64, OpenMP over independent vectors)."""
    with _lock:
        stale = (not os.path.exists(_LIB)) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC)
        if force or stale:
            tmp = _LIB + ".tmp%d" % os.getpid()
            cmd = ["gcc", "-O2", "-std=gnu11", "-fopenmp", "-ffp-contract=off", "-fPIC",
                   "-shared", _SRC, "-o", tmp, "-lm"]
            subprocess.run(cmd, check=True)
            os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is not None:
        return _lib
    build()
    lib = ctypes.CDLL(_LIB)
    P = ctypes.c_void_p
    i32, u64, u32 = ctypes.c_int, ctypes.c_uint64, ctypes.c_uint32
    sig = {
        "oracle_half_to_double": (ctypes.c_double, [ctypes.c_uint16]),
        "oracle_bf16_to_double": (ctypes.c_double, [ctypes.c_uint16]),
        "oracle_double_to_half": (ctypes.c_uint16, [ctypes.c_double]),
        "oracle_draw": (u64, [u64, u32, u64]),
        "oracle_splitmix64_next": (u64, [P]),
        "oracle_gauss": (ctypes.c_double, [u64, u32, u64]),
        "oracle_rotation_signs": (None, [i32, u64, P]),
        "oracle_qjl_matrix": (None, [i32, i32, u64, P]),
        "oracle_lloyd_max_unit": (i32, [i32, P, P]),
        "oracle_quantizer_mse_unit": (ctypes.c_double, [i32, P]),
        "oracle_codebook": (i32, [i32, i32, P, P]),
        "oracle_beta_marginal_pdf": (ctypes.c_double, [i32, ctypes.c_double]),
        "oracle_lloyd_max_beta": (i32, [i32, i32, P]),
        "oracle_quantizer_mse_beta": (ctypes.c_double, [i32, i32, P]),
        "oracle_codebook_beta": (i32, [i32, i32, P, P]),
        "oracle_rotate": (None, [i32, P, P, P]),
        "oracle_rotate_inverse": (None, [i32, P, P, P]),
        "oracle_encode": (i32, [ctypes.c_double, P, i32]),
        "oracle_quantize_keys": (None, [i32, i32, P, P, P, P, P, i32, i32, P, P, P, P, P, P, P]),
        "oracle_quantize_values": (None, [i32, i32, P, P, P, P, i32, P, P, P, P]),
        "oracle_tile_bytes": (ctypes.c_int64, [i32, i32, i32, i32]),
        "oracle_pack_stream": (None, [i32, i32, i32, i32, i32, P, P, P, P, P, P, P]),
        "oracle_unpack_stream": (None, [i32, i32, i32, i32, i32, P, P, P, P, P, P, P]),
        "oracle_attend_head": (None, [i32, i32, P, i32, i32, P, P, P, P, P, P, P, P, P, P, P, P]),
        "oracle_attend_batch": (None, [i32, i32, i32, i32, i32, P, P, i32, i32, P, P, P, P,
                                        P, P, P, P, P, P, P, P]),
        "oracle_distortion_mc": (ctypes.c_double, [i32, i32, i32, u64]),
        "oracle_ip_trials": (None, [i32, i32, i32, u64, P, P, P, P]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    _lib = lib
    return lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "arrays passed to the oracle must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


# --------------------------------------------------------------------------
# scalars and tables
# --------------------------------------------------------------------------

def half_to_double(h: int) -> float:
    return _load().oracle_half_to_double(int(h) & 0xFFFF)


def bf16_to_double(h: int) -> float:
    return _load().oracle_bf16_to_double(int(h) & 0xFFFF)


def double_to_half(x: float) -> int:
    return int(_load().oracle_double_to_half(float(x)))


def draw(seed: int, stream: int, k: int) -> int:
    return int(_load().oracle_draw(seed, stream, k))


def splitmix64_outputs(state: int, n: int) -> list:
    s = ctypes.c_uint64(state)
    lib = _load()
    return [int(lib.oracle_splitmix64_next(ctypes.byref(s))) for _ in range(n)]


def gauss(seed: int, stream: int, e: int) -> float:
    return float(_load().oracle_gauss(seed, stream, e))


def rotation_signs(d: int, seed: int) -> np.ndarray:
    D = np.zeros(d, dtype=np.int8)
    _load().oracle_rotation_signs(d, seed, _p(D))
    return D


def qjl_matrix(m: int, d: int, seed: int) -> np.ndarray:
    S = np.zeros((m, d), dtype=np.float64)
    _load().oracle_qjl_matrix(m, d, seed, _p(S))
    return S


def lloyd_max_unit(B: int):
    c = np.zeros(1 << B, dtype=np.float64)
    it = ctypes.c_int(0)
    rc = _load().oracle_lloyd_max_unit(B, _p(c), ctypes.byref(it))
    return c, rc, it.value


def quantizer_mse_unit(B: int, c: np.ndarray) -> float:
    c = np.ascontiguousarray(c, dtype=np.float64)
    return float(_load().oracle_quantizer_mse_unit(B, _p(c)))


def codebook(B: int, d: int, kind: str = "gauss"):
    """fp32 centroids and boundaries of the B-bit codebook for head dim d:
    kind "gauss" models a rotated coordinate as N(0, 1/d); "beta" uses its
    exact marginal (beta_marginal_pdf)."""
    c = np.zeros(1 << B, dtype=np.float32)
    t = np.zeros(max((1 << B) - 1, 1), dtype=np.float32)
    fn = _load().oracle_codebook if kind == "gauss" else _load().oracle_codebook_beta
    rc = fn(B, d, _p(c), _p(t))
    assert rc == 0
    return c, t[: (1 << B) - 1]


def beta_marginal_pdf(d: int, y: float) -> float:
    return float(_load().oracle_beta_marginal_pdf(d, float(y)))


def lloyd_max_beta(d: int, B: int):
    c = np.zeros(1 << B, dtype=np.float64)
    rc = _load().oracle_lloyd_max_beta(d, B, _p(c))
    return c, rc


def quantizer_mse_beta(d: int, B: int, c: np.ndarray) -> float:
    """MSE under the exact marginal of the quantizer with centroids c."""
    c = np.ascontiguousarray(c, dtype=np.float64)
    return float(_load().oracle_quantizer_mse_beta(d, B, _p(c)))


def rotate(D: np.ndarray, u: np.ndarray) -> np.ndarray:
    d = D.shape[0]
    u = np.ascontiguousarray(u, dtype=np.float64)
    y = np.zeros(d, dtype=np.float64)
    _load().oracle_rotate(d, _p(np.ascontiguousarray(D)), _p(u), _p(y))
    return y


def rotate_inverse(D: np.ndarray, y: np.ndarray) -> np.ndarray:
    d = D.shape[0]
    y = np.ascontiguousarray(y, dtype=np.float64)
    u = np.zeros(d, dtype=np.float64)
    _load().oracle_rotate_inverse(d, _p(np.ascontiguousarray(D)), _p(y), _p(u))
    return u


def encode(y: float, bounds: np.ndarray) -> int:
    b = np.ascontiguousarray(bounds, dtype=np.float32)
    return int(_load().oracle_encode(float(y), _p(b), b.shape[0] + 1))


class Tables:
    """The method's tables for (d, bits, seed), built by the oracle itself.

    fmt = (B_K, B_V, qjl): key and value cell bits and whether keys carry the
    1-bit QJL sketch. The default is TurboQuant at b bits, (b - 1, b, 1); the
    MSE-only key formats ("nc", [MUNINN §MSE-Only vs QJL]) have qjl = 0."""

    def __init__(self, d: int, bits: int, seed: int, fmt: tuple | None = None,
                 kind: str = "gauss"):
        self.d, self.bits, self.seed, self.m = d, bits, seed, d
        self.fmt = fmt_of(bits) if fmt is None else tuple(int(x) for x in fmt)
        self.BK, self.BV, self.qjl = self.fmt
        self.kind = kind   # the codebooks' coordinate model (see codebook)
        self.D = rotation_signs(d, seed)
        self.S = qjl_matrix(d, d, seed)
        self.cK, self.tK = codebook(self.BK, d, kind)
        self.cV, self.tV = codebook(self.BV, d, kind)


def fmt_of(x) -> tuple:
    """(B_K, B_V, qjl) of a format given as b (TurboQuant at b bits), a tuple or Tables."""
    if isinstance(x, Tables):
        return x.fmt
    if isinstance(x, tuple):
        return tuple(int(v) for v in x)
    b = int(x)
    return (b - 1, b, 1)


# --------------------------------------------------------------------------
# quantization, packing, attention
# --------------------------------------------------------------------------

def quantize_keys(tab: Tables, x: np.ndarray):
    """x: [N, d] float16 (or its uint16 bits). Returns a dict of numpy arrays."""
    x = np.ascontiguousarray(x).view(np.uint16)
    N, d = x.shape
    out = dict(
        kidx=np.zeros((N, d), np.uint8), ksign=np.zeros((N, d), np.uint8),
        knorm=np.zeros(N, np.uint16), rnorm=np.zeros(N, np.uint16),
        kydist=np.zeros((N, d), np.float64), zabs=np.zeros((N, d), np.float64),
        ksat=np.zeros(N, np.uint8))
    _load().oracle_quantize_keys(d, N, _p(x), _p(tab.D), _p(tab.S), _p(tab.cK), _p(tab.tK),
                                 tab.BK, tab.qjl, _p(out["kidx"]), _p(out["ksign"]), _p(out["knorm"]),
                                 _p(out["rnorm"]), _p(out["kydist"]), _p(out["zabs"]),
                                 _p(out["ksat"]))
    return out


def quantize_values(tab: Tables, x: np.ndarray):
    x = np.ascontiguousarray(x).view(np.uint16)
    N, d = x.shape
    out = dict(vidx=np.zeros((N, d), np.uint8), vnorm=np.zeros(N, np.uint16),
               vydist=np.zeros((N, d), np.float64), vsat=np.zeros(N, np.uint8))
    _load().oracle_quantize_values(d, N, _p(x), _p(tab.D), _p(tab.cV), _p(tab.tV), tab.BV,
                                   _p(out["vidx"]), _p(out["vnorm"]), _p(out["vydist"]),
                                   _p(out["vsat"]))
    return out


def quantize(tab: Tables, k: np.ndarray, v: np.ndarray):
    out = quantize_keys(tab, k)
    out.update(quantize_values(tab, v))
    return out


def tile_bytes(d: int, fmt) -> int:
    """Bytes of a 16-token tile; fmt as for fmt_of (b, (B_K, B_V, qjl) or Tables)."""
    kb, vb, qjl = fmt_of(fmt)
    return int(_load().oracle_tile_bytes(d, kb, vb, qjl))


def pack_stream(d: int, fmt, codes: dict, N: int | None = None) -> np.ndarray:
    """Pack tokens [0, N) of one (batch, kv-head) stream into 16-token tiles."""
    kb, vb, qjl = fmt_of(fmt)
    N = codes["kidx"].shape[0] if N is None else N
    nt = (N + TILE - 1) // TILE
    out = np.zeros(nt * tile_bytes(d, (kb, vb, qjl)), dtype=np.uint8)
    c = {k: np.ascontiguousarray(codes[k]) for k in
         ("kidx", "ksign", "knorm", "rnorm", "vidx", "vnorm")}
    _load().oracle_pack_stream(d, kb, vb, qjl, N, _p(c["kidx"]), _p(c["ksign"]), _p(c["knorm"]),
                               _p(c["rnorm"]), _p(c["vidx"]), _p(c["vnorm"]), _p(out))
    return out


def unpack_stream(d: int, fmt, N: int, tiles: np.ndarray) -> dict:
    tiles = np.ascontiguousarray(tiles, dtype=np.uint8)
    out = dict(kidx=np.zeros((N, d), np.uint8), ksign=np.zeros((N, d), np.uint8),
               knorm=np.zeros(N, np.uint16), rnorm=np.zeros(N, np.uint16),
               vidx=np.zeros((N, d), np.uint8), vnorm=np.zeros(N, np.uint16))
    kb, vb, qjl = fmt_of(fmt)
    _load().oracle_unpack_stream(d, kb, vb, qjl, N, _p(tiles), _p(out["kidx"]), _p(out["ksign"]),
                                 _p(out["knorm"]), _p(out["rnorm"]), _p(out["vidx"]),
                                 _p(out["vnorm"]))
    return out


def attend_head(tab: Tables, q_bits: np.ndarray, q_is_bf16: bool, codes: dict, N: int):
    """One query head over tokens [0, N) of decoded codes. Returns (o, logits)."""
    d = tab.d
    q_bits = np.ascontiguousarray(q_bits).view(np.uint16)
    o = np.zeros(d, np.float64)
    lg = np.zeros(max(N, 1), np.float64)
    c = {k: np.ascontiguousarray(codes[k]) for k in
         ("kidx", "ksign", "knorm", "rnorm", "vidx", "vnorm")}
    _load().oracle_attend_head(d, N, _p(q_bits), int(q_is_bf16), tab.qjl, _p(tab.D), _p(tab.S),
                               _p(tab.cK), _p(tab.cV), _p(c["kidx"]), _p(c["ksign"]),
                               _p(c["knorm"]), _p(c["rnorm"]), _p(c["vidx"]), _p(c["vnorm"]),
                               _p(o), _p(lg))
    return o, lg[:N]


def attend_batch(tab: Tables, q_bits: np.ndarray, q_is_bf16: bool, codes: dict,
                 seq_len: np.ndarray, Hkv: int, want_logits: bool = False):
    """q_bits: [B, Hq, d] uint16; codes: arrays shaped [B, Hkv, cap, ...]."""
    q_bits = np.ascontiguousarray(q_bits).view(np.uint16)
    B, Hq, d = q_bits.shape
    cap = codes["knorm"].shape[2]
    out = np.zeros((B, Hq, d), np.float64)
    lg = np.zeros((B, Hq, cap), np.float64) if want_logits else None
    sl = np.ascontiguousarray(seq_len, dtype=np.int32)
    c = {k: np.ascontiguousarray(codes[k]) for k in
         ("kidx", "ksign", "knorm", "rnorm", "vidx", "vnorm")}
    _load().oracle_attend_batch(d, B, Hq, Hkv, cap, _p(sl), _p(q_bits), int(q_is_bf16), tab.qjl,
                                _p(tab.D), _p(tab.S), _p(tab.cK), _p(tab.cV), _p(c["kidx"]),
                                _p(c["ksign"]), _p(c["knorm"]), _p(c["rnorm"]), _p(c["vidx"]),
                                _p(c["vnorm"]), _p(out), _p(lg) if lg is not None else None)
    return (out, lg) if want_logits else out


def distortion_mc(d: int, B: int, nvec: int, seed: int = 12345) -> float:
    return float(_load().oracle_distortion_mc(d, B, nvec, seed))


def ip_trials(d: int, bits: int, ntrials: int, seed0: int, q: np.ndarray, k: np.ndarray):
    q = np.ascontiguousarray(q, dtype=np.float64)
    k = np.ascontiguousarray(k, dtype=np.float64)
    em = np.zeros(ntrials, np.float64)
    eq = np.zeros(ntrials, np.float64)
    _load().oracle_ip_trials(d, bits, ntrials, seed0, _p(q), _p(k), _p(em), _p(eq))
    return em, eq


def reconstruct(tab: Tables, codes: dict, N: int):
    """Dequantized vectors implied by stored codes (fp64):
    k^_n = |k_n| Pi^T (cK[idx_n] + rho_n kappa S^T (2 s_n - 1)),
    v^_n = |v_n| Pi^T cV[vidx_n]. Used to pin attention to textbook SDPA."""
    d, m = tab.d, tab.m
    kappa = np.sqrt(np.pi / 2) / m
    kh = np.zeros((N, d))
    vh = np.zeros((N, d))
    for n in range(N):
        kn = half_to_double(codes["knorm"][n])
        rn = half_to_double(codes["rnorm"][n])
        vn = half_to_double(codes["vnorm"][n])
        yk = tab.cK[codes["kidx"][n]].astype(np.float64) + rn * kappa * (
            tab.S.T @ (2.0 * codes["ksign"][n].astype(np.float64) - 1.0))
        kh[n] = kn * rotate_inverse(tab.D, yk)
        vh[n] = vn * rotate_inverse(tab.D, tab.cV[codes["vidx"][n]].astype(np.float64))
    return kh, vh
