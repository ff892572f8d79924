"""ctypes binding of the TurboQuant C ABI (include/tq.h).

Argument marshalling only: every step of quantization and attention runs in
the CUDA kernels of ``libtq.so``. PyTorch supplies device memory and streams.
Functions carry the names of the C entry points; tensors are passed as raw
pointers after checking dtype, device, shape and contiguity. If the shared
library is missing, importing this module raises: there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libtq.so")

TQ_OK = 0
TQ_ERR_INVALID_ARG = -1
TQ_ERR_UNSUPPORTED = -2
TQ_ERR_CUDA = -3
TQ_ERR_WORKSPACE = -4
TQ_ERR_DEVICE = -5
TQ_STATUS_CAPACITY = 0x1
TQ_STATUS_SEQ_LEN = 0x2
TQ_STATUS_NORM_SAT = 0x4
TQ_STATUS_WAIT_TIMEOUT = 0x8
TQ_CC_QJL_NIBBLE = 1
TQ_CC_QJL_POPCOUNT = 2
TQ_TILE = 16
TQ_CODEBOOK_GAUSS = 0
TQ_CODEBOOK_BETA = 1
TQ_DTYPE_F16 = 0
TQ_DTYPE_BF16 = 1

# every symbol include/tq.h declares
EXPORTS = ("tq_init", "tq_init_ex", "tq_build_codebook", "tq_destroy", "tq_cache_layout", "tq_cache_bytes", "tq_get_tables",
           "tq_build_tables", "tq_quantize", "tq_attend_workspace", "tq_attend", "tq_scores",
           "tq_attend_noalloc", "tq_append_attend", "tq_attend_cudacore", "tq_status", "tq_copy",
           "tq_strerror")
TQ_NOALLOC_SCRATCH_BYTES = 16 << 20


class TQError(RuntimeError):
    def __init__(self, code: int, what: str = ""):
        self.code = code
        super().__init__("%s: %s (%d)" % (what, _strerror(code), code))


class _Layout(ctypes.Structure):
    _fields_ = [("d", ctypes.c_int32), ("bits", ctypes.c_int32), ("m", ctypes.c_int32),
                ("kbits", ctypes.c_int32), ("vbits", ctypes.c_int32), ("tile", ctypes.c_int32),
                ("k_bytes_per_token", ctypes.c_int64), ("v_bytes_per_token", ctypes.c_int64),
                ("tile_bytes", ctypes.c_int64), ("code_bytes", ctypes.c_int64),
                ("chunk_bytes", ctypes.c_int32), ("qjl", ctypes.c_int32)]


class _Cache(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("B", ctypes.c_int32), ("Hkv", ctypes.c_int32),
                ("capacity", ctypes.c_int32)]


def _load(path: str = LIB_PATH):
    if not os.path.exists(path):
        raise ImportError("libtq.so not found at %s: build it with "
                          "`python kv_cache_vector_04_b200/build.py`" % path)
    lib = ctypes.CDLL(path)
    P, I, U64, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_uint64, ctypes.c_size_t
    sig = {
        "tq_init": (I, [I, I, U64, ctypes.POINTER(P)]),
        "tq_init_ex": (I, [I, I, I, I, I, U64, ctypes.POINTER(P)]),
        "tq_build_codebook": (I, [I, I, I, P, P]),
        "tq_destroy": (None, [P]),
        "tq_cache_layout": (I, [P, ctypes.POINTER(_Layout)]),
        "tq_cache_bytes": (I, [P, I, I, I, ctypes.POINTER(SZ)]),
        "tq_get_tables": (I, [P, P, P, P, P, P, P]),
        "tq_build_tables": (I, [I, I, U64, P, P, P, P, P, P]),
        "tq_quantize": (I, [P, P, P, I, I, I, P, ctypes.POINTER(_Cache), P]),
        "tq_attend_workspace": (I, [P, I, I, I, I, ctypes.POINTER(SZ)]),
        "tq_attend": (I, [P, P, I, I, I, ctypes.POINTER(_Cache), P, I, P, P, SZ, P]),
        "tq_scores": (I, [P, P, I, I, I, ctypes.POINTER(_Cache), P, I, P, P, SZ, P]),
        "tq_attend_noalloc": (I, [P, P, I, I, I, ctypes.POINTER(_Cache), P, I, P, P]),
        "tq_attend_cudacore": (I, [P, P, I, I, I, ctypes.POINTER(_Cache), P, I, P, P, SZ, I, P]),
        "tq_append_attend": (I, [P, P, I, P, P, I, I, I, P, ctypes.POINTER(_Cache), P, I, P, P,
                                 SZ, P]),
        "tq_status": (I, [P, ctypes.POINTER(ctypes.c_uint32)]),
        "tq_copy": (I, [P, P, SZ, P]),
        "tq_strerror": (ctypes.c_char_p, [I]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    return lib


class _LazyLib:
    """The CUDA library, loaded on first use (a missing library then raises
    ImportError at that first call): importing the package for its workload
    shapes alone maps no GPU code."""
    _handle = None

    def __getattr__(self, name):
        if _LazyLib._handle is None:
            _LazyLib._handle = _load()
        return getattr(_LazyLib._handle, name)


_lib = _LazyLib()


def _strerror(code: int) -> str:
    return _lib.tq_strerror(int(code)).decode()


def tq_strerror(code: int) -> str:
    return _strerror(code)


def _check(rc: int, what: str):
    if rc != TQ_OK:
        raise TQError(rc, what)


def _stream_ptr(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _dev(t: torch.Tensor, name: str, dtype=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor" % name)
    if dtype is not None and t.dtype != dtype:
        raise ValueError("%s must have dtype %s, got %s" % (name, dtype, t.dtype))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    return ctypes.c_void_p(t.data_ptr())


# ------------------------------------------------------------------ context

class Context:
    """Handle of a tq_ctx: the tables of one (d, format, seed) on one device.
    fmt = (B_K, B_V, qjl); TurboQuant at b bits is (b - 1, b, 1)."""

    def __init__(self, handle: int, d: int, bits: int, seed: int, device: int,
                 fmt: tuple | None = None):
        self._h = ctypes.c_void_p(handle)
        self.d, self.bits, self.seed, self.device = d, bits, seed, device
        self.fmt = (bits - 1, bits, 1) if fmt is None else tuple(fmt)

    @property
    def handle(self):
        return self._h

    def close(self):
        if self._h and self._h.value:
            _lib.tq_destroy(self._h)
            self._h = ctypes.c_void_p(0)

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


@dataclass
class Cache:
    """A packed cache: ``data`` is a uint8 CUDA tensor of tq_cache_bytes."""
    data: torch.Tensor
    B: int
    Hkv: int
    capacity: int

    def struct(self) -> _Cache:
        return _Cache(ctypes.c_void_p(self.data.data_ptr()), self.B, self.Hkv, self.capacity)


def tq_init(d: int, bits: int, seed: int) -> Context:
    h = ctypes.c_void_p()
    _check(_lib.tq_init(int(d), int(bits), ctypes.c_uint64(seed), ctypes.byref(h)), "tq_init")
    return Context(h.value, d, bits, seed, torch.cuda.current_device())


def tq_init_ex(d: int, kbits: int, vbits: int, qjl: int, seed: int,
               codebook: int = TQ_CODEBOOK_GAUSS) -> Context:
    """A context of any built format: (kbits, vbits, qjl) = (B_K, B_V, QJL on
    keys); codebook TQ_CODEBOOK_GAUSS or TQ_CODEBOOK_BETA (exact marginal)."""
    h = ctypes.c_void_p()
    _check(_lib.tq_init_ex(int(d), int(kbits), int(vbits), int(qjl), int(codebook),
                           ctypes.c_uint64(seed), ctypes.byref(h)), "tq_init_ex")
    return Context(h.value, d, vbits, seed, torch.cuda.current_device(),
                   fmt=(int(kbits), int(vbits), int(qjl)))


def tq_build_codebook(B: int, d: int, codebook: int = TQ_CODEBOOK_GAUSS):
    """Host-only codebook: (fp32 centroids [2^B], fp32 boundaries [2^B - 1])."""
    import numpy as np
    c = np.zeros(1 << B, np.float32)
    t = np.zeros(max((1 << B) - 1, 1), np.float32)
    _check(_lib.tq_build_codebook(int(B), int(d), int(codebook), c.ctypes.data_as(ctypes.c_void_p),
                                  t.ctypes.data_as(ctypes.c_void_p)), "tq_build_codebook")
    return c, t[: (1 << B) - 1]


def tq_destroy(ctx: Context):
    ctx.close()


def tq_cache_layout(ctx: Context) -> dict:
    L = _Layout()
    _check(_lib.tq_cache_layout(ctx.handle, ctypes.byref(L)), "tq_cache_layout")
    return {name: getattr(L, name) for name, _ in _Layout._fields_}


def tq_cache_bytes(ctx: Context, B: int, Hkv: int, capacity: int) -> int:
    n = ctypes.c_size_t()
    _check(_lib.tq_cache_bytes(ctx.handle, B, Hkv, capacity, ctypes.byref(n)), "tq_cache_bytes")
    return n.value


def new_cache(ctx: Context, B: int, Hkv: int, capacity: int, device=None) -> Cache:
    """Allocate (torch) a packed cache; capacity is rounded up to a tile."""
    capacity = (capacity + TQ_TILE - 1) // TQ_TILE * TQ_TILE
    n = tq_cache_bytes(ctx, B, Hkv, capacity)
    dev = torch.device("cuda", ctx.device) if device is None else device
    return Cache(torch.zeros(n, dtype=torch.uint8, device=dev), B, Hkv, capacity)


def _tables(fn, d: int, kbits: int, vbits: int, args_prefix):
    import numpy as np
    ck = np.zeros(1 << kbits, np.float32)
    tk = np.zeros(max((1 << kbits) - 1, 1), np.float32)
    cv = np.zeros(1 << vbits, np.float32)
    tv = np.zeros((1 << vbits) - 1, np.float32)
    sg = np.zeros(d, np.int8)
    S = np.zeros((d, d), np.float32)
    p = lambda a: a.ctypes.data_as(ctypes.c_void_p)
    _check(fn(*args_prefix, p(ck), p(tk), p(cv), p(tv), p(sg), p(S)), fn.__name__)
    return dict(centroids_k=ck, bounds_k=tk[: (1 << kbits) - 1], centroids_v=cv,
                bounds_v=tv, signs=sg, S=S)


def tq_get_tables(ctx: Context) -> dict:
    """Host copies of a context's tables (arrays sized by its format)."""
    return _tables(_lib.tq_get_tables, ctx.d, ctx.fmt[0], ctx.fmt[1], (ctx.handle,))


def tq_build_tables(d: int, bits: int, seed: int) -> dict:
    """TurboQuant tables at b = bits computed on the host only."""
    return _tables(_lib.tq_build_tables, d, bits - 1, bits, (int(d), int(bits), ctypes.c_uint64(seed)))


# ------------------------------------------------------------------ quantize / attend

def tq_quantize(ctx: Context, k: torch.Tensor, v: torch.Tensor, start_pos: torch.Tensor,
                cache: Cache, stream=None):
    """Append T tokens: k, v fp16 [B, Hkv, T, d]; start_pos int32 [B] (device)."""
    if k.dim() != 4 or k.shape != v.shape or k.shape[3] != ctx.d:
        raise ValueError("k and v must both be [B, Hkv, T, d] with d = %d" % ctx.d)
    B, Hkv, T, _ = k.shape
    if start_pos.numel() != B:
        raise ValueError("start_pos must have B entries")
    c = cache.struct()
    _check(_lib.tq_quantize(ctx.handle, _dev(k, "k", torch.float16), _dev(v, "v", torch.float16),
                            B, Hkv, T, _dev(start_pos, "start_pos", torch.int32), ctypes.byref(c),
                            ctypes.c_void_p(_stream_ptr(stream))), "tq_quantize")


def tq_attend_workspace(ctx: Context, B: int, Hq: int, Hkv: int, max_len: int) -> int:
    n = ctypes.c_size_t()
    _check(_lib.tq_attend_workspace(ctx.handle, B, Hq, Hkv, max_len, ctypes.byref(n)),
           "tq_attend_workspace")
    return n.value


def new_workspace(ctx: Context, B: int, Hq: int, Hkv: int, max_len: int) -> torch.Tensor:
    n = tq_attend_workspace(ctx, B, Hq, Hkv, max_len)
    return torch.empty(max(n, 256), dtype=torch.uint8, device=torch.device("cuda", ctx.device))


def _q_dtype(q: torch.Tensor) -> int:
    if q.dtype == torch.bfloat16:
        return TQ_DTYPE_BF16
    if q.dtype == torch.float16:
        return TQ_DTYPE_F16
    raise ValueError("q must be bfloat16 or float16")


def _attend_like(fn, what, ctx, q, cache, seq_len, max_len, out, workspace, stream):
    if q.dim() != 3 or q.shape[2] != ctx.d:
        raise ValueError("q must be [B, Hq, d] with d = %d" % ctx.d)
    B, Hq, _ = q.shape
    if workspace is None:
        workspace = new_workspace(ctx, B, Hq, cache.Hkv, max_len)
    c = cache.struct()
    _check(fn(ctx.handle, _dev(q, "q"), _q_dtype(q), B, Hq, ctypes.byref(c),
              _dev(seq_len, "seq_len", torch.int32), int(max_len), _dev(out, "out", torch.float32),
              _dev(workspace, "workspace"), workspace.numel() * workspace.element_size(),
              ctypes.c_void_p(_stream_ptr(stream))), what)
    return out


def tq_attend(ctx: Context, q: torch.Tensor, cache: Cache, seq_len: torch.Tensor, max_len: int,
              out: torch.Tensor | None = None, workspace: torch.Tensor | None = None, stream=None):
    """One decode step: q [B, Hq, d] (bf16/fp16) -> out fp32 [B, Hq, d]."""
    if out is None:
        out = torch.empty(q.shape, dtype=torch.float32, device=q.device)
    return _attend_like(_lib.tq_attend, "tq_attend", ctx, q, cache, seq_len, max_len, out,
                        workspace, stream)


def tq_attend_cudacore(ctx: Context, q: torch.Tensor, cache: Cache, seq_len: torch.Tensor,
                       max_len: int, qjl_mode: int = 1, out: torch.Tensor | None = None,
                       workspace: torch.Tensor | None = None, stream=None):
    """tq_attend with the split kernel on CUDA cores (lookup tables; QJL term by
    sign-nibble tables, qjl_mode 1, or bit-plane popcounts, qjl_mode 2): the
    measured comparison for the tensor-core kernel. d = 128, 4-bit TurboQuant only."""
    if q.dim() != 3 or q.shape[2] != ctx.d:
        raise ValueError("q must be [B, Hq, d] with d = %d" % ctx.d)
    if out is None:
        out = torch.empty(q.shape, dtype=torch.float32, device=q.device)
    B, Hq, _ = q.shape
    if workspace is None:
        workspace = new_workspace(ctx, B, Hq, cache.Hkv, max_len)
    c = cache.struct()
    _check(_lib.tq_attend_cudacore(ctx.handle, _dev(q, "q"), _q_dtype(q), B, Hq, ctypes.byref(c),
                                   _dev(seq_len, "seq_len", torch.int32), int(max_len),
                                   _dev(out, "out", torch.float32), _dev(workspace, "workspace"),
                                   workspace.numel() * workspace.element_size(), int(qjl_mode),
                                   ctypes.c_void_p(_stream_ptr(stream))), "tq_attend_cudacore")
    return out


def tq_scores(ctx: Context, q: torch.Tensor, cache: Cache, seq_len: torch.Tensor, max_len: int,
              out: torch.Tensor | None = None, workspace: torch.Tensor | None = None, stream=None):
    """Estimated logits: fp32 [B, Hq, max_len] (-inf past seq_len)."""
    if out is None:
        out = torch.empty((q.shape[0], q.shape[1], max_len), dtype=torch.float32, device=q.device)
    return _attend_like(_lib.tq_scores, "tq_scores", ctx, q, cache, seq_len, max_len, out,
                        workspace, stream)


def tq_attend_noalloc(ctx: Context, q: torch.Tensor, cache: Cache, seq_len: torch.Tensor,
                      max_len: int, out: torch.Tensor | None = None, stream=None):
    """tq_attend with the library's static device scratch instead of a
    workspace: for callers that cannot allocate device memory (their device
    memory belongs to another allocator, or allocation is forbidden after
    start-up; see tq.h). Overlapping calls on one GPU race on that scratch."""
    if q.dim() != 3 or q.shape[2] != ctx.d:
        raise ValueError("q must be [B, Hq, d] with d = %d" % ctx.d)
    if out is None:
        out = torch.empty(q.shape, dtype=torch.float32, device=q.device)
    B, Hq, _ = q.shape
    c = cache.struct()
    _check(_lib.tq_attend_noalloc(ctx.handle, _dev(q, "q"), _q_dtype(q), B, Hq, ctypes.byref(c),
                                  _dev(seq_len, "seq_len", torch.int32), int(max_len),
                                  _dev(out, "out", torch.float32),
                                  ctypes.c_void_p(_stream_ptr(stream))), "tq_attend_noalloc")
    return out


def tq_append_attend(ctx: Context, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                     start_pos: torch.Tensor, cache: Cache, seq_len: torch.Tensor, max_len: int,
                     out: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
                     stream=None):
    """One layer's decode step: append k, v (fp16 [B, Hkv, T, d]) at start_pos,
    then attend q [B, Hq, d] over tokens [0, seq_len[b]) -> fp32 [B, Hq, d]."""
    if q.dim() != 3 or q.shape[2] != ctx.d:
        raise ValueError("q must be [B, Hq, d] with d = %d" % ctx.d)
    if k.dim() != 4 or k.shape != v.shape or k.shape[3] != ctx.d:
        raise ValueError("k and v must both be [B, Hkv, T, d] with d = %d" % ctx.d)
    B, Hq, _ = q.shape
    if k.shape[0] != B or k.shape[1] != cache.Hkv or start_pos.numel() != B:
        raise ValueError("k, v, start_pos must match q's batch and the cache's kv heads")
    T = k.shape[2]
    if out is None:
        out = torch.empty(q.shape, dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = new_workspace(ctx, B, Hq, cache.Hkv, max_len)
    c = cache.struct()
    _check(_lib.tq_append_attend(ctx.handle, _dev(q, "q"), _q_dtype(q), _dev(k, "k", torch.float16),
                                 _dev(v, "v", torch.float16), B, Hq, T,
                                 _dev(start_pos, "start_pos", torch.int32), ctypes.byref(c),
                                 _dev(seq_len, "seq_len", torch.int32), int(max_len),
                                 _dev(out, "out", torch.float32), _dev(workspace, "workspace"),
                                 workspace.numel() * workspace.element_size(),
                                 ctypes.c_void_p(_stream_ptr(stream))), "tq_append_attend")
    return out


def tq_status(ctx: Context) -> int:
    f = ctypes.c_uint32()
    _check(_lib.tq_status(ctx.handle, ctypes.byref(f)), "tq_status")
    return f.value


def tq_copy(src: torch.Tensor, dst: torch.Tensor, stream=None):
    n = src.numel() * src.element_size()
    if dst.numel() * dst.element_size() < n:
        raise ValueError("dst smaller than src")
    _check(_lib.tq_copy(_dev(src, "src"), _dev(dst, "dst"), n,
                        ctypes.c_void_p(_stream_ptr(stream))), "tq_copy")


def attend_host(ctx: Context, q_host: torch.Tensor, cache: Cache, seq_len: torch.Tensor,
                max_len: int, out_host: torch.Tensor, workspace: torch.Tensor,
                q_dev: torch.Tensor, out_dev: torch.Tensor, stream=None):
    """tq_attend with host (pinned) input and output: H2D copy of q, the
    attention step, D2H copy of the result, all on one stream."""
    q_dev.copy_(q_host, non_blocking=True)
    tq_attend(ctx, q_dev, cache, seq_len, max_len, out=out_dev, workspace=workspace, stream=stream)
    out_host.copy_(out_dev, non_blocking=True)
    return out_host
