"""Host-side checks of the CUDA library that need no GPU: the shared library
loads and exports every entry point include/tq.h declares, argument errors are
reported without a launch, and the host-built tables equal the oracle's."""
import ctypes
import os
import re

import numpy as np
import pytest

import kv_cache_vector_04_b200 as tq
from kv_cache_vector_04_b200 import binding
from oracle import oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    src = open(os.path.join(ROOT, "include", "tq.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(tq_[a-z_]+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    names = declared_functions()
    assert len(names) >= 12
    lib = ctypes.CDLL(binding.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(binding.EXPORTS) == names


def test_binding_constants_equal_header_defines():
    src = open(os.path.join(ROOT, "include", "tq.h")).read()
    defs = dict(re.findall(r"#define\s+(TQ_[A-Z0-9_]+)\s+\(?(-?(?:0x)?[0-9a-fA-F]+)u?\)?\s*(?:/\*|\n)", src))
    assert binding.TQ_NOALLOC_SCRATCH_BYTES == 16 << 20 and "(16u << 20)" in src
    assert len(defs) >= 12
    for name, val in defs.items():
        if hasattr(binding, name):
            assert getattr(binding, name) == int(val, 0), name
    for name in ("TQ_STATUS_CAPACITY", "TQ_STATUS_SEQ_LEN", "TQ_STATUS_NORM_SAT",
                 "TQ_STATUS_WAIT_TIMEOUT", "TQ_ERR_WORKSPACE", "TQ_TILE"):
        assert name in defs and hasattr(binding, name), name


def test_unsupported_formats_are_refused_before_any_cuda_call():
    h = ctypes.c_void_p()
    for f in ((2, 4, 1), (5, 5, 0), (4, 3, 0), (1, 1, 0), (3, 4, 2), (2, 3, 0)):
        assert binding._lib.tq_init_ex(128, f[0], f[1], f[2], 0, 1, ctypes.byref(h)) == \
            tq.TQ_ERR_UNSUPPORTED, f
    assert binding._lib.tq_init_ex(96, 3, 4, 0, 0, 1, ctypes.byref(h)) == tq.TQ_ERR_UNSUPPORTED
    assert binding._lib.tq_init_ex(128, 3, 4, 0, 2, 1, ctypes.byref(h)) == tq.TQ_ERR_UNSUPPORTED


def test_missing_library_fails_loudly(tmp_path):
    with pytest.raises(ImportError):
        binding._load(str(tmp_path / "libtq.so"))


def test_argument_errors_without_launch():
    lib = binding._lib
    assert lib.tq_cache_layout(None, None) == tq.TQ_ERR_INVALID_ARG
    h = ctypes.c_void_p()
    assert lib.tq_init(100, 3, 1, ctypes.byref(h)) == tq.TQ_ERR_UNSUPPORTED
    assert lib.tq_init(128, 5, 1, ctypes.byref(h)) == tq.TQ_ERR_UNSUPPORTED
    assert lib.tq_init(128, 3, 1, None) == tq.TQ_ERR_INVALID_ARG
    assert lib.tq_quantize(None, None, None, 1, 1, 1, None, None, None) == tq.TQ_ERR_INVALID_ARG
    assert lib.tq_copy(None, None, 16, None) == tq.TQ_ERR_INVALID_ARG
    for code in (0, -1, -2, -3, -4, -5):
        assert isinstance(tq.tq_strerror(code), str) and tq.tq_strerror(code)


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("bits", [2, 3, 4])
@pytest.mark.parametrize("seed", [1, 0xDEADBEEF12345678])
def test_host_tables_equal_oracle_tables(d, bits, seed):
    # The library builds its tables with its own fp64 code; the oracle with
    # its own. Both follow the same definition, so they must agree to the bit.
    t = tq.tq_build_tables(d, bits, seed)
    o = O.Tables(d, bits, seed)
    assert np.array_equal(t["centroids_k"], o.cK)
    assert np.array_equal(t["bounds_k"], o.tK)
    assert np.array_equal(t["centroids_v"], o.cV)
    assert np.array_equal(t["bounds_v"], o.tV)
    assert np.array_equal(t["signs"], o.D)
    assert np.array_equal(t["S"].astype(np.float64), o.S)


def test_k8v4_is_a_built_format_and_its_neighbours_are_not():
    # (7, 4, 1) passes the format check (on a machine without a GPU the call then
    # fails at the device, with another code); its near misses are refused first
    h = ctypes.c_void_p()
    rc = binding._lib.tq_init_ex(128, 7, 4, 1, 0, 1, ctypes.byref(h))
    assert rc != tq.TQ_ERR_UNSUPPORTED
    if rc == tq.TQ_OK:
        binding._lib.tq_destroy(h)
    for f in ((6, 4, 1), (7, 3, 1), (7, 4, 0), (8, 4, 1), (7, 2, 1)):
        assert binding._lib.tq_init_ex(128, f[0], f[1], f[2], 0, 1, ctypes.byref(h)) == \
            tq.TQ_ERR_UNSUPPORTED, f
    for d in (64, 256):
        rc = binding._lib.tq_init_ex(d, 7, 4, 1, 0, 1, ctypes.byref(h))
        assert rc != tq.TQ_ERR_UNSUPPORTED
        if rc == tq.TQ_OK:
            binding._lib.tq_destroy(h)
