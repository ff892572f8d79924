"""tq_attend_noalloc: attention with the library's static device scratch.

Some callers cannot allocate device memory (for example code running inside a
CUDA-graph stream capture, or a runtime whose memory belongs to another
allocator), so this entry point takes no workspace. These tests call it
through the C ABI and check that it gives what tq_attend gives with a
caller-allocated workspace, on two calls in a row (the second call reuses the
scratch the first one left behind), and that a call needing more scratch than
the static array holds is refused without running.

The file is named to be collected last; every test here also passes when run
alone in a fresh process.
"""
import numpy as np
import pytest
import torch

import kv_cache_vector_04_b200 as tq
from kv_cache_vector_04_b200 import inputs
from tests import parity as P

pytestmark = pytest.mark.gpu


def _case(ctx, B, Hkv, Hq, N, seed):
    k = inputs.kv_tensor((B, Hkv, N, ctx.d), "lognormal_norm", seed)
    v = inputs.kv_tensor((B, Hkv, N, ctx.d), "lognormal_norm", seed + 1)
    cache = tq.new_cache(ctx, B, Hkv, N)
    tq.tq_quantize(ctx, k.cuda(), v.cuda(), torch.zeros(B, dtype=torch.int32, device="cuda"), cache)
    q = torch.randn((B, Hq, ctx.d), generator=torch.Generator().manual_seed(seed)).to(torch.bfloat16)
    return cache, q.cuda()


def test_noalloc_matches_workspace_call_twice():
    torch.cuda.set_device(0)
    ctx = tq.tq_init(128, 3, 1)
    runs = [(_case(ctx, 2, 4, 16, 1000, 7), [1000, 377]),
            (_case(ctx, 3, 2, 10, 300, 9), [300, 0, 151])]
    for (cache, q), seq in runs:
        sl = torch.tensor(seq, dtype=torch.int32, device="cuda")
        max_len = max(seq)
        ref = tq.tq_attend(ctx, q, cache, sl, max_len)
        got = tq.tq_attend_noalloc(ctx, q, cache, sl, max_len)
        torch.cuda.synchronize()
        err = P.attn_error(got.cpu().numpy().astype(np.float64), ref.cpu().numpy().astype(np.float64))
        assert err.max() <= P.ATTN_TOL, err.max()
    assert tq.tq_status(ctx) == 0


def test_noalloc_refuses_more_than_its_scratch():
    torch.cuda.set_device(0)
    ctx = tq.tq_init(128, 4, 1)
    B, Hkv, Hq, N = 256, 8, 64, 32768
    need = tq.tq_attend_workspace(ctx, B, Hq, Hkv, N)
    assert need > tq.binding.TQ_NOALLOC_SCRATCH_BYTES
    # the request is refused before anything is launched, so a stand-in cache
    # buffer of any size will do
    cache = tq.Cache(torch.zeros(16, dtype=torch.uint8, device="cuda"), B, Hkv, N)
    q = torch.zeros((B, Hq, 128), dtype=torch.bfloat16, device="cuda")
    sl = torch.full((B,), N, dtype=torch.int32, device="cuda")
    with pytest.raises(tq.TQError) as e:
        tq.tq_attend_noalloc(ctx, q, cache, sl, N)
    assert e.value.code == tq.binding.TQ_ERR_WORKSPACE
