"""tq_attend_noalloc: attention with the library's static device scratch.

Some callers cannot allocate device memory (a runtime whose device memory
belongs to an allocator it does not control, a serving loop that forbids
allocation after start-up), so this entry point takes no workspace. These
tests call it through the C ABI and check that it gives what tq_attend gives
with a caller-allocated workspace, and what the fp64 oracle gives, on two calls
in a row (the second call reuses the scratch the first one left behind), and
that a call needing more scratch than the static array holds is refused
without running.

The file is named to be collected last; every test here also passes when run
alone in a fresh process.
"""
import numpy as np
import pytest
import torch

import kv_cache_vector_04_b200 as tq
from kv_cache_vector_04_b200 import inputs
from oracle import oracle as O
from tests import parity as P

pytestmark = pytest.mark.gpu


def _case(ctx, tab, B, Hkv, Hq, N, seed):
    """A cache holding the oracle's packing of its own codes (so the GPU and the
    oracle attend over the same codes), the codes, and bf16 queries."""
    k = inputs.kv_tensor((B, Hkv, N, ctx.d), "lognormal_norm", seed)
    v = inputs.kv_tensor((B, Hkv, N, ctx.d), "lognormal_norm", seed + 1)
    codes = P.oracle_codes(tab, k, v)
    cache = tq.Cache(P.pack_cache(tab, codes, N, ctx.d, ctx.bits), B, Hkv, N)
    q = torch.randn((B, Hq, ctx.d), generator=torch.Generator().manual_seed(seed)).to(torch.bfloat16)
    return cache, codes, q


def test_noalloc_matches_workspace_call_and_oracle_twice():
    torch.cuda.set_device(0)
    ctx, tab = tq.tq_init(128, 3, 1), O.Tables(128, 3, 1)
    runs = [(_case(ctx, tab, 2, 4, 16, 1008, 7), [1000, 377]),
            (_case(ctx, tab, 3, 2, 10, 304, 9), [300, 0, 151])]
    for (cache, codes, q), seq in runs:
        sl = torch.tensor(seq, dtype=torch.int32, device="cuda")
        max_len = max(seq)
        ref = tq.tq_attend(ctx, q.cuda(), cache, sl, max_len)
        got = tq.tq_attend_noalloc(ctx, q.cuda(), cache, sl, max_len)
        torch.cuda.synchronize()
        got = got.cpu().numpy().astype(np.float64)
        err = P.attn_error(got, ref.cpu().numpy().astype(np.float64))
        assert err.max() <= P.ATTN_TOL, err.max()
        ora = O.attend_batch(tab, P.q_bits(q), True, P.stack_codes(codes, cache.capacity),
                             np.array(seq, np.int32), cache.Hkv)
        err = P.attn_error(got, ora)
        assert err.max() <= P.ATTN_TOL, err.max()
    assert tq.tq_status(ctx) == 0


def test_noalloc_refuses_more_than_its_scratch():
    torch.cuda.set_device(0)
    ctx = tq.tq_init(128, 4, 1)
    # the workspace grows with the number of (sequence, kv head, head group)
    # units, not with the context: 256 x 8 units need more than the 16 MiB
    # array even at 16 tokens. The cache is a real one of that size, so a
    # refusal that regressed would still read inside its buffers.
    B, Hkv, Hq, N = 256, 8, 64, 16
    need = tq.tq_attend_workspace(ctx, B, Hq, Hkv, N)
    assert need > tq.binding.TQ_NOALLOC_SCRATCH_BYTES
    cache = tq.new_cache(ctx, B, Hkv, N)
    q = torch.zeros((B, Hq, 128), dtype=torch.bfloat16, device="cuda")
    sl = torch.full((B,), N, dtype=torch.int32, device="cuda")
    with pytest.raises(tq.TQError) as e:
        tq.tq_attend_noalloc(ctx, q, cache, sl, N)
    assert e.value.code == tq.binding.TQ_ERR_WORKSPACE
