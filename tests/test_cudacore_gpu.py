"""tq_attend_cudacore, the CUDA-core comparison kernel (shared-memory lookup
tables for the codebook logits, the QJL term by sign-nibble tables or by
bit-plane popcounts, P V as FMAs), against the fp64 oracle over the same codes
and against the tensor-core tq_attend, through the C ABI. Cases span several
tiles with ragged tails, an empty sequence, GQA group sizes below 8, and a
unit split over many CTAs; the argument checks refuse other formats and modes."""
import numpy as np
import pytest
import torch

import kv_cache_vector_04_b200 as tq
from kv_cache_vector_04_b200 import inputs
from oracle import oracle as O
from tests import parity as P

pytestmark = pytest.mark.gpu


def _case(ctx, tab, B, Hkv, Hq, N, seed, dist="lognormal_norm"):
    k = inputs.kv_tensor((B, Hkv, N, ctx.d), dist, seed)
    v = inputs.kv_tensor((B, Hkv, N, ctx.d), dist, seed + 1)
    codes = P.oracle_codes(tab, k, v)
    cache = tq.Cache(P.pack_cache(tab, codes, N, ctx.d, ctx.bits), B, Hkv, N)
    q = torch.randn((B, Hq, ctx.d), generator=torch.Generator().manual_seed(seed)).to(torch.bfloat16)
    return cache, codes, q


@pytest.mark.parametrize("mode", [tq.binding.TQ_CC_QJL_NIBBLE, tq.binding.TQ_CC_QJL_POPCOUNT])
@pytest.mark.parametrize("shape", [(2, 4, 16, 1008, [1000, 377], "lognormal_norm"),
                                   (3, 2, 10, 304, [300, 0, 151], "spiky_tokens"),
                                   (1, 1, 8, 4096, [4093], "outlier_channels")])
def test_cudacore_matches_oracle_and_tensor_core_path(mode, shape):
    torch.cuda.set_device(0)
    B, Hkv, Hq, N, seq, dist = shape
    ctx, tab = tq.tq_init(128, 4, 1), O.Tables(128, 4, 1)
    cache, codes, q = _case(ctx, tab, B, Hkv, Hq, N, 11, dist)
    sl = torch.tensor(seq, dtype=torch.int32, device="cuda")
    got = tq.tq_attend_cudacore(ctx, q.cuda(), cache, sl, max(seq), qjl_mode=mode)
    ref = tq.tq_attend(ctx, q.cuda(), cache, sl, max(seq))
    torch.cuda.synchronize()
    assert tq.tq_status(ctx) == 0
    got = got.cpu().numpy().astype(np.float64)
    ora = O.attend_batch(tab, P.q_bits(q), True, P.stack_codes(codes, cache.capacity),
                         np.array(seq, np.int32), cache.Hkv)
    err = P.attn_error(got, ora)
    assert err.max() <= P.ATTN_TOL, err.max()
    err = P.attn_error(got, ref.cpu().numpy().astype(np.float64))
    assert err.max() <= P.ATTN_TOL, err.max()
    for b in range(B):
        if seq[b] == 0:
            assert np.all(got[b] == 0.0)


def test_cudacore_refuses_other_formats_and_modes():
    torch.cuda.set_device(0)
    ctx = tq.tq_init(128, 3, 1)
    cache = tq.new_cache(ctx, 1, 1, 16)
    q = torch.zeros((1, 8, 128), dtype=torch.bfloat16, device="cuda")
    sl = torch.full((1,), 16, dtype=torch.int32, device="cuda")
    with pytest.raises(tq.TQError) as e:
        tq.tq_attend_cudacore(ctx, q, cache, sl, 16)
    assert e.value.code == tq.binding.TQ_ERR_UNSUPPORTED
    ctx4 = tq.tq_init(128, 4, 1)
    cache4 = tq.new_cache(ctx4, 1, 1, 16)
    for mode in (0, 3):
        with pytest.raises(tq.TQError) as e:
            tq.tq_attend_cudacore(ctx4, q, cache4, sl, 16, qjl_mode=mode)
        assert e.value.code == tq.binding.TQ_ERR_INVALID_ARG
