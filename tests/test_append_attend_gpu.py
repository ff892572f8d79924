"""GPU parity of tq_append_attend: one layer's decode step (append T new
tokens, then attend) against the oracle.

For 1 <= T <= 16 the new tokens are quantized inside the attention prologue
from shared-memory copies of their tiles; for T > 16 the quantize kernel runs
first. Either way the cache must hold the oracle's codes for the new tokens,
every other token's bits must be left as they were (the tiles start out as
random bytes), and the attention output must match the oracle's over the
prefix plus the new tokens.
"""
import numpy as np
import pytest
import torch

import kv_cache_vector_04_b200 as tq
from oracle import oracle as O
from tests import parity as P
from tests.test_parity_gpu import ctx_for, kv, qtensor

pytestmark = pytest.mark.gpu

DB = [(d, b) for d in (64, 128, 256) for b in (2, 3, 4)]


def _run(d, bits, T, starts, Hq=8, seed=0, fmt=None):
    ctx, tab = ctx_for(d, bits, fmt=fmt)
    B, Hkv, cap = len(starts), 2, 96
    pre = max(starts)
    cache = tq.new_cache(ctx, B, Hkv, cap)
    g = torch.Generator().manual_seed(seed + 77)
    cache.data.copy_(torch.randint(0, 256, (cache.data.numel(),), generator=g,
                                   dtype=torch.uint8).cuda())
    k0, v0 = kv(B, Hkv, max(pre, 1), d, seed=seed + 11)
    if pre > 0:
        tq.tq_quantize(ctx, k0.cuda(), v0.cuda(), torch.zeros(B, dtype=torch.int32).cuda(), cache)
    before = cache.data.cpu().numpy()
    k1, v1 = kv(B, Hkv, T, d, seed=seed + 23, dist="outlier_channels")
    q = qtensor(B, Hq, d, seed=seed + 5)
    sp = torch.tensor(starts, dtype=torch.int32)
    seq = sp + T
    out = tq.tq_append_attend(ctx, q.cuda(), k1.cuda(), v1.cuda(), sp.cuda(), cache,
                              seq.cuda(), int(seq.max()))
    torch.cuda.synchronize()
    assert tq.tq_status(ctx) == 0
    after = cache.data.cpu().numpy()
    lay = tq.tq_cache_layout(ctx)
    per = (cap // 16) * lay["tile_bytes"]
    c0 = P.oracle_codes(tab, k0, v0)
    c1 = P.oracle_codes(tab, k1, v1)
    stats = P.QuantStats()
    streams = []
    for b in range(B):
        row = []
        for h in range(Hkv):
            s0 = (b * Hkv + h) * per
            new = O.unpack_stream(d, tab, cap, after[s0: s0 + per])
            old = O.unpack_stream(d, tab, cap, before[s0: s0 + per])
            sel = np.zeros(cap, bool)
            sel[starts[b]: starts[b] + T] = True
            for key in new:
                assert np.array_equal(new[key][~sel], old[key][~sel]), (b, h, key)
            P.compare_stream(tab, {kk: vv[starts[b]: starts[b] + T] for kk, vv in new.items()},
                             c1[b][h], T, stats)
            # the oracle's own codes for tokens [0, start + T): prefix, then the new tokens
            full = {}
            for key in ("kidx", "ksign", "knorm", "rnorm", "vidx", "vnorm"):
                full[key] = np.concatenate([c0[b][h][key][:starts[b]], c1[b][h][key]])
            row.append(full)
        streams.append(row)
    stats.check()
    ref = O.attend_batch(tab, P.q_bits(q), True, P.stack_codes(streams, cap), seq.numpy(), Hkv)
    err = P.attn_error(out.cpu().numpy().astype(np.float64), ref)
    assert err.max() <= P.ATTN_TOL, err.max()


@pytest.mark.parametrize("d,bits", DB)
def test_append_one_token_then_attend(d, bits):
    # the decode step proper: one token per sequence, at a tile start, mid-tile and a tile end
    _run(d, bits, 1, [32, 37, 47], seed=d + bits)


@pytest.mark.parametrize("d,bits", [(128, 4), (64, 2), (256, 3)])
@pytest.mark.parametrize("T", [5, 16])
def test_append_several_tokens_across_tiles(d, bits, T):
    # T new tokens that straddle a tile boundary in some sequences; an empty prefix in one
    _run(d, bits, T, [0, 13, 60], seed=3 * T + d)


def test_append_more_than_a_tile_uses_the_quantize_kernel():
    _run(128, 3, 21, [7, 40], seed=9)


def test_append_out_of_capacity_sets_status_and_writes_nothing():
    d, bits = 128, 4
    ctx, tab = ctx_for(d, bits)
    B, Hkv, cap = 2, 1, 32
    cache = tq.new_cache(ctx, B, Hkv, cap)
    k0, v0 = kv(B, Hkv, 30, d, seed=4)
    tq.tq_quantize(ctx, k0.cuda(), v0.cuda(), torch.zeros(B, dtype=torch.int32).cuda(), cache)
    before = cache.data.clone()
    k1, v1 = kv(B, Hkv, 4, d, seed=5)
    q = qtensor(B, 4, d, seed=6)
    sp = torch.tensor([30, 2], dtype=torch.int32)   # 30 + 4 > 32: sequence 0 is skipped
    seq = torch.tensor([30, 6], dtype=torch.int32)
    tq.tq_append_attend(ctx, q.cuda(), k1.cuda(), v1.cuda(), sp.cuda(), cache, seq.cuda(), 30)
    torch.cuda.synchronize()
    assert tq.tq_status(ctx) & tq.TQ_STATUS_CAPACITY
    lay = tq.tq_cache_layout(ctx)
    per = (cap // 16) * lay["tile_bytes"]
    assert torch.equal(before[:per], cache.data[:per])
    assert not torch.equal(before[per:], cache.data[per:])
