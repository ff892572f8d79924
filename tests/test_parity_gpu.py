"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on the
same seeded inputs, element by element. Sizes span several tiles plus a
ragged tail; every supported (d, bits) is covered."""
import numpy as np
import pytest
import torch

import kv_cache_vector_04_b200 as tq
from kv_cache_vector_04_b200 import inputs
from oracle import oracle as O
from tests import parity as P

pytestmark = pytest.mark.gpu

DB = [(d, b) for d in (64, 128, 256) for b in (2, 3, 4)]
_ctx_cache = {}


def ctx_for(d, bits, seed=1, fmt=None, kind="gauss"):
    """(library context, oracle tables) of TurboQuant at `bits`, or of the
    format fmt = (B_K, B_V, qjl) when given; kind "beta" selects the
    exact-marginal codebooks."""
    key = (d, bits, seed, fmt, kind)
    if key not in _ctx_cache:
        if fmt is None and kind == "gauss":
            _ctx_cache[key] = (tq.tq_init(d, bits, seed), O.Tables(d, bits, seed))
        else:
            f = (bits - 1, bits, 1) if fmt is None else fmt
            code = tq.TQ_CODEBOOK_BETA if kind == "beta" else tq.TQ_CODEBOOK_GAUSS
            _ctx_cache[key] = (tq.tq_init_ex(d, f[0], f[1], f[2], seed, codebook=code),
                               O.Tables(d, f[1], seed, fmt=f, kind=kind))
    return _ctx_cache[key]


def kv(B, Hkv, T, d, seed, dist="lognormal_norm"):
    k = inputs.kv_tensor((B, Hkv, T, d), dist, seed)
    v = inputs.kv_tensor((B, Hkv, T, d), dist, seed + 1)
    return k, v


def qtensor(B, Hq, d, seed, dtype=torch.bfloat16):
    g = torch.Generator().manual_seed(seed)
    return torch.randn((B, Hq, d), generator=g).to(dtype)


def check_quantize(ctx, tab, k, v, cache, start=0, stats=None):
    B, Hkv, T, d = k.shape
    lay = tq.tq_cache_layout(ctx)
    host = cache.data.cpu().numpy()
    codes = P.oracle_codes(tab, k, v)
    st = P.QuantStats() if stats is None else stats
    for b in range(B):
        for h in range(Hkv):
            sb = P.stream_bytes(host, lay["tile_bytes"], cache.capacity, Hkv, b, h, start + T)
            gpu = O.unpack_stream(d, tab, start + T, sb)
            gpu = {kk: vv[start:] for kk, vv in gpu.items()}
            P.compare_stream(tab, gpu, codes[b][h], T, st)
    if stats is None:
        st.check()
    return codes


@pytest.mark.parametrize("d,bits", DB)
def test_quantize_matches_oracle(d, bits):
    ctx, tab = ctx_for(d, bits)
    stats = P.QuantStats()
    for T, dist in ((257, "lognormal_norm"), (33, "outlier_channels"), (48, "spiky_tokens")):
        k, v = kv(2, 3, T, d, seed=d * 10 + bits + T, dist=dist)
        cache = P.quantize_on_gpu(ctx, k, v, capacity=T + 40)
        check_quantize(ctx, tab, k, v, cache, stats=stats)
    stats.check()
    assert tq.tq_status(ctx) == 0


@pytest.mark.parametrize("d,bits", [(128, 3), (64, 2), (256, 4)])
def test_quantize_packed_bytes_equal_oracle_packer(d, bits):
    # With no boundary case in the batch, the packed tiles are byte-identical.
    ctx, tab = ctx_for(d, bits)
    k, v = kv(1, 2, 64, d, seed=7)
    cache = P.quantize_on_gpu(ctx, k, v, capacity=64)
    codes = P.oracle_codes(tab, k, v)
    host = cache.data.cpu().numpy()
    lay = tq.tq_cache_layout(ctx)
    for h in range(2):
        near = (codes[0][h]["kydist"] < P.BAND).any() or (codes[0][h]["zabs"] < P.BAND).any() \
            or (codes[0][h]["vydist"] < P.BAND).any()
        if near:
            continue
        ref = O.pack_stream(d, bits, codes[0][h])
        got = P.stream_bytes(host, lay["tile_bytes"], 64, 2, 0, h, 64)
        assert np.array_equal(got, ref)


@pytest.mark.parametrize("d,bits", [(128, 3), (64, 4), (256, 2)])
def test_append_one_token_at_a_time_equals_bulk(d, bits):
    ctx, tab = ctx_for(d, bits)
    B, Hkv, T = 2, 2, 37
    k, v = kv(B, Hkv, T, d, seed=11)
    bulk = P.quantize_on_gpu(ctx, k, v, capacity=48)
    step = tq.new_cache(ctx, B, Hkv, 48)
    kd, vd = k.cuda(), v.cuda()
    for t in range(T):
        sp = torch.full((B,), t, dtype=torch.int32, device="cuda")
        tq.tq_quantize(ctx, kd[:, :, t:t + 1].contiguous(), vd[:, :, t:t + 1].contiguous(), sp, step)
    torch.cuda.synchronize()
    # compare only the slots that were written (the rest of the last tile is
    # zero in both caches since both start zeroed)
    assert torch.equal(bulk.data, step.data)


def test_partial_tiles_keep_other_slots():
    d, bits = 128, 4
    ctx, tab = ctx_for(d, bits)
    B, Hkv, cap = 2, 1, 96
    cache = tq.new_cache(ctx, B, Hkv, cap)
    g = torch.Generator().manual_seed(3)
    canary = torch.randint(0, 256, (cache.data.numel(),), generator=g, dtype=torch.uint8)
    cache.data.copy_(canary.cuda())
    start = [5, 40]
    T = 29
    k, v = kv(B, Hkv, T, d, seed=5)
    tq.tq_quantize(ctx, k.cuda(), v.cuda(), torch.tensor(start, dtype=torch.int32).cuda(), cache)
    host = cache.data.cpu().numpy()
    base = canary.numpy()
    lay = tq.tq_cache_layout(ctx)
    codes = P.oracle_codes(tab, k, v)
    stats = P.QuantStats()
    for b in range(B):
        s0 = b * (cap // 16) * lay["tile_bytes"]
        new = O.unpack_stream(d, bits, cap, host[s0: s0 + (cap // 16) * lay["tile_bytes"]])
        old = O.unpack_stream(d, bits, cap, base[s0: s0 + (cap // 16) * lay["tile_bytes"]])
        sel = np.zeros(cap, bool)
        sel[start[b]: start[b] + T] = True
        for key in new:
            assert np.array_equal(new[key][~sel], old[key][~sel]), key
        P.compare_stream(tab, {kk: vv[start[b]: start[b] + T] for kk, vv in new.items()},
                         codes[b][0], T, stats)
    stats.check()


def test_capacity_overflow_sets_status_and_writes_nothing():
    ctx, tab = ctx_for(128, 3)
    cache = tq.new_cache(ctx, 2, 1, 32)
    before = cache.data.clone()
    k, v = kv(2, 1, 8, 128, seed=9)
    tq.tq_quantize(ctx, k.cuda(), v.cuda(), torch.tensor([28, -1], dtype=torch.int32).cuda(), cache)
    assert tq.tq_status(ctx) & tq.TQ_STATUS_CAPACITY
    assert torch.equal(before, cache.data)
    assert tq.tq_status(ctx) == 0   # read-and-clear


def test_norm_saturation_and_zero_vectors():
    d, bits = 128, 3
    ctx, tab = ctx_for(d, bits)
    k, v = kv(1, 1, 16, d, seed=21)
    k[0, 0, 3] = 60000.0
    v[0, 0, 4] = -60000.0
    k[0, 0, 5] = 0.0
    v[0, 0, 6] = 0.0
    cache = P.quantize_on_gpu(ctx, k, v, capacity=16)
    assert tq.tq_status(ctx) & tq.TQ_STATUS_NORM_SAT
    codes = check_quantize(ctx, tab, k, v, cache)
    assert codes[0][0]["knorm"][3] == 0x7BFF and codes[0][0]["vnorm"][4] == 0x7BFF
    assert codes[0][0]["knorm"][5] == 0 and codes[0][0]["vnorm"][6] == 0


# ---------------------------------------------------------------- attention

def run_attend(ctx, tab, cache, q, seq, max_len, Hkv):
    out = tq.tq_attend(ctx, q.cuda(), cache, torch.tensor(seq, dtype=torch.int32).cuda(), max_len)
    torch.cuda.synchronize()
    return out.cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("d,bits", DB)
def test_attend_on_oracle_packed_cache(d, bits):
    # Attention alone: the GPU attends over the oracle's packed codes.
    ctx, tab = ctx_for(d, bits)
    B, Hkv, Hq, N = 2, 2, 8, 257
    cap = 272
    k, v = kv(B, Hkv, N, d, seed=100 + d + bits, dist="outlier_channels")
    codes = P.oracle_codes(tab, k, v)
    cache = tq.Cache(P.pack_cache(tab, codes, cap, d, bits), B, Hkv, cap)
    seq = [257, 100]
    for dtype in (torch.bfloat16, torch.float16):
        q = qtensor(B, Hq, d, seed=bits, dtype=dtype)
        got = run_attend(ctx, tab, cache, q, seq, N, Hkv)
        ref = O.attend_batch(tab, P.q_bits(q), dtype == torch.bfloat16, P.stack_codes(codes, cap),
                             np.array(seq, np.int32), Hkv)
        err = P.attn_error(got, ref)
        assert err.max() <= P.ATTN_TOL, err.max()


@pytest.mark.parametrize("d,bits", [(128, 3), (64, 2), (256, 4), (128, 4)])
def test_quantize_then_attend_end_to_end(d, bits):
    ctx, tab = ctx_for(d, bits)
    B, Hkv, Hq, N = 2, 2, 4, 300
    k, v = kv(B, Hkv, N, d, seed=200 + d)
    cache = P.quantize_on_gpu(ctx, k, v, capacity=304)
    codes = P.oracle_codes(tab, k, v)
    q = qtensor(B, Hq, d, seed=1)
    seq = [300, 173]
    got = run_attend(ctx, tab, cache, q, seq, 300, Hkv)
    ref = O.attend_batch(tab, P.q_bits(q), True, P.stack_codes(codes, 304), np.array(seq, np.int32), Hkv)
    assert P.attn_error(got, ref).max() <= P.ATTN_TOL


@pytest.mark.parametrize("N", [1, 15, 16, 17, 33])
def test_attend_short_and_ragged(N):
    d, bits = 128, 3
    ctx, tab = ctx_for(d, bits)
    B, Hkv, Hq = 1, 2, 10   # 5 query heads per kv head (GQA group smaller than 8)
    k, v = kv(B, Hkv, N, d, seed=N)
    codes = P.oracle_codes(tab, k, v)
    cap = ((N + 15) // 16) * 16
    cache = tq.Cache(P.pack_cache(tab, codes, cap, d, bits), B, Hkv, cap)
    q = qtensor(B, Hq, d, seed=N)
    got = run_attend(ctx, tab, cache, q, [N], N, Hkv)
    ref = O.attend_batch(tab, P.q_bits(q), True, P.stack_codes(codes, cap), np.array([N], np.int32), Hkv)
    assert P.attn_error(got, ref).max() <= P.ATTN_TOL
    if N == 1:   # a single token: the output is its dequantized value
        kh, vh = O.reconstruct(tab, codes[0][0], 1)
        assert np.allclose(got[0, 0], vh[0], atol=2e-3 * np.abs(vh[0]).max())


def test_attend_many_heads_per_group_and_empty_sequence():
    d, bits = 128, 3
    ctx, tab = ctx_for(d, bits)
    B, Hkv, Hq, N = 3, 1, 20, 70       # 20 query heads: 3 groups of up to 8
    k, v = kv(B, Hkv, N, d, seed=4)
    codes = P.oracle_codes(tab, k, v)
    cap = 80
    cache = tq.Cache(P.pack_cache(tab, codes, cap, d, bits), B, Hkv, cap)
    q = qtensor(B, Hq, d, seed=3)
    seq = [70, 0, 31]
    got = run_attend(ctx, tab, cache, q, seq, 70, Hkv)
    ref = O.attend_batch(tab, P.q_bits(q), True, P.stack_codes(codes, cap), np.array(seq, np.int32), Hkv)
    assert np.all(got[1] == 0.0)
    assert P.attn_error(got, ref).max() <= P.ATTN_TOL


@pytest.mark.parametrize("d", [64, 128, 256])
def test_attend_one_unit_over_the_whole_grid(d):
    # One sequence, one kv head, one group of query heads, 188 tiles: the unit
    # is split over every CTA of the grid, so the reduce merges one partial per
    # CTA: more partials than its D threads take at once at d = 64 and 128.
    ctx, tab = ctx_for(d, 3)
    B, Hkv, Hq, N = 1, 1, 6, 3001
    cap = 3008
    k, v = kv(B, Hkv, N, d, seed=900 + d)
    codes = P.oracle_codes(tab, k, v)
    cache = tq.Cache(P.pack_cache(tab, codes, cap, d, 3), B, Hkv, cap)
    q = qtensor(B, Hq, d, seed=d)
    got = run_attend(ctx, tab, cache, q, [N], N, Hkv)
    ref = O.attend_batch(tab, P.q_bits(q), True, P.stack_codes(codes, cap), np.array([N], np.int32), Hkv)
    assert P.attn_error(got, ref).max() <= P.ATTN_TOL
    assert tq.tq_status(ctx) == 0


@pytest.mark.parametrize("d,bits,max_len", [(64, 4, 600), (128, 3, 600), (128, 2, 4096)])
def test_attend_many_ragged_sequences(d, bits, max_len):
    # Many sequences of mixed lengths (empty, one token, tile edges, a few
    # hundred): the split kernel's equal ranges of the laid-out tiles then
    # start and end inside units, span several units, and (max_len far above
    # every length) some CTAs get no tiles at all.
    ctx, tab = ctx_for(d, bits)
    B, Hkv, Hq = 40, 2, 12
    rng = np.random.default_rng(d + bits)
    top = min(max_len, 600)
    seq = [int(x) for x in rng.choice([0, 1, 15, 16, 17, 33, top], size=B)]
    seq[:8] = [int(x) for x in rng.integers(0, top + 1, size=8)]
    seq = [min(s, 40) for s in seq] if max_len > 600 else seq
    N = max(seq)
    cap = ((max(max_len, N) + 15) // 16) * 16
    k, v = kv(B, Hkv, N, d, seed=300 + d + bits)
    codes = P.oracle_codes(tab, k, v)
    cache = tq.Cache(P.pack_cache(tab, codes, cap, d, bits), B, Hkv, cap)
    q = qtensor(B, Hq, d, seed=5)
    got = run_attend(ctx, tab, cache, q, seq, max_len, Hkv)
    ref = O.attend_batch(tab, P.q_bits(q), True, P.stack_codes(codes, cap), np.array(seq, np.int32), Hkv)
    for b in range(B):
        if seq[b] == 0:
            assert np.all(got[b] == 0.0)
    assert P.attn_error(got, ref).max() <= P.ATTN_TOL
    assert tq.tq_status(ctx) == 0


def test_seq_len_out_of_range_is_clamped_and_flagged():
    d, bits = 64, 3
    ctx, tab = ctx_for(d, bits)
    k, v = kv(1, 1, 32, d, seed=8)
    codes = P.oracle_codes(tab, k, v)
    cache = tq.Cache(P.pack_cache(tab, codes, 32, d, bits), 1, 1, 32)
    q = qtensor(1, 2, d, seed=8)
    got = run_attend(ctx, tab, cache, q, [40], 20, 1)   # seq 40 > max_len 20
    assert tq.tq_status(ctx) & tq.TQ_STATUS_SEQ_LEN
    ref = O.attend_batch(tab, P.q_bits(q), True, P.stack_codes(codes, 32), np.array([20], np.int32), 1)
    assert P.attn_error(got, ref).max() <= P.ATTN_TOL


@pytest.mark.parametrize("d,bits", [(128, 3), (64, 4), (256, 2)])
def test_scores_match_oracle_logits(d, bits):
    ctx, tab = ctx_for(d, bits)
    B, Hkv, Hq, N = 2, 2, 6, 90
    k, v = kv(B, Hkv, N, d, seed=31, dist="outlier_channels")
    codes = P.oracle_codes(tab, k, v)
    cap = 96
    cache = tq.Cache(P.pack_cache(tab, codes, cap, d, bits), B, Hkv, cap)
    q = qtensor(B, Hq, d, seed=2)
    seq = [90, 50]
    s = tq.tq_scores(ctx, q.cuda(), cache, torch.tensor(seq, dtype=torch.int32).cuda(), 96)
    s = s.cpu().numpy().astype(np.float64)
    _, ref = O.attend_batch(tab, P.q_bits(q), True, P.stack_codes(codes, cap), np.array(seq, np.int32),
                            Hkv, want_logits=True)
    for b in range(B):
        assert np.all(np.isneginf(s[b, :, seq[b]:]))
        err = np.abs(s[b, :, :seq[b]] - ref[b, :, :seq[b]]).max()
        assert err <= P.ATTN_TOL * (np.abs(ref[b, :, :seq[b]]).max() + 1.0), err


def test_single_head_workload_full_size():
    # d=128, 3 bits, 8192 keys, 64 fp16 queries on one kv head: full size.
    w = inputs.WORKLOADS["single_head_d128_b3"]
    ctx, tab = ctx_for(w.d, w.bits)
    k, v = inputs.kv_pair(w, w.N)
    cache = P.quantize_on_gpu(ctx, k, v, capacity=w.N)
    codes = check_quantize(ctx, tab, k, v, cache)
    q = inputs.queries(w)
    got = run_attend(ctx, tab, cache, q, [w.N], w.N, 1)
    ref = O.attend_batch(tab, P.q_bits(q), False, P.stack_codes(codes, w.N),
                         np.array([w.N], np.int32), 1)
    assert P.attn_error(got, ref).max() <= P.ATTN_TOL
