"""GPU parity of the MSE-only key formats ("nc": no QJL sketch) and the
asymmetric 3/4-bit format, against the oracle with the same format.

The formats are those of the method table in the vLLM section of
turboquant-kvquant-vllm-benchmark ("vLLM 工程師的實測"): 2/3/4-bit "nc" and
k3v4-nc, read as keys without the QJL correction. Each is checked the way
TurboQuant itself is:
* codes and norms against the oracle's;
* packed bytes against the oracle packer;
* attention and logits over an oracle-packed cache;
* the fused one-token decode step.
"""
import numpy as np
import pytest
import torch

import kv_cache_vector_04_b200 as tq
from oracle import oracle as O
from tests import parity as P
from tests.test_append_attend_gpu import _run as run_append
from tests.test_parity_gpu import check_quantize, ctx_for, kv, qtensor

pytestmark = pytest.mark.gpu

NC = [(2, 2, 0), (3, 3, 0), (4, 4, 0), (3, 4, 0)]
DF = [(d, f) for d in (64, 128, 256) for f in NC]


def test_layout_of_each_format():
    for d, f in DF:
        ctx, _ = ctx_for(d, f[1], fmt=f)
        lay = tq.tq_cache_layout(ctx)
        assert (lay["kbits"], lay["vbits"], lay["qjl"]) == f
        assert lay["tile_bytes"] == O.tile_bytes(d, f)
        assert lay["k_bytes_per_token"] == f[0] * d // 8 + 2
        assert lay["v_bytes_per_token"] == f[1] * d // 8 + 2


@pytest.mark.parametrize("d,fmt", DF)
def test_quantize_matches_oracle(d, fmt):
    ctx, tab = ctx_for(d, fmt[1], fmt=fmt)
    stats = P.QuantStats()
    for T, dist in ((131, "lognormal_norm"), (33, "outlier_channels")):
        k, v = kv(2, 2, T, d, seed=d + 10 * fmt[0] + fmt[1] + T, dist=dist)
        cache = P.quantize_on_gpu(ctx, k, v, capacity=T + 24)
        codes = check_quantize(ctx, tab, k, v, cache, stats=stats)
        for b in range(2):
            for h in range(2):
                assert not codes[b][h]["ksign"].any() and not codes[b][h]["rnorm"].any()
    stats.check()
    assert tq.tq_status(ctx) == 0


@pytest.mark.parametrize("d,fmt", [(64, (3, 4, 0)), (128, (4, 4, 0)), (256, (2, 2, 0))])
def test_packed_bytes_equal_oracle_packer(d, fmt):
    ctx, tab = ctx_for(d, fmt[1], fmt=fmt)
    k, v = kv(1, 2, 48, d, seed=3)
    cache = P.quantize_on_gpu(ctx, k, v, capacity=48)
    codes = P.oracle_codes(tab, k, v)
    host = cache.data.cpu().numpy()
    lay = tq.tq_cache_layout(ctx)
    for h in range(2):
        if (codes[0][h]["kydist"] < P.BAND).any() or (codes[0][h]["vydist"] < P.BAND).any():
            continue
        ref = O.pack_stream(d, tab, codes[0][h])
        got = P.stream_bytes(host, lay["tile_bytes"], 48, 2, 0, h, 48)
        assert np.array_equal(got, ref)


@pytest.mark.parametrize("d,fmt", DF)
def test_attend_on_oracle_packed_cache(d, fmt):
    ctx, tab = ctx_for(d, fmt[1], fmt=fmt)
    B, Hkv, Hq, N, cap = 2, 2, 8, 203, 208
    k, v = kv(B, Hkv, N, d, seed=50 + d, dist="outlier_channels")
    codes = P.oracle_codes(tab, k, v)
    cache = tq.Cache(P.pack_cache(tab, codes, cap, d, fmt[1]), B, Hkv, cap)
    seq = [203, 90]
    q = qtensor(B, Hq, d, seed=fmt[0] + fmt[1])
    got = tq.tq_attend(ctx, q.cuda(), cache, torch.tensor(seq, dtype=torch.int32).cuda(), N)
    torch.cuda.synchronize()
    ref = O.attend_batch(tab, P.q_bits(q), True, P.stack_codes(codes, cap), np.array(seq, np.int32),
                         Hkv)
    err = P.attn_error(got.cpu().numpy().astype(np.float64), ref)
    assert err.max() <= P.ATTN_TOL, err.max()
    assert tq.tq_status(ctx) == 0


@pytest.mark.parametrize("d,fmt", [(128, (3, 3, 0)), (64, (3, 4, 0)), (256, (4, 4, 0))])
def test_scores_match_oracle_logits(d, fmt):
    ctx, tab = ctx_for(d, fmt[1], fmt=fmt)
    B, Hkv, Hq, N, cap = 1, 2, 4, 77, 80
    k, v = kv(B, Hkv, N, d, seed=9)
    codes = P.oracle_codes(tab, k, v)
    cache = tq.Cache(P.pack_cache(tab, codes, cap, d, fmt[1]), B, Hkv, cap)
    q = qtensor(B, Hq, d, seed=2)
    got = tq.tq_scores(ctx, q.cuda(), cache, torch.tensor([N], dtype=torch.int32).cuda(), N)
    torch.cuda.synchronize()
    _, lg = O.attend_batch(tab, P.q_bits(q), True, P.stack_codes(codes, cap),
                           np.array([N], np.int32), Hkv, want_logits=True)
    g = got.cpu().numpy().astype(np.float64)
    ref = lg[:, :, :N]
    assert np.abs(g - ref).max() <= P.ATTN_TOL * (np.abs(ref).max() + 1.0)


@pytest.mark.parametrize("d,fmt", [(64, (2, 2, 0)), (128, (3, 4, 0)), (256, (3, 3, 0))])
def test_append_one_token_then_attend(d, fmt):
    run_append(d, fmt[1], 1, [32, 37, 47], seed=d + fmt[0], fmt=fmt)


# ---------------------------------------------------------------- exact-marginal codebooks

BETA = [(64, (1, 2, 1)), (128, (3, 4, 1)), (128, (3, 3, 0)), (256, (2, 3, 1))]


@pytest.mark.parametrize("d,fmt", BETA)
def test_beta_codebook_tables_quantize_and_attend(d, fmt):
    # The exact Beta-marginal codebooks ride on the same kernels: the device
    # tables hold the oracle's codebooks, quantization and attention match.
    ctx, tab = ctx_for(d, fmt[1], fmt=fmt, kind="beta")
    t = tq.tq_get_tables(ctx)
    assert np.array_equal(t["centroids_k"], tab.cK) and np.array_equal(t["centroids_v"], tab.cV)
    assert np.array_equal(t["bounds_k"], tab.tK) and np.array_equal(t["bounds_v"], tab.tV)
    stats = P.QuantStats()
    k, v = kv(2, 2, 97, d, seed=d + fmt[1], dist="spiky_tokens")
    cache = P.quantize_on_gpu(ctx, k, v, capacity=112)
    codes = check_quantize(ctx, tab, k, v, cache, stats=stats)
    stats.check()
    q = qtensor(2, 8, d, seed=4)
    seq = [97, 40]
    got = tq.tq_attend(ctx, q.cuda(), cache, torch.tensor(seq, dtype=torch.int32).cuda(), 97)
    torch.cuda.synchronize()
    ref = O.attend_batch(tab, P.q_bits(q), True, P.stack_codes(codes, 112), np.array(seq, np.int32), 2)
    assert P.attn_error(got.cpu().numpy().astype(np.float64), ref).max() <= P.ATTN_TOL
    assert tq.tq_status(ctx) == 0


# ---------------------------------------------------------------- k8v4: 8-bit TurboQuant keys

# "TQ k8v4" of the same vLLM table, read as TurboQuant keys at 8 bits (7-bit
# Lloyd-Max cells plus the 1-bit QJL sketch) with 4-bit values: (7, 4, 1). The
# decoder takes the 7-bit key levels code by code, each as fp16 hi + lo parts.
K8V4 = (7, 4, 1)


@pytest.mark.parametrize("d", [64, 128, 256])
def test_k8v4_layout_and_quantize(d):
    # check_quantize unpacks the device's bytes with the oracle's packer layout
    # and compares every code with the oracle's: the layout and the decisions
    ctx, tab = ctx_for(d, 4, fmt=K8V4)
    lay = tq.tq_cache_layout(ctx)
    assert (lay["kbits"], lay["vbits"], lay["qjl"]) == K8V4
    assert lay["tile_bytes"] == O.tile_bytes(d, K8V4)
    assert lay["k_bytes_per_token"] == d + 4 and lay["v_bytes_per_token"] == d // 2 + 2
    stats = P.QuantStats()
    for T, dist in ((77, "lognormal_norm"), (40, "outlier_channels"), (33, "spiky_tokens")):
        k, v = kv(2, 2, T, d, seed=d + T, dist=dist)
        cache = P.quantize_on_gpu(ctx, k, v, capacity=T + 19)
        check_quantize(ctx, tab, k, v, cache, stats=stats)
    stats.check()
    assert tq.tq_status(ctx) == 0


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("dist", ["lognormal_norm", "outlier_channels", "spiky_tokens"])
def test_k8v4_attend_on_oracle_packed_cache(d, dist):
    ctx, tab = ctx_for(d, 4, fmt=K8V4)
    B, Hkv, Hq, N, cap = 2, 2, 8, 203, 208
    k, v = kv(B, Hkv, N, d, seed=70 + d, dist=dist)
    codes = P.oracle_codes(tab, k, v)
    cache = tq.Cache(P.pack_cache(tab, codes, cap, d, 4), B, Hkv, cap)
    seq = [203, 90]
    for qs in (1.0, 3.0):
        q = (qtensor(B, Hq, d, seed=8).float() * qs).to(torch.bfloat16)
        got = tq.tq_attend(ctx, q.cuda(), cache, torch.tensor(seq, dtype=torch.int32).cuda(), N)
        torch.cuda.synchronize()
        ref = O.attend_batch(tab, P.q_bits(q), True, P.stack_codes(codes, cap), np.array(seq, np.int32),
                             Hkv)
        err = P.attn_error(got.cpu().numpy().astype(np.float64), ref)
        assert err.max() <= P.ATTN_TOL, (qs, err.max())
    assert tq.tq_status(ctx) == 0


def test_k8v4_scores_match_oracle_logits():
    d = 128
    ctx, tab = ctx_for(d, 4, fmt=K8V4)
    B, Hkv, Hq, N, cap = 1, 2, 4, 77, 80
    k, v = kv(B, Hkv, N, d, seed=12, dist="outlier_channels")
    codes = P.oracle_codes(tab, k, v)
    cache = tq.Cache(P.pack_cache(tab, codes, cap, d, 4), B, Hkv, cap)
    q = qtensor(B, Hq, d, seed=3)
    got = tq.tq_scores(ctx, q.cuda(), cache, torch.tensor([N], dtype=torch.int32).cuda(), N)
    torch.cuda.synchronize()
    _, lg = O.attend_batch(tab, P.q_bits(q), True, P.stack_codes(codes, cap),
                           np.array([N], np.int32), Hkv, want_logits=True)
    g = got.cpu().numpy().astype(np.float64)
    ref = lg[:, :, :N]
    assert np.abs(g - ref).max() <= P.ATTN_TOL * (np.abs(ref).max() + 1.0)


@pytest.mark.parametrize("d", [128, 256])
def test_k8v4_append_one_token_then_attend(d):
    run_append(d, 4, 1, [32, 37, 47], seed=d + 7, fmt=K8V4)
