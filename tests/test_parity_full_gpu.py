"""Full-size parity on sampled slices.

Each workload's layer is drawn at its real size on the GPU and quantized
there; the oracle recomputes sampled (batch, kv-head) streams from the same
fp16 inputs, copied to the host, and every token's codes, signs and norms are
compared. Attention then runs in the launch configuration the bench uses
(every sequence and head, the full context) after the sampled streams of the
cache are replaced by the oracle's packing of its own codes, so the GPU and
the oracle attend over the same codes; every query head reading a sampled
stream is compared.
"""
import numpy as np
import pytest
import torch

import kv_cache_vector_04_b200 as tq
from kv_cache_vector_04_b200 import inputs
from oracle import oracle as O
from tests import parity as P

pytestmark = pytest.mark.gpu


def _run_layer(w, samples, seq_fn=None, decode_step=False):
    """Quantize + attend one layer of workload `w` on the GPU, then check the
    sampled (b, kv head) streams against the oracle."""
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    ctx = tq.tq_init(w.d, w.bits, 1)
    tab = O.Tables(w.d, w.bits, 1)
    k, v = inputs.kv_pair(w, w.N, layer=0, device=dev)
    cache = tq.new_cache(ctx, w.B, w.Hkv, w.N + (16 if decode_step else 0))
    tq.tq_quantize(ctx, k, v, torch.zeros(w.B, dtype=torch.int32, device=dev), cache)
    assert tq.tq_status(ctx) == 0
    host = cache.data.cpu().numpy()
    lay = tq.tq_cache_layout(ctx)
    per_stream = (cache.capacity // 16) * lay["tile_bytes"]
    g = w.Hq // w.Hkv
    stats = P.QuantStats()
    oracle_streams = {}
    for (b, h) in samples:
        ora = O.quantize(tab, k[b, h].cpu().numpy(), v[b, h].cpu().numpy())
        sb = P.stream_bytes(host, lay["tile_bytes"], cache.capacity, w.Hkv, b, h, w.N)
        gpu = O.unpack_stream(w.d, w.bits, w.N, sb)
        P.compare_stream(tab, gpu, ora, w.N, stats)
        oracle_streams[(b, h)] = ora
        packed = torch.from_numpy(O.pack_stream(w.d, w.bits, ora)).to(dev)
        s0 = (b * w.Hkv + h) * per_stream
        cache.data[s0: s0 + packed.numel()].copy_(packed)
    stats.check()
    del k, v
    q = inputs.queries(w, device=dev)
    if decode_step:
        # the bench's step: tq_append_attend of one new token per sequence at
        # position N, captured in a CUDA graph and replayed
        nk, nv = inputs.kv_pair(w, 1, layer=10_000, device=dev)
        start = torch.full((w.B,), w.N, dtype=torch.int32, device=dev)
        seq = torch.full((w.B,), w.N + 1, dtype=torch.int32)
        ws = tq.new_workspace(ctx, w.B, w.Hq, w.Hkv, w.N + 1)
        outd = torch.empty((w.B, w.Hq, w.d), dtype=torch.float32, device=dev)
        seqd = seq.to(dev)
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            tq.tq_append_attend(ctx, q, nk, nv, start, cache, seqd, w.N + 1, out=outd, workspace=ws)
        torch.cuda.current_stream().wait_stream(side)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            tq.tq_append_attend(ctx, q, nk, nv, start, cache, seqd, w.N + 1, out=outd, workspace=ws)
        outd.zero_()
        graph.replay()
        torch.cuda.synchronize()
        out = outd.cpu().numpy().astype(np.float64)
        del graph
        assert tq.tq_status(ctx) == 0
        host = cache.data.cpu().numpy()
        for (b, h) in samples:
            new = O.quantize(tab, nk[b, h].cpu().numpy(), nv[b, h].cpu().numpy())
            sb = P.stream_bytes(host, lay["tile_bytes"], cache.capacity, w.Hkv, b, h, w.N + 1)
            gpu = O.unpack_stream(w.d, tab, w.N + 1, sb)
            P.compare_stream(tab, {kk: vv[w.N:] for kk, vv in gpu.items()}, new, 1, stats)
            ora = oracle_streams[(b, h)]
            oracle_streams[(b, h)] = {kk: np.concatenate([ora[kk], new[kk]]) for kk in ora}
        stats.check()
    else:
        seq = torch.full((w.B,), w.N, dtype=torch.int32) if seq_fn is None else seq_fn(w)
        out = tq.tq_attend(ctx, q, cache, seq.to(dev), w.N).cpu().numpy().astype(np.float64)
        assert tq.tq_status(ctx) == 0
    qbits_all = P.q_bits(q.cpu())
    for (b, h) in samples:
        ora = oracle_streams[(b, h)]
        n = int(seq[b])
        codes = {key: ora[key][None, None] for key in ("kidx", "ksign", "knorm", "rnorm", "vidx",
                                                      "vnorm")}
        qb = np.ascontiguousarray(qbits_all[b:b + 1, h * g:(h + 1) * g])
        ref = O.attend_batch(tab, qb, w.q_dtype == torch.bfloat16, codes,
                             np.array([n], np.int32), 1)
        err = P.attn_error(out[b:b + 1, h * g:(h + 1) * g], ref)
        assert err.max() <= P.ATTN_TOL, (b, h, err.max())
    return stats


def test_llama70b_shaped_layer_32k():
    # 16 sequences x 8 kv heads x 32768 tokens, K 3-bit + QJL, V 4-bit; 64 query heads
    w = inputs.WORKLOADS["llama3.3-70b_decode_32k"]
    _run_layer(w, samples=[(0, 0), (15, 7), (9, 3)])


def test_llama70b_shaped_decode_step_in_a_cuda_graph():
    # the benchmarked path: one tq_append_attend per layer, replayed from a graph
    w = inputs.WORKLOADS["llama3.3-70b_decode_32k"]
    _run_layer(w, samples=[(3, 1), (12, 6)], decode_step=True)


def test_qwen32b_shaped_layer_128k():
    # one sequence x 8 kv heads x 131072 tokens, 3 bits, 2% spiky tokens; 40 query heads
    w = inputs.WORKLOADS["qwen2.5-32b_prefill_decode_128k"]
    _run_layer(w, samples=[(0, 2)])


def test_qwen3b_shaped_layer_8k():
    # one sequence x 2 kv heads x 8192 tokens, 3 bits, outlier channels x15
    w = inputs.WORKLOADS["qwen2.5-3b_decode_8k"]
    _run_layer(w, samples=[(0, 0), (0, 1)])


@pytest.mark.parametrize("name", [w.name for w in inputs.sweep_workloads()])
def test_sweep_points(name):
    # every point of the d x bits x context sweep at its full size (batch 8,
    # 8 kv heads, 32 query heads), with unequal lengths across the batch; one
    # sampled stream per point
    w = {x.name: x for x in inputs.sweep_workloads()}[name]
    _run_layer(w, samples=[(7, 5)],
               seq_fn=lambda w: torch.tensor([w.N - 37 * i for i in range(w.B)], dtype=torch.int32))


def test_qwen32b_shaped_prefill_then_32_decode_steps():
    # The long-context workload as specified: bulk tq_quantize of all 131072
    # prefill tokens of one layer, then 32 decode steps, each one
    # tq_append_attend (append the step's token at position N + s, attend over
    # N + s + 1 tokens). On one sampled (batch, kv head) stream, every appended
    # token's codes and every step's output (its 5 query heads) are compared
    # with the oracle's, the oracle attending over its own codes of the prefix
    # and of the appended tokens.
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    w = inputs.WORKLOADS["qwen2.5-32b_prefill_decode_128k"]
    assert w.decode_steps == 32
    steps, (b, h) = w.decode_steps, (0, 6)
    ctx = tq.tq_init(w.d, w.bits, 1)
    tab = O.Tables(w.d, w.bits, 1)
    k, v = inputs.kv_pair(w, w.N, layer=0, device=dev)
    cap = w.N + steps
    cache = tq.new_cache(ctx, w.B, w.Hkv, cap)
    tq.tq_quantize(ctx, k, v, torch.zeros(w.B, dtype=torch.int32, device=dev), cache)
    assert tq.tq_status(ctx) == 0
    lay = tq.tq_cache_layout(ctx)
    per_stream = (cap // 16) * lay["tile_bytes"]
    stats = P.QuantStats()
    ora = O.quantize(tab, k[b, h].cpu().numpy(), v[b, h].cpu().numpy())
    host = cache.data.cpu().numpy()
    P.compare_stream(tab, O.unpack_stream(w.d, w.bits, w.N,
                                          P.stream_bytes(host, lay["tile_bytes"], cap, w.Hkv, b, h, w.N)),
                     ora, w.N, stats)
    # the sampled stream holds the oracle's packing of its own codes from here on
    s0 = (b * w.Hkv + h) * per_stream
    packed = torch.from_numpy(O.pack_stream(w.d, w.bits, ora)).to(dev)
    cache.data[s0: s0 + packed.numel()].copy_(packed)
    del k, v
    g = w.Hq // w.Hkv
    ws = tq.new_workspace(ctx, w.B, w.Hq, w.Hkv, cap)
    out = torch.empty((w.B, w.Hq, w.d), dtype=torch.float32, device=dev)
    for s in range(steps):
        n = w.N + s
        q = inputs.queries(w, layer=s, device=dev)
        nk, nv = inputs.kv_pair(w, 1, layer=10_000 + s, device=dev)
        start = torch.full((w.B,), n, dtype=torch.int32, device=dev)
        seq = torch.full((w.B,), n + 1, dtype=torch.int32, device=dev)
        tq.tq_append_attend(ctx, q, nk, nv, start, cache, seq, n + 1, out=out, workspace=ws)
        torch.cuda.synchronize()
        assert tq.tq_status(ctx) == 0
        new = O.quantize(tab, nk[b, h].cpu().numpy(), nv[b, h].cpu().numpy())
        tb0 = s0 + (n // 16) * lay["tile_bytes"]   # the tile holding token n
        gpu = O.unpack_stream(w.d, tab, 16, cache.data[tb0: tb0 + lay["tile_bytes"]].cpu().numpy())
        P.compare_stream(tab, {kk: vv[n % 16: n % 16 + 1] for kk, vv in gpu.items()}, new, 1, stats)
        ora = {kk: np.concatenate([ora[kk], new[kk]]) for kk in ora}
        codes = {key: ora[key][None, None] for key in ("kidx", "ksign", "knorm", "rnorm", "vidx", "vnorm")}
        qb = np.ascontiguousarray(P.q_bits(q.cpu())[b:b + 1, h * g:(h + 1) * g])
        ref = O.attend_batch(tab, qb, True, codes, np.array([n + 1], np.int32), 1)
        err = P.attn_error(out[b:b + 1, h * g:(h + 1) * g].cpu().numpy().astype(np.float64), ref)
        assert err.max() <= P.ATTN_TOL, (s, err.max())
    stats.check()
