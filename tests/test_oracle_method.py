"""Pins for the oracle's encoder, QJL estimator, packed format and attention.

Checks against brute force, statistics the method guarantees, textbook
softmax attention (torch, fp64) over reconstructed keys and values, and the
byte counts printed on the pages.
"""
import math

import numpy as np
import pytest
import torch

from oracle import oracle as O


# ---------------------------------------------------------------- encoder

@pytest.mark.parametrize("B", [1, 2, 3, 4])
@pytest.mark.parametrize("d", [4, 8, 128])
def test_encode_is_nearest_centroid(B, d):
    c, t = O.codebook(B, d)
    lim = 4.0 / math.sqrt(d)
    ys = np.linspace(-lim, lim, 4001)
    for y in ys:
        dist = np.abs(y - c.astype(np.float64))
        j = int(np.argmin(dist))
        if np.sort(dist)[1] - dist[j] < 1e-12:   # an exact tie: either is nearest
            continue
        assert O.encode(y, t) == j
    # ties go to the lower cell (strict '>')
    for j, tb in enumerate(t):
        assert O.encode(float(tb), t) == j


def test_quantize_keys_brute_force_small():
    # d = 8: recompute every step by brute force from the definition.
    d, bits = 8, 3
    tab = O.Tables(d, bits, seed=7)
    rng = np.random.default_rng(1)
    x = (rng.standard_normal((64, d)) * 3).astype(np.float16)
    x[0] = 0  # zero vector
    out = O.quantize(tab, x, x)
    H = np.array([[(-1) ** bin(i & j).count("1") for j in range(d)] for i in range(d)], float)
    for n in range(x.shape[0]):
        xv = x[n].astype(np.float64)
        nrm = np.linalg.norm(xv)
        u = xv / nrm if nrm > 0 else np.zeros(d)
        y = H @ (tab.D * u) / math.sqrt(d)
        kid = np.array([np.argmin(np.abs(yi - tab.cK.astype(np.float64))) for yi in y])
        vid = np.array([np.argmin(np.abs(yi - tab.cV.astype(np.float64))) for yi in y])
        assert np.array_equal(out["kidx"][n], kid)
        assert np.array_equal(out["vidx"][n], vid)
        r = y - tab.cK[kid].astype(np.float64)
        z = tab.S @ r
        assert np.array_equal(out["ksign"][n], (z >= 0).astype(np.uint8))
        assert out["knorm"][n] == np.float16(nrm).view(np.uint16)
        assert out["rnorm"][n] == np.float16(np.linalg.norm(r)).view(np.uint16)


@pytest.mark.parametrize("fmt", [(3, 3, 0), (2, 4, 0)])
def test_quantize_keys_mse_only_brute_force_small(fmt):
    # the MSE-only key format: nearest B_K-bit cell, |k| stored, no sketch
    d = 8
    tab = O.Tables(d, 3, seed=4, fmt=fmt)
    rng = np.random.default_rng(2)
    x = (rng.standard_normal((40, d)) * 2).astype(np.float16)
    out = O.quantize(tab, x, x)
    H = np.array([[(-1) ** bin(i & j).count("1") for j in range(d)] for i in range(d)], float)
    for n in range(x.shape[0]):
        xv = x[n].astype(np.float64)
        y = H @ (tab.D * xv) / math.sqrt(d) / np.linalg.norm(xv)
        kid = np.array([np.argmin(np.abs(yi - tab.cK.astype(np.float64))) for yi in y])
        vid = np.array([np.argmin(np.abs(yi - tab.cV.astype(np.float64))) for yi in y])
        assert np.array_equal(out["kidx"][n], kid)
        assert np.array_equal(out["vidx"][n], vid)
        assert kid.max() < (1 << fmt[0]) and vid.max() < (1 << fmt[1])
        assert not out["ksign"][n].any() and out["rnorm"][n] == 0
        assert out["knorm"][n] == np.float16(np.linalg.norm(xv)).view(np.uint16)


def test_exact_cancellation_meets_the_tie_rule():
    # D o x = (1, 1, 0, ...) gives Walsh-Hadamard sums 1 + (-1)^(i&1): every
    # odd coordinate of the rotated vector is exactly 0, which the strict '>'
    # rule puts in the cell below the middle boundary (which is exactly 0).
    d, bits = 64, 3
    tab = O.Tables(d, bits, seed=3)
    x = np.zeros((1, d), np.float16)
    x[0, 0] = tab.D[0]
    x[0, 1] = tab.D[1]
    out = O.quantize(tab, x, x)
    L_k, L_v = 1 << tab.BK, 1 << tab.BV
    assert np.all(out["kidx"][0, 1::2] == L_k // 2 - 1)
    assert np.all(out["vidx"][0, 1::2] == L_v // 2 - 1)
    assert np.all(out["kydist"][0, 1::2] == 0.0)


def test_norm_saturation_flag():
    tab = O.Tables(64, 3, seed=1)
    x = np.full((2, 64), 60000.0, dtype=np.float16)
    x[1] = 1.0
    out = O.quantize(tab, x, x)
    assert out["ksat"][0] == 1 and out["vsat"][0] == 1
    assert out["knorm"][0] == 0x7BFF and out["vnorm"][0] == 0x7BFF
    assert out["ksat"][1] == 0


# ---------------------------------------------------------------- QJL estimator

@pytest.mark.slow
@pytest.mark.parametrize("bits", [2, 3])
def test_qjl_unbiased_and_mse_only_shrinks(bits):
    # 1e5 fresh (rotation, S) draws for a fixed pair with cos = 0.5. The
    # QJL-corrected estimate is unbiased (within 3 sigma); the MSE-only
    # estimate at the same bit budget is biased towards 0 by about D_b <q,k>
    # (a positive bias for <q,k> > 0, as the pages report).
    d, n = 64, 100_000
    rng = np.random.default_rng(bits)
    a = rng.standard_normal(d)
    a /= np.linalg.norm(a)
    b = rng.standard_normal(d)
    b -= (b @ a) * a
    b /= np.linalg.norm(b)
    q = 3.0 * a
    k = 2.0 * (0.5 * a + math.sqrt(0.75) * b)
    ip = float(q @ k)
    em, eq = O.ip_trials(d, bits, n, 1000 * bits, q, k)
    bias_q = ip - eq.mean()
    se_q = eq.std(ddof=1) / math.sqrt(n)
    assert abs(bias_q) < 3.0 * se_q, (bias_q, se_q)
    bias_m = ip - em.mean()
    se_m = em.std(ddof=1) / math.sqrt(n)
    assert bias_m > 5.0 * se_m
    c, _, _ = O.lloyd_max_unit(bits)
    Db = O.quantizer_mse_unit(bits, c)
    assert abs(bias_m / ip - Db) < 0.35 * Db, (bias_m / ip, Db)


def test_qjl_unbiased_quick():
    # the same property at a CPU-cheap size (runs without -m slow filtering)
    d, n = 64, 20_000
    q = np.zeros(d)
    q[:2] = [2.0, 1.0]
    k = np.zeros(d)
    k[:2] = [1.0, 1.5]
    em, eq = O.ip_trials(d, 3, n, 77, q, k)
    ip = float(q @ k)
    assert abs(ip - eq.mean()) < 3.0 * eq.std(ddof=1) / math.sqrt(n)
    assert ip - em.mean() > 0


# ---------------------------------------------------------------- packed format

@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("b", [2, 3, 4])
def test_pack_round_trip(d, b):
    rng = np.random.default_rng(d * 10 + b)
    for N in (1, 15, 16, 17, 48):
        codes = dict(
            kidx=rng.integers(0, 1 << (b - 1), (N, d), dtype=np.uint8),
            ksign=rng.integers(0, 2, (N, d), dtype=np.uint8),
            knorm=rng.integers(0, 0x7BFF, N, dtype=np.uint16),
            rnorm=rng.integers(0, 0x7BFF, N, dtype=np.uint16),
            vidx=rng.integers(0, 1 << b, (N, d), dtype=np.uint8),
            vnorm=rng.integers(0, 0x7BFF, N, dtype=np.uint16))
        tiles = O.pack_stream(d, b, codes)
        assert tiles.size == ((N + 15) // 16) * 16 * (b * d // 4 + 6)
        back = O.unpack_stream(d, b, N, tiles)
        for key in codes:
            assert np.array_equal(back[key], codes[key]), (key, N)
        # every code bit of a full tile is used exactly once: random codes fill it
        if N % 16 == 0:
            code_bytes = 4 * b * d
            for tl in range(N // 16):
                blk = tiles[tl * tiles.size // (N // 16):][:code_bytes]
                assert np.unpackbits(blk).mean() > 0.4


FORMATS = [(1, 2, 1), (2, 3, 1), (3, 4, 1), (7, 4, 1), (2, 2, 0), (3, 3, 0), (4, 4, 0), (3, 4, 0)]


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("fmt", FORMATS)
def test_pack_round_trip_formats(d, fmt):
    kb, vb, qjl = fmt
    rng = np.random.default_rng(d + 7 * kb + vb)
    for N in (1, 17, 32):
        codes = dict(
            kidx=rng.integers(0, 1 << kb, (N, d), dtype=np.uint8),
            ksign=rng.integers(0, 2, (N, d), dtype=np.uint8) * qjl,
            knorm=rng.integers(0, 0x7BFF, N, dtype=np.uint16),
            rnorm=rng.integers(0, 0x7BFF, N, dtype=np.uint16) * qjl,
            vidx=rng.integers(0, 1 << vb, (N, d), dtype=np.uint8),
            vnorm=rng.integers(0, 0x7BFF, N, dtype=np.uint16))
        tiles = O.pack_stream(d, fmt, codes)
        # per head-token: key cells + sketch + |k| (+ rho), value cells + |v|
        per_token = (kb + qjl) * d / 8 + 2 + 2 * qjl + vb * d / 8 + 2
        assert tiles.size == ((N + 15) // 16) * 16 * per_token
        back = O.unpack_stream(d, fmt, N, tiles)
        for key in codes:
            assert np.array_equal(back[key], codes[key]), (key, N)


@pytest.mark.parametrize("fmt", FORMATS)
def test_pack_fields_tile_the_tile(fmt):
    # Packing one field at a time: every field sets exactly its own bits, no
    # two fields share a bit, and together they cover the whole tile.
    d = 64
    kb, vb, qjl = fmt
    N = 16
    zero = dict(kidx=np.zeros((N, d), np.uint8), ksign=np.zeros((N, d), np.uint8),
                knorm=np.zeros(N, np.uint16), rnorm=np.zeros(N, np.uint16),
                vidx=np.zeros((N, d), np.uint8), vnorm=np.zeros(N, np.uint16))
    TB = O.tile_bytes(d, fmt)
    owner = np.full(TB * 8, -1)
    fields = [("kidx", (1 << kb) - 1, kb), ("vidx", (1 << vb) - 1, vb)]
    if qjl:
        fields.append(("ksign", 1, 1))
    fid = 0
    for name, val, width in fields:
        for n in range(N):
            for i in range(d):
                c = {k: v.copy() for k, v in zero.items()}
                c[name][n, i] = val
                bits = np.flatnonzero(np.unpackbits(O.pack_stream(d, fmt, c), bitorder="little"))
                assert bits.size == width
                assert np.all(owner[bits] == -1)
                owner[bits] = fid
                fid += 1
    for name in ("knorm", "vnorm") + (("rnorm",) if qjl else ()):
        for n in range(N):
            c = {k: v.copy() for k, v in zero.items()}
            c[name][n] = 0xFFFF
            bits = np.flatnonzero(np.unpackbits(O.pack_stream(d, fmt, c), bitorder="little"))
            assert bits.size == 16 and np.all(owner[bits] == -1)
            owner[bits] = fid
            fid += 1
    assert np.all(owner >= 0)


@pytest.mark.parametrize("d", [64, 128])
def test_pack_key_sign_bytes_of_3bit_keys(d):
    # Format (3, 4, 1) keeps each key pair with two sign bits in one byte of a
    # lane string: every key code lies in bits 0..5 of a byte, every sign in
    # bit 6 or 7 of a byte of the same region, and the two signs of a sign
    # pair sit 16 bits apart in one 32-bit word (a decoder's single shift).
    fmt, N = (3, 4, 1), 16
    zero = dict(kidx=np.zeros((N, d), np.uint8), ksign=np.zeros((N, d), np.uint8),
                knorm=np.zeros(N, np.uint16), rnorm=np.zeros(N, np.uint16),
                vidx=np.zeros((N, d), np.uint8), vnorm=np.zeros(N, np.uint16))
    key_region = 2 * 4 * d                 # bytes of the key+sign words of a tile (of 2*W*d)
    C = 16                                 # chunk bytes: a lane string is W*d/16 = d/2 bytes

    def lane_bit(byte_in_tile, bit):
        chunk, lane, off = byte_in_tile // (32 * C), (byte_in_tile // C) % 32, byte_in_tile % C
        return lane, (chunk * C + off) * 8 + bit

    for n in (0, 5, 8, 15):
        for i in range(0, d, 3):
            c = {k: v.copy() for k, v in zero.items()}
            c["kidx"][n, i] = 7
            bits = np.flatnonzero(np.unpackbits(O.pack_stream(d, fmt, c), bitorder="little"))
            assert bits.size == 3 and len({b // 8 for b in bits}) == 1
            assert all(b % 8 <= 5 for b in bits) and bits[0] // 8 < key_region
            c = {k: v.copy() for k, v in zero.items()}
            c["ksign"][n, i] = 1
            sb = np.flatnonzero(np.unpackbits(O.pack_stream(d, fmt, c), bitorder="little"))
            assert sb.size == 1 and sb[0] % 8 in (6, 7) and sb[0] // 8 < key_region
            # its partner (the neighbouring coordinate of the pair) is 16 bits away
            j = i ^ 1
            c["ksign"][n, i] = 0
            c["ksign"][n, j] = 1
            sj = np.flatnonzero(np.unpackbits(O.pack_stream(d, fmt, c), bitorder="little"))[0]
            li, bi = lane_bit(sb[0] // 8, sb[0] % 8)
            lj, bj = lane_bit(sj // 8, sj % 8)
            assert li == lj and abs(bi - bj) == 16 and bi // 32 == bj // 32


def test_pack_sizes_match_pages(golden):
    vals = {r[0]: float(r[1]) for r in golden("pages_numbers.txt")}
    d = 128
    # 8192 keys, 3 bits: fp16 2048 KB; codes (2-bit indices + 1 sign bit) 384 KB
    assert 8192 * d * 2 / 1024 == vals["keys_8192_fp16_kb"]
    key_code_bytes = 8192 * (3 * d // 8)
    assert key_code_bytes / 1024 == vals["keys_8192_tq3_kb"]
    # the tile stores exactly b*d/4 code bytes + 6 norm bytes per token (K + V)
    for b in (2, 3, 4):
        per_token = O.tile_bytes(d, b) / 16
        assert per_token == b * d / 4 + 6
        ratio = (2 * d * 2) / per_token
        assert round(ratio, 1) == vals["ratio_b%d" % b]
    # 36 layers x 2 kv heads x 8192 tokens at 3 bits: the pages' 289 MB -> 57.6 MB
    tq3 = 36 * 2 * 8192 * O.tile_bytes(d, 3) / 16
    fp16 = 36 * 2 * 8192 * d * 2 * 2
    assert abs(vals["kv_8k_fp16_mb"] * tq3 / fp16 - vals["kv_8k_tq3_mb"]) < 0.05


# ---------------------------------------------------------------- attention

def _random_codes(tab, N, seed, kscale=1.0):
    rng = np.random.default_rng(seed)
    k = (rng.standard_normal((N, tab.d)) * kscale).astype(np.float16)
    v = rng.standard_normal((N, tab.d)).astype(np.float16)
    return O.quantize(tab, k, v)


@pytest.mark.parametrize("d,bits,fmt", [(64, 2, None), (128, 3, None), (256, 4, None),
                                        (128, 3, (3, 3, 0)), (64, 4, (3, 4, 0)), (128, 4, (7, 4, 1))])
def test_attention_equals_sdpa_over_reconstructed(d, bits, fmt):
    # with fmt (B_K, B_V, 0) the keys are the MSE-only reconstructions
    tab = O.Tables(d, bits, seed=5, fmt=fmt)
    N = 77
    codes = _random_codes(tab, N, seed=d + bits, kscale=2.0)
    kh, vh = O.reconstruct(tab, codes, N)
    rng = np.random.default_rng(3)
    for q_is_bf16 in (True, False):
        qf = rng.standard_normal(d)
        if q_is_bf16:
            qt = torch.tensor(qf, dtype=torch.bfloat16)
            qbits = qt.view(torch.int16).numpy().view(np.uint16)
        else:
            qt = torch.tensor(qf, dtype=torch.float16)
            qbits = qt.numpy().view(np.uint16)
        o, logits = O.attend_head(tab, qbits, q_is_bf16, codes, N)
        Q = qt.to(torch.float64)[None, None, None, :]
        K = torch.from_numpy(kh)[None, None]
        V = torch.from_numpy(vh)[None, None]
        ref = torch.nn.functional.scaled_dot_product_attention(Q, K, V)[0, 0, 0].numpy()
        assert np.allclose(o, ref, atol=1e-12, rtol=1e-10)
        ref_logits = (kh @ qt.to(torch.float64).numpy()) / math.sqrt(d)
        assert np.allclose(logits, ref_logits, atol=1e-12, rtol=1e-10)


def test_attention_special_cases():
    d, bits = 128, 3
    tab = O.Tables(d, bits, seed=9)
    codes = _random_codes(tab, 8, seed=1)
    kh, vh = O.reconstruct(tab, codes, 8)
    q = torch.randn(d, generator=torch.Generator().manual_seed(0)).to(torch.bfloat16)
    qbits = q.view(torch.int16).numpy().view(np.uint16)
    # N = 1: the output is the single reconstructed value
    o, _ = O.attend_head(tab, qbits, True, codes, 1)
    assert np.allclose(o, vh[0], atol=1e-13)
    # N = 0: defined as zero
    o0, _ = O.attend_head(tab, qbits, True, codes, 0)
    assert np.all(o0 == 0)
    # identical keys: uniform weights, the mean of the values
    same = {kk: vv.copy() for kk, vv in codes.items()}
    for kk in ("kidx", "ksign", "knorm", "rnorm"):
        same[kk][:] = same[kk][0]
    o, lg = O.attend_head(tab, qbits, True, same, 8)
    assert np.allclose(lg, lg[0])
    assert np.allclose(o, vh.mean(axis=0), atol=1e-13)


def test_attend_batch_matches_per_head():
    d, bits, B, Hq, Hkv, cap = 64, 3, 2, 4, 2, 40
    tab = O.Tables(d, bits, seed=2)
    rng = np.random.default_rng(0)
    streams = [_random_codes(tab, cap, seed=s) for s in range(B * Hkv)]
    codes = {k: np.stack([s[k] for s in streams]).reshape((B, Hkv) + streams[0][k].shape)
             for k in ("kidx", "ksign", "knorm", "rnorm", "vidx", "vnorm")}
    q = torch.from_numpy(rng.standard_normal((B, Hq, d))).to(torch.bfloat16)
    qbits = q.view(torch.int16).numpy().view(np.uint16)
    seq = np.array([40, 23], np.int32)
    out, lg = O.attend_batch(tab, qbits, True, codes, seq, Hkv, want_logits=True)
    for b in range(B):
        for h in range(Hq):
            s = streams[b * Hkv + h // (Hq // Hkv)]
            o, l1 = O.attend_head(tab, qbits[b, h], True, s, int(seq[b]))
            assert np.array_equal(out[b, h], o)
            assert np.array_equal(lg[b, h, :seq[b]], l1)


@pytest.mark.parametrize("d", [64, 128])
def test_pack_value_sign_bytes_of_3bit_values(d):
    # Format (2, 3, 1) (TurboQuant at 3 bits) keeps each value pair with two
    # sign bits in one byte of the region after the key codes: every value code
    # lies in bits 0..5 of a byte there, every sign in bit 6 or 7 of a byte
    # there, the two signs of a sign pair sit 16 bits apart in one 32-bit word,
    # and the key codes keep the first 2*d/2 bits of each lane string.
    fmt, N = (2, 3, 1), 16
    zero = dict(kidx=np.zeros((N, d), np.uint8), ksign=np.zeros((N, d), np.uint8),
                knorm=np.zeros(N, np.uint16), rnorm=np.zeros(N, np.uint16),
                vidx=np.zeros((N, d), np.uint8), vnorm=np.zeros(N, np.uint16))
    C = 16 if (6 * d // 16) % 16 == 0 else 8   # chunk bytes of a lane string of 6d/16 bytes
    key_bytes = 2 * d // 2 // 8                # key codes: the first kb*d/2 bits of a lane string

    def lane_pos(bit_in_tile):
        byte = bit_in_tile // 8
        chunk, lane, off = byte // (32 * C), (byte // C) % 32, byte % C
        return lane, (chunk * C + off) * 8 + bit_in_tile % 8

    for n in (0, 5, 8, 15):
        for i in range(0, d, 3):
            c = {k: v.copy() for k, v in zero.items()}
            c["vidx"][n, i] = 7
            bits = np.flatnonzero(np.unpackbits(O.pack_stream(d, fmt, c), bitorder="little"))
            assert bits.size == 3 and len({b // 8 for b in bits}) == 1
            lane, pos = lane_pos(bits[0])
            assert all(lane_pos(b)[1] % 8 <= 5 for b in bits) and pos // 8 >= key_bytes
            c = {k: v.copy() for k, v in zero.items()}
            c["kidx"][n, i] = 3
            kbits = np.flatnonzero(np.unpackbits(O.pack_stream(d, fmt, c), bitorder="little"))
            assert kbits.size == 2 and all(lane_pos(b)[1] // 8 < key_bytes for b in kbits)
            c = {k: v.copy() for k, v in zero.items()}
            c["ksign"][n, i] = 1
            sb = np.flatnonzero(np.unpackbits(O.pack_stream(d, fmt, c), bitorder="little"))
            li, bi = lane_pos(sb[0])
            assert sb.size == 1 and bi % 8 in (6, 7) and bi // 8 >= key_bytes
            c["ksign"][n, i] = 0
            c["ksign"][n, i ^ 1] = 1
            lj, bj = lane_pos(np.flatnonzero(np.unpackbits(O.pack_stream(d, fmt, c), bitorder="little"))[0])
            assert li == lj and abs(bi - bj) == 16 and bi // 32 == bj // 32
