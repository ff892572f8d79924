"""Pins for the oracle's scalar conversions, generator, rotation and codebook.

Each test checks the oracle against something other than itself: published
SplitMix64 outputs, numpy/torch dtype conversions, scipy's Hadamard matrix and
numerical integration, the textbook Gaussian Lloyd–Max table, closed forms,
and the distortion values printed on the pages.
"""
import math

import numpy as np
import pytest
import scipy.integrate
import scipy.linalg
import scipy.stats
import torch

from oracle import oracle as O


# ---------------------------------------------------------------- conversions

def test_half_to_double_matches_numpy_for_all_bit_patterns():
    bits = np.arange(65536, dtype=np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([O.half_to_double(int(b)) for b in bits])
    finite = np.isfinite(ref)
    assert np.array_equal(got[finite], ref[finite])
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    assert np.array_equal(np.isinf(got), np.isinf(ref))


def test_double_to_half_rounds_like_numpy():
    rng = np.random.default_rng(0)
    x = np.concatenate([
        rng.standard_normal(20000) * 10.0 ** rng.uniform(-9, 5, 20000),
        # exact ties between neighbouring fp16 values, subnormals, the overflow edge
        (np.arange(0, 2048, dtype=np.float64) + 0.5) * 2.0 ** -24,
        (np.arange(1024, 2048, dtype=np.float64) + 0.5) * 2.0 ** -10,
        np.array([65504.0, 65519.99, 65520.0, 70000.0, 2.0 ** -25, 2.0 ** -26, 0.0, -0.0]),
    ])
    with np.errstate(over="ignore"):
        ref = x.astype(np.float16).view(np.uint16)
    got = np.array([O.double_to_half(float(v)) for v in x], dtype=np.uint16)
    assert np.array_equal(got, ref)


def test_bf16_to_double_matches_torch():
    bits = np.arange(0, 65536, 7, dtype=np.uint16)
    t = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    got = np.array([O.bf16_to_double(int(b)) for b in bits])
    ok = np.isfinite(t)
    assert np.array_equal(got[ok], t[ok])


# ---------------------------------------------------------------- generator

def test_splitmix64_published_outputs():
    # SplitMix64 from state 0: the first outputs of the reference generator.
    assert O.splitmix64_outputs(0, 4) == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4,
                                          0x06C45D188009454F, 0xF88BB8A8724C81EC]


def test_counter_draws_equal_sequential_generator():
    seed = 0x1234_5678_9ABC_DEF0
    for stream in (0, 1, 7):
        state0 = seed ^ ((0x5851F42D4C957F2D * (stream + 1)) & (2 ** 64 - 1))
        seq = O.splitmix64_outputs(state0, 50)
        assert [O.draw(seed, stream, k) for k in range(50)] == seq


def test_gaussian_stream_statistics():
    n = 200_000
    g = np.array([O.gauss(99, 5, e) for e in range(n)])
    assert abs(g.mean()) < 5.0 / math.sqrt(n)
    assert abs(g.var() - 1.0) < 5.0 * math.sqrt(2.0 / n)
    assert scipy.stats.kstest(g, "norm").pvalue > 1e-4


def test_rotation_signs_and_qjl_matrix():
    D = O.rotation_signs(256, 1)
    assert set(np.unique(D)) <= {-1, 1}
    assert abs(int(D.sum())) < 4 * math.sqrt(256)
    S = O.qjl_matrix(128, 128, 1)
    # every entry is an fp16 value (rounded once), distributed as N(0, 1)
    assert np.array_equal(S.astype(np.float16).astype(np.float64), S)
    assert scipy.stats.kstest(S.ravel(), "norm").pvalue > 1e-4
    assert abs(S.mean()) < 5.0 / 128
    # different seeds give different tables
    assert not np.array_equal(O.qjl_matrix(64, 64, 1), O.qjl_matrix(64, 64, 2))


# ---------------------------------------------------------------- rotation

@pytest.mark.parametrize("d", [4, 8, 64, 128, 256])
def test_rotation_is_scaled_sylvester_hadamard(d):
    # With D = +1 the rotation is H / sqrt(d), H = scipy's Sylvester Hadamard.
    ones = np.ones(d, np.int8)
    H = scipy.linalg.hadamard(d).astype(np.float64)
    M = np.stack([O.rotate(ones, e) for e in np.eye(d)], axis=1)
    assert np.allclose(M, H / math.sqrt(d), atol=1e-14)
    # and with random signs it is H diag(D) / sqrt(d)
    D = O.rotation_signs(d, 3)
    M2 = np.stack([O.rotate(D, e) for e in np.eye(d)], axis=1)
    assert np.allclose(M2, H * D[None, :] / math.sqrt(d), atol=1e-14)


@pytest.mark.parametrize("d", [64, 128, 256])
def test_rotation_orthogonal(d):
    rng = np.random.default_rng(d)
    D = O.rotation_signs(d, 11)
    for _ in range(5):
        x = rng.standard_normal(d)
        y = O.rotate(D, x)
        assert abs(np.linalg.norm(y) - np.linalg.norm(x)) < 1e-14 * np.linalg.norm(x) * 10
        assert np.allclose(O.rotate_inverse(D, y), x, atol=1e-13)
    e1 = np.zeros(d)
    e1[0] = 1.0
    assert np.allclose(np.abs(O.rotate(D, e1)), 1.0 / math.sqrt(d), atol=1e-15)


# ---------------------------------------------------------------- codebook

def test_one_bit_codebook_closed_form():
    c, rc, _ = O.lloyd_max_unit(1)
    assert rc == 0
    assert np.allclose(c, [-math.sqrt(2 / math.pi), math.sqrt(2 / math.pi)], atol=1e-12)
    cK, tK = O.codebook(1, 128)
    assert abs(float(cK[1]) - 0.0705237) < 1e-6
    assert tK[0] == 0.0


def test_codebook_matches_textbook_table(golden):
    for row in golden("lloyd_max_gaussian.txt"):
        L, mse_ref, levels = int(row[0]), float(row[1]), [float(v) for v in row[2:]]
        B = L.bit_length() - 1
        c, rc, _ = O.lloyd_max_unit(B)
        assert rc == 0
        # the table prints 4 significant digits: allow half a unit of the 4th
        tol = np.array([0.5e-3 * 10 ** math.floor(math.log10(v)) + 1e-4 for v in levels])
        assert np.all(np.abs(c[L // 2:] - levels) <= tol), (L, c)
        assert abs(O.quantizer_mse_unit(B, c) - mse_ref) < 1e-3 * mse_ref + 2e-5


@pytest.mark.parametrize("B", [1, 2, 3, 4, 7])
def test_codebook_centroid_condition_by_quadrature(B):
    # Independent numerical integration: each centroid is the mean of N(0,1)
    # over its cell, and MSE = 1 - sum_j c_j^2 P_j at the optimum.
    c, _, _ = O.lloyd_max_unit(B)
    L = 1 << B
    t = np.concatenate([[-np.inf], 0.5 * (c[1:] + c[:-1]), [np.inf]])
    s = 0.0
    for j in range(L):
        mass = scipy.stats.norm.cdf(t[j + 1]) - scipy.stats.norm.cdf(t[j])
        mean = scipy.integrate.quad(lambda x: x * scipy.stats.norm.pdf(x), t[j], t[j + 1],
                                    epsabs=1e-14, epsrel=1e-13)[0] / mass
        assert abs(mean - c[j]) < 1e-9
        s += c[j] ** 2 * mass
    mse_q = scipy.integrate.quad(
        lambda x: (x - c[np.searchsorted(t[1:-1], x)]) ** 2 * scipy.stats.norm.pdf(x),
        -12, 12, points=list(t[1:-1]), limit=4000, epsabs=1e-13)[0]
    assert abs(O.quantizer_mse_unit(B, c) - mse_q) < 1e-9
    assert abs(O.quantizer_mse_unit(B, c) - (1.0 - s)) < 1e-9


@pytest.mark.parametrize("B", [1, 2, 3, 4, 7])
@pytest.mark.parametrize("d", [64, 128, 256])
def test_codebook_scaling_and_boundaries(B, d):
    c, t = O.codebook(B, d)
    cu, _, _ = O.lloyd_max_unit(B)
    L = 1 << B
    assert c.dtype == np.float32 and t.shape == (L - 1,)
    assert np.array_equal(c, (cu / math.sqrt(d)).astype(np.float32))
    assert np.array_equal(c, -c[::-1])                       # exactly symmetric
    assert t[L // 2 - 1] == 0.0                              # middle boundary is 0
    mid = ((c[:-1].astype(np.float64) + c[1:].astype(np.float64)) / 2).astype(np.float32)
    assert np.array_equal(t, mid)
    assert np.all(np.diff(c) > 0) and np.all(np.diff(t) > 0)


def test_codebook_high_rate_limit():
    # Panter-Dite: the optimal B-bit quantizer of N(0, 1) has MSE -> (pi sqrt(3) / 2) 4^-B
    # as B grows, approached from below. The 7-bit key cells of k8v4 sit within 2 % of it.
    limit = math.pi * math.sqrt(3.0) / 2.0
    scaled = []
    for B in (4, 5, 6, 7):
        c, _, _ = O.lloyd_max_unit(B)
        scaled.append(O.quantizer_mse_unit(B, c) * 4.0 ** B)
    assert all(x < limit for x in scaled)
    assert all(b > a for a, b in zip(scaled, scaled[1:]))
    assert scaled[-1] > 0.98 * limit


def test_distortion_matches_pages(golden):
    vals = {r[0]: float(r[1]) for r in golden("pages_numbers.txt")}
    c3, _, _ = O.lloyd_max_unit(3)
    D3 = O.quantizer_mse_unit(3, c3)
    for d in (128, 256):
        ref = vals["distortion_per_coord_d%d_b3" % d]
        # the Gaussian-model distortion per coordinate prints as the pages' value
        assert round(D3 / d, 6) == ref
        # Monte Carlo on uniformly random unit vectors lands within 2%
        mc = O.distortion_mc(d, 3, 20000, seed=2024)
        assert abs(mc - ref) < 0.02 * ref, (d, mc)
    # d = 64 is not printed; the same model predicts twice the d = 128 value
    assert abs(O.distortion_mc(64, 3, 20000, seed=5) - D3 / 64) < 0.05 * D3 / 64
