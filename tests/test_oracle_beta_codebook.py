"""Pins for the exact-marginal (Beta) codebook of the oracle, and the library's
independent host computation of it.

One coordinate y of a uniformly random unit vector in R^d has density
proportional to (1 - y^2)^((d-3)/2) ("TurboQuant 是什麼", step 1, in
turboquant-kvquant-vllm-benchmark: the rotation concentrates the coordinates
as a Beta distribution); N(0, 1/d) is its large-d limit and the model the
Gaussian codebook uses. Pins:
* d = 3: the density is uniform on [-1, 1], so Lloyd–Max is the uniform
  quantizer;
* d = 4: a semicircle, whose 1-bit centroids are +-E|y| = +-4/(3 pi);
* the density's normalisation and variance 1/d;
* optimality against the Gaussian codebook under the exact density;
* a Monte-Carlo check on random unit vectors;
* convergence to the Gaussian codebook as d grows;
* the library's codebook (incomplete beta by continued fraction, closed-form
  first moment) equal to the oracle's (Simpson quadrature in angle) in fp32.
"""
import math

import numpy as np
import pytest

import kv_cache_vector_04_b200 as tq
from oracle import oracle as O


@pytest.mark.parametrize("B", [1, 2, 3, 4])
def test_d3_is_the_uniform_quantizer(B):
    c, rc = O.lloyd_max_beta(3, B)
    L = 1 << B
    assert rc == 0
    assert np.allclose(c, -1.0 + (2.0 * np.arange(L) + 1.0) / L, atol=1e-12)
    assert abs(O.quantizer_mse_beta(3, B, c) - (2.0 / L) ** 2 / 12.0) < 1e-12


def test_d4_one_bit_is_the_semicircle_mean():
    c, rc = O.lloyd_max_beta(4, 1)
    assert rc == 0
    assert np.allclose(c, [-4.0 / (3.0 * math.pi), 4.0 / (3.0 * math.pi)], atol=1e-12)


@pytest.mark.parametrize("d", [3, 4, 10, 64, 128])
def test_density_is_normalised_with_variance_one_over_d(d):
    # the variance of one coordinate of a unit vector is 1/d by symmetry
    th = np.linspace(-math.pi / 2, math.pi / 2, 200001)
    y = np.sin(th)
    f = np.array([O.beta_marginal_pdf(d, v) for v in y[1:-1]])
    w = np.cos(th[1:-1]) * (th[1] - th[0])
    assert abs((f * w).sum() - 1.0) < 1e-9
    assert abs((f * w * y[1:-1] ** 2).sum() - 1.0 / d) < 1e-9


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("B", [1, 2, 3, 4])
def test_beta_codebook_never_worse_and_gaussian_close(d, B):
    cb, rc = O.lloyd_max_beta(d, B)
    assert rc == 0
    cg = O.lloyd_max_unit(B)[0] / math.sqrt(d)
    mb, mg = O.quantizer_mse_beta(d, B, cb), O.quantizer_mse_beta(d, B, cg)
    assert mb <= mg * (1 + 1e-12)
    # the Gaussian model is within half a percent in MSE at these head dims
    assert (mg - mb) / mg < 5e-3


def test_converges_to_the_gaussian_codebook_like_one_over_d():
    B = 3
    cg = O.lloyd_max_unit(B)[0]
    gaps = [np.abs(O.lloyd_max_beta(d, B)[0] * math.sqrt(d) - cg).max() for d in (64, 128, 256)]
    assert 1.8 < gaps[0] / gaps[1] < 2.2 and 1.8 < gaps[1] / gaps[2] < 2.2


def test_monte_carlo_distortion_matches():
    d, B, n = 64, 3, 40000
    c, _ = O.lloyd_max_beta(d, B)
    rng = np.random.default_rng(11)
    x = rng.standard_normal((n, d))
    y = (x / np.linalg.norm(x, axis=1, keepdims=True)).ravel()
    t = 0.5 * (c[1:] + c[:-1])
    e = (y - c[np.searchsorted(t, y)]) ** 2
    exact = O.quantizer_mse_beta(d, B, c)
    assert abs(e.mean() - exact) < 4 * e.std() / math.sqrt(e.size) * 3   # coordinates are weakly dependent


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("B", [1, 2, 3, 4, 7])
def test_library_codebooks_equal_oracle(d, B):
    # 7 bits (the key cells of k8v4): the Gaussian model only; the oracle's
    # exact-marginal iteration integrates every cell by quadrature, minutes at 7 bits
    kinds = (("gauss", tq.TQ_CODEBOOK_GAUSS),) if B > 4 else \
        (("gauss", tq.TQ_CODEBOOK_GAUSS), ("beta", tq.TQ_CODEBOOK_BETA))
    for kind, code in kinds:
        c_lib, t_lib = tq.tq_build_codebook(B, d, code)
        c_ora, t_ora = O.codebook(B, d, kind)
        assert np.array_equal(c_lib, c_ora), (kind, c_lib, c_ora)
        assert np.array_equal(t_lib, t_ora), kind
