"""Pins for the oracle's randomized token spectrum ("A JoLT for the KV Cache",
Section 3.1, FlashJoLT: the leading q_cap token singular values from a
randomized SVD, plus one synthetic tail entry that restores the total
energy). The expected values are theorems about randomized subspace
iteration with Rayleigh-Ritz, not the oracle's own formulas:
  * if X has rank r <= k, the sketch spans the column space and the computed
    values are the exact ones (Halko, Martinsson, Tropp 2011, Section 1.3);
  * Ritz values never exceed the true singular values (Cauchy interlacing for
    B = Q^T A), so the tail is at least the true discarded energy (Ky Fan);
  * power iterations drive the leading values toward the exact ones."""
import numpy as np
import pytest

from oracle import jolt_oracle as o


def _cache(T, H, D, spectrum, rng):
    """[1, H, T, D] with token unfolding U diag(s) V^T (U, V orthonormal)."""
    r = len(spectrum)
    U = np.linalg.qr(rng.standard_normal((T, r)))[0]
    V = np.linalg.qr(rng.standard_normal((H * D, r)))[0]
    A = (U * np.asarray(spectrum)[None, :]) @ V.T
    return A.reshape(T, H, D).transpose(1, 0, 2)[None]


def test_low_rank_input_is_recovered_exactly():
    rng = np.random.default_rng(0)
    s = np.linspace(5.0, 1.0, 12)
    X = _cache(200, 2, 32, s, rng)
    Om = rng.standard_normal((64, 24))
    w, U = o.randomized_token_spectrum(X, Om, 0, 12)
    assert np.allclose(w[:12], s ** 2, rtol=1e-10)
    assert w[12] < 1e-10 * np.sum(s ** 2)
    wx, Ux = o.token_spectrum(X, 12)
    assert np.abs(np.abs(U.T @ Ux) - np.eye(12)).max() < 1e-8


@pytest.mark.parametrize("n_iter", [0, 1, 2])
def test_ritz_values_interlace_and_tail_bounds_discarded_energy(n_iter):
    rng = np.random.default_rng(1 + n_iter)
    X = rng.standard_normal((1, 2, 150, 32))
    Om = rng.standard_normal((64, 24))
    q = 16
    w, _ = o.randomized_token_spectrum(X, Om, n_iter, q)
    exact, _ = o.token_spectrum(X)
    assert np.all(w[:q] <= exact[:q] * (1 + 1e-12))
    assert w[q] >= np.sum(exact[q:]) * (1 - 1e-12)
    assert abs(np.sum(w) - np.sum(X * X)) <= 1e-9 * np.sum(X * X)


def test_power_iterations_approach_the_exact_values():
    rng = np.random.default_rng(5)
    s = np.arange(1, 61, dtype=np.float64) ** -0.8
    X = _cache(300, 2, 32, s, rng)
    Om = rng.standard_normal((64, 24))
    err = []
    for n_iter in (0, 1, 3):
        w, _ = o.randomized_token_spectrum(X, Om, n_iter, 8)
        err.append(np.abs(w[:8] - s[:8] ** 2).max() / s[0] ** 2)
    assert err[2] < err[1] < err[0]
    assert err[2] < 1e-4


def test_library_sketch_layout_and_rounding():
    N, k = 40, 16
    a = o.library_sketch(N, k, N, 7, 0)
    z = o.gaussian_f64(k * N, 7, o.STREAM_SKETCH)
    assert np.array_equal(a, o.bf16_rne(z).reshape(k, N).T)
    # values are bf16: 8 significant bits
    m, _ = np.frexp(a[a != 0])
    assert np.all(np.rint(m * 256) == m * 256)
    # a wider pitch takes the first N of each row of length ld
    b = o.library_sketch(N, k, 48, 7, 0)
    z48 = o.bf16_rne(o.gaussian_f64(k * 48, 7, o.STREAM_SKETCH)).reshape(k, 48)
    assert np.array_equal(b, z48[:, :N].T)
    # the counter word separates cells
    assert not np.array_equal(o.library_sketch(N, k, N, 7, 1), a)
