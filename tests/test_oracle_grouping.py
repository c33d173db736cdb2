"""Pins for the oracle's data-driven layer grouping ("A JoLT for the KV
Cache", Section 3: layers split into contiguous groups by the alignment of
their top-8 token-mode singular vectors, a new group below the median score,
and the size bounds of that paragraph's footnote).

Every expected value comes from the construction of the input or from the
rule as the page states it, never from the oracle itself:
  * subspace overlaps of bases built with a known number of shared columns
    (the score is then m/8 exactly) or known principal angles;
  * the page's own statements about the size bounds (groups close at eight
    layers; a trailing single layer joins its predecessor, so the last group
    can hold nine);
  * caches whose token factors are known, with and without RoPE.
"""
import numpy as np
import pytest

from oracle import jolt_oracle as o


def _orthonormal(n, r, rng):
    q, rr = np.linalg.qr(rng.standard_normal((n, r)))
    return q * np.sign(np.diag(rr))[None, :]


def _layer_from_factors(A, s, Fm, H, D):
    """[H, T, D] with token unfolding A diag(s) Fm^T (column index h*D + d)."""
    T = A.shape[0]
    XT = (A * s[None, :]) @ Fm.T
    return XT.reshape(T, H, D).transpose(1, 0, 2)


# ------------------------------------------------------------------- rule
def test_equal_scores_close_groups_at_eight():
    # no score is strictly below the median: only the size bound splits
    assert o.group_layers([0.7] * 31) == [0, 8, 16, 24, 32]


def test_trailing_single_layer_joins_predecessor():
    # 17 layers: 8 + 8 + 1, the last single layer merges -> a group of nine
    assert o.group_layers([0.5] * 16) == [0, 8, 17]
    # 2 layers: a group cannot open before the first holds two layers
    assert o.group_layers([0.0]) == [0, 2]
    assert o.group_layers([]) == [0, 1]


def test_low_score_ignored_until_group_holds_two_layers():
    # median of (0, 1, 1, 1) is 1; the 0 at (0, 1) meets a group of size 1
    assert o.group_layers([0.0, 1.0, 1.0, 1.0]) == [0, 5]
    # a dip after two layers opens a group
    assert o.group_layers([1.0, 0.0, 1.0, 1.0, 1.0]) == [0, 2, 6]


def test_even_count_median_is_mean_of_middle_pair():
    # median of (0.2, 0.4, 0.6, 0.8) is 0.5: 0.4 < 0.5 opens a group at 2;
    # the lower middle (0.4) would not, the strict "<" matters too
    assert o.group_layers([0.2, 0.4, 0.6, 0.8]) == [0, 2, 5]
    assert o.group_layers([0.3, 0.5, 0.5, 0.7]) == [0, 5]


def test_equal_to_median_does_not_split():
    # median of (0, .5, .5, .5, .9, 1) is 0.5: the three scores equal to it
    # keep the group, the 0 at (4, 5) opens one
    assert o.group_layers([1.0, 0.5, 0.5, 0.5, 0.0, 0.9]) == [0, 5, 7]


# ------------------------------------------------------------------ score
@pytest.mark.parametrize("m", [0, 1, 3, 5, 8])
def test_score_of_bases_sharing_m_columns(m):
    rng = np.random.default_rng(10 + m)
    Q = _orthonormal(200, 16, rng)
    Ua = Q[:, :8]
    Ub = np.concatenate([Q[:, :m], Q[:, 8:16 - m]], axis=1)
    assert o.basis_score(Ua, Ub) == pytest.approx(m / 8, abs=1e-12)


def test_score_is_mean_cos2_of_principal_angles_and_basis_invariant():
    rng = np.random.default_rng(3)
    Q = _orthonormal(300, 16, rng)
    th = rng.uniform(0, np.pi / 2, 8)
    Ua = Q[:, :8]
    Ub = Q[:, :8] * np.cos(th)[None, :] + Q[:, 8:] * np.sin(th)[None, :]
    expect = float(np.mean(np.cos(th) ** 2))
    assert o.basis_score(Ua, Ub) == pytest.approx(expect, abs=1e-12)
    R = _orthonormal(8, 8, rng)          # another basis of the same subspaces
    assert o.basis_score(Ua @ R, Ub @ R.T) == pytest.approx(expect, abs=1e-12)


# ------------------------------------------------------------ whole cache
def _cache(T, H, D, overlaps, rng, L=None):
    """Key cache [1, L, H, T, D]: layer l+1's top-8 token subspace shares
    overlaps[l] directions with layer l's; every layer uses the SAME feature
    factor, so a feature-mode basis would score 1 everywhere."""
    L = len(overlaps) + 1
    Fm = _orthonormal(H * D, 8, rng)
    s = np.array([8.0, 7.0, 6.0, 5.0, 4.0, 3.0, 2.5, 2.0])
    basis = _orthonormal(T, 8, rng)
    layers = [basis]
    for m in overlaps:
        prev = layers[-1]
        # m columns of prev kept, the rest replaced by directions orthogonal
        # to prev (projected-out Gaussian, orthonormalized)
        g = rng.standard_normal((T, 8 - m))
        g -= prev @ (prev.T @ g)
        new = np.linalg.qr(g)[0]
        layers.append(np.concatenate([prev[:, :m], new], axis=1))
    X = np.stack([_layer_from_factors(A, s, Fm, H, D) for A in layers])[None]
    expect = [o.basis_score(layers[i], layers[i + 1]) for i in range(L - 1)]
    return X, expect, layers


def test_layer_scores_recover_planted_overlaps():
    rng = np.random.default_rng(5)
    ov = [8, 6, 2, 0, 8, 4]
    X, expect, _ = _cache(96, 2, 32, ov, rng)
    s = o.layer_scores(X)
    assert np.allclose(s, [m / 8 for m in ov], atol=1e-9)
    assert np.allclose(s, expect, atol=1e-9)


def test_layer_scores_token_side_when_tokens_exceed_features():
    # T > H*D takes token_spectrum's other branch (Gram of the features)
    rng = np.random.default_rng(6)
    ov = [7, 1, 5]
    X, _, _ = _cache(160, 2, 32, ov, rng)
    assert np.allclose(o.layer_scores(X), [m / 8 for m in ov], atol=1e-9)


def test_layer_basis_spans_the_svd_subspace():
    rng = np.random.default_rng(7)
    X = rng.standard_normal((1, 3, 50, 16))
    U = o.layer_token_basis(X)
    u, _, _ = np.linalg.svd(o.token_unfolding(X), full_matrices=False)
    P1, P2 = U @ U.T, u[:, :8] @ u[:, :8].T
    assert np.abs(P1 - P2).max() < 1e-9
    assert np.allclose(U.T @ U, np.eye(8), atol=1e-12)


def test_rope_keys_scored_before_rope():
    rng = np.random.default_rng(8)
    T, H, D, theta = 128, 2, 64, 1e4
    ov = [8, 3, 0, 5]
    X, _, _ = _cache(T, H, D, ov, rng)
    cs, sn = o.rope_table(T, D, theta)
    Y = o.rope_f32(X.astype(np.float32), cs, sn)
    s_rope = o.layer_scores(Y, rope_theta_k=theta)
    assert np.allclose(s_rope, [m / 8 for m in ov], atol=2e-5)
    # scoring the post-RoPE keys as they are gives other subspaces
    assert np.abs(o.layer_scores(Y) - np.array(ov) / 8).max() > 0.05


def test_zero_layer_scores_zero():
    rng = np.random.default_rng(9)
    X, _, _ = _cache(64, 2, 32, [8, 8, 8], rng)
    X[0, 2] = 0.0
    s = o.layer_scores(X)
    assert s[1] == 0.0 and s[2] == 0.0
    assert s[0] == pytest.approx(1.0, abs=1e-9)


def test_batch_score_is_mean_over_sequences():
    X1, _, _ = _cache(64, 2, 32, [2, 8], np.random.default_rng(11))
    X2, _, _ = _cache(64, 2, 32, [6, 0], np.random.default_rng(12))
    s = o.layer_scores(np.concatenate([X1, X2]))
    assert np.allclose(s, [(2 + 6) / 16, (8 + 0) / 16], atol=1e-9)


def test_groups_of_planted_cache():
    # scores 1, 7/8, 1, 0, 1, 3/4, 1, 7/8, 1, 5/8: median (7/8 + 1)/2 =
    # 15/16, every score at least 1/16 away from it. Each score below the
    # median meets a group of two layers and opens a new one; the last (at
    # layer 10) would leave a single trailing layer, which merges back.
    ov = [8, 7, 8, 0, 8, 6, 8, 7, 8, 5]
    X, _, _ = _cache(64, 1, 64, ov, np.random.default_rng(13))
    starts, s = o.layer_groups(X)
    assert np.allclose(s, np.array(ov) / 8, atol=1e-9)
    assert starts == [0, 2, 4, 6, 8, 11]


def test_score_against_library_principal_angles():
    # scipy computes principal angles by its own (SVD-based, sine/cosine
    # switching) method; the score is the mean squared cosine over them
    from scipy.linalg import subspace_angles
    rng = np.random.default_rng(21)
    for _ in range(5):
        Ua = _orthonormal(120, 8, rng)
        Ub = _orthonormal(120, 8, rng)
        mix = 0.3 * Ua + Ub                          # partial alignment
        Ub = np.linalg.qr(mix)[0]
        th = subspace_angles(Ua, Ub)
        assert o.basis_score(Ua, Ub) == pytest.approx(float(np.mean(np.cos(th) ** 2)), abs=1e-12)
