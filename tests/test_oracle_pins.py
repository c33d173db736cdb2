"""Pins for the CPU oracle: each test ties one oracle function to something
other than itself -- a value the paper prints, a closed form, a theorem, a
library routine on a special case, or brute force on a tiny input."""
import itertools
import json
import math
import os

import numpy as np
import pytest
import scipy.linalg
import torch

from oracle import jolt_oracle as o

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "paper_values.json")))
RNG = np.random.default_rng(1234)


# ---------------------------------------------------------------- generators
def test_philox_words_are_uniform_and_distinct():
    w = o.philox_block(1 << 16, seed=7, stream=3)
    assert w.dtype == np.uint32 and w.shape == (1 << 16, 4)
    u = (w.astype(np.float64) + 0.5) / 2 ** 32
    # mean and variance of U(0,1) to ~5 sigma
    assert abs(u.mean() - 0.5) < 5 * math.sqrt(1 / 12 / u.size)
    assert abs(u.var() - 1 / 12) < 0.002
    # each bit is fair
    bits = (w[:, 0][:, None] >> np.arange(32, dtype=np.uint32)) & 1
    assert np.all(np.abs(bits.mean(axis=0) - 0.5) < 0.01)
    # keyed: another seed or stream changes every word
    assert np.mean(o.philox_block(1024, 8, 3) == o.philox_block(1024, 7, 3)) < 0.01
    assert np.mean(o.philox_block(1024, 7, 4) == o.philox_block(1024, 7, 3)) < 0.01


def test_philox_known_answer_vectors():
    kat = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "philox4x32_10_kat.json")))
    for v in kat["vectors"]:
        ctr = np.array([int(x, 16) for x in v["ctr"]], dtype=np.uint32)
        key = tuple(int(x, 16) for x in v["key"])
        out = o.philox4x32_10(ctr, key)
        assert [int(x) for x in out] == [int(x, 16) for x in v["out"]]


def test_gaussian_moments_and_tails():
    z = o.gaussian_f64(1 << 18, seed=0, stream=o.STREAM_CALIB)
    assert abs(z.mean()) < 0.01 and abs(z.var() - 1) < 0.01
    assert abs(np.mean(z ** 4) - 3.0) < 0.05          # Gaussian kurtosis
    assert abs(np.mean(np.abs(z) > 1.96) - 0.05) < 0.003


def test_hadamard_signs_balanced_and_seeded():
    s = o.hadamard_signs(4096, seed=3)
    assert set(np.unique(s)) == {-1.0, 1.0}
    assert abs(s.mean()) < 0.06
    assert not np.array_equal(s[:128], o.hadamard_signs(128, seed=4))
    assert np.array_equal(s[:128], o.hadamard_signs(128, seed=3))


# ----------------------------------------------------------------- rounding
def test_bf16_rne_matches_torch_on_fp32_inputs():
    x = (RNG.standard_normal(200000) * np.exp(RNG.uniform(-20, 20, 200000))).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(o.bf16_rne(x), ref)


def test_bf16_rne_ties_to_even_from_fp64():
    # 1 + 2^-8 is halfway between 1 and 1 + 2^-7: ties to even -> 1
    assert o.bf16_rne(np.array([1 + 2.0 ** -8]))[0] == 1.0
    # 1 + 3 * 2^-8 is halfway between 1+2^-7 and 1+2^-6: even is 1+2^-6
    assert o.bf16_rne(np.array([1 + 3 * 2.0 ** -8]))[0] == 1 + 2.0 ** -6
    # just above the tie rounds up; direct rounding, no fp32 double rounding
    assert o.bf16_rne(np.array([1 + 2.0 ** -8 + 2.0 ** -40]))[0] == 1 + 2.0 ** -7
    assert o.bf16_rne(np.array([-(1 + 2.0 ** -8 + 2.0 ** -40)]))[0] == -(1 + 2.0 ** -7)


# ---------------------------------------------------------------- rotation
@pytest.mark.parametrize("D", [64, 128])
def test_fwht_of_unit_vectors_is_sylvester_hadamard(D):
    H = o.fwht_f32(np.eye(D, dtype=np.float32))
    assert np.array_equal(H, scipy.linalg.hadamard(D).astype(np.float32))


@pytest.mark.parametrize("D", [64, 128])
def test_rotation_is_orthogonal_and_inverted(D):
    s = o.hadamard_signs(D, 11)
    R = o.rotate(np.eye(D, dtype=np.float32), s).T.astype(np.float64)   # columns = R e_i
    assert np.max(np.abs(R @ R.T - np.eye(D))) < 1e-6
    E = RNG.standard_normal((500, D)).astype(np.float32)
    r = o.rotate(E, s)
    assert abs(np.linalg.norm(r) / np.linalg.norm(E) - 1) < 1e-6
    assert np.max(np.abs(o.unrotate(r, s) - E)) < 1e-5
    # the matrix form: r = D^-1/2 H diag(s) E
    ref = (E.astype(np.float64) * s) @ scipy.linalg.hadamard(D).T / math.sqrt(D)
    assert np.max(np.abs(r - ref)) < 1e-5


# --------------------------------------------------------------- quantizer
@pytest.mark.parametrize("b", [2, 3, 4, 8])
@pytest.mark.parametrize("g", [64, 128])
def test_quantizer_error_bound_and_range(b, g):
    r = (RNG.standard_normal((300, 128)) * RNG.uniform(0.01, 10, (300, 1))).astype(np.float32)
    r[5] = 0.0
    codes, sc = o.quantize(r, b, g)
    q = o.qmax(b)
    assert codes.min() >= -q and codes.max() <= q
    deq = o.dequantize(codes, sc, g)
    err = np.abs(r.astype(np.float64) - deq).reshape(300, 128 // g, g)
    bound = sc.astype(np.float64)[..., None] / 2
    assert np.all(err <= bound * (1 + 1e-6) + 1e-30)
    # the absmax element of every nonzero group lands on +-q_max
    grp = np.abs(r.reshape(300, 128 // g, g))
    top = np.take_along_axis(np.abs(codes.reshape(300, 128 // g, g)), np.argmax(grp, -1)[..., None], -1)
    nz = sc > 0
    assert np.all(top[..., 0][nz] == q)
    assert np.all(codes[5] == 0) and np.all(sc[5] == 0)


def test_quantizer_rounds_half_to_even():
    # absmax 3 with q_max 3 gives scale 1: 0.5 -> 0, 1.5 -> 2, -2.5 -> -2
    r = np.zeros((1, 64), np.float32)
    r[0, :4] = [3.0, 0.5, 1.5, -2.5]
    c, s = o.quantize(r, 3, 64)
    assert s[0, 0] == 1.0 and list(c[0, :4]) == [3, 0, 2, -2]


@pytest.mark.parametrize("b", [2, 3, 4, 8])
def test_pack_unpack_round_trip_and_bit_order(b):
    q = o.qmax(b)
    codes = RNG.integers(-q, q + 1, (7, 128)).astype(np.int32)
    p = o.pack_bits(codes, b)
    assert p.shape == (7, 128 * b // 8) and p.dtype == np.uint8
    assert np.array_equal(o.unpack_bits(p, b, 128), codes)
    # hand-made row: u_i = code_i + 2^(b-1) laid LSB first
    row = np.zeros((1, 64), np.int32)
    row[0, 0] = 1 - (1 << (b - 1))          # u0 = 1
    row[0, 1] = 0                           # u1 = 2^(b-1)
    stream = 1 | ((1 << (b - 1)) << b)
    for i in range(2, 64):
        stream |= (1 << (b - 1)) << (i * b)
    ref = np.frombuffer(stream.to_bytes(64 * b // 8, "little"), np.uint8)
    assert np.array_equal(o.pack_bits(row, b)[0], ref)


# ------------------------------------------------------- eps^2 calibration
def test_eps2_matches_the_printed_calibration():
    tab = o.eps2_table((0, 2, 4, 8), 128)
    for b, vt in GOLD["eps2_at_dh128"].items():
        if b.startswith("_"):
            continue
        val, tol = vt
        assert abs(tab[int(b)] - val) <= tol, (b, tab[int(b)])


def test_eps2_b8_is_uniform_noise_level():
    # 8-bit: step = absmax/127, noise variance step^2/12 relative to E[x^2]=1;
    # for 128 Gaussians E[absmax^2] ~ 2.65^2 -> ~ 3.6e-5 .. 4.6e-5
    tab = o.eps2_table((8,), 128)
    assert 3.0e-5 < tab[8] < 5.0e-5


def test_other_quantizer_forms_do_not_reproduce_the_printed_eps2():
    """The mid-tread symmetric reading is the one the printed values fix."""
    x = o.f32(o.gaussian_f64(1 << 18, 0, o.STREAM_CALIB)).reshape(-1, 128)
    a = np.max(np.abs(x), axis=1, keepdims=True)
    # mid-rise alternative with 2^b levels
    step = 2 * a / 4
    xr = (np.floor(x / step) + 0.5) * step
    e_rise = float(np.sum((x - xr) ** 2) / np.sum(x ** 2))
    assert abs(e_rise - 0.59) > 0.3


# ---------------------------------------------------------- Eq. (1), Eq. (5)
def test_eq1_worked_example_and_zero_bit_case():
    ex = GOLD["eq1_effective_bits"]
    assert o.residual_row_bytes(ex["b"], ex["d_h"], ex["d_h"]) * 8 / ex["d_h"] == ex["bits_per_element"]
    assert o.residual_row_bytes(0, 128, 128) == 0
    Lg, H, T, D = 4, 8, 1024, 128
    # b = 0: only core and factors
    assert o.cost_bytes(Lg, H, T, D, 10, 20, 0, D) == (Lg * H * 10 * 20 + T * 10 + D * 20) * 2
    # the residual term at b=4 is 4.25 bits per element of the cell
    extra = o.cost_bytes(Lg, H, T, D, 10, 20, 4, D) - o.cost_bytes(Lg, H, T, D, 10, 20, 0, D)
    assert extra * 8 == 4.25 * Lg * H * T * D


def test_one_scale_per_row_convention_gives_the_int8_ratio():
    for T in GOLD["int8_per_channel_ratio"]["T"]:
        ratio = 2 * T / o.residual_row_bytes(8, T, T)
        assert ratio == pytest.approx(2 * T / (T + 4))


def test_eq5_qcap():
    for T, C, q in GOLD["eq5_qcap"]["cases"]:
        assert o.q_cap(T, C) == q


# ----------------------------------------------------------------- spectra
def _lowrank_cell(Lg, H, T, D, s_tok):
    """Cell whose token unfolding is U diag(s) V^T with known U, s, V."""
    N = Lg * H * D
    r = len(s_tok)
    U = np.linalg.qr(RNG.standard_normal((T, r)))[0]
    V = np.linalg.qr(RNG.standard_normal((N, r)))[0]
    XT = (U * s_tok) @ V.T
    X = XT.reshape(T, Lg, H, D).transpose(1, 2, 0, 3).copy()
    return X, U


@pytest.mark.parametrize("T,Lg,H,D", [(40, 2, 2, 16), (200, 1, 2, 16)])
def test_token_spectrum_recovers_known_svd(T, Lg, H, D):
    s = np.array([9.0, 5.0, 3.0, 2.0, 1.0, 0.5])
    X, U = _lowrank_cell(Lg, H, T, D, s)
    w, UT = o.token_spectrum(X)
    assert np.allclose(w[:6], s ** 2, rtol=1e-10)
    assert np.max(np.abs(w[6:])) < 1e-9
    assert np.allclose(np.abs(UT[:, :6].T @ U), np.eye(6), atol=1e-8)
    # the library SVD of the unfolding (a textbook special case)
    sv = np.linalg.svd(o.token_unfolding(X), compute_uv=False)
    assert np.allclose(w[: len(sv)], sv ** 2, rtol=1e-10, atol=1e-9)
    assert abs(w.sum() - np.sum(X * X)) < 1e-8 * np.sum(X * X)


def test_unfolding_index_order():
    X = RNG.standard_normal((2, 3, 5, 4))
    XT = o.token_unfolding(X)
    for l, h, t, d in [(1, 2, 3, 1), (0, 1, 4, 3)]:
        assert XT[t, (l * 3 + h) * 4 + d] == X[l, h, t, d]


def test_feature_spectrum_is_the_feature_unfolding_svd():
    X = RNG.standard_normal((2, 3, 30, 8))
    Xd = np.transpose(X, (3, 0, 1, 2)).reshape(8, -1)
    sv = np.linalg.svd(Xd, compute_uv=False)
    assert np.allclose(np.sqrt(o.feature_spectrum(X)), sv, rtol=1e-10)


def test_tail_fractions():
    w = np.array([4.0, 3.0, 2.0, 1.0])
    t = o.tail_fractions(w, 10.0)
    assert np.allclose(t, [1.0, 0.6, 0.3, 0.1, 0.0])


def test_sign_convention():
    U = np.array([[0.1, -0.9], [-0.8, 0.3], [0.2, 0.9]])
    F = o.fix_signs(U)
    assert F[1, 0] > 0 and F[0, 1] > 0      # tie |-.9| = |.9| -> first entry


# -------------------------------------------------- ST-HOSVD (fp64 storage)
def _noisy_cell(Lg=2, H=3, T=48, D=16):
    X, _ = _lowrank_cell(Lg, H, T, D, np.array([10.0, 6.0, 4.0, 3.0, 2.0, 1.0]))
    return X + 0.05 * RNG.standard_normal(X.shape)


def test_full_ranks_reconstruct_exactly():
    X = _noisy_cell()
    Lg, H, T, D = X.shape
    w, U = o.token_spectrum(X)
    f = o.fit(X, U, min(T, Lg * H * D), D, store_f64=True)
    assert np.max(np.abs(o.backbone(f) - X)) < 1e-10 * np.max(np.abs(X))


def test_factors_orthonormal():
    X = _noisy_cell()
    w, U = o.token_spectrum(X)
    f = o.fit(X, U, 7, 5, store_f64=True)
    assert np.max(np.abs(f.UT.T @ f.UT - np.eye(7))) < 1e-12
    assert np.max(np.abs(f.Ud.T @ f.Ud - np.eye(5))) < 1e-12


@pytest.mark.parametrize("rT,rd", [(3, 4), (6, 10), (12, 2), (1, 16)])
def test_st_hosvd_error_identity_and_bounds(rT, rd):
    X = _noisy_cell()
    Lg, H, T, D = X.shape
    w, U = o.token_spectrum(X)
    f = o.fit(X, U, rT, rd, store_f64=True)
    err2 = float(np.sum((X - o.backbone(f)) ** 2))
    # exact: token tail + feature tail of the PROJECTED tensor
    Y = np.einsum("tr,lhtd->lhrd", f.UT, X)
    wp = np.sort(np.linalg.eigvalsh(o.feature_gram(Y)))[::-1]
    assert err2 == pytest.approx(float(np.sum(w[rT:]) + np.sum(wp[rd:])), rel=1e-9)
    # bounded by the surrogate's unprojected tails (so by sqrt(2) x optimum)
    wd = o.feature_spectrum(X)
    tT, tD = float(np.sum(w[rT:])), float(np.sum(wd[rd:]))
    assert err2 <= (tT + tD) * (1 + 1e-9)
    assert err2 <= 2 * max(tT, tD) * (1 + 1e-9)
    # and no better than either single-mode Eckart-Young optimum
    assert err2 >= max(tT, tD) * (1 - 1e-9)


def test_full_feature_rank_is_eckart_young_on_token_unfolding():
    X = _noisy_cell()
    Lg, H, T, D = X.shape
    w, U = o.token_spectrum(X)
    f = o.fit(X, U, 4, D, store_f64=True)
    XT = o.token_unfolding(X)
    u, s, vt = np.linalg.svd(XT, full_matrices=False)
    best = (u[:, :4] * s[:4]) @ vt[:4]
    assert np.max(np.abs(o.token_unfolding(o.backbone(f)) - best)) < 1e-9


# --------------------------------------------------------------------- RoPE
def test_rope_round_trip_norm_and_complex_form():
    T, D = 64, 32
    cs, sn = o.rope_table(T, D, 1e4)
    x = RNG.standard_normal((3, T, D)).astype(np.float32)
    y = o.rope_f32(x, cs, sn)
    assert np.max(np.abs(o.unrope_f32(y, cs, sn) - x)) < 1e-5
    assert np.linalg.norm(y) == pytest.approx(np.linalg.norm(x), rel=1e-6)
    # rotate-half RoPE is complex multiplication of (x_i + i x_{i+D/2}) by e^{i angle}
    inv = 1e4 ** (-2.0 * np.arange(D // 2) / D)
    ang = np.arange(T)[:, None] * inv[None]
    z = (x[..., : D // 2] + 1j * x[..., D // 2:]) * np.exp(1j * ang)
    assert np.max(np.abs(y[..., : D // 2] - z.real)) < 1e-5
    assert np.max(np.abs(y[..., D // 2:] - z.imag)) < 1e-5


# -------------------------------------------------------------- allocation
def _tiny_tables():
    from tucker_quantized_residual_b200 import synth
    spec = synth.SPECS["tiny"]
    K, V = synth.make_cache(spec, 0)
    opt = o.Options(bits=(0, 2, 3, 4, 8), rt_grid=(8, 16, 32, 64), rd_grid=(16, 32, 48))
    eps = o.eps2_table(opt.bits, 64)
    tabs = []
    for src in (K.numpy(), V.numpy()):
        X = src[0, 0:2].astype(np.float64)
        tabs.append(o.build_table(X, opt, eps)[0])
    return tabs


def test_lagrangian_matches_exhaustive_search_at_attained_budget():
    tabs = _tiny_tables()
    arrs = [t.arrays() for t in tabs]
    n0, n1 = len(arrs[0][3]), len(arrs[1][3])
    assert n0 == n1 == 60
    E = arrs[0][3][:, None] + arrs[1][3][None, :]
    S = arrs[0][4][:, None] + arrs[1][4][None, :]
    dense = 2 * 2 * 2 * 256 * 64 * 2
    for C in (1.5, 2.0, 3.0, 4.0, 6.0):
        B = o.budget_for_ratio(dense // 2, C)
        al = o.allocate(tabs, B)
        attained = sum(al.bytes)
        assert attained <= B
        best = float(np.min(np.where(S <= attained, E, np.inf)))
        assert sum(al.errors) == pytest.approx(best, rel=1e-12, abs=1e-15)


def test_total_cost_monotone_in_lambda():
    tabs = _tiny_tables()
    arrs = [t.arrays() for t in tabs]
    prev = None
    for lam in np.geomspace(1e-12, 1e-2, 60):
        S = sum(int(a[4][o.argmin_cell(t, lam, a)]) for t, a in zip(tabs, arrs))
        if prev is not None:
            assert S <= prev
        prev = S


def test_allocation_edges():
    tabs = _tiny_tables()
    huge = o.allocate(tabs, 10 ** 9)
    assert huge.lam == 1e-30 and huge.iters == 0
    # the best-quality choice of each cell at a negligible price
    for t, ch in zip(tabs, huge.choice):
        b, rT, rd, e, s = t.arrays()
        i = o.argmin_cell(t, 1e-30)
        assert ch == (int(rT[i]), int(rd[i]), int(b[i]))
    with pytest.raises(ValueError):
        o.allocate(tabs, 100)


def test_greedy_never_beats_enumeration_on_integer_grids():
    X = _noisy_cell(2, 2, 40, 16)
    opt = o.Options(bits=(0, 2, 4, 8))
    eps = o.eps2_table(opt.bits, 16)
    tab = o.build_table(X, opt, eps)[0]
    arr = tab.arrays()
    for lam in (1e-9, 1e-7, 1e-5, 1e-4):
        i = o.argmin_cell(tab, lam, arr)
        v_enum = arr[3][i] + lam * arr[4][i]
        rT, rd, b, v_g = o.greedy_cell(tab, lam)
        assert v_g >= v_enum - 1e-15


def test_greedy_ends_at_a_local_minimum_of_its_grid():
    """No single grid step from the greedy choice lowers e + lam*s, and at a
    prohibitive price it stays at the smallest ranks."""
    X = _noisy_cell(2, 2, 40, 16)
    opt = o.Options(bits=(0, 2, 4, 8))
    eps = o.eps2_table(opt.bits, 16)
    tab = o.build_table(X, opt, eps)[0]

    def value(bi, ti, di):
        rT, rd = int(tab.rt_grid[ti]), int(tab.rd_grid[di])
        if not tab.valid(rT, rd):
            return math.inf
        e = float(tab.eps2[bi]) * (float(tab.tT[rT]) + float(tab.tD[rd]))
        return e + lam * o.cost_bytes(tab.Lg, tab.H, tab.T, tab.D, rT, rd, int(tab.bits[bi]), tab.g)

    for lam in (1e-9, 1e-7, 1e-5, 1e-4):
        rT, rd, b, v = o.greedy_cell(tab, lam)
        bi = list(tab.bits).index(b)
        ti, di = list(tab.rt_grid).index(rT), list(tab.rd_grid).index(rd)
        assert v == value(bi, ti, di)
        if ti + 1 < len(tab.rt_grid):
            assert value(bi, ti + 1, di) >= v
        if di + 1 < len(tab.rd_grid):
            assert value(bi, ti, di + 1) >= v
    lam = 1e3
    rT, rd, b, v = o.greedy_cell(tab, lam)
    assert (rT, rd, b) == (int(tab.rt_grid[0]), int(tab.rd_grid[0]), int(tab.bits[0]))


def test_greedy_allocation_respects_the_budget():
    tabs = _tiny_tables()
    dense = 2 * 2 * 2 * 256 * 64 * 2
    for C in (2.0, 3.0):
        B = o.budget_for_ratio(dense // 2, C)
        g = o.allocate(tabs, B, minimizer="greedy")
        e = o.allocate(tabs, B)
        assert sum(g.bytes) <= B
        assert all(ch[0] in tabs[0].rt_grid and ch[1] in tabs[0].rd_grid for ch in g.choice)
        # enumeration is the exact per-cell minimizer: at its own attained budget
        # it is at least as good as any allocation that fits in that budget
        if sum(g.bytes) <= sum(e.bytes):
            assert sum(e.errors) <= sum(g.errors) * (1 + 1e-12)


# --------------------------------------------------------------- full path
def test_full_ranks_no_residual_is_bf16_storage_exact_level():
    from tucker_quantized_residual_b200 import synth
    spec = synth.SPECS["tiny"]
    K, V = synth.make_cache(spec, 0)
    K, V = K.numpy(), V.numpy()
    opt = o.Options(bits=(0,), rt_grid=(256,), rd_grid=(64,))
    c = o.compress(K, V, [0, 2], 10 ** 9, 0, opt)
    Kh, Vh = o.decompress(c)
    # bf16 factors, core and output: error at the bf16 rounding level
    assert o.rel_frobenius(K, Kh) < 2 ** -7
    assert o.rel_frobenius(V, Vh) < 2 ** -7


def test_residual_bits_lower_the_error():
    from tucker_quantized_residual_b200 import synth
    spec = synth.SPECS["tiny"]
    K, V = synth.make_cache(spec, 0)
    K, V = K.numpy(), V.numpy()
    errs = []
    for b in (0, 2, 4, 8):
        c = o.compress(K, V, [0, 2], 10 ** 9, 0, o.Options(bits=(b,), rt_grid=(8,), rd_grid=(16,)))
        errs.append(o.rel_frobenius(V, o.decompress(c)[1]))
    assert errs[0] > errs[1] > errs[2] > errs[3]
    # each level follows the calibrated eps^2 of the residual (scale 64)
    # once the output's own bf16 rounding (independent noise) is taken out
    eps = o.eps2_table((2, 4, 8), 64)
    floor2 = o.rel_frobenius(V, o.bf16_rne(V)) ** 2
    for b, e in zip((2, 4, 8), errs[1:]):
        ratio = (e ** 2 - floor2) / (errs[0] ** 2 - floor2)
        assert 0.5 * eps[b] < ratio < 2.0 * eps[b]


# ------------------------------------------------------- QR-Gaussian rotation
# ("Rotated low-bit residual": the page rotates by the Q of a seeded
# Gaussian's QR factorization; reading R17 fixes the sign convention)
@pytest.mark.parametrize("D", [64, 128])
def test_qr_rotation_is_the_positive_diagonal_factor_of_its_gaussian(D):
    Q = o.qr_rotation(D, 11)
    assert np.abs(Q.T @ Q - np.eye(D)).max() < 1e-13
    # uniqueness: with R upper triangular and R_ii > 0, R^T R = G^T G, so R is
    # the transposed Cholesky factor of G^T G and Q = G R^-1
    G = o.gaussian_f64(D * D, 11, o.STREAM_QRGAUSS).reshape(D, D)
    R = np.linalg.cholesky(G.T @ G).T
    assert np.abs(Q - G @ np.linalg.inv(R)).max() < 1e-9
    assert np.abs(o.qr_rotation(D, 12) - Q).max() > 0.1


def test_qr_rotation_orientation_and_round_trip():
    D = 64
    Q = o.qr_rotation(D, 5)
    # rotating a unit vector e_j gives column j of Q (r = Q e)
    E = np.eye(D, dtype=np.float32)[:3]
    r = o.rotate_qr(E, Q)
    for j in range(3):
        assert np.abs(r[j] - Q[:, j].astype(np.float32)).max() < 1e-7
    x = np.random.default_rng(0).standard_normal((50, D)).astype(np.float32)
    y = o.rotate_qr(x, Q)
    assert np.allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), rtol=1e-6)
    back = o.unrotate_qr(y, Q)
    # each r_i carries one fp32 rounding (|d r_i| <= 2^-24 |r_i|); Q^T spreads
    # them by at most ||r||_2 = ||x||_2 per element (unit columns), plus the
    # final rounding of e_j
    bound = 2.0 ** -24 * (np.linalg.norm(x, axis=1)[:, None] + np.abs(x)) * 1.01
    assert np.all(np.abs(back - x) <= bound)


def test_qr_rotation_residual_round_trip_error_bound():
    # encode/decode through the rotation: the error is the quantizer's,
    # rotated back, so its norm is bounded by the per-row bound sqrt(D) s/2
    D, b = 64, 8
    Q = o.rotation_for(D, 3, "qr")
    E = np.random.default_rng(1).standard_normal((40, D)).astype(np.float32)
    res = o.encode_residual(E, b, D, Q)
    back = o.decode_residual(res, D, Q, D)
    err = np.linalg.norm(back - E, axis=1)
    bound = np.sqrt(D) * res.scales[:, 0] / 2 * 1.001 + 1e-5
    assert np.all(err <= bound)


# --------------------------------------------------------------------------
# Reading R9: which (r_T, r_d) pairs are admissible options
# --------------------------------------------------------------------------
@pytest.mark.parametrize("rT", [2, 3, 5])
def test_admissible_feature_ranks_end_where_the_projected_gram_runs_out_of_rank(rT):
    """The token-projected tensor Y = X x_T U_T^T has a feature unfolding of
    D rows and L_g*H*r_T columns, so its feature Gram has rank at most
    L_g*H*r_T: feature ranks beyond that add null-space columns and cannot
    lower the backbone error (Section 3, "Partial Tucker backbone"). With fp64
    storage, fit() shows the error falling strictly up to that rank and flat
    after it; CellTable.valid must admit exactly the ranks up to the first
    r_d at which the error reaches its floor."""
    rng = np.random.default_rng(rT)
    Lg, H, T, D = 1, 2, 40, 16
    X = rng.standard_normal((Lg, H, T, D))
    _, U = o.token_spectrum(X)
    errs = []
    for rd in range(1, D + 1):
        f = o.fit(X, U, rT, rd, store_f64=True)
        errs.append(float(np.sum((X - o.backbone(f)) ** 2)))
    floor = errs[-1]
    r_floor = next(rd for rd in range(1, D + 1) if errs[rd - 1] <= floor * (1 + 1e-10))
    assert all(errs[i + 1] < errs[i] * (1 - 1e-8) for i in range(r_floor - 1))
    assert r_floor == Lg * H * rT          # the boundary the algebra fixes
    tab = o.CellTable(Lg, H, T, D, D, 1.0, np.zeros(T + 1), np.zeros(D + 1), np.arange(1, 9),
                      np.arange(1, D + 1), np.array([0]), np.array([1.0]))
    assert [bool(tab.valid(rT, rd)) for rd in range(1, D + 1)] == [rd <= r_floor for rd in range(1, D + 1)]


def test_tiny_grid_excludes_exactly_one_pair_per_bit_width():
    """On the tiny grid (L_g = H = 2: r_d <= 4 r_T), only (r_T, r_d) = (8, 48)
    is ruled out, for each of the 5 bit widths: 5 of the 60 options carry
    e = +inf and the enumeration skips exactly them."""
    tab = _tiny_tables()[0]
    full = {(int(b), int(t), int(d)) for b in tab.bits for t in tab.rt_grid for d in tab.rd_grid}
    listed = {(b, t, d) for b, t, d, _, _ in tab.options()}
    assert full - listed == {(int(b), 8, 48) for b in tab.bits}
    b, t, d, e, s = tab.arrays()
    assert sorted(zip(b[np.isinf(e)].tolist(), t[np.isinf(e)].tolist(), d[np.isinf(e)].tolist())) == \
        sorted((int(x), 8, 48) for x in tab.bits)
