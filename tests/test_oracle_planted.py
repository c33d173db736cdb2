"""Planted mistakes: each test swaps one oracle function for a plausible
wrong variant (a dropped term, a wrong sign or index, a transposed operand)
and checks that at least one pin in test_oracle_pins.py then fails. A pin
set that let such a mistake through would not pin the oracle."""
import numpy as np
import pytest

import test_oracle_pins as pins
from oracle import jolt_oracle as o


def _fails(fn, *args):
    with pytest.raises(AssertionError):
        fn(*args)


def test_butterfly_sign(monkeypatch):
    def bad(v):
        v = np.array(v, dtype=np.float32, copy=True)
        D = v.shape[-1]
        h = 1
        while h < D:
            w = v.reshape(*v.shape[:-1], D // (2 * h), 2, h)
            a, b = w[..., 0, :].copy(), w[..., 1, :].copy()
            w[..., 0, :] = a + b
            w[..., 1, :] = b - a          # wrong: (a + b, b - a)
            h *= 2
        return v
    monkeypatch.setattr(o, "fwht_f32", bad)
    _fails(pins.test_fwht_of_unit_vectors_is_sylvester_hadamard, 64)


def test_dropped_rotation_scale(monkeypatch):
    monkeypatch.setattr(o, "rot_scale", lambda D: np.float32(1.0))
    _fails(pins.test_rotation_is_orthogonal_and_inverted, 64)


def test_floor_instead_of_round(monkeypatch):
    orig = o.quantize

    def bad(r, b, g):
        codes, sc = orig(r, b, g)
        rr = np.asarray(r, np.float32).reshape(r.shape[0], -1, g)
        s = sc[..., None].astype(np.float32)
        with np.errstate(divide="ignore", invalid="ignore"):
            q = np.where(s > 0, np.floor(rr / np.where(s > 0, s, 1)), 0)
        q = np.clip(q, -o.qmax(b), o.qmax(b)).astype(np.int32)
        return q.reshape(codes.shape), sc
    monkeypatch.setattr(o, "quantize", bad)
    _fails(pins.test_quantizer_error_bound_and_range, 4, 64)


def test_wrong_qmax(monkeypatch):
    monkeypatch.setattr(o, "qmax", lambda b: (1 << b) - 1)
    _fails(pins.test_eps2_matches_the_printed_calibration)


def test_missing_scale_bytes(monkeypatch):
    monkeypatch.setattr(o, "residual_row_bytes", lambda b, D, g: (b * D) // 8)
    _fails(pins.test_eq1_worked_example_and_zero_bit_case)


def test_tail_off_by_one(monkeypatch):
    orig = o.tail_fractions

    def bad(sig2, normsq):
        t = orig(sig2, normsq)
        return np.concatenate([t[1:], t[-1:]])
    monkeypatch.setattr(o, "tail_fractions", bad)
    _fails(pins.test_tail_fractions)


def test_swapped_layer_head_order(monkeypatch):
    def bad(X):
        Lg, H, T, D = X.shape
        return np.transpose(X, (2, 1, 0, 3)).reshape(T, H * Lg * D)
    monkeypatch.setattr(o, "token_unfolding", bad)
    _fails(pins.test_unfolding_index_order)


def test_infeasible_side_returned(monkeypatch):
    orig = o.allocate

    def bad(tables, budget, *a, **k):
        # a bisection that keeps the lower multiplier returns more bytes
        return orig(tables, int(budget * 1.3), *a, **k)
    monkeypatch.setattr(o, "allocate", bad)
    _fails(pins.test_lagrangian_matches_exhaustive_search_at_attained_budget)


def test_msb_first_packing(monkeypatch):
    def bad(codes, b):
        u = (np.asarray(codes, np.int64) + (1 << (b - 1))).astype(np.uint64)
        rows, D = u.shape
        out = np.zeros((rows, D * b // 8), np.uint8)
        for r in range(rows):
            bits = "".join(format(int(x), f"0{b}b") for x in u[r])
            out[r] = np.frombuffer(int(bits, 2).to_bytes(D * b // 8, "big"), np.uint8)
        return out
    monkeypatch.setattr(o, "pack_bits", bad)
    _fails(pins.test_pack_unpack_round_trip_and_bit_order, 4)


def test_wrong_philox_multiplier(monkeypatch):
    monkeypatch.setattr(o, "_PHILOX_M0", np.uint64(0xD2511F55))
    _fails(pins.test_philox_known_answer_vectors)


def test_rope_sign(monkeypatch):
    orig = o.rope_f32

    def bad(x, cos, sin):
        return orig(x, cos, -sin)
    monkeypatch.setattr(o, "rope_f32", bad)
    _fails(pins.test_rope_round_trip_norm_and_complex_form)


def test_backbone_without_feature_factor(monkeypatch):
    orig = o.fit

    def bad(X, U_T, rT, rd, store_f64=False):
        f = orig(X, U_T, rT, rd, store_f64)
        f.Ud = f.Ud * 1.01              # factor scaled: no longer orthonormal
        return f
    monkeypatch.setattr(o, "fit", bad)
    _fails(pins.test_factors_orthonormal)


# ----------------------------------------------------- layer grouping plants
import test_oracle_grouping as gpins


def test_feature_mode_basis(monkeypatch):
    def bad(X, r=o.GROUP_VECTORS):
        # right singular vectors (feature mode) instead of token mode
        _, _, vt = np.linalg.svd(o.token_unfolding(X), full_matrices=False)
        return vt[:r].T
    monkeypatch.setattr(o, "layer_token_basis", bad)
    _fails(gpins.test_layer_scores_recover_planted_overlaps)


def test_score_summed_not_averaged(monkeypatch):
    monkeypatch.setattr(o, "basis_score", lambda a, b: float(np.sum((a.T @ b) ** 2)))
    _fails(gpins.test_score_of_bases_sharing_m_columns, 3)


def test_rope_not_undone(monkeypatch):
    monkeypatch.setattr(o, "layer_keys", lambda K, b, l, th: np.asarray(K[b, l:l + 1], np.float64))
    _fails(gpins.test_rope_keys_scored_before_rope)


def _rule(lower_median=False, le=False, merge=True, min_size=2, max_size=8):
    def rule(scores):
        L = len(scores) + 1
        if L == 1:
            return [0, 1]
        srt = sorted(scores)
        med = srt[(len(srt) - 1) // 2] if lower_median else float(np.median(scores))
        starts, size = [0], 1
        for l in range(1, L):
            s = scores[l - 1]
            below = s <= med if le else s < med
            if size >= max_size or (size >= min_size and below):
                starts.append(l)
                size = 1
            else:
                size += 1
        if merge and len(starts) > 1 and L - starts[-1] == 1:
            starts.pop()
        return starts + [L]
    return rule


def test_rule_lower_median(monkeypatch):
    monkeypatch.setattr(o, "group_layers", _rule(lower_median=True))
    _fails(gpins.test_even_count_median_is_mean_of_middle_pair)


def test_rule_not_strict(monkeypatch):
    monkeypatch.setattr(o, "group_layers", _rule(le=True))
    _fails(gpins.test_equal_to_median_does_not_split)


def test_rule_no_trailing_merge(monkeypatch):
    monkeypatch.setattr(o, "group_layers", _rule(merge=False))
    _fails(gpins.test_trailing_single_layer_joins_predecessor)


def test_rule_no_minimum_size(monkeypatch):
    monkeypatch.setattr(o, "group_layers", _rule(min_size=1))
    _fails(gpins.test_low_score_ignored_until_group_holds_two_layers)


def test_rule_size_cap_off_by_one(monkeypatch):
    monkeypatch.setattr(o, "group_layers", _rule(max_size=9))
    _fails(gpins.test_equal_scores_close_groups_at_eight)


# ------------------------------------------------- QR rotation plants
def test_qr_without_sign_fix(monkeypatch):
    def bad(D, seed):
        G = o.gaussian_f64(D * D, seed, o.STREAM_QRGAUSS).reshape(D, D)
        return np.linalg.qr(G)[0]
    monkeypatch.setattr(o, "qr_rotation", bad)
    _fails(pins.test_qr_rotation_is_the_positive_diagonal_factor_of_its_gaussian, 64)


def test_qr_rotation_transposed(monkeypatch):
    monkeypatch.setattr(o, "rotate_qr", lambda E, Q: o.f32(np.asarray(E, np.float64) @ Q))
    _fails(pins.test_qr_rotation_orientation_and_round_trip)


def test_qr_unrotation_transposed(monkeypatch):
    monkeypatch.setattr(o, "unrotate_qr", lambda r, Q: o.f32(np.asarray(r, np.float64) @ Q.T))
    _fails(pins.test_qr_rotation_residual_round_trip_error_bound)


# ------------------------------------------------- decode attention plants
import math as _math

import test_oracle_decode as dpins


def _bad_decode(head_of, scale):
    def bad(comp, b, l, q, tail_k=None, tail_v=None):
        K, V = o.layer_kv_f32(comp, b, l)
        K, V = np.asarray(K, np.float64), np.asarray(V, np.float64)
        if tail_k is not None and tail_k.shape[1] > 0:
            K = np.concatenate([K, tail_k], axis=1)
            V = np.concatenate([V, tail_v], axis=1)
        H, _, D = K.shape
        out = np.zeros((q.shape[0], D))
        for j in range(q.shape[0]):
            h = head_of(j, q.shape[0], H)
            s = K[h] @ q[j] * scale(D)
            p = np.exp(s - s.max())
            out[j] = (p / p.sum()) @ V[h]
        return out
    return bad


def test_decode_head_mapping_modulo(monkeypatch, comp):
    monkeypatch.setattr(o, "decode_attention", _bad_decode(lambda j, Hq, H: j % H, lambda D: 1 / _math.sqrt(D)))
    _fails(dpins.test_grouped_query_heads_read_their_kv_head, comp)


def test_decode_without_scale(monkeypatch, comp):
    monkeypatch.setattr(o, "decode_attention", _bad_decode(lambda j, Hq, H: j // (Hq // H), lambda D: 1.0))
    _fails(dpins.test_matches_library_attention_with_tail, comp, 2)


@pytest.fixture(scope="module")
def comp():
    return dpins.make_comp()


# --------------------------------------------- randomized spectrum plants
import test_oracle_randomized as rpins

_rand_orig = o.randomized_token_spectrum


def test_randomized_without_tail(monkeypatch):
    def bad(X, Om, n_iter, q):
        w, U = _rand_orig(X, Om, n_iter, q)
        w = w.copy()
        w[-1] = 0.0
        return w, U
    monkeypatch.setattr(o, "randomized_token_spectrum", bad)
    _fails(rpins.test_ritz_values_interlace_and_tail_bounds_discarded_energy, 1)


def test_randomized_values_not_squared(monkeypatch):
    def bad(X, Om, n_iter, q):
        w, U = _rand_orig(X, Om, n_iter, q)
        head = np.sqrt(w[:q])
        A = o.token_unfolding(X)
        return np.concatenate([head, [max(0.0, float(np.sum(A * A)) - float(np.sum(head)))]]), U
    monkeypatch.setattr(o, "randomized_token_spectrum", bad)
    _fails(rpins.test_low_rank_input_is_recovered_exactly)


def test_randomized_power_iterations_skipped(monkeypatch):
    monkeypatch.setattr(o, "randomized_token_spectrum", lambda X, Om, n_iter, q: _rand_orig(X, Om, 0, q))
    _fails(rpins.test_power_iterations_approach_the_exact_values)


def test_admissible_pairs_strict(monkeypatch):
    monkeypatch.setattr(o.CellTable, "valid", lambda self, rT, rd: rd < self.Lg * self.H * rT)
    _fails(pins.test_tiny_grid_excludes_exactly_one_pair_per_bit_width)
    _fails(pins.test_admissible_feature_ranks_end_where_the_projected_gram_runs_out_of_rank, 3)


def test_admissible_pairs_without_heads(monkeypatch):
    monkeypatch.setattr(o.CellTable, "valid", lambda self, rT, rd: rd <= self.Lg * rT)
    _fails(pins.test_tiny_grid_excludes_exactly_one_pair_per_bit_width)
    _fails(pins.test_admissible_feature_ranks_end_where_the_projected_gram_runs_out_of_rank, 3)
