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
