"""Pins for the oracle's decode attention over the compressed cache ("A JoLT
for the KV Cache", Section 3.1: the decode kernel attends directly over the
stored factors and packed residual, with one softmax over the compressed
prefix and a dense tail of new tokens).

Expected values come from an independent library routine (torch's
scaled_dot_product_attention in fp64 on the same tensors), from closed forms
(a zero query averages the values, tail tokens included; a key far more
aligned with the query than any other selects its value), and from the
decompression path the other pins cover (the fp32 reconstruction rounds to
decompress's bf16 output)."""
import numpy as np
import pytest
import torch

from oracle import jolt_oracle as o
from tucker_quantized_residual_b200 import synth


def make_comp():
    """2 layers x 2 KV heads x 96 tokens x D = 64 keys with RoPE, compressed
    exactly at 2.5x by the oracle."""
    spec = synth.CacheSpec("dec", 1, 2, 2, 96, 64, 2, 16, 1.0, 0.02, rope_theta_k=1e4, dtype="f32")
    K, V = synth.make_cache(spec, 2)
    gs = synth.group_starts(spec)
    B = o.budget_for_ratio(K.numel() * 2, 2.5)
    opt = o.Options(bits=(0, 2, 4, 8), rt_grid=(4, 8, 16, 32), rd_grid=(8, 16, 32))
    return o.compress(K.numpy(), V.numpy(), gs, B, 0, opt, spec.rope_theta_k)


@pytest.fixture(scope="module")
def comp():
    return make_comp()


def _sdpa(q, K, V):
    """torch SDPA, fp64: q [Hq, D], K/V [H, T, D], heads repeated for GQA."""
    Hq, H = q.shape[0], K.shape[0]
    Kr = torch.from_numpy(np.repeat(K, Hq // H, axis=0))[None]
    Vr = torch.from_numpy(np.repeat(V, Hq // H, axis=0))[None]
    qq = torch.from_numpy(q)[None, :, None, :]
    return torch.nn.functional.scaled_dot_product_attention(qq, Kr, Vr)[0, :, 0, :].numpy()


def test_reconstruction_rounds_to_the_decompressed_cache(comp):
    D = comp.shape[4]
    Kd, Vd = o.decompress(comp)
    for l in range(comp.shape[1]):
        K, V = o.layer_kv_f32(comp, 0, l)
        assert np.array_equal(o.bf16_rne(K), Kd[0, l])
        assert np.array_equal(o.bf16_rne(V), Vd[0, l])


@pytest.mark.parametrize("Hq", [2, 4])
def test_matches_library_attention_with_tail(comp, Hq):
    rng = np.random.default_rng(Hq)
    D = comp.shape[4]
    q = rng.standard_normal((Hq, D))
    tk = rng.standard_normal((2, 5, D))
    tv = rng.standard_normal((2, 5, D))
    out = o.decode_attention(comp, 0, 1, q, tk, tv)
    K, V = o.layer_kv_f32(comp, 0, 1)
    Kc = np.concatenate([K.astype(np.float64), tk], axis=1)
    Vc = np.concatenate([V.astype(np.float64), tv], axis=1)
    assert np.abs(out - _sdpa(q, Kc, Vc)).max() < 1e-12
    # without a tail: the prefix alone
    out0 = o.decode_attention(comp, 0, 1, q)
    assert np.abs(out0 - _sdpa(q, K.astype(np.float64), V.astype(np.float64))).max() < 1e-12


def test_zero_query_averages_values_tail_included(comp):
    D = comp.shape[4]
    K, V = o.layer_kv_f32(comp, 0, 0)
    out = o.decode_attention(comp, 0, 0, np.zeros((2, D)))
    assert np.abs(out - V.astype(np.float64).mean(axis=1)).max() < 1e-12
    tk = np.zeros((2, 3, D))
    tv = np.zeros((2, 3, D))
    out = o.decode_attention(comp, 0, 0, np.zeros((2, D)), tk, tv)
    T = K.shape[1]
    assert np.abs(out - V.astype(np.float64).sum(axis=1) / (T + 3)).max() < 1e-12


def test_dominant_tail_key_selects_its_value(comp):
    D = comp.shape[4]
    rng = np.random.default_rng(9)
    q = rng.standard_normal((2, D))
    tk = np.stack([[q[0] * 100.0], [q[1] * 100.0]])       # [H=2, 1, D]
    tv = rng.standard_normal((2, 1, D))
    out = o.decode_attention(comp, 0, 0, q, tk, tv)
    assert np.abs(out - tv[:, 0]).max() < 1e-9


def test_grouped_query_heads_read_their_kv_head(comp):
    D = comp.shape[4]
    rng = np.random.default_rng(4)
    q = rng.standard_normal((4, D))
    q[1] = q[0]
    out = o.decode_attention(comp, 0, 1, q)
    assert np.array_equal(out[0], out[1])
    # heads 0, 1 read KV head 0 and heads 2, 3 read KV head 1: the same query
    # in head 2 gives KV head 1's answer
    q2 = q.copy()
    q2[2] = q[0]
    out2 = o.decode_attention(comp, 0, 1, q2)
    K, V = o.layer_kv_f32(comp, 0, 1)
    ref = _sdpa(q[0:1], K[1:2].astype(np.float64), V[1:2].astype(np.float64))[0]
    assert np.abs(out2[2] - ref).max() < 1e-12
