"""Bit-exact codes and scales of the production residual kernel.

jolt_compress quantizes every bf16 cache with the tensor-core stream kernel
(backbone tile on tcgen05, un-RoPE, seeded Hadamard rotation, absmax codes,
LSB-first packing; Section 3, "Rotated low-bit residual"). Its quantizer takes
r * RN(1/scale) and switches to the IEEE quotient near rounding boundaries, so
it is different code from the row encoder that the other bit-exact test uses.
jolt_residual_stream_encode runs that very kernel on given factors.

The factors are chosen so that the backbone U_T^ M^ is exact in fp32 whatever
the order of the tensor cores' additions: U_T^ entries are -1, 0 or 1 and M^
entries are multiples of 2^-8 below 1 in magnitude, so every partial sum is a
multiple of 2^-8 smaller than r in magnitude, which fp32 holds exactly. The
residual E = fl32(X - U_T^ M^)
is then the same number on both sides, and the oracle's rotation, quantizer
and packer must give the same bytes. With a few hundred thousand elements per
case, tens to hundreds of quotients land within 1e-4 of a rounding tie, which
is where a multiply-by-reciprocal quantizer would flip a code; the test counts
them. RoPE cases use base 1 (every pair rotated by the angle t), whose angles
are exact on both sides, so the fp32 cos/sin tables agree and the fused
un-RoPE arithmetic is compared bit for bit too."""
import numpy as np
import pytest
import torch

from oracle import jolt_oracle as o
from tucker_quantized_residual_b200 import jolt

pytestmark = pytest.mark.gpu

CASES = [(D, b, g, rope) for D in (64, 128) for b in (2, 3, 4, 8) for g in sorted({32, 64, D})
         for rope in (0.0, 1.0)]


def _bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.asarray(a, np.float32)).to(torch.bfloat16)


@pytest.mark.parametrize("D,b,g,rope", CASES)
def test_stream_kernel_codes_and_scales_bit_exact(D, b, g, rope):
    rng = np.random.default_rng(1000 * D + 10 * b + g + int(rope))
    LH, T, r = 5, 1000, 96                       # ragged last token tile; r spans two 64-rank blocks
    seed = 77
    X = _bf16(rng.standard_normal((LH, T, D)) * 3.0)
    U = _bf16(rng.integers(-1, 2, size=(T, r)))
    M = _bf16(rng.integers(-255, 256, size=(LH, r, D)) / 256.0)
    Xd, Ud, Md = X.cuda(), U.t().contiguous().cuda(), M.cuda()
    codes = torch.zeros((LH, T, b * D // 8), dtype=torch.uint8, device="cuda")
    scales = torch.zeros((LH, T, D // g), dtype=torch.float32, device="cuda")
    jolt.jolt_residual_stream_encode(Xd, Ud, Md, b, g, seed, rope, codes, scales)
    torch.cuda.synchronize()

    # the oracle on the same inputs
    x = X.float().numpy()
    if rope:
        cs, sn = o.rope_table(T, D, rope)
        x = o.unrope_f32(x, cs, sn)
    Xt = np.einsum("tr,lrd->ltd", U.double().numpy(), M.double().numpy())
    # the backbone is exactly representable in fp32 (see the module docstring)
    assert np.array_equal(Xt, o.f32(Xt).astype(np.float64))
    E = o.residual_from(x, Xt)
    res = o.encode_residual(E, b, g, o.hadamard_signs(D, seed))
    got_codes = codes.cpu().numpy()
    got_scales = scales.cpu().numpy()
    assert np.array_equal(got_scales.view(np.uint32), res.scales.view(np.uint32))
    assert np.array_equal(got_codes, res.packed)
    # how many quotients sat near a tie (reported; they are inside the compared set)
    rot = o.apply_rotation(E, o.hadamard_signs(D, seed)).reshape(LH, T, D // g, g)
    q = np.abs(rot / np.where(res.scales > 0, res.scales, 1)[..., None])
    near = int(np.sum(np.abs(q - np.floor(q) - 0.5) < 1e-4))
    print(f"D={D} b={b} g={g} rope={rope}: {LH * T} rows bit-exact, {near} quotients within 1e-4 of a tie")


def test_stream_kernel_rejects_bad_arguments():
    x = torch.zeros((1, 16, 64), dtype=torch.bfloat16, device="cuda")
    u = torch.zeros((4, 16), dtype=torch.bfloat16, device="cuda")
    m = torch.zeros((1, 4, 64), dtype=torch.bfloat16, device="cuda")
    c = torch.zeros((1, 16, 32), dtype=torch.uint8, device="cuda")
    s = torch.zeros((1, 16, 1), dtype=torch.float32, device="cuda")
    c5 = torch.zeros((1, 16, 40), dtype=torch.uint8, device="cuda")
    with pytest.raises(jolt.JoltError):
        jolt.jolt_residual_stream_encode(x, u, m, 5, 64, 0, 0.0, c5, s)    # 5 bits
    with pytest.raises(ValueError):
        jolt.jolt_residual_stream_encode(x, u, m, 4, 64, 0, 0.0, c[:, :, :16], s)
