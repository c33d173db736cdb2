"""Randomized mode (Section 3.1, FlashJoLT) at the sizes where its kernels take
their full-size paths, against the fp64 oracle.

* k = 528: one layer of 8 KV heads at D = 128 and T = 16384, so N = 1024 and
  q_cap = 512 by Eq. (5): the sketch width k = 512 + 8 rounded up to 16 is the
  one of the 64K-token LLaMA-3.1-8B-shaped cache, the CTA-pair GEMM splits it
  into N tiles of 272 and 256 columns, and CholeskyQR and the eigensolver run
  on 528 x 528 matrices.
* k = 272: the same layer at T = 8192 (q_cap = 256): one N tile of 272
  columns, two MMAs of 144 and 128 per K step.
* LLaMA-2-13B shape: 4 layers of 40 KV heads (N_c = 20480) at T = 4096,
  q_cap = 128, k = 144.
* the MoE/GQA batch: 16 sequences in one call (groups of 6 layers, 4 KV heads,
  T = 1024), every sequence with its own cells, seeds and allocation under one
  shared 3x budget (two layer groups per sequence, 64 cells).

Each case checks the end-to-end gate err_gpu <= 1.02 err_oracle + 1e-4 per
kind against exact JoLT with the same token-rank cap, and the two k = 528 /
k = 144 cases also compare the spectrum the allocator sees with the oracle's
randomized SVD on the library's own sketch (library_sketch)."""
import numpy as np
import pytest
import torch

from oracle import jolt_oracle as o
from tucker_quantized_residual_b200 import jolt, synth

from gpu_helpers import gpu_compress, oracle_compress

pytestmark = pytest.mark.gpu

K528 = synth.SPECS["llama31_8b_64k"].replace(n_layers=1, group_size=1, seq_len=16384)
K272 = synth.SPECS["llama31_8b_64k"].replace(n_layers=1, group_size=1, seq_len=8192)
LLAMA2 = synth.SPECS["llama2_13b"].replace(n_layers=4)
MOE16 = synth.SPECS["moe_t1024"].replace(n_layers=12)


def _gate(spec, C_ratio):
    K, V = synth.make_cache(spec, 0)
    gs = synth.group_starts(spec)
    B = o.budget_for_ratio(K.numel() * 2, C_ratio)
    q = o.q_cap(spec.seq_len, C_ratio)
    Kh, Vh, cells, lam, it, nbytes = gpu_compress(K, V, gs, B, 0, spec.rope_theta_k, mode=jolt.JOLT_RANDOMIZED)
    assert nbytes <= B
    assert all(c.r_t <= q for c in cells)
    Kn, Vn, Ko, Vo, comp = oracle_compress(K, V, gs, B, 0, spec.rope_theta_k, rt_max=q)
    eg = (o.rel_frobenius(Kn, Kh), o.rel_frobenius(Vn, Vh))
    eo = (o.rel_frobenius(Kn, Ko), o.rel_frobenius(Vn, Vo))
    print(f"{spec.name} {spec.n_layers}L T={spec.seq_len} B={spec.batch} {C_ratio}x: randomized K/V "
          f"{eg[0]:.5f}/{eg[1]:.5f}, capped exact {eo[0]:.5f}/{eo[1]:.5f}")
    for g, r in zip(eg, eo):
        assert g <= 1.02 * r + 1e-4, (g, r)
    return cells, comp


def _same_sketch(spec, C_ratio):
    """jolt_rd_table's token spectrum against oracle.randomized_token_spectrum
    on the library's sketch. The bf16 GEMM operands move the Ritz values by a
    small multiple of 2^-9 relative to sigma_1^2; 1e-2 leaves a wide margin."""
    K, V = synth.make_cache(spec, 0)
    gs = synth.group_starts(spec)
    B = o.budget_for_ratio(K.numel() * 2, C_ratio)
    Kd, Vd = K.cuda(), V.cuda()
    lay, keep = jolt.make_layout(Kd, gs, spec.rope_theta_k)
    opt, k2 = jolt.make_options(mode=jolt.JOLT_RANDOMIZED)
    plan = jolt.jolt_plan(lay, B, opt)
    qc = o.q_cap(spec.seq_len, C_ratio)
    try:
        n = jolt.jolt_num_cells(plan)
        ns, st, nt, sd = jolt.jolt_rd_table(plan, Kd, Vd, n, qc + 1, spec.head_dim)
    finally:
        jolt.jolt_free_plan(plan)
    del Kd, Vd
    k = ((qc + 8 + 15) // 16) * 16
    refs = o.cells_of(1, gs)
    ld = max((c.l1 - c.l0) * spec.n_heads * spec.head_dim for c in refs)
    worst = 0.0
    for i, c in enumerate(refs[:2]):
        X = o.cell_tensor(K.float().numpy(), V.float().numpy(), c, spec.rope_theta_k)
        N = (c.l1 - c.l0) * spec.n_heads * spec.head_dim
        Om = o.library_sketch(N, k, ld, c.b, 2 * c.g + c.kind)
        w, _ = o.randomized_token_spectrum(X, Om, 2, qc)
        # randomized mode reads keys with a RoPE base as the un-RoPE'd values
        # rounded to bf16 (the tensor-core operand); values are read as stored
        Xop = o.bf16_rne(X) if (c.kind == 0 and spec.rope_theta_k > 0) else X
        nsq = float(np.sum(Xop * Xop))
        # the feature Gram (and its trace) is summed by the tensor cores 256 rows
        # at a time, then in fp32 with round-to-nearest; inside the tensor cores
        # each row's product can lose up to one ulp toward zero
        assert abs(ns[i] - nsq) <= 256 * 2.0 ** -23 * nsq
        rel = np.abs(np.array(st[i][:qc]) - w[:qc]) / w[0]
        worst = max(worst, float(rel.max()))
        assert rel.max() < 1e-2, (i, rel.max())
        # the tail entry closes the energy budget
        assert abs(sum(st[i][:qc + 1]) - ns[i]) <= 1e-9 * ns[i]
    print(f"{spec.name} k={k}: worst |sigma~^2 - oracle| / sigma_1^2 = {worst:.2e}")


def test_k528_spectrum_on_the_same_sketch():
    _same_sketch(K528, 2.0)


@pytest.mark.parametrize("C_ratio", [2.0, 3.0])
def test_k528_gate(C_ratio):
    _gate(K528, C_ratio)


def test_k272_spectrum_on_the_same_sketch():
    _same_sketch(K272, 2.0)


def test_k272_gate():
    _gate(K272, 2.0)


def test_llama2_13b_shape_spectrum_on_the_same_sketch():
    _same_sketch(LLAMA2, 2.0)


def test_llama2_13b_shape_gate():
    _gate(LLAMA2, 2.0)


def test_moe_batch_of_16_sequences_in_one_call():
    cells, comp = _gate(MOE16, 3.0)
    # one allocation per cell, every sequence represented, shared budget
    assert len(cells) == 16 * 2 * 2
    assert sorted({c.seq for c in cells}) == list(range(16))
