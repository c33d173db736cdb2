"""The sketch Omega of the randomized range finder (Section 3.1) drawn by the
library, against the oracle's library_sketch: the same Philox4x32-10 counter
layout and Box-Muller transform, rounded to bf16. This is the independent pin
of library_sketch (the oracle never reads the library's values; the library
never calls the oracle): two cells of different width N = L_g*H*D in one plan,
with the row pitch ld set to the largest N, and two sequences of a batch."""
import numpy as np
import pytest
import torch

from oracle import jolt_oracle as o
from tucker_quantized_residual_b200 import jolt

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("seed", [0, 12345])
def test_library_sketch_bit_exact(seed):
    # groups of 1 and 2 layers: N = 1*2*64 = 128 and 2*2*64 = 256; batch of 2
    gs = [0, 1, 3]
    K = torch.zeros((2, 3, 2, 512, 64), dtype=torch.bfloat16, device="cuda")
    lay, keep = jolt.make_layout(K, gs)
    opt, k2 = jolt.make_options(mode=jolt.JOLT_RANDOMIZED)
    B = o.budget_for_ratio(K.numel() * 2, 3.0)
    plan = jolt.jolt_plan(lay, B, opt)
    try:
        n = jolt.jolt_num_cells(plan)
        W = jolt.jolt_sketch(plan, seed, n)
        torch.cuda.synchronize()
    finally:
        jolt.jolt_free_plan(plan)
    got = W.cpu().numpy().view(np.uint16)
    refs = o.cells_of(2, gs)
    Ns = [(c.l1 - c.l0) * 2 * 64 for c in refs]
    ld = max(Ns)
    k = got.shape[1]
    assert got.shape == (len(refs), k, ld)
    assert k == ((o.q_cap(512, 3.0) + 8 + 15) // 16) * 16
    for i, (c, N) in enumerate(zip(refs, Ns)):
        Om = o.library_sketch(N, k, ld, seed + c.b, 2 * c.g + c.kind)       # N x k, bf16 values
        want = (np.asarray(Om.T, np.float32).view(np.uint32) >> 16).astype(np.uint16)
        assert np.array_equal(got[i, :, :N], want), i
        assert not np.any(got[i, :, N:]), i
    # cells differ from each other (distinct counter words and keys)
    assert not np.array_equal(got[0, :, :128], got[1, :, :128])
    assert not np.array_equal(got[0], got[4])
