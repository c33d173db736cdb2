"""jolt_eps2_noalloc: the calibration entry point for callers that cannot
allocate GPU memory while they run (for example an engine that reserved all
of HBM for its KV pool). It must give what jolt_eps2 gives, call after call,
with its partial sums in the library's fixed device array instead of an
allocation. This file is collected last so that a run stopping at the first
failure has run every other test already; it also passes on its own."""
import ctypes as C
import math

import pytest
import torch

from tucker_quantized_residual_b200 import jolt

pytestmark = pytest.mark.gpu

BITS = (0, 2, 3, 4, 8)


ALLOC_FN = C.CFUNCTYPE(C.c_void_p, C.c_size_t, C.c_void_p, C.c_void_p)
FREE_FN = C.CFUNCTYPE(None, C.c_void_p, C.c_void_p, C.c_void_p)


@pytest.mark.parametrize("group", [128, 64, 32])
def test_noalloc_matches_the_allocating_entry_point_twice(group):
    ref = jolt.jolt_eps2(BITS, group)
    outs = [torch.full((len(BITS),), float("nan"), dtype=torch.float64, device="cuda") for _ in range(2)]
    torch.cuda.synchronize()
    # every device allocation of the library goes through its allocator
    # callback: count the requests while the entry point runs
    requests = []
    af = ALLOC_FN(lambda n, s, ctx: requests.append(n) or None)
    ff = FREE_FN(lambda p, s, ctx: None)
    lib = jolt.load_library()
    before = torch.cuda.memory_allocated()
    assert lib.jolt_set_allocator(C.cast(af, C.c_void_p), C.cast(ff, C.c_void_p), None) == 0
    try:
        for out in outs:
            jolt.jolt_eps2_noalloc(BITS, group, out)
        torch.cuda.synchronize()
    finally:
        lib.jolt_set_allocator(None, None, None)
    assert requests == []
    assert torch.cuda.memory_allocated() == before
    for out in outs:
        got = out.cpu().tolist()
        for g, r in zip(got, ref):
            assert math.isfinite(g)
            assert abs(g - r) <= 1e-12 * abs(r), (g, r)


def test_noalloc_rejects_sizes_beyond_its_scratch():
    out = torch.zeros(9, dtype=torch.float64, device="cuda")
    with pytest.raises(jolt.JoltError) as ei:
        jolt.jolt_eps2_noalloc((0, 2, 3, 4, 8, 0, 2, 3, 4), 128, out)
    assert "bit widths" in str(ei.value)
    with pytest.raises(jolt.JoltError):
        jolt.jolt_eps2_noalloc((2,), 48, out)
