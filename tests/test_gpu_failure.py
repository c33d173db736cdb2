"""Failure paths through the C ABI on the GPU, none of which faults the GPU:
a cache holding NaN or Inf (JOLT_ERR_NONFINITE from the status word at the
next synchronising call), an allocator that fails part-way (JOLT_ERR_OOM, and
every block the library did get back is returned), and inputs whose base
pointer the tensor-memory-accelerator path cannot take (the per-row kernels
take over and still match the oracle)."""
import ctypes as C

import numpy as np
import pytest
import torch

from oracle import jolt_oracle as o
from tucker_quantized_residual_b200 import jolt, synth

from gpu_helpers import oracle_compress

pytestmark = pytest.mark.gpu

ALLOC_FN = C.CFUNCTYPE(C.c_void_p, C.c_size_t, C.c_void_p, C.c_void_p)
FREE_FN = C.CFUNCTYPE(None, C.c_void_p, C.c_void_p, C.c_void_p)


class CountingAllocator:
    """torch's caching allocator behind jolt_set_allocator; fails from the
    `fail_at`-th request on (1-based; 0 = never)."""

    def __init__(self, fail_at=0):
        self.fail_at = fail_at
        self.requests = 0
        self.live = {}
        self.freed = 0
        self._a = ALLOC_FN(self._alloc)
        self._f = FREE_FN(self._free)

    def _alloc(self, nbytes, stream, ctx):
        self.requests += 1
        if self.fail_at and self.requests >= self.fail_at:
            return None
        p = torch.cuda.caching_allocator_alloc(int(nbytes), torch.cuda.current_device(), stream)
        self.live[p] = nbytes
        return p

    def _free(self, ptr, stream, ctx):
        if ptr in self.live:
            del self.live[ptr]
            self.freed += 1
            torch.cuda.caching_allocator_delete(ptr)

    def __enter__(self):
        lib = jolt.load_library()
        assert lib.jolt_set_allocator(C.cast(self._a, C.c_void_p), C.cast(self._f, C.c_void_p), None) == 0
        return self

    def __exit__(self, *exc):
        torch.cuda.synchronize()
        jolt.load_library().jolt_set_allocator(None, None, None)


def _tiny(kind="f32"):
    spec = synth.SPECS["tiny"]
    if kind == "bf16":
        spec = spec.replace(dtype="bf16", seq_len=512)
    K, V = synth.make_cache(spec, 0)
    return spec, K, V


@pytest.mark.parametrize("mode,bad", [(jolt.JOLT_EXACT, float("nan")), (jolt.JOLT_EXACT, float("inf")),
                                      (jolt.JOLT_RANDOMIZED, float("nan"))])
def test_nonfinite_cache_reports_nonfinite(mode, bad):
    spec, K, V = _tiny("f32" if mode == jolt.JOLT_EXACT else "bf16")
    K = K.clone()
    K[0, 1, 0, 17, 5] = bad
    gs = synth.group_starts(spec)
    B = o.budget_for_ratio(K.numel() * 2, 3.0)
    Kd, Vd = K.cuda(), V.cuda()
    lay, keep = jolt.make_layout(Kd, gs)
    opt, k2 = jolt.make_options(mode=mode)
    plan = jolt.jolt_plan(lay, B, opt)
    try:
        h = jolt.jolt_compress(plan, Kd, Vd, B, 0)
        with pytest.raises(jolt.JoltError) as ei:
            jolt.jolt_bytes(h)
        assert ei.value.status == 7, ei.value
        jolt.jolt_free_handle(h)
        # the context is still usable: a clean cache compresses afterwards
        Kd.copy_(V.cuda())
        h = jolt.jolt_compress(plan, Kd, Vd, B, 0)
        assert 0 < jolt.jolt_bytes(h) <= B
        jolt.jolt_free_handle(h)
    finally:
        torch.cuda.synchronize()
        jolt.jolt_free_plan(plan)


def test_allocator_failure_returns_oom_and_leaks_nothing():
    spec, K, V = _tiny()
    gs = synth.group_starts(spec)
    B = o.budget_for_ratio(K.numel() * 2, 2.0)
    Kd, Vd = K.cuda(), V.cuda()
    lay, keep = jolt.make_layout(Kd, gs)
    opt, k2 = jolt.make_options(bits=(0, 2, 3, 4, 8), rt_grid=(8, 16, 32, 64), rd_grid=(16, 32, 48))
    # request 1 is the plan's workspace; the handle (request 2) fails
    with CountingAllocator(fail_at=2) as al:
        plan = jolt.jolt_plan(lay, B, opt)
        with pytest.raises(jolt.JoltError) as ei:
            jolt.jolt_compress(plan, Kd, Vd, B, 0)
        assert ei.value.status == 4
        jolt.jolt_free_plan(plan)
        torch.cuda.synchronize()
        assert al.requests == 2 and not al.live and al.freed == 1
    # the plan itself failing: nothing allocated, nothing freed
    with CountingAllocator(fail_at=1) as al:
        with pytest.raises(jolt.JoltError) as ei:
            jolt.jolt_plan(lay, B, opt)
        assert ei.value.status == 4
        assert al.requests == 1 and not al.live and al.freed == 0
    # and a whole compress + decompress through the counting allocator
    # returns every block once the handle and the plan are freed
    with CountingAllocator() as al:
        plan = jolt.jolt_plan(lay, B, opt)
        h = jolt.jolt_compress(plan, Kd, Vd, B, 0)
        Ko = torch.empty(K.shape, dtype=torch.bfloat16, device="cuda")
        Vo = torch.empty_like(Ko)
        jolt.jolt_decompress(h, Ko, Vo)
        assert jolt.jolt_bytes(h) <= B
        jolt.jolt_free_handle(h)
        jolt.jolt_free_plan(plan)
        torch.cuda.synchronize()
        assert al.requests >= 2 and not al.live


@pytest.mark.parametrize("which", ["k", "v"])
def test_unaligned_base_pointer_takes_the_per_row_path(which):
    """A cache view that starts 2 bytes past a 16-byte boundary cannot be read
    by TMA; exact mode then runs the residual on the per-row kernels and must
    still match the oracle within 1e-4."""
    spec = synth.SPECS["mistral"].replace(n_layers=4, seq_len=512)
    K, V = synth.make_cache(spec, 0)
    gs = synth.group_starts(spec)
    B = o.budget_for_ratio(K.numel() * 2, 3.0)
    buf = torch.zeros(K.numel() + 8, dtype=torch.bfloat16, device="cuda")
    shifted = buf[1:1 + K.numel()].view(K.shape)
    shifted.copy_((K if which == "k" else V).cuda())
    assert shifted.data_ptr() % 16 == 2
    Kd = shifted if which == "k" else K.cuda()
    Vd = shifted if which == "v" else V.cuda()
    lay, keep = jolt.make_layout(Kd, gs, spec.rope_theta_k)
    opt, k2 = jolt.make_options()
    plan = jolt.jolt_plan(lay, B, opt)
    try:
        h = jolt.jolt_compress(plan, Kd, Vd, B, 0)
        Ko = torch.empty(K.shape, dtype=torch.bfloat16, device="cuda")
        Vo = torch.empty_like(Ko)
        jolt.jolt_decompress(h, Ko, Vo)
        cells, lam, it = jolt.jolt_handle_info(h, jolt.jolt_num_cells(plan))
        jolt.jolt_free_handle(h)
    finally:
        torch.cuda.synchronize()
        jolt.jolt_free_plan(plan)
    Kn, Vn, Kr, Vr, comp = oracle_compress(K, V, gs, B, 0, spec.rope_theta_k)
    assert [(c.r_t, c.r_d, c.bits) for c in cells] == comp.alloc.choice
    for got, ref in ((Ko, Kr), (Vo, Vr)):
        assert o.rel_frobenius(ref, got.double().cpu().numpy()) <= 1e-4


def test_randomized_mode_rejects_an_unaligned_base_pointer():
    spec = synth.SPECS["mistral"].replace(n_layers=4, seq_len=512)
    K, V = synth.make_cache(spec, 0)
    buf = torch.zeros(V.numel() + 8, dtype=torch.bfloat16, device="cuda")
    Vs = buf[1:1 + V.numel()].view(V.shape)
    Vs.copy_(V.cuda())
    Kd = K.cuda()
    gs = synth.group_starts(spec)
    lay, keep = jolt.make_layout(Kd, gs, spec.rope_theta_k)
    opt, k2 = jolt.make_options(mode=jolt.JOLT_RANDOMIZED)
    B = o.budget_for_ratio(K.numel() * 2, 3.0)
    plan = jolt.jolt_plan(lay, B, opt)
    try:
        with pytest.raises(jolt.JoltError) as ei:
            jolt.jolt_compress(plan, Kd, Vs, B, 0)
        assert ei.value.status == 2
    finally:
        torch.cuda.synchronize()
        jolt.jolt_free_plan(plan)
