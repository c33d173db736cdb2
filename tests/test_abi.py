"""The C-ABI library loads on a machine without a GPU and exports every
function include/jolt.h declares; host-side argument checks answer with
status codes (no kernel runs)."""
import ctypes as C

import pytest

from tucker_quantized_residual_b200 import jolt


def test_library_exports_every_declared_symbol():
    lib = jolt.load_library()
    names = jolt.header_symbols()
    assert len(names) >= 16
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(jolt._SIGS), "binding and header disagree"


def test_default_options_are_the_papers():
    o, _ = jolt.make_options()
    assert list(o.bits[: o.n_bits]) == [0, 2, 4, 8]
    assert o.budget_tol == 0.005 and o.max_iters == 50
    assert o.oversample_p == 8 and o.power_iters == 2 and o.scale_group == 0
    assert o.minimizer == jolt.JOLT_MIN_ENUMERATE


def _layout(D=64, theta=0.0, groups=(0, 2)):
    gs = (C.c_int32 * len(groups))(*groups)
    L = jolt.jolt_layout(1, groups[-1], 2, 256, D, len(groups) - 1, C.cast(gs, C.POINTER(C.c_int32)),
                         jolt.JOLT_F32, groups[-1] * 2 * 256 * D, 2 * 256 * D, 256 * D, D, theta)
    return L, gs


@pytest.mark.parametrize("bad", ["D", "bits", "group", "grid", "groups", "minimizer", "rotation", "dtype", "stride",
                                 "rope", "mode", "n_bits", "bits_order", "tol", "iters", "seq_base", "cap_ratio",
                                 "rd_grid", "budget"])
def test_plan_rejects_bad_arguments_before_touching_the_device(bad):
    L, keep = _layout()
    o, k2 = jolt.make_options()
    budget = 10 ** 6
    if bad == "dtype":
        L.dtype = 7
    elif bad == "stride":
        L.stride_t = L.head_dim - 1
    elif bad == "rope":
        L.rope_theta_k = -1.0
    elif bad == "mode":
        o.mode = 5
    elif bad == "n_bits":
        o.n_bits = 0
    elif bad == "bits_order":
        o, k2 = jolt.make_options(bits=(4, 2))
    elif bad == "tol":
        o.budget_tol = 1.0
    elif bad == "iters":
        o.max_iters = 0
    elif bad == "seq_base":
        o.seq_base = -1
    elif bad == "cap_ratio":
        o.cap_ratio = float("nan")
    elif bad == "rd_grid":
        o, k2 = jolt.make_options(rd_grid=[0, 8])
    elif bad == "budget":
        budget = 0
    elif bad == "D":
        L.head_dim = 96
    elif bad == "bits":
        o.bits[1] = 5
    elif bad == "group":
        o.scale_group = 48
    elif bad == "grid":
        o, k2 = jolt.make_options(rt_grid=[4, 2])
    elif bad == "groups":
        L, keep = _layout(groups=(0, 1))
        L.n_layers = 2
    elif bad == "minimizer":
        o.minimizer = 7
    elif bad == "rotation":
        o.rotation = 2
    with pytest.raises(jolt.JoltError) as ei:
        jolt.jolt_plan(L, budget, o)
    assert ei.value.status in (1, 2)


def test_plan_rejects_infeasible_budget():
    L, keep = _layout()
    o, k2 = jolt.make_options()
    with pytest.raises(jolt.JoltError) as ei:
        jolt.jolt_plan(L, 100, o)
    assert ei.value.status == 3


def _groups_call(L, k=0x10000, iters=4):
    lib = jolt.load_library()
    n = max(L.n_layers + 1, 2)
    starts = (C.c_int32 * n)()
    ng = C.c_int32(-1)
    st = lib.jolt_layer_groups(C.byref(L), k, iters, 0, None, starts, C.byref(ng), None)
    return st, list(starts), ng.value


@pytest.mark.parametrize("bad", ["null", "short", "odd_stride", "iters", "layers", "D", "align", "theta"])
def test_layer_groups_rejects_bad_arguments_before_touching_the_device(bad):
    L, keep = _layout(groups=(0, 4))
    k, iters = 0x10000, 4
    if bad == "null":
        k = None
    elif bad == "short":
        L.seq_len = 15
    elif bad == "odd_stride":
        L.stride_t = 65
    elif bad == "iters":
        iters = 33
    elif bad == "layers":
        L.n_layers = 1025
    elif bad == "D":
        L.head_dim = 96
    elif bad == "align":
        k = 0x10004
    elif bad == "theta":
        L.rope_theta_k = -1.0
    st, _, _ = _groups_call(L, k, iters)
    assert st in (1, 2), bad             # JOLT_ERR_INVALID_ARG, JOLT_ERR_UNSUPPORTED_SHAPE
    assert jolt.jolt_last_error()


def test_layer_groups_single_layer_needs_no_device():
    L, keep = _layout(groups=(0, 1))
    st, starts, ng = _groups_call(L)
    assert st == 0 and ng == 1 and starts[:2] == [0, 1]


@pytest.mark.parametrize("bad", ["not_tensor", "dtype", "strided", "short", "cpu"])
def test_noalloc_wrapper_rejects_outputs_the_library_cannot_write(bad):
    """The C entry point only sees a raw pointer and writes len(bits) doubles
    there from a kernel; the binding refuses anything else before the call."""
    import torch
    bits = (0, 2, 4, 8)
    out = {"not_tensor": [0.0] * 4,
           "dtype": torch.zeros(4, dtype=torch.float32),
           "strided": torch.zeros(8, dtype=torch.float64)[::2],
           "short": torch.zeros(3, dtype=torch.float64),
           "cpu": torch.zeros(4, dtype=torch.float64)}[bad]
    with pytest.raises((TypeError, ValueError)):
        jolt.jolt_eps2_noalloc(bits, 128, out)


def test_plan_reports_oom_from_a_failing_allocator_without_touching_the_device():
    """jolt_plan asks the registered allocator for its workspace before any
    CUDA call; a NULL answer is JOLT_ERR_OOM and nothing is freed."""
    lib = jolt.load_library()
    calls = {"alloc": 0, "free": 0}
    AF = C.CFUNCTYPE(C.c_void_p, C.c_size_t, C.c_void_p, C.c_void_p)
    FF = C.CFUNCTYPE(None, C.c_void_p, C.c_void_p, C.c_void_p)

    def a(n, s, ctx):
        calls["alloc"] += 1
        return None

    def f(p, s, ctx):
        calls["free"] += 1

    af, ff = AF(a), FF(f)
    assert lib.jolt_set_allocator(C.cast(af, C.c_void_p), C.cast(ff, C.c_void_p), None) == 0
    try:
        L, keep = _layout()
        o, k2 = jolt.make_options()
        with pytest.raises(jolt.JoltError) as ei:
            jolt.jolt_plan(L, 10 ** 6, o)
        assert ei.value.status == 4
        assert calls == {"alloc": 1, "free": 0}
    finally:
        assert lib.jolt_set_allocator(None, None, None) == 0
    # only one of the two callbacks is an error
    assert lib.jolt_set_allocator(C.cast(af, C.c_void_p), None, None) == 1


@pytest.mark.parametrize("call", ["compress", "compress_begin", "decompress", "rd_table", "residual_encode",
                                  "residual_decode", "layer_groups"])
def test_wrappers_refuse_host_tensors_for_device_buffers(call):
    """Every entry point hands its buffers to kernels as device addresses; the
    binding refuses host tensors before the call (a host address read as a
    device one is a memory fault), so no plan or handle is needed here."""
    import torch
    x = torch.zeros(1, 2, 2, 64, 64)
    codes = torch.zeros(4, 32, dtype=torch.uint8)
    scales = torch.zeros(4, 1)
    with pytest.raises(ValueError):
        if call == "compress":
            jolt.jolt_compress(0, x, x, 1000, 0)
        elif call == "compress_begin":
            jolt.jolt_compress_begin(0, x, x, 1000, 0, None)
        elif call == "decompress":
            jolt.jolt_decompress(0, x, x)
        elif call == "rd_table":
            jolt.jolt_rd_table(0, x, x, 1, 8, 64)
        elif call == "residual_encode":
            jolt.jolt_residual_encode(torch.zeros(4, 64), 64, 4, 64, 0, codes, scales)
        elif call == "residual_decode":
            jolt.jolt_residual_decode(codes, scales, 4, 64, 4, 64, 0, torch.zeros(4, 64))
        else:
            jolt.jolt_layer_groups(x)
