"""ctypes binding of libjolt (include/jolt.h), same names as the C ABI.

Argument marshalling only: every step of compression and decompression runs
in the CUDA kernels of libjolt.so. PyTorch supplies device memory and streams.
Importing this module does not need a GPU; calling into the library does.
"""
from __future__ import annotations

import ctypes as C
import os
import re
from typing import List, Optional, Sequence, Tuple

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libjolt.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "jolt.h")

JOLT_BF16, JOLT_F32 = 0, 1
JOLT_EXACT, JOLT_RANDOMIZED = 0, 1
JOLT_MIN_ENUMERATE, JOLT_MIN_GREEDY = 0, 1
JOLT_ROT_HADAMARD, JOLT_ROT_QR_GAUSS = 0, 1
STATUS = {0: "JOLT_OK", 1: "JOLT_ERR_INVALID_ARG", 2: "JOLT_ERR_UNSUPPORTED_SHAPE",
          3: "JOLT_ERR_BUDGET_INFEASIBLE", 4: "JOLT_ERR_OOM", 5: "JOLT_ERR_CUDA",
          6: "JOLT_ERR_TIMEOUT", 7: "JOLT_ERR_NONFINITE"}


class JoltError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS.get(status, status)}: {msg}")
        self.status = status


class jolt_layout(C.Structure):
    _fields_ = [("batch", C.c_int32), ("n_layers", C.c_int32), ("n_heads", C.c_int32),
                ("seq_len", C.c_int32), ("head_dim", C.c_int32), ("n_groups", C.c_int32),
                ("group_start", C.POINTER(C.c_int32)), ("dtype", C.c_int32),
                ("stride_b", C.c_int64), ("stride_l", C.c_int64), ("stride_h", C.c_int64),
                ("stride_t", C.c_int64), ("rope_theta_k", C.c_float)]


class jolt_options(C.Structure):
    _fields_ = [("mode", C.c_int32), ("n_bits", C.c_int32), ("bits", C.c_int32 * 8),
                ("n_rt", C.c_int32), ("rt_grid", C.POINTER(C.c_int32)),
                ("n_rd", C.c_int32), ("rd_grid", C.POINTER(C.c_int32)),
                ("rt_max", C.c_int32), ("oversample_p", C.c_int32), ("power_iters", C.c_int32),
                ("scale_group", C.c_int32), ("rotation", C.c_int32),
                ("budget_tol", C.c_double), ("max_iters", C.c_int32), ("minimizer", C.c_int32),
                ("seq_base", C.c_int32), ("group_base", C.c_int32), ("cap_ratio", C.c_double)]


class jolt_cell_info(C.Structure):
    _fields_ = [("seq", C.c_int32), ("group", C.c_int32), ("kind", C.c_int32),
                ("r_t", C.c_int32), ("r_d", C.c_int32), ("bits", C.c_int32),
                ("bytes", C.c_int64), ("err_model", C.c_double), ("norm_sq", C.c_double)]


class jolt_cell_view(C.Structure):
    _fields_ = [("r_t", C.c_int32), ("r_d", C.c_int32), ("bits", C.c_int32),
                ("scale_group", C.c_int32), ("L", C.c_int32), ("H", C.c_int32),
                ("T", C.c_int32), ("D", C.c_int32), ("t_pitch", C.c_int32),
                ("ut", C.c_void_p), ("ud", C.c_void_p), ("core", C.c_void_p),
                ("codes", C.c_void_p), ("scales", C.c_void_p)]


_lib = None
_VP, _I32, _I64, _U64, _D = C.c_void_p, C.c_int32, C.c_int64, C.c_uint64, C.c_double
_SIGS = {
    "jolt_default_options": (None, [C.POINTER(jolt_options)]),
    "jolt_plan": (C.c_int, [C.POINTER(jolt_layout), _I64, C.POINTER(jolt_options), C.POINTER(_VP)]),
    "jolt_free_plan": (None, [_VP]),
    "jolt_compress": (C.c_int, [_VP, _VP, _VP, _I64, _U64, _VP, C.POINTER(_VP)]),
    "jolt_summary_bytes": (_I64, [_VP]),
    "jolt_compress_begin": (C.c_int, [_VP, _VP, _VP, _I64, _U64, _VP, _VP, C.POINTER(_VP)]),
    "jolt_compress_end": (C.c_int, [_VP, _VP, _I32, _I32, _VP]),
    "jolt_decompress": (C.c_int, [_VP, _VP, _VP, C.POINTER(jolt_layout), _VP]),
    "jolt_decode_attention": (C.c_int, [_VP, _I32, _VP, _I32, _VP, _VP, _I32, _VP, _VP]),
    "jolt_bytes": (C.c_int, [_VP, C.POINTER(_I64)]),
    "jolt_handle_info": (C.c_int, [_VP, C.POINTER(jolt_cell_info), _I32, C.POINTER(_D), C.POINTER(_I32)]),
    "jolt_handle_cell": (C.c_int, [_VP, _I32, C.POINTER(jolt_cell_view)]),
    "jolt_num_cells": (_I32, [_VP]),
    "jolt_free_handle": (None, [_VP]),
    "jolt_rd_table": (C.c_int, [_VP, _VP, _VP, C.POINTER(_D), C.POINTER(_D), _I32, C.POINTER(_I32),
                                C.POINTER(_D), _VP]),
    "jolt_allocate": (C.c_int, [_VP, C.POINTER(_D), _I32, C.POINTER(_D), _I32, C.POINTER(_D), _I64,
                                C.POINTER(_I32), C.POINTER(_I64), C.POINTER(_D), C.POINTER(_I32), _VP]),
    "jolt_eps2": (C.c_int, [C.POINTER(_I32), _I32, _I32, C.POINTER(_D), _VP]),
    "jolt_eps2_noalloc": (C.c_int, [C.POINTER(_I32), _I32, _I32, _VP, _VP]),
    "jolt_residual_encode": (C.c_int, [_VP, _I64, _I32, _I32, _I32, _U64, _VP, _VP, _VP]),
    "jolt_residual_decode": (C.c_int, [_VP, _VP, _I64, _I32, _I32, _I32, _U64, _VP, _VP]),
    "jolt_residual_stream_encode": (C.c_int, [_VP, _I32, _I32, _I32, _VP, _I32, _VP, _I32, _I32, _U64,
                                              C.c_float, _VP, _VP, _VP]),
    "jolt_sketch": (C.c_int, [_VP, _U64, _VP, C.POINTER(_I32), C.POINTER(_I32), _VP]),
    "jolt_layer_groups": (C.c_int, [C.POINTER(jolt_layout), _VP, _I32, _U64, C.POINTER(C.c_double),
                                    C.POINTER(C.c_int32), C.POINTER(C.c_int32), _VP]),
    "jolt_set_allocator": (C.c_int, [_VP, _VP, _VP]),
    "jolt_last_error": (C.c_char_p, []),
    "jolt_launch_count": (_U64, []),
    "jolt_profile_enable": (None, [_I32]),
    "jolt_profile_read": (C.c_int, [C.c_void_p, _I32]),
}

STAGES = ["copy", "fgram", "token_gram", "gemm_xw", "gemm_xty", "orth", "gemm_gram", "eig", "alloc", "fit",
          "residual", "decompress"]


class jolt_stage_stats(C.Structure):
    _fields_ = [("ms", C.c_double), ("calls", C.c_int64), ("launches", C.c_int64)]


def load_library():
    """Load libjolt.so from the package directory (built by build.py)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                           "`python -m tucker_quantized_residual_b200.build`")
    lib = C.CDLL(LIB_PATH)
    for name, (res, args) in _SIGS.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def header_symbols() -> List[str]:
    """Every function include/jolt.h declares."""
    txt = open(HEADER).read()
    return sorted(set(re.findall(r"^JOLT_API\s+[\w\s\*]*?\b(jolt_\w+)\s*\(", txt, re.M)))


def _check(st: int) -> None:
    if st != 0:
        raise JoltError(st, load_library().jolt_last_error().decode())


def _stream(stream) -> Optional[int]:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _dev(**tensors) -> None:
    """The library reads and writes these buffers from its kernels: refuse host
    tensors before their addresses reach the device."""
    for name, t in tensors.items():
        if t is not None and not getattr(t, "is_cuda", False):
            raise ValueError(f"{name} must be a CUDA tensor (the library reads and writes it on the device)")


# ------------------------------------------------------------------ helpers
def make_layout(t, group_start: Sequence[int], rope_theta_k: float = 0.0) -> Tuple[jolt_layout, object]:
    """Layout of a [B, L, H, T, D] torch tensor (d contiguous). Returns the
    struct and the ctypes array it points to (keep it alive while in use)."""
    import torch
    assert t.dim() == 5 and t.stride(4) == 1
    B, L, H, T, D = t.shape
    gs = (C.c_int32 * len(group_start))(*group_start)
    dt = JOLT_F32 if t.dtype == torch.float32 else JOLT_BF16
    lay = jolt_layout(B, L, H, T, D, len(group_start) - 1, C.cast(gs, C.POINTER(C.c_int32)), dt,
                      t.stride(0), t.stride(1), t.stride(2), t.stride(3), float(rope_theta_k))
    return lay, gs


def make_options(mode: int = JOLT_EXACT, bits: Sequence[int] = (0, 2, 4, 8),
                 rt_grid: Optional[Sequence[int]] = None, rd_grid: Optional[Sequence[int]] = None,
                 rt_max: int = 0, oversample_p: int = 8, power_iters: int = 2,
                 scale_group: int = 0, budget_tol: float = 0.005,
                 max_iters: int = 50, minimizer: int = 0,
                 rotation: int = JOLT_ROT_HADAMARD, seq_base: int = 0,
                 group_base: int = 0, cap_ratio: float = 0.0) -> Tuple[jolt_options, list]:
    lib = load_library()
    o = jolt_options()
    lib.jolt_default_options(C.byref(o))
    o.mode = mode
    o.n_bits = len(bits)
    for i, b in enumerate(bits):
        o.bits[i] = b
    keep = []
    if rt_grid:
        a = (C.c_int32 * len(rt_grid))(*rt_grid)
        keep.append(a)
        o.n_rt, o.rt_grid = len(rt_grid), C.cast(a, C.POINTER(C.c_int32))
    if rd_grid:
        a = (C.c_int32 * len(rd_grid))(*rd_grid)
        keep.append(a)
        o.n_rd, o.rd_grid = len(rd_grid), C.cast(a, C.POINTER(C.c_int32))
    o.rt_max, o.oversample_p, o.power_iters = rt_max, oversample_p, power_iters
    o.scale_group, o.budget_tol, o.max_iters = scale_group, budget_tol, max_iters
    o.minimizer = minimizer
    o.rotation = rotation
    o.seq_base, o.group_base, o.cap_ratio = seq_base, group_base, cap_ratio
    return o, keep


# --------------------------------------------------------------- C-ABI names
def jolt_plan(layout: jolt_layout, byte_budget: int, options: jolt_options) -> int:
    lib = load_library()
    out = C.c_void_p()
    _check(lib.jolt_plan(C.byref(layout), int(byte_budget), C.byref(options), C.byref(out)))
    return out.value


def jolt_free_plan(plan: int) -> None:
    load_library().jolt_free_plan(plan)


def jolt_num_cells(plan: int) -> int:
    return load_library().jolt_num_cells(plan)


def jolt_compress(plan: int, k, v, byte_budget: int = 0, seed: int = 0, stream=None) -> int:
    _dev(k=k, v=v)
    lib = load_library()
    out = C.c_void_p()
    _check(lib.jolt_compress(plan, _ptr(k), _ptr(v), int(byte_budget), int(seed), _stream(stream),
                             C.byref(out)))
    return out.value


def jolt_summary_bytes(plan: int) -> int:
    return load_library().jolt_summary_bytes(plan)


def jolt_compress_begin(plan: int, k, v, byte_budget: int, seed: int, summary, stream=None) -> int:
    _dev(k=k, v=v)
    """Phase 1 of a shared-budget compression; `summary` is a CUDA uint8
    tensor of jolt_num_cells(plan) * jolt_summary_bytes(plan) bytes."""
    need = jolt_num_cells(plan) * jolt_summary_bytes(plan)
    if not (summary.is_cuda and summary.is_contiguous() and summary.numel() * summary.element_size() >= need):
        raise ValueError(f"summary must be a contiguous CUDA buffer of at least {need} bytes")
    out = C.c_void_p()
    _check(load_library().jolt_compress_begin(plan, _ptr(k), _ptr(v), int(byte_budget), int(seed), _ptr(summary),
                                              _stream(stream), C.byref(out)))
    return out.value


def jolt_compress_end(handle: int, all_summaries, n_total: int, first_cell: int, stream=None) -> None:
    """Phase 2: the allocation over the gathered records of every process,
    then this plan's fit and residual."""
    if not (all_summaries.is_cuda and all_summaries.is_contiguous()):
        raise ValueError("all_summaries must be a contiguous CUDA buffer")
    _check(load_library().jolt_compress_end(handle, _ptr(all_summaries), int(n_total), int(first_cell),
                                            _stream(stream)))


def jolt_decompress(handle: int, k_out, v_out, out_layout: Optional[jolt_layout] = None, stream=None) -> None:
    _dev(k_out=k_out, v_out=v_out)
    lib = load_library()
    _check(lib.jolt_decompress(handle, _ptr(k_out), _ptr(v_out),
                               C.byref(out_layout) if out_layout is not None else None, _stream(stream)))


def jolt_decode_attention(handle: int, layer: int, q, out, tail_k=None, tail_v=None, stream=None) -> None:
    """One fused decode step of `layer`: q fp32 [B, Hq, D] -> out fp32 [B, Hq, D];
    optional dense tail bf16 [B, H, n_tail, D] (CUDA, contiguous)."""
    import torch
    for t, dt in ((q, torch.float32), (out, torch.float32)):
        if not (t.is_cuda and t.dtype == dt and t.is_contiguous() and t.dim() == 3):
            raise ValueError("q and out must be contiguous CUDA float32 tensors [B, Hq, D]")
    n_tail = 0
    if tail_k is not None:
        for t in (tail_k, tail_v):
            if not (t.is_cuda and t.dtype == torch.bfloat16 and t.is_contiguous() and t.dim() == 4):
                raise ValueError("tail_k and tail_v must be contiguous CUDA bfloat16 tensors [B, H, n, D]")
        n_tail = tail_k.shape[2]
    _check(load_library().jolt_decode_attention(handle, int(layer), _ptr(q), q.shape[1], _ptr(tail_k),
                                                _ptr(tail_v), n_tail, _ptr(out), _stream(stream)))


def jolt_bytes(handle: int) -> int:
    n = C.c_int64()
    _check(load_library().jolt_bytes(handle, C.byref(n)))
    return n.value


def jolt_handle_info(handle: int, n_cells: int):
    cells = (jolt_cell_info * n_cells)()
    lam = C.c_double()
    it = C.c_int32()
    _check(load_library().jolt_handle_info(handle, cells, n_cells, C.byref(lam), C.byref(it)))
    return list(cells), lam.value, it.value


def jolt_handle_cell(handle: int, cell: int) -> jolt_cell_view:
    v = jolt_cell_view()
    _check(load_library().jolt_handle_cell(handle, cell, C.byref(v)))
    return v


def jolt_free_handle(handle: int) -> None:
    load_library().jolt_free_handle(handle)


def jolt_rd_table(plan: int, k, v, n_cells: int, max_t: int, D: int, stream=None):
    """Returns (norm_sq[n], sig_t[n][max_t], n_t, sig_d[n][D]) as Python lists."""
    _dev(k=k, v=v)
    ns = (C.c_double * n_cells)()
    st = (C.c_double * (n_cells * max_t))()
    sd = (C.c_double * (n_cells * D))()
    nt = C.c_int32()
    _check(load_library().jolt_rd_table(plan, _ptr(k), _ptr(v), ns, st, max_t, C.byref(nt), sd,
                                        _stream(stream)))
    return (list(ns), [list(st[i * max_t:(i + 1) * max_t]) for i in range(n_cells)], nt.value,
            [list(sd[i * D:(i + 1) * D]) for i in range(n_cells)])


def jolt_allocate(plan: int, t_t: Sequence[Sequence[float]], t_d: Sequence[Sequence[float]],
                  eps2: Sequence[float], byte_budget: int, stream=None):
    """t_t[c] / t_d[c]: tail fractions per cell (padded to equal length)."""
    nc = len(t_t)
    ld_t, ld_d = max(len(x) for x in t_t), max(len(x) for x in t_d)
    tt = (C.c_double * (nc * ld_t))()
    td = (C.c_double * (nc * ld_d))()
    for i in range(nc):
        for j, x in enumerate(t_t[i]):
            tt[i * ld_t + j] = x
        for j, x in enumerate(t_d[i]):
            td[i * ld_d + j] = x
    e = (C.c_double * len(eps2))(*eps2)
    ch = (C.c_int32 * (3 * nc))()
    by = (C.c_int64 * nc)()
    lam = C.c_double()
    it = C.c_int32()
    _check(load_library().jolt_allocate(plan, tt, ld_t, td, ld_d, e, int(byte_budget), ch, by,
                                        C.byref(lam), C.byref(it), _stream(stream)))
    return [tuple(ch[3 * i:3 * i + 3]) for i in range(nc)], list(by), lam.value, it.value


def jolt_eps2(bits: Sequence[int], group: int, stream=None) -> List[float]:
    b = (C.c_int32 * len(bits))(*bits)
    out = (C.c_double * len(bits))()
    _check(load_library().jolt_eps2(b, len(bits), group, out, _stream(stream)))
    return list(out)


def jolt_eps2_noalloc(bits: Sequence[int], group: int, out, stream=None) -> None:
    """Same values as jolt_eps2, written to the device tensor `out` (float64,
    len(bits) entries) without any device allocation inside the library.

    The library only sees a raw pointer and writes len(bits) doubles there,
    so the tensor is checked here: a CUDA float64 tensor, contiguous, with
    room for every bit width."""
    import torch
    if not isinstance(out, torch.Tensor):
        raise TypeError("out must be a torch.Tensor")
    if out.dtype != torch.float64:
        raise ValueError(f"out must be float64, not {out.dtype}")
    if not out.is_contiguous():
        raise ValueError("out must be contiguous")
    if out.numel() < len(bits):
        raise ValueError(f"out holds {out.numel()} values, {len(bits)} needed")
    if not out.is_cuda:
        raise ValueError("out must be a CUDA tensor (the library writes it from a kernel)")
    b = (C.c_int32 * len(bits))(*bits)
    _check(load_library().jolt_eps2_noalloc(b, len(bits), group, _ptr(out), _stream(stream)))


def jolt_residual_stream_encode(x, ut_t, m, bits: int, group: int, seed: int, rope_theta: float,
                                codes, scales, stream=None) -> None:
    """The compress path's residual kernel on given factors. x: bf16 [LH, T, D];
    ut_t: bf16 [r, T]; m: bf16 [LH, r, D]; codes: uint8 [LH, T, bits*D/8];
    scales: float32 [LH, T, D/group] (all CUDA, contiguous)."""
    import torch
    LH, T, D = x.shape
    r = ut_t.shape[0]
    for t, dt, shape in ((x, torch.bfloat16, (LH, T, D)), (ut_t, torch.bfloat16, (r, T)),
                         (m, torch.bfloat16, (LH, r, D)), (codes, torch.uint8, (LH, T, bits * D // 8)),
                         (scales, torch.float32, (LH, T, D // group))):
        if not (t.is_cuda and t.dtype == dt and t.is_contiguous() and tuple(t.shape) == shape):
            raise ValueError(f"expected a contiguous CUDA {dt} tensor of shape {shape}")
    _check(load_library().jolt_residual_stream_encode(_ptr(x), LH, T, D, _ptr(ut_t), r, _ptr(m), bits, group,
                                                      int(seed), float(rope_theta), _ptr(codes), _ptr(scales),
                                                      _stream(stream)))


def jolt_sketch(plan: int, seed: int, n_cells: int, stream=None):
    """The randomized plan's sketch: a CUDA int16 tensor [n_cells, k, ld] of
    bf16 bit patterns (row j of cell c = column j of that cell's Omega)."""
    import torch
    lib = load_library()
    k, ld = C.c_int32(), C.c_int32()
    _check(lib.jolt_sketch(plan, int(seed), None, C.byref(k), C.byref(ld), _stream(stream)))
    out = torch.zeros((n_cells, k.value, ld.value), dtype=torch.int16, device="cuda")
    _check(lib.jolt_sketch(plan, int(seed), _ptr(out), None, None, _stream(stream)))
    return out


def jolt_residual_encode(e, D: int, bits: int, group: int, seed: int, codes, scales, stream=None) -> None:
    _dev(e=e, codes=codes, scales=scales)
    rows = e.numel() // D
    _check(load_library().jolt_residual_encode(_ptr(e), rows, D, bits, group, int(seed), _ptr(codes),
                                               _ptr(scales), _stream(stream)))


def jolt_residual_decode(codes, scales, rows: int, D: int, bits: int, group: int, seed: int, e_hat,
                         stream=None) -> None:
    _dev(codes=codes, scales=scales, e_hat=e_hat)
    _check(load_library().jolt_residual_decode(_ptr(codes), _ptr(scales), rows, D, bits, group, int(seed),
                                               _ptr(e_hat), _stream(stream)))


def jolt_layer_groups(k, rope_theta_k: float = 0.0, power_iters: int = 4, seed: int = 0,
                      stream=None) -> Tuple[List[int], List[float]]:
    """Data-driven layer grouping of a [B, L, H, T, D] device key tensor:
    (group starts including 0 and L, the L-1 consecutive-layer scores)."""
    _dev(k=k)
    L = k.shape[1]
    lay, keep = make_layout(k, [0, L], rope_theta_k)
    starts = (C.c_int32 * (L + 1))()
    scores = (C.c_double * max(L - 1, 1))()
    ng = C.c_int32(0)
    _check(load_library().jolt_layer_groups(C.byref(lay), _ptr(k), int(power_iters), int(seed), scores, starts,
                                            C.byref(ng), _stream(stream)))
    del keep
    return list(starts[:ng.value + 1]), list(scores[:L - 1])


def jolt_profile_enable(on: bool) -> None:
    load_library().jolt_profile_enable(1 if on else 0)


def jolt_profile_read() -> dict:
    """{stage: (ms, calls, launches)} summed since the last enable."""
    arr = (jolt_stage_stats * len(STAGES))()
    _check(load_library().jolt_profile_read(C.cast(arr, C.c_void_p), len(STAGES)))
    return {name: (arr[i].ms, arr[i].calls, arr[i].launches) for i, name in enumerate(STAGES)}


def jolt_last_error() -> str:
    return load_library().jolt_last_error().decode()


def jolt_launch_count() -> int:
    return load_library().jolt_launch_count()
