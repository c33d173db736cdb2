"""Shared helpers for the GPU parity tests: run the CUDA path through the
C-ABI binding, and the oracle on the same seeded inputs."""
from __future__ import annotations

import numpy as np
import torch

from oracle import jolt_oracle as o
from tucker_quantized_residual_b200 import jolt


def gpu_compress(K: torch.Tensor, V: torch.Tensor, group_starts, budget: int, seed: int = 0,
                 rope_theta_k: float = 0.0, **opt_kw):
    """Compress + decompress on cuda:0. Returns (K_hat, V_hat, cells, lambda,
    iters, bytes, plan, handle) with K_hat/V_hat as float64 numpy arrays."""
    Kd, Vd = K.cuda().contiguous(), V.cuda().contiguous()
    lay, keep = jolt.make_layout(Kd, group_starts, rope_theta_k)
    kw = dict(opt_kw)
    if isinstance(kw.get("minimizer"), str):
        kw["minimizer"] = jolt.JOLT_MIN_GREEDY if kw["minimizer"] == "greedy" else jolt.JOLT_MIN_ENUMERATE
    if isinstance(kw.get("rotation"), str):
        kw["rotation"] = jolt.JOLT_ROT_QR_GAUSS if kw["rotation"] == "qr" else jolt.JOLT_ROT_HADAMARD
    opt, keep2 = jolt.make_options(**kw)
    plan = jolt.jolt_plan(lay, budget, opt)
    try:
        h = jolt.jolt_compress(plan, Kd, Vd, budget, seed)
        Ko = torch.empty(K.shape, dtype=torch.bfloat16, device="cuda")
        Vo = torch.empty(V.shape, dtype=torch.bfloat16, device="cuda")
        jolt.jolt_decompress(h, Ko, Vo)
        torch.cuda.synchronize()
        n = jolt.jolt_num_cells(plan)
        cells, lam, it = jolt.jolt_handle_info(h, n)
        nbytes = jolt.jolt_bytes(h)
        out = (Ko.double().cpu().numpy(), Vo.double().cpu().numpy(), cells, lam, it, nbytes)
        jolt.jolt_free_handle(h)
    finally:
        torch.cuda.synchronize()
        jolt.jolt_free_plan(plan)
    return out


def oracle_compress(K: torch.Tensor, V: torch.Tensor, group_starts, budget: int, seed: int = 0,
                    rope_theta_k: float = 0.0, **opt_kw):
    Kn, Vn = K.float().numpy(), V.float().numpy()
    kw = dict(opt_kw)
    if "scale_group" not in kw:
        kw["scale_group"] = 0
    opt = o.Options(bits=tuple(kw.pop("bits", (0, 2, 4, 8))),
                    rt_grid=tuple(kw["rt_grid"]) if kw.get("rt_grid") else None,
                    rd_grid=tuple(kw["rd_grid"]) if kw.get("rd_grid") else None,
                    rt_max=kw.get("rt_max", 0), scale_group=kw["scale_group"],
                    tol=kw.get("budget_tol", 0.005), max_iters=kw.get("max_iters", 50),
                    minimizer=kw.get("minimizer", "enumerate"),
                    rotation=kw.get("rotation", "hadamard"))
    comp = o.compress(Kn, Vn, group_starts, budget, seed, opt, rope_theta_k)
    Kh, Vh = o.decompress(comp)
    return Kn, Vn, Kh, Vh, comp
