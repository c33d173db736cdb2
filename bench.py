#!/usr/bin/env python
"""Benchmark of the JoLT compress -> decompress path on B200.

Metric: GB/s of dense bf16 KV cache (K and V) compressed and decompressed,
at a global byte budget of dense / ratio. One step = jolt_compress (spectra,
allocation, fit, residual) + jolt_decompress of the whole cache; inputs are
resident in HBM and larger than L2. Default workload: the LLaMA-3.1-8B-shaped
64K-token cache (32 layers in groups of 4, 8 KV heads, D = 128), randomized
token-mode SVD (q_cap = Eq. (5), p = 8, 2 power iterations), 2x budget.

Under torchrun the job compresses N times the cache, one sequence block per
rank, under ONE shared byte budget: every rank computes its cells' spectra and
rate-distortion records, one all-gather of the records (NCCL), the same
multiplier bisection on every rank, then each rank fits, encodes and decodes
its own cells. Scaling is weak (fixed work per GPU); the value is the total
over ranks divided by the slowest rank's time.

--impl reference runs the CPU oracle (exact JoLT, fp64) on a bounded sample of
the same workload on the host cores.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return PEAKS_FALLBACK, "fallback"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="jolt", choices=["jolt", "reference"])
    ap.add_argument("--config", default="llama31_8b_64k")
    ap.add_argument("--ratio", type=float, default=2.0)
    ap.add_argument("--mode", default="randomized", choices=["randomized", "exact"])
    ap.add_argument("--e2e-steps", type=int, default=8)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--groups", type=int, default=0,
                    help="only the first N layer groups of the config (small profiling cases)")
    ap.add_argument("--cpu-tokens", type=int, default=1024, help="tokens in the CPU baseline sample")
    ap.add_argument("--cpu-reps", type=int, default=8, help="repetitions of the CPU baseline sample")
    ap.add_argument("--extra-ratios", default="3,4,5",
                    help="further budgets timed after the headline one (comma list; empty: none)")
    ap.add_argument("--extra-steps", type=int, default=3)
    ap.add_argument("--no-decode", action="store_true", help="skip the fused decode-attention measurement")
    ap.add_argument("--stages", action="store_true", help="print the per-stage table to stderr")
    ap.add_argument("--no-grouping", action="store_true", help="skip the layer-grouping measurement")
    return ap.parse_args()


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during a region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.f = None

    def start(self):
        try:
            self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.flush()
        rows = [r.split(",") for r in open(self.f.name).read().strip().splitlines() if r.strip()]
        os.unlink(self.f.name)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[1]))
                smax.append(float(r[2]))
                for n, v in zip(names, r[5:9]):
                    if v.strip().lower() == "active":
                        reasons.add(n)
            except (ValueError, IndexError):
                continue
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "samples": len(sm), "reasons": sorted(reasons)}


# ------------------------------------------------------------ workload
# DRAM bytes per launch of the dominant kernel from an ncu capture
# (dram__bytes_read.sum + dram__bytes_write.sum) of the first layer group of
# the 64K-token cache, scaled to the full 16-cell launch by the cells it
# processes (mean of the X W and X^T Y launches); None once the kernel has
# changed since the capture.
GEMM_TRAFFIC = {"llama31_8b_64k": 9.85e9}


def sketch_width(spec, ratio, p=8):
    """k = q_cap (Eq. 5) + p, rounded up to a multiple of 16."""
    q = min(max(32 if ratio <= 4 else 64, -(-spec.seq_len // 32)), 512)
    return ((q + p + 15) // 16) * 16


def stage_work(spec, cells, k, power_iters=2):
    """Algorithmic work of one step, per stage: (flops, HBM bytes, launches).

    Tensor-core GEMM passes over X (2k flops and one 2-byte read per element
    each): the sketch X W0, then per power iteration X^T Y and X W, then the
    final X^T Y; the Gram Y^T Y of the last sketch. Residual pass: read X
    (2 B/elem), write codes + scales, 2 r_T flops/elem for the backbone.
    Decode: read the payload, write 2 B/elem, 2 r_T flops/elem."""
    Lg, H, D, T = spec.group_size, spec.n_heads, spec.head_dim, spec.seq_len
    ncell = len(cells)
    elems = Lg * H * T * D                     # per cell
    N = Lg * H * D
    w = {}
    w["gemm_xw"] = (2.0 * T * N * k * ncell * (power_iters + 1),
                    (2.0 * elems + 2.0 * (N + T) * k) * ncell * (power_iters + 1), power_iters + 1)
    w["gemm_xty"] = (2.0 * T * N * k * ncell * (power_iters + 1),
                     (2.0 * elems + 2.0 * T * k + 4.0 * N * k) * ncell * (power_iters + 1), power_iters + 1)
    w["gemm_gram"] = (2.0 * k * k * T * ncell, 2.0 * T * k * ncell, 1)
    res_f = res_b = dec_f = dec_b = 0.0
    rows = Lg * H * T
    for c in cells:
        back = 2.0 * c.r_t * elems
        dec_f += back
        dec_b += c.bytes + 2.0 * elems
        if c.bits:
            res_f += back
            res_b += 2.0 * elems + rows * (c.bits * D // 8 + 4)
    w["residual"] = (res_f, res_b, 1)
    w["decompress"] = (dec_f, dec_b, 1)
    return w


def max_over_ranks(x, world, dist=None, device=None):
    """The largest value of x over all ranks (each rank's own device time)."""
    if world <= 1:
        return float(x)
    import torch
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def throughput_gbs(world, dense_bytes, steps, ms):
    """Whole-job GB/s: every rank's dense bytes over the slowest rank's time."""
    return world * dense_bytes * steps / (ms / 1e3) / 1e9


# fp32 lanes per SM (4 partitions x 32) on B200; with 148 SMs and the 1965 MHz
# boost clock this is the fp32 FMA ceiling of the grouping's sketch passes
FP32_LANES_PER_SM = 128


def time_grouping(jolt, K, spec, stream, power_iters=4, reps=3):
    """jolt_layer_groups on the resident key cache: device time per call
    (CUDA events on the launching stream, one warm-up call). Each call makes
    2 * power_iters + 2 passes over the keys (X Z and X^T Q, 16 columns, fp32
    FMAs); the roofline is that FMA work against the fp32 ALU peak."""
    import torch
    jolt.jolt_layer_groups(K, spec.rope_theta_k, power_iters, 0, stream)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        starts, _s = jolt.jolt_layer_groups(K, spec.rope_theta_k, power_iters, 0, stream)
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / reps
    sm = torch.cuda.get_device_properties(K.device).multi_processor_count
    out = {"ms_per_call": round(ms, 3), "power_iters": power_iters, "passes_over_keys": 2 * power_iters + 2,
           "n_groups": len(starts) - 1}
    out["roofline"] = grouping_roofline(ms, K.numel(), K.element_size(), power_iters, sm)
    return out


def grouping_roofline(ms, n_keys, elem_bytes, power_iters, sm_count, sketch=16, clock_hz=1.965e9):
    """The grouping's sketch passes against the fp32 FMA peak: 2 * power_iters
    + 2 passes over the keys, each 2 * sketch flops per key element."""
    passes = 2 * power_iters + 2
    flops = passes * 2.0 * n_keys * sketch
    peak = sm_count * FP32_LANES_PER_SM * 2 * clock_hz / 1e12
    ach = flops / (ms / 1e3) / 1e12
    return {"bound": "alu", "achieved": round(ach, 2), "peak": round(peak, 1), "unit": "TFLOP/s",
            "frac": round(ach / peak, 3),
            "peak_source": f"derived: {sm_count} SMs x {FP32_LANES_PER_SM} fp32 lanes x 2 x {clock_hz / 1e6:.0f} MHz",
            "key_gb_read": round(passes * n_keys * elem_bytes / 1e9, 2)}


def decode_roofline(ms, cells_k, cells_v, spec, G, pk, src, sm_count, clock_hz=1.965e9):
    """The fused decode kernel of one layer against its bounds: the bytes it
    must read (each sequence's U_T^ rows of K and V once, every head's codes
    and scales), the tensor-core flops of the key backbone (2 r_T D per
    token-head) and the fp32 flops of the scores and the rank-space values
    (2 G (D + r_T^V + D) per token-head). The slowest bound is the roofline."""
    H, T, D = spec.n_heads, spec.seq_len, spec.head_dim
    nbytes = tc = alu = 0.0
    for ck, cv in zip(cells_k, cells_v):
        for c in (ck, cv):
            # U_T^ rows, then per head and token b*D/8 code bytes and one fp32
            # scale (one scale group per row, the default)
            nbytes += 2.0 * c.r_t * T + H * T * (c.bits * D / 8 + (4.0 if c.bits else 0.0))
        tc += 2.0 * ck.r_t * D * T * H
        alu += 2.0 * G * (2 * D + cv.r_t) * T * H
    alu_peak = sm_count * 128 * 2 * clock_hz
    t_bytes = nbytes / (pk["hbm_gbs"] * 1e9)
    t_tc = tc / (pk["bf16_tflops"] * 1e12)
    t_alu = alu / alu_peak
    bound = max((t_bytes, "hbm"), (t_tc, "tensor"), (t_alu, "alu"))
    return {"bound": bound[1], "bound_ms": round(1e3 * bound[0], 4), "frac": round(1e3 * bound[0] / ms, 3),
            "payload_gb": round(nbytes / 1e9, 4), "payload_gb_s": round(nbytes / (ms / 1e3) / 1e9, 1),
            "peaks": f"{src} HBM {pk['hbm_gbs']} GB/s, {src} bf16 burst {pk['bf16_tflops']} TF/s, "
                     f"fp32 FMA {alu_peak / 1e12:.1f} TF/s (derived)"}


def time_decode(jolt, h, K, V, Ko, Vo, spec, stream, cells, ncell_per_seq, pk, src, reps=20):
    """One fused decode step of layer 0 (every sequence, G = 4 query heads per
    KV head as in LLaMA-3.1-8B, no tail) against reconstruct-then-attend:
    decompress of the whole cache per step amortised over the layers, plus
    torch's attention over the dense bf16 layer."""
    import torch
    B, H, D = spec.batch, spec.n_heads, spec.head_dim
    G = 4
    q = torch.randn((B, H * G, D), device=K.device, dtype=torch.float32)
    out = torch.empty_like(q)
    for _ in range(3):
        jolt.jolt_decode_attention(h, 0, q, out, None, None, stream)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        jolt.jolt_decode_attention(h, 0, q, out, None, None, stream)
    e1.record(stream)
    torch.cuda.synchronize()
    ms_fused = e0.elapsed_time(e1) / reps
    # dense attention over the (already decompressed) bf16 layer
    qq = q.to(torch.bfloat16)[:, :, None, :]
    Kl = Ko[:, 0].repeat_interleave(G, 1)
    Vl = Vo[:, 0].repeat_interleave(G, 1)
    for _ in range(3):
        torch.nn.functional.scaled_dot_product_attention(qq, Kl, Vl)
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(reps):
        torch.nn.functional.scaled_dot_product_attention(qq, Kl, Vl)
    e1.record(stream)
    torch.cuda.synchronize()
    ms_dense = e0.elapsed_time(e1) / reps
    e0.record(stream)
    for _ in range(3):
        jolt.jolt_decompress(h, Ko, Vo, None, stream)
    e1.record(stream)
    torch.cuda.synchronize()
    ms_decomp_layer = e0.elapsed_time(e1) / 3 / spec.n_layers
    # layer 0 lives in group 0: the K and V cells of group 0 of every sequence
    ck = [cells[b * ncell_per_seq + 0] for b in range(B)]
    cv = [cells[b * ncell_per_seq + 1] for b in range(B)]
    sm = torch.cuda.get_device_properties(K.device).multi_processor_count
    return {"layer": 0, "query_heads_per_kv_head": G, "ms_per_layer": round(ms_fused, 4),
            "reconstruct_then_attend_ms": round(ms_decomp_layer + ms_dense, 4),
            "dense_attention_only_ms": round(ms_dense, 4),
            "roofline": decode_roofline(ms_fused, ck, cv, spec, G, pk, src, sm)}


def time_e2e(jolt, shard, plan, B, ncell, K, V, Ko, Vo, stream, world, dist, dev, dense, steps):
    """The step end to end: every step copies its K and V from pinned host
    memory to the device, compresses and decompresses them through the C ABI,
    and copies the decompressed K and V back to pinned host memory.

    Two figures. `serial`: copy in, compute, copy out, one after the other on
    one stream. `value`: the same steps double-buffered, as a server that
    compresses a stream of prefill caches would run them: the copy in of step
    i+1 (one copy stream) and the copy out of step i-1 (another) overlap the
    kernels of step i; the timed region spans the first copy in to the last
    copy out, so it holds every step's copies."""
    import torch

    Kh = torch.empty(K.shape, dtype=K.dtype, pin_memory=True)
    Vh = torch.empty(V.shape, dtype=V.dtype, pin_memory=True)
    Kh.copy_(K)
    Vh.copy_(V)
    Koh = torch.empty_like(Kh, pin_memory=True)
    Voh = torch.empty_like(Vh, pin_memory=True)
    # slot 0 reuses the bench's own buffers, slot 1 is a second set
    kin = [K, torch.empty_like(K)]
    vin = [V, torch.empty_like(V)]
    kout = [Ko, torch.empty_like(Ko)]
    vout = [Vo, torch.empty_like(Vo)]
    torch.cuda.synchronize()

    def compress(k, v):
        if world > 1:
            h, _, _ = shard.compress_sharded(plan, k, v, B, 1234, None, stream, counts=[ncell] * world)
        else:
            h = jolt.jolt_compress(plan, k, v, B, 1234, stream)
        return h

    def run_serial():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        for _ in range(steps):
            kin[0].copy_(Kh, non_blocking=True)
            vin[0].copy_(Vh, non_blocking=True)
            hh = compress(kin[0], vin[0])
            jolt.jolt_decompress(hh, kout[0], vout[0], None, stream)
            Koh.copy_(kout[0], non_blocking=True)
            Voh.copy_(vout[0], non_blocking=True)
            jolt.jolt_free_handle(hh)
        f1.record(stream)
        torch.cuda.synchronize()
        return max_over_ranks(f0.elapsed_time(f1), world, dist, dev)

    def run_pipelined():
        s_in = torch.cuda.Stream(device=dev)
        s_out = torch.cuda.Stream(device=dev)
        ev = lambda: torch.cuda.Event()  # noqa: E731
        in_ready = [ev(), ev()]
        in_free = [None, None]      # compress of the slot's previous step done
        out_ready = [ev(), ev()]
        out_free = [None, None]     # copy out of the slot's previous step done
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        s_in.wait_event(f0)
        s_out.wait_event(f0)

        def copy_in(i):
            j = i % 2
            with torch.cuda.stream(s_in):
                if in_free[j] is not None:
                    s_in.wait_event(in_free[j])
                kin[j].copy_(Kh, non_blocking=True)
                vin[j].copy_(Vh, non_blocking=True)
                in_ready[j].record(s_in)

        copy_in(0)
        last = None
        for i in range(steps):
            j = i % 2
            if i + 1 < steps:
                copy_in(i + 1)
            stream.wait_event(in_ready[j])
            if out_free[j] is not None:
                stream.wait_event(out_free[j])
            hh = compress(kin[j], vin[j])
            in_free[j] = torch.cuda.Event()
            in_free[j].record(stream)
            jolt.jolt_decompress(hh, kout[j], vout[j], None, stream)
            out_ready[j].record(stream)
            jolt.jolt_free_handle(hh)
            with torch.cuda.stream(s_out):
                s_out.wait_event(out_ready[j])
                Koh.copy_(kout[j], non_blocking=True)
                Voh.copy_(vout[j], non_blocking=True)
                out_free[j] = torch.cuda.Event()
                out_free[j].record(s_out)
                last = out_free[j]
        stream.wait_event(last)
        f1.record(stream)
        torch.cuda.synchronize()
        return max_over_ranks(f0.elapsed_time(f1), world, dist, dev)

    run_pipelined()                      # one untimed pass: streams, pinned pages, pool
    sms = run_serial()
    pms = run_pipelined()
    n = min(Koh.numel(), 1 << 20)
    last = kout[(steps - 1) % 2].reshape(-1)
    ok = bool(torch.equal(Koh.reshape(-1)[:n], last[:n].cpu()) and torch.equal(Koh.reshape(-1)[-n:], last[-n:].cpu()))
    del kin[1], vin[1], kout[1], vout[1]
    return {"value": round(throughput_gbs(world, dense, steps, pms), 3), "unit": "GB/s",
            "h2d_bytes_per_step": 2 * K.numel() * K.element_size(),
            "d2h_bytes_per_step": 2 * Ko.numel() * Ko.element_size(),
            "steps": steps, "ms_per_step": round(pms / steps, 3),
            "overlap": "double-buffered: step i+1's copy in and step i-1's copy out run on two copy streams "
                       "beside step i's kernels; pinned host buffers",
            "serial": {"value": round(throughput_gbs(world, dense, steps, sms), 3),
                       "ms_per_step": round(sms / steps, 3)},
            "copy_out_matches_device": ok}


def run_jolt(args):
    import torch
    import torch.distributed as dist
    from tucker_quantized_residual_b200 import jolt, shard, synth

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    spec = synth.SPECS[args.config]
    if args.groups:
        spec = spec.replace(n_layers=min(spec.n_layers, args.groups * spec.group_size))
    gs = synth.group_starts(spec)
    # with N ranks the job compresses N times the cache under ONE shared
    # budget: rank r holds sequences [r*B, (r+1)*B) of the whole batch
    K, V = synth.make_cache(spec, seed=1000 * rank, device="cuda")
    torch.cuda.synchronize()
    dense = synth.dense_bf16_bytes(spec)
    mode = jolt.JOLT_RANDOMIZED if args.mode == "randomized" else jolt.JOLT_EXACT
    lay, keep = jolt.make_layout(K, gs, spec.rope_theta_k)
    Ko = torch.empty_like(K)
    Vo = torch.empty_like(V)
    stream = torch.cuda.current_stream()

    def make_plan(ratio):
        B_all = int(math.floor(dense * world / ratio))
        opt, keep2 = jolt.make_options(mode=mode, seq_base=rank * spec.batch, cap_ratio=ratio)
        return jolt.jolt_plan(lay, B_all, opt), B_all

    def step_fn(plan, B_all):
        def step():
            if world > 1:
                h, _, _ = shard.compress_sharded(plan, K, V, B_all, 1234, None, stream,
                                                 counts=[jolt.jolt_num_cells(plan)] * world)
            else:
                h = jolt.jolt_compress(plan, K, V, B_all, 1234, stream)
            jolt.jolt_decompress(h, Ko, Vo, None, stream)
            return h
        return step

    def timed(step, steps):
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(steps):
            jolt.jolt_free_handle(step())
        e1.record(stream)
        torch.cuda.synchronize()
        return max_over_ranks(e0.elapsed_time(e1), world, dist, dev)

    plan, B = make_plan(args.ratio)
    ncell = jolt.jolt_num_cells(plan)
    step = step_fn(plan, B)
    for _ in range(args.warmup):
        jolt.jolt_free_handle(step())
    torch.cuda.synchronize()
    # one synchronised step for the allocation report
    h = step()
    cells, lam, iters = jolt.jolt_handle_info(h, ncell)
    nbytes = jolt.jolt_bytes(h)
    jolt.jolt_free_handle(h)

    # ---- timed region (device time, CUDA events on the launching stream)
    clocks = ClockSampler(local)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    jolt.jolt_profile_enable(True)
    l0 = jolt.jolt_launch_count()
    clocks.start()
    ms = timed(step, args.steps)
    clk = clocks.stop()
    launches = jolt.jolt_launch_count() - l0
    prof = jolt.jolt_profile_read()
    jolt.jolt_profile_enable(False)
    value = throughput_gbs(world, dense, args.steps, ms)
    errK = errV = None
    if rank == 0:
        errK = rel_err(K, Ko)
        errV = rel_err(V, Vo)

    # ---- the other budgets of the workload (same cache, same step)
    budgets = {}
    ratios = [float(x) for x in args.extra_ratios.split(",") if x.strip()] if args.extra_ratios else []
    for r in ratios:
        pr, Br = make_plan(r)
        st = step_fn(pr, Br)
        for _ in range(2):
            jolt.jolt_free_handle(st())
        msr = timed(st, args.extra_steps)
        hh = st()
        nb = jolt.jolt_bytes(hh)
        jolt.jolt_free_handle(hh)
        budgets[f"{r:g}x"] = {"value": round(throughput_gbs(world, dense, args.extra_steps, msr), 3),
                              "ms_per_step": round(msr / args.extra_steps, 3), "bytes": nb, "budget": Br,
                              "rel_frobenius_err": {"K": rel_err(K, Ko), "V": rel_err(V, Vo)} if rank == 0 else None}
        jolt.jolt_free_plan(pr)

    # ---- end to end through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        e2e = time_e2e(jolt, shard, plan, B, ncell, K, V, Ko, Vo, stream, world, dist, dev, dense, args.e2e_steps)

    pk, src = peaks()
    # ---- data-driven layer grouping and fused decode attention (outside the
    # timed region, rank 0)
    grouping = decode = None
    if rank == 0 and not args.no_grouping:
        grouping = time_grouping(jolt, K, spec, stream)
    if rank == 0 and world == 1 and not args.no_decode:
        h = step()
        decode = time_decode(jolt, h, K, V, Ko, Vo, spec, stream, cells, ncell // spec.batch, pk, src)
        jolt.jolt_free_handle(h)

    # ---- roofline: the dominant kernel, and the whole path per stage
    work = stage_work(spec, cells, sketch_width(spec, args.ratio))
    per_step = {s_: prof[s_][0] / args.steps for s_ in prof}
    tc = pk["bf16_tflops_sustained"] * 1e12
    bw = pk["hbm_gbs"] * 1e9
    # the tcgen05 GEMM kernel (its X W and X^T Y launches) against the stream passes
    gemm_ms = per_step.get("gemm_xw", 0.0) + per_step.get("gemm_xty", 0.0)
    cand = {"gemm": gemm_ms, "residual": per_step.get("residual", 0.0),
            "decompress": per_step.get("decompress", 0.0)}
    dom = max(cand, key=cand.get)
    if dom == "gemm":
        fl = work["gemm_xw"][0] + work["gemm_xty"][0]
        nl = work["gemm_xw"][2] + work["gemm_xty"][2]
        per_launch_s = gemm_ms / 1e3 / nl
        ach = fl / nl / per_launch_s / 1e12
        traffic = GEMM_TRAFFIC.get(args.config) if (GEMM_TRAFFIC and not args.groups and args.ratio == 2.0) else None
        roof = {"bound": "tensor", "kernel": "k_umma_gemm_pair (X W and X^T Y launches)", "achieved": round(ach, 1),
                "peak": pk["bf16_tflops_sustained"], "unit": "TFLOP/s", "frac": round(ach / pk["bf16_tflops_sustained"], 3),
                "peak_source": f"{src} bf16 sustained", "flops_per_launch": fl / nl,
                "traffic": traffic}
    else:
        fl, by, nl = work[dom]
        per_launch_s = cand[dom] / 1e3 / nl
        if fl / tc > by / bw:
            ach = fl / nl / per_launch_s / 1e12
            roof = {"bound": "tensor", "kernel": f"k_stream ({dom})", "achieved": round(ach, 1),
                    "peak": pk["bf16_tflops_sustained"], "unit": "TFLOP/s",
                    "frac": round(ach / pk["bf16_tflops_sustained"], 3), "peak_source": f"{src} bf16 sustained",
                    "traffic": None}
        else:
            ach = by / nl / per_launch_s / 1e9
            roof = {"bound": "hbm", "kernel": f"k_stream ({dom})", "achieved": round(ach, 1), "peak": pk["hbm_gbs"],
                    "unit": "GB/s", "frac": round(ach / pk["hbm_gbs"], 3), "peak_source": f"{src} copy bandwidth",
                    "traffic": None}
    bound_ms = 0.0
    for st_, (fl, by, nl) in work.items():
        bound_ms += 1e3 * max(fl / tc, by / bw)
    path_roof = {"bound_ms": round(bound_ms, 3), "ms_per_step": round(ms / args.steps, 3),
                 "frac": round(bound_ms / (ms / args.steps), 3),
                 "rule": "sum over GEMM passes, residual and decode of max(flops / sustained bf16, bytes / HBM)"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(spec, args.ratio, args.cpu_tokens, args.cpu_reps)

    if args.stages and rank == 0:
        for s in jolt.STAGES:
            msx, calls, ln = prof[s]
            if calls:
                sys.stderr.write(f"{s:12s} {msx / args.steps:9.3f} ms/step  calls {calls / args.steps:5.1f}  "
                                 f"launches {ln / args.steps:6.1f}\n")
        sys.stderr.write(f"alloc: lambda {lam:.3e} iters {iters} bytes {nbytes} budget {B}\n")
        for c in cells[:6]:
            sys.stderr.write(f"  cell g{c.group} {'KV'[c.kind]}: r_T {c.r_t} r_d {c.r_d} b {c.bits}\n")

    if rank == 0:
        line = {
            "metric": "GB/s of bf16 KV cache compressed+decompressed at 2x/3x budget; rel. Frobenius err",
            "value": round(value, 3), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms / args.steps, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": arm_config(args, spec, world),
            "rel_frobenius_err": {"K": errK, "V": errV}, "bytes": nbytes, "budget": B,
            "budgets": budgets,
            "roofline": roof, "path_roofline": path_roof, "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": int(launches),
            "clocks": clk, "layer_grouping": grouping, "decode_attention": decode,
            "stages_ms_per_step": {s: round(v, 3) for s, v in per_step.items() if v > 0},
        }
        print(json.dumps(line), flush=True)
    jolt.jolt_free_plan(plan)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def rel_err(X, Xh):
    import torch
    num = 0.0
    den = 0.0
    for l in range(X.shape[1]):
        a = X[:, l].float()
        b = Xh[:, l].float()
        num += float(((a - b) ** 2).sum())
        den += float((a * a).sum())
    return round(math.sqrt(num / den), 6)


# ---------------------------------------------------------- CPU baseline
# Both CPU legs (the cpu_baseline object and --impl reference) time the same
# sample: layer group 0 (its K and V cells) of sequence 0 of the workload's
# cache, its first CPU_TOKENS tokens, regenerated on the host from the same
# seeded generator, compressed and decompressed by the oracle (exact JoLT in
# fp64) with the token rank capped at Eq. (5)'s q_cap of the full sequence.
CPU_TOKENS = 1024


def cpu_sample(spec, T_sample):
    from tucker_quantized_residual_b200 import synth
    spec_s = spec.replace(seq_len=T_sample, n_layers=spec.group_size, batch=1)
    K, V = synth.make_cache(spec_s, seed=0)
    return K.float().numpy(), V.float().numpy()


def run_oracle_sample(Ks, Vs, spec, ratio):
    from oracle import jolt_oracle as o
    n = Ks.size + Vs.size
    B = o.budget_for_ratio(n, ratio)
    q = o.q_cap(spec.seq_len, ratio)
    opt = o.Options(rt_max=q)
    t0 = time.perf_counter()
    comp = o.compress(Ks, Vs, [0, spec.group_size], B, 0, opt, spec.rope_theta_k)
    o.decompress(comp)
    return time.perf_counter() - t0, 2 * n


def sample_text(spec, T_sample, reps):
    return (f"layer group 0 (K and V cells) of sequence 0 of a {spec.name}-shaped cache, first {T_sample} tokens "
            f"(regenerated on the host from the same seeded generator), exact JoLT in fp64 (numpy/OpenBLAS) with "
            f"the token rank capped at q_cap = {min(max(32, -(-spec.seq_len // 32)), 512)}; {reps} repetition(s) "
            f"per measurement")


def cpu_baseline(spec, ratio, T_sample=CPU_TOKENS, reps=8):
    Ks, Vs = cpu_sample(spec, T_sample)
    total = 0.0
    nb = 0
    for _ in range(reps):
        sec, nbytes = run_oracle_sample(Ks, Vs, spec, ratio)
        total += sec
        nb += nbytes
    return {"value": round(nb / total / 1e9, 6), "unit": "GB/s", "cores": os.cpu_count(), "kind": "oracle",
            "sample": sample_text(spec, T_sample, reps) + f", {nb / 1e6:.1f} MB dense bf16 in {total:.2f} s"}


def arm_config(args, spec, world):
    """The workload both arms report (the reference arm times a bounded sample
    of it, described in its cpu_baseline)."""
    from tucker_quantized_residual_b200 import synth
    dense = synth.dense_bf16_bytes(spec)
    par = (f"one shared byte budget over {world} GPUs: rank r compresses sequences [r*{spec.batch}, "
           f"(r+1)*{spec.batch}), one all-gather of per-cell rate-distortion records per step (NCCL)"
           if world > 1 else "one GPU")
    return {"workload": f"{args.config} ({spec.n_layers} layers / groups of {spec.group_size}, "
                        f"{spec.n_heads} KV heads, D={spec.head_dim}, T={spec.seq_len}, "
                        f"batch {spec.batch} per GPU), {args.ratio:g}x budget, {args.mode} token SVD",
            "global_batch": spec.batch * world, "seq_len": spec.seq_len,
            "parallelism": par,
            "l2": f"inputs {dense / 1e9:.2f} GB per GPU" + (
                ", larger than L2; no flush" if dense > 126e6 else ", smaller than L2")}


def run_reference(args):
    """The oracle arm: the same bounded sample as the cpu_baseline leg, on the
    host cores, one sample per step."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from tucker_quantized_residual_b200 import synth
    spec = synth.SPECS[args.config]
    if args.groups:
        spec = spec.replace(n_layers=min(spec.n_layers, args.groups * spec.group_size))
    T_sample = args.cpu_tokens
    Ks, Vs = cpu_sample(spec, T_sample)
    for _ in range(args.warmup):
        run_oracle_sample(Ks, Vs, spec, args.ratio)
    total = 0.0
    nb = 0
    for _ in range(args.steps):
        sec, nbytes = run_oracle_sample(Ks, Vs, spec, args.ratio)
        total += sec
        nb += nbytes
    value = nb / total / 1e9
    line = {"impl": "reference",
            "metric": "GB/s of bf16 KV cache compressed+decompressed at 2x/3x budget; rel. Frobenius err",
            "value": round(value, 6), "unit": "GB/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(1e3 * total / args.steps, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": arm_config(args, spec, int(os.environ.get("WORLD_SIZE", "1"))),
            "cpu_baseline": {"value": round(value, 6), "unit": "GB/s", "cores": os.cpu_count(), "kind": "oracle",
                             "sample": sample_text(spec, T_sample, 1)},
            "e2e": {"value": round(value, 6), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_jolt(args)


if __name__ == "__main__":
    main()
