"""The shared-budget protocol through the C ABI on one GPU: the cache is split
into two shards (by sequence, or by layer group), each shard has its own plan
(seq_base / group_base set) and runs jolt_compress_begin; the two record
buffers are concatenated in rank order, which is what the all-gather of two
ranks produces; then each shard runs jolt_compress_end on the whole buffer.
The shards run one after the other on one stream, so no kernel waits for
another process. Every cell's allocation, the multiplier and the
decompressed cache must equal a single jolt_compress over the whole cache
bit for bit (the same kernels on the same cells, and the same deterministic
bisection over the same records)."""
import numpy as np
import pytest
import torch

from oracle import jolt_oracle as o
from tucker_quantized_residual_b200 import jolt, shard, synth

pytestmark = pytest.mark.gpu


def _whole(K, V, gs, B, seed, theta, **kw):
    lay, keep = jolt.make_layout(K, gs, theta)
    opt, k2 = jolt.make_options(**kw)
    plan = jolt.jolt_plan(lay, B, opt)
    h = jolt.jolt_compress(plan, K, V, B, seed)
    Ko, Vo = torch.empty_like(K, dtype=torch.bfloat16), torch.empty_like(V, dtype=torch.bfloat16)
    jolt.jolt_decompress(h, Ko, Vo)
    cells, lam, it = jolt.jolt_handle_info(h, jolt.jolt_num_cells(plan))
    jolt.jolt_free_handle(h)
    jolt.jolt_free_plan(plan)
    return Ko, Vo, [(c.seq, c.group, c.kind, c.r_t, c.r_d, c.bits, c.bytes) for c in cells], lam


def _sharded(shards, B, seed, theta, **kw):
    """shards: list of (K view, V view, group starts, seq_base, group_base).
    Every shard's plan gets the whole cache's compression ratio for Eq. (5)."""
    dense = sum(2 * 2 * Ks.numel() for Ks, _, _, _, _ in shards)
    kw = dict(kw, cap_ratio=dense / B)
    plans, handles, bufs, keeps = [], [], [], []
    for Ks, Vs, gs, sb, gb in shards:
        lay, keep = jolt.make_layout(Ks, gs, theta)
        opt, k2 = jolt.make_options(seq_base=sb, group_base=gb, **kw)
        keeps += [keep, k2]
        plan = jolt.jolt_plan(lay, B, opt)
        n, rb = jolt.jolt_num_cells(plan), jolt.jolt_summary_bytes(plan)
        buf = torch.zeros(n * rb, dtype=torch.uint8, device="cuda")
        handles.append(jolt.jolt_compress_begin(plan, Ks, Vs, B, seed, buf))
        plans.append(plan)
        bufs.append(buf)
    allrec = torch.cat(bufs)                 # what an all-gather in rank order gives
    n_total = sum(jolt.jolt_num_cells(p) for p in plans)
    firsts = shard.first_cells([jolt.jolt_num_cells(p) for p in plans])
    outs, cells, lams = [], [], []
    for (Ks, Vs, gs, sb, gb), plan, h, f in zip(shards, plans, handles, firsts):
        jolt.jolt_compress_end(h, allrec, n_total, f)
        Ko, Vo = torch.empty_like(Ks, dtype=torch.bfloat16), torch.empty_like(Vs, dtype=torch.bfloat16)
        jolt.jolt_decompress(h, Ko, Vo)
        ci, lam, it = jolt.jolt_handle_info(h, jolt.jolt_num_cells(plan))
        outs.append((Ko, Vo))
        cells += [(c.seq, c.group, c.kind, c.r_t, c.r_d, c.bits, c.bytes) for c in ci]
        lams.append(lam)
    torch.cuda.synchronize()
    recs = shard.decode_records(allrec.cpu().numpy().tobytes(), jolt.jolt_summary_bytes(plans[0]))
    for h in handles:
        jolt.jolt_free_handle(h)
    for p in plans:
        jolt.jolt_free_plan(p)
    return outs, cells, lams, recs


@pytest.mark.parametrize("mode", [jolt.JOLT_EXACT, jolt.JOLT_RANDOMIZED])
def test_split_by_sequence_equals_one_process(mode):
    spec = synth.SPECS["mistral"].replace(n_layers=8, batch=3, seq_len=512)
    K, V = synth.make_cache(spec, 0, device="cuda")
    gs = synth.group_starts(spec)
    B = o.budget_for_ratio(K.numel() * 2, 3.0)
    theta = spec.rope_theta_k
    Kw, Vw, cells_w, lam_w = _whole(K, V, gs, B, 5, theta, mode=mode)
    outs, cells_s, lams, recs = _sharded([(K[0:2], V[0:2], gs, 0, 0), (K[2:3], V[2:3], gs, 2, 0)], B, 5, theta,
                                         mode=mode)
    assert cells_s == cells_w
    assert lams == [lam_w, lam_w]
    assert [(r["seq"], r["group"], r["kind"]) for r in recs] == [(c[0], c[1], c[2]) for c in cells_w]
    assert torch.equal(torch.cat([outs[0][0], outs[1][0]]), Kw)
    assert torch.equal(torch.cat([outs[0][1], outs[1][1]]), Vw)


def test_split_by_layer_group_equals_one_process():
    spec = synth.SPECS["mistral"].replace(n_layers=12, seq_len=1024)
    K, V = synth.make_cache(spec, 0, device="cuda")
    gs = synth.group_starts(spec)                                 # [0, 4, 8, 12]
    B = o.budget_for_ratio(K.numel() * 2, 2.0)
    theta = spec.rope_theta_k
    Kw, Vw, cells_w, lam_w = _whole(K, V, gs, B, 9, theta, mode=jolt.JOLT_RANDOMIZED)
    shards = [(K[:, 0:4].contiguous(), V[:, 0:4].contiguous(), [0, 4], 0, 0),
              (K[:, 4:12].contiguous(), V[:, 4:12].contiguous(), [0, 4, 8], 0, 1)]
    outs, cells_s, lams, recs = _sharded(shards, B, 9, theta, mode=jolt.JOLT_RANDOMIZED)
    # cell order of the gathered records is rank order, which here is the
    # single plan's order too (sequence, then group, then kind)
    assert cells_s == cells_w
    assert lams == [lam_w, lam_w]
    assert torch.equal(torch.cat([outs[0][0], outs[1][0]], dim=1), Kw)
    assert torch.equal(torch.cat([outs[0][1], outs[1][1]], dim=1), Vw)


def _begun(K, V, gs, B, theta, i, **kw):
    lay, keep = jolt.make_layout(K[i:i + 1], gs, theta)
    opt, k2 = jolt.make_options(seq_base=i, **kw)
    plan = jolt.jolt_plan(lay, B, opt)
    buf = torch.zeros(jolt.jolt_num_cells(plan) * jolt.jolt_summary_bytes(plan), dtype=torch.uint8, device="cuda")
    h = jolt.jolt_compress_begin(plan, K[i:i + 1], V[i:i + 1], B, 0, buf)
    return plan, h, buf


def test_mismatched_settings_or_slice_are_reported():
    spec = synth.SPECS["mistral"].replace(n_layers=8, batch=2, seq_len=512)
    K, V = synth.make_cache(spec, 0, device="cuda")
    gs = synth.group_starts(spec)
    B = o.budget_for_ratio(K.numel() * 2, 3.0)
    th = spec.rope_theta_k
    made = [_begun(K, V, gs, B, th, 0), _begun(K, V, gs, B, th, 1, bits=(0, 4, 8)),
            _begun(K, V, gs, B, th, 1)]
    (p0, h0, b0), (p1, h1, b1), (p2, h2, b2) = made
    n = jolt.jolt_num_cells(p0)
    try:
        # before end, the handle is not a compressed cache
        with pytest.raises(jolt.JoltError) as ei:
            jolt.jolt_bytes(h0)
        assert ei.value.status == 1
        # records of a plan with other bit widths
        jolt.jolt_compress_end(h0, torch.cat([b0, b1]), 2 * n, 0)
        with pytest.raises(jolt.JoltError) as ei:
            jolt.jolt_bytes(h0)
        assert ei.value.status == 1 and "records" in str(ei.value)
        # same settings, but this plan's slice points at the other plan's cells
        jolt.jolt_compress_end(h2, torch.cat([b0, b2]), 2 * n, 0)
        with pytest.raises(jolt.JoltError) as ei:
            jolt.jolt_bytes(h2)
        assert ei.value.status == 1
        # a slice outside the buffer is refused before any work
        with pytest.raises(jolt.JoltError):
            jolt.jolt_compress_end(h1, b1, n, 1)
    finally:
        torch.cuda.synchronize()
        for p, h, b in made:
            jolt.jolt_free_handle(h)
            jolt.jolt_free_plan(p)
