"""The shared-budget protocol across processes (host side, CPU, two gloo
ranks): cells split by sequence over the ranks, one summary record per cell,
one all-gather of records whose count differs between ranks, and the same
multiplier bisection on every rank. The device steps (spectra, tables) are
stood in for by the oracle's tables packed into the library's record format;
what is tested is the exchange: the split, the gather order with uneven
counts, the record codec (fp64 tables bit for bit) and that every rank then
reaches the single-process allocation exactly (Section 3, "Solving the
allocation": the problem separates across cells once lambda is fixed)."""
import datetime
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

OPT = dict(bits=(0, 2, 3, 4, 8), rt_grid=(8, 16, 32, 64), rd_grid=(16, 32, 48))
NSEQ = 3


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _cache():
    from tucker_quantized_residual_b200 import synth
    spec = synth.SPECS["tiny"].replace(batch=NSEQ)
    K, V = synth.make_cache(spec, 0)
    return spec, K.numpy(), V.numpy()


def _tables(K, V, spec, seqs):
    from oracle import jolt_oracle as o
    opt = o.Options(**OPT)
    eps = o.eps2_table(opt.bits, spec.head_dim)
    gs = [0, spec.n_layers]
    out = []
    for c in o.cells_of(NSEQ, gs):
        if c.b in seqs:
            X = o.cell_tensor(K, V, c, 0.0)
            out.append((c, o.build_table(X, opt, eps)[0]))
    return out


def _record(c, tab, ntp, rec_bytes):
    from tucker_quantized_residual_b200 import shard
    return shard.encode_record(dict(Lg=tab.Lg, H=tab.H, T=tab.T, D=tab.D, n_rt=len(tab.rt_grid),
                                    nt=len(tab.tT) - 1, ntp=ntp, fingerprint=0xC0FFEE, norm_sq=tab.normsq,
                                    seq=c.b, group=c.g, kind=c.kind, tT=list(tab.tT), tD=list(tab.tD)), rec_bytes)


def _table_from(rec, like):
    from oracle import jolt_oracle as o
    return o.CellTable(rec["Lg"], rec["H"], rec["T"], rec["D"], like.g, rec["norm_sq"],
                       np.array(rec["tT"][:rec["nt"] + 1]), np.array(rec["tD"]), like.rt_grid, like.rd_grid,
                       like.bits, like.eps2)


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import torch
    import torch.distributed as dist
    from oracle import jolt_oracle as o
    from tucker_quantized_residual_b200 import shard
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        spec, K, V = _cache()
        s0, s1 = shard.shard_range(NSEQ, world, rank)
        mine = _tables(K, V, spec, range(s0, s1))
        ntp = spec.seq_len + 1
        rb = (64 + 8 * ntp + 8 * (spec.head_dim + 1) + 255) // 256 * 256
        local = torch.frombuffer(bytearray(b"".join(_record(c, t, ntp, rb) for c, t in mine)), dtype=torch.uint8)
        allrec, counts = shard.gather_records(local, len(mine), rb)
        first = shard.first_cells(counts)[rank]
        recs = shard.decode_records(allrec.numpy().tobytes(), rb)
        # this rank's own records sit at its offset, unchanged
        for i, (c, t) in enumerate(mine):
            r = recs[first + i]
            assert (r["seq"], r["group"], r["kind"]) == (c.b, c.g, c.kind)
            assert np.array_equal(np.array(r["tT"][:len(t.tT)]), t.tT)
            assert np.array_equal(np.array(r["tD"]), t.tD)
        like = mine[0][1]
        tabs = [_table_from(r, like) for r in recs]
        B = o.budget_for_ratio(2 * K.size, 2.5)
        al = o.allocate(tabs, B)
        q.put((rank, counts, first, [(r["seq"], r["kind"]) for r in recs], al.choice, al.lam, al.bytes))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_reach_the_single_process_allocation():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
    alive = [p for p in procs if p.is_alive()]
    for p in alive:
        p.kill()
    assert not alive and all(p.exitcode == 0 for p in procs)
    got = sorted(q.get(timeout=10) for _ in range(2))
    # the single-process allocation over every cell
    sys.path.insert(0, ROOT)
    from oracle import jolt_oracle as o
    spec, K, V = _cache()
    tabs = [t for _, t in _tables(K, V, spec, range(NSEQ))]
    ref = o.allocate(tabs, o.budget_for_ratio(2 * K.size, 2.5))
    for rank, counts, first, order, choice, lam, nbytes in got:
        assert counts == [4, 2]                      # sequences 0-1 on rank 0, sequence 2 on rank 1
        assert first == [0, 4][rank]
        assert order == [(b, k) for b in range(NSEQ) for k in (0, 1)]
        assert choice == ref.choice and lam == ref.lam and nbytes == ref.bytes


def test_shard_range_covers_every_unit_once():
    from tucker_quantized_residual_b200 import shard
    for n in range(1, 40):
        for world in range(1, min(n, 9) + 1):
            spans = [shard.shard_range(n, world, r) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == n
            assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
            sizes = [b - a for a, b in spans]
            assert max(sizes) - min(sizes) <= 1 and min(sizes) >= 1
    with pytest.raises(ValueError):
        shard.shard_range(2, 3, 0)
    assert shard.first_cells([4, 2, 3]) == [0, 4, 6]


def test_record_codec_round_trip():
    from tucker_quantized_residual_b200 import shard
    rec = dict(Lg=4, H=8, T=1024, D=128, n_rt=32, nt=33, ntp=34, fingerprint=2 ** 63 + 5, norm_sq=1.5e6,
               seq=3, group=7, kind=1, tT=[1.0 / (i + 3) for i in range(34)], tD=[2.0 ** -i for i in range(129)])
    rb = (64 + 8 * 34 + 8 * 129 + 255) // 256 * 256
    buf = shard.encode_record(rec, rb)
    assert len(buf) == rb
    back = shard.decode_records(buf + buf, rb)
    assert len(back) == 2
    for k, val in rec.items():
        assert back[1][k] == val, k
    assert back[0]["magic"] == shard.RD_MAGIC and back[0]["rec_bytes"] == rb
