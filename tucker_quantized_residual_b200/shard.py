"""One byte budget shared by several processes, one per GPU.

"A JoLT for the KV Cache" (Section 3, "Solving the allocation") picks every
cell's ranks and bit width with one Lagrange multiplier: once the multiplier
is fixed, the problem separates across cells. So the cells of a cache can be
split over GPUs, and only each cell's rate-distortion summary has to travel:
  1. every rank computes the spectra and rate-distortion tables of its own
     cells (jolt_compress_begin), one summary record per cell;
  2. one all-gather of the records (NCCL over NVLink, or gloo on CPU);
  3. every rank runs the same deterministic multiplier bisection over all
     cells, gets the same allocation bit for bit, and fits and encodes its
     own cells (jolt_compress_end).
The compressed cells stay where they were computed; decompression is local.

This module is the host side of that exchange: the split of units over
ranks, the gather of records whose count differs between ranks, and a
decoder of the record format (the library writes records on the device; the
decoder is for inspection and tests). The compress steps themselves run in
libjolt's kernels."""
from __future__ import annotations

import struct
from typing import Dict, List, Optional, Sequence, Tuple

RD_MAGIC = 0x3144524A
HEADER = struct.Struct("<I7iQd4i")          # 64 bytes, the library's RDRecordHdr
assert HEADER.size == 64


def shard_range(n_units: int, world: int, rank: int) -> Tuple[int, int]:
    """Contiguous, balanced split of n_units (sequences or layer groups) over
    `world` ranks: rank r gets [start, stop); the first n_units % world ranks
    get one more unit."""
    if world < 1 or not 0 <= rank < world or n_units < world:
        raise ValueError(f"cannot split {n_units} units over {world} ranks (rank {rank})")
    base, extra = divmod(n_units, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def first_cells(counts: Sequence[int]) -> List[int]:
    """Index of each rank's first record in the gathered buffer (records are
    gathered in rank order)."""
    out, acc = [], 0
    for c in counts:
        out.append(acc)
        acc += c
    return out


def gather_records(local, n_local: int, rec_bytes: int, group=None, counts=None):
    """All-gather every rank's records into one contiguous buffer in rank
    order, for any mix of per-rank counts. `local` is a uint8 tensor holding
    n_local records of rec_bytes each (on the device for NCCL, on the host for
    gloo). `counts` (every rank's record count) may be given when known, which
    saves an exchange and a host synchronisation. Returns (all_records,
    counts): all_records holds sum(counts) records, rank r's at
    first_cells(counts)[r]."""
    import torch
    import torch.distributed as dist
    world = dist.get_world_size(group)
    dev = local.device
    if counts is None:
        cnt = torch.tensor([n_local], dtype=torch.int64, device=dev)
        counts_t = torch.zeros(world, dtype=torch.int64, device=dev)
        dist.all_gather_into_tensor(counts_t, cnt, group=group)
        counts = [int(c) for c in counts_t.cpu().tolist()]
    counts = list(counts)
    if len(counts) != world or counts[dist.get_rank(group)] != n_local:
        raise ValueError("counts must list every rank's record count, this rank's included")
    cmax = max(counts)
    # equal-size contributions for the collective: pad to the largest count
    send = torch.zeros(cmax * rec_bytes, dtype=torch.uint8, device=dev)
    send[: n_local * rec_bytes] = local.reshape(-1)[: n_local * rec_bytes]
    recv = torch.empty(world * cmax * rec_bytes, dtype=torch.uint8, device=dev)
    dist.all_gather_into_tensor(recv, send, group=group)
    if all(c == cmax for c in counts):
        return recv, counts
    parts = [recv[r * cmax * rec_bytes: (r * cmax + counts[r]) * rec_bytes] for r in range(world)]
    return torch.cat(parts), counts


def decode_records(buf: bytes, rec_bytes: int) -> List[Dict]:
    """The records of a buffer as dictionaries: shape, grid length, global
    (seq, group, kind), fingerprint, ||X||^2 and the t_T / t_D tables."""
    out = []
    n = len(buf) // rec_bytes
    for i in range(n):
        rec = buf[i * rec_bytes:(i + 1) * rec_bytes]
        (magic, Lg, H, T, D, n_rt, nt, ntp, fp, nsq, seq, grp, kind, rb) = HEADER.unpack_from(rec, 0)
        tT = struct.unpack_from(f"<{ntp}d", rec, 64) if magic == RD_MAGIC else ()
        tD = struct.unpack_from(f"<{D + 1}d", rec, 64 + 8 * ntp) if magic == RD_MAGIC else ()
        out.append(dict(magic=magic, Lg=Lg, H=H, T=T, D=D, n_rt=n_rt, nt=nt, ntp=ntp, fingerprint=fp,
                        norm_sq=nsq, seq=seq, group=grp, kind=kind, rec_bytes=rb, tT=list(tT), tD=list(tD)))
    return out


def encode_record(rec: Dict, rec_bytes: int) -> bytes:
    """Inverse of decode_records for one record (for tests and tools that
    build records on the host)."""
    ntp, D = rec["ntp"], rec["D"]
    body = bytearray(rec_bytes)
    HEADER.pack_into(body, 0, RD_MAGIC, rec["Lg"], rec["H"], rec["T"], D, rec["n_rt"], rec["nt"], ntp,
                     rec["fingerprint"], rec["norm_sq"], rec["seq"], rec["group"], rec["kind"], rec_bytes)
    tT = list(rec["tT"]) + [0.0] * (ntp - len(rec["tT"]))
    struct.pack_into(f"<{ntp}d", body, 64, *tT)
    struct.pack_into(f"<{D + 1}d", body, 64 + 8 * ntp, *rec["tD"])
    return bytes(body)


def compress_sharded(plan: int, k, v, byte_budget: int, seed: int, group=None, stream=None, counts=None):
    """The whole protocol on this rank: begin (local spectra and records),
    all-gather of the records, end (shared allocation, local fit and
    residual). `counts`: every rank's cell count, when known. Returns
    (handle, counts, first_cell)."""
    import torch
    import torch.distributed as dist
    from . import jolt
    n = jolt.jolt_num_cells(plan)
    rb = jolt.jolt_summary_bytes(plan)
    local = torch.empty(n * rb, dtype=torch.uint8, device=k.device)
    h = jolt.jolt_compress_begin(plan, k, v, byte_budget, seed, local, stream)
    try:
        # the collective runs on the current stream: order it after begin's kernels
        if stream is not None and stream != torch.cuda.current_stream():
            torch.cuda.current_stream().wait_stream(stream)
        allrec, counts = gather_records(local, n, rb, group, counts)
        first = first_cells(counts)[dist.get_rank(group)]
        if stream is not None and stream != torch.cuda.current_stream():
            stream.wait_stream(torch.cuda.current_stream())
            allrec.record_stream(stream)        # read by end's kernels on `stream`
        jolt.jolt_compress_end(h, allrec, sum(counts), first, stream)
    except Exception:
        jolt.jolt_free_handle(h)
        raise
    return h, counts, first
