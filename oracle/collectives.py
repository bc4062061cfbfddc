"""The collectives, as the pages define them, on N virtual ranks (host arrays).

Test infrastructure only (see ``oracle/__init__.py``).

Each rank is a 1-D numpy array in storage type (bf16/fp16 as uint16 bits,
fp32, int32).  Functions return NEW arrays; where a collective leaves a rank's
buffer unspecified (gather / reduce on non-destination ranks) the caller's
buffer is the rank's result, untouched.

Citations are to the vLLM collectives tutorial (gsyq.cn/news/307221) by
section, to "From NCCL Ring LL to PCIe IPC AllReduce" (hjcheng0602.cn) by
section title, to the TP communication essay (52jiny.com thread-1337) and to
the sglang PR 27492 summary (prhub, ``all_to_all_single``).
"""
from __future__ import annotations

import numpy as np

from .numerics import ESIZE, combine, narrow, reduce_ranks, widen


def _copy(xs):
    return [np.array(x, copy=True) for x in xs]


# ---------------------------------------------------------- Broadcast ----

def broadcast(bufs, src: int):
    """Tutorial 1.1: the root's data is copied to every rank; afterwards all
    ranks hold identical data (no concatenation, no sum).  The sglang PR
    33307 summary ("key code") relies on every rank ending bit-identical."""
    return [np.array(bufs[src], copy=True) for _ in bufs]


# ------------------------------------------------------------- Gather ----

def gather(xs, dst_buf, rows: int = 1):
    """Tutorial 2.1 / 2.2.1: dst receives every rank's block concatenated in
    rank order; other ranks receive nothing.

    ``rows == 1``: flat concatenation.  ``rows > 1``: every rank holds a
    [rows, cols] block and the blocks are joined along the LAST dimension
    (the vocab-parallel logits picture ``logits[*, vocab_r]`` of 2.2.1).
    Returns the destination's buffer.
    """
    n = len(xs)
    cols = xs[0].size // rows
    out = np.array(dst_buf, copy=True).reshape(rows, n * cols)
    for r in range(n):
        out[:, r * cols:(r + 1) * cols] = np.asarray(xs[r]).reshape(rows, cols)
    return out.reshape(-1)


# ------------------------------------------------------------- Reduce ----

def reduce(xs, op: int, dtype: str):
    """Tutorial 3.1: same-shape data from every rank combined with SUM / MAX /
    MIN / PROD; only the destination holds the result (returned here)."""
    return reduce_ranks(xs, op, dtype)


# ------------------------------------------------------------ Scatter ----

def scatter(src_buf, nranks: int):
    """Tutorial 4.1: the root's full buffer is cut into N equal blocks and
    rank r receives block r (the inverse of Gather).  Reading: the length must
    be a multiple of N."""
    src_buf = np.asarray(src_buf)
    assert src_buf.size % nranks == 0
    c = src_buf.size // nranks
    return [np.array(src_buf[r * c:(r + 1) * c], copy=True) for r in range(nranks)]


# ------------------------------------------------------ ReduceScatter ----

def reduce_scatter(xs, op: int, dtype: str):
    """Tutorial 5.1 / 5.3: reduce, then cut the global result into N blocks;
    rank r keeps block r (the 2-GPU example: GPU0 gets [y0, y1], GPU1 gets
    [y2, y3])."""
    n = len(xs)
    full = reduce_ranks(xs, op, dtype)
    assert full.size % n == 0
    c = full.size // n
    return [np.array(full[r * c:(r + 1) * c], copy=True) for r in range(n)]


# ---------------------------------------------------------- AllReduce ----

def all_reduce(xs, op: int, dtype: str):
    """Tutorial 6.1: every rank receives the same complete reduction."""
    full = reduce_ranks(xs, op, dtype)
    return [np.array(full, copy=True) for _ in xs]


def segment_elems(count: int, nranks: int, dtype: str) -> int:
    """Length of one owner segment / ring chunk: ceil(count / N) rounded up to
    a whole 16-byte group.  The last segments may be short or empty.

    Reading: "From NCCL Ring LL ..." ("Pro5000 ?") splits each input into
    segments A, B, C, D without saying how a length that does not divide
    evenly is cut.
    """
    g = 16 // ESIZE[dtype]
    per = -(-count // nranks)
    return -(-per // g) * g


def all_reduce_two_shot(xs, op: int, dtype: str, trace=None):
    """"From NCCL Ring LL to PCIe IPC AllReduce", section "Pro5000 ?": every
    input is split into N segments; owner s collects segment s from all ranks,
    reduces it, and sends the result to all the others."""
    n = len(xs)
    count = xs[0].size
    seg = segment_elems(count, n, dtype)
    outs = [np.empty_like(np.asarray(xs[0])) for _ in range(n)]
    for s in range(n):  # owner s
        lo, hi = min(s * seg, count), min((s + 1) * seg, count)
        reduced = reduce_ranks([np.asarray(x)[lo:hi] for x in xs], op, dtype)
        if trace is not None:
            trace.append((s, lo, hi))
        for q in range(n):
            outs[q][lo:hi] = reduced
    return outs


def all_reduce_one_shot(xs, op: int, dtype: str):
    """"From NCCL Ring LL ..." (one-shot all-reduce, "Pro5000 ?"): every rank
    reads all N inputs and reduces them itself."""
    return [reduce_ranks(xs, op, dtype) for _ in xs]


def all_reduce_ring(xs, op: int, dtype: str, trace=None):
    """Ring all-reduce (TP communication essay; NCCL's Ring kernel named in
    "From NCCL Ring LL ...").  2(N-1) steps on the ring r -> r+1.

    Reduce-scatter phase: chunk c starts as rank c+1's values; at each of the
    next N-1 steps every chunk moves one rank on and the receiving rank adds
    its own values, so chunk c is accumulated in the order c+1, c+2, ...,
    N-1, 0, ..., c and is complete on rank c.  Partials travel in the
    arithmetic type (fp32 for the float types) and are rounded once, on
    rank c.  All-gather phase: N-1 further steps in which rank c+j copies
    chunk c from rank c+j-1.

    Reading: the pages give neither the ring's chunk order nor the partials'
    type; this is the order above with fp32 partials, so the result differs
    from the rank-order reduction by rounding only.
    """
    n = len(xs)
    count = xs[0].size
    seg = segment_elems(count, n, dtype)
    bounds = [(min(c * seg, count), min((c + 1) * seg, count)) for c in range(n)]
    outs = [np.empty_like(np.asarray(xs[0])) for _ in range(n)]
    if n == 1:
        outs[0][:] = np.asarray(xs[0])
        return outs
    # rank c+1 starts chunk c
    partial = [widen(np.asarray(xs[(c + 1) % n])[lo:hi], dtype).copy() for c, (lo, hi) in enumerate(bounds)]
    for k in range(1, n):  # reduce-scatter steps
        for c, (lo, hi) in enumerate(bounds):
            r = (c + 1 + k) % n  # chunk c arrives at rank r
            if trace is not None:
                trace.append(("rs", k, c, (r - 1) % n, r))
            partial[c] = combine(partial[c], widen(np.asarray(xs[r])[lo:hi], dtype), op, dtype)
    for c, (lo, hi) in enumerate(bounds):  # complete on rank c
        outs[c][lo:hi] = narrow(partial[c], dtype)
    for j in range(1, n):  # all-gather steps
        for c, (lo, hi) in enumerate(bounds):
            if trace is not None:
                trace.append(("ag", j, c, (c + j - 1) % n, (c + j) % n))
            outs[(c + j) % n][lo:hi] = outs[(c + j - 1) % n][lo:hi]
    return outs


def all_reduce_ring_wire(xs, op: int, dtype: str):
    """The same ring (chunk order and the 2(N-1) steps of ``all_reduce_ring``)
    with the partial travelling in the buffers' own type: every rank that
    receives a chunk's partial widens it, combines its own values in the
    arithmetic type, and rounds the result back to the storage type before
    passing it on, as a ring whose messages carry the buffer dtype does.

    Reading: the pages fix no wire type for the ring (NCCL's ring kernel is
    only named in "From NCCL Ring LL ..."); this is the variant in which
    every hop rounds, reported beside the fp32-partial ring.  For fp32 and
    int32 the storage and arithmetic types agree, and for MAX / MIN rounding
    a winner's own bits is exact, so there it equals ``all_reduce_ring``.
    """
    n = len(xs)
    count = xs[0].size
    seg = segment_elems(count, n, dtype)
    bounds = [(min(c * seg, count), min((c + 1) * seg, count)) for c in range(n)]
    outs = [np.empty_like(np.asarray(xs[0])) for _ in range(n)]
    if n == 1:
        outs[0][:] = np.asarray(xs[0])
        return outs
    # rank c+1 starts chunk c with its own (storage-type) values
    msg = [np.array(np.asarray(xs[(c + 1) % n])[lo:hi], copy=True) for c, (lo, hi) in enumerate(bounds)]
    for k in range(1, n):  # reduce-scatter steps: each hop delivers a storage-type message
        for c, (lo, hi) in enumerate(bounds):
            r = (c + 1 + k) % n
            msg[c] = narrow(combine(widen(msg[c], dtype), widen(np.asarray(xs[r])[lo:hi], dtype), op, dtype), dtype)
    for c, (lo, hi) in enumerate(bounds):  # complete on rank c
        outs[c][lo:hi] = msg[c]
    for j in range(1, n):  # all-gather steps, as in all_reduce_ring
        for c, (lo, hi) in enumerate(bounds):
            outs[(c + j) % n][lo:hi] = outs[(c + j - 1) % n][lo:hi]
    return outs


# ---------------------------------------------------------- AllGather ----

def all_gather(xs):
    """Tutorial 7.1 / 7.3: every rank receives the rank-ordered concatenation
    ([t0, t1] and [t2, t3] -> both ranks hold [t0, t1, t2, t3])."""
    full = np.concatenate([np.asarray(x) for x in xs])
    return [np.array(full, copy=True) for _ in xs]


# ---------------------------------------------------------- All-to-All ----

def all_to_all(xs):
    """Tutorial 8.1: every rank lays out its send buffer as [to 0, to 1, ...];
    afterwards rank d holds [from 0, from 1, ...].  Equal blocks (alltoall).
    The world-size-1 case is a copy (sglang PR 27492 summary, step 3)."""
    n = len(xs)
    c = xs[0].size // n
    return [np.concatenate([np.asarray(xs[s])[d * c:(d + 1) * c] for s in range(n)]) for d in range(n)]


def all_to_all_v(send, recv_bufs, send_counts, send_displs, recv_displs, row_elems: int):
    """Tutorial 8.2 (alltoallv: per-peer lengths differ).

    ``send_counts[s][d]`` rows of ``row_elems`` elements leave rank s from row
    ``send_displs[s][d]`` and land on rank d at row ``recv_displs[d][s]``.
    Rows of ``recv_bufs`` not written keep their contents.
    """
    n = len(send)
    outs = _copy(recv_bufs)
    for s in range(n):
        for d in range(n):
            k = int(send_counts[s][d])
            if k == 0:
                continue
            so, ro = int(send_displs[s][d]) * row_elems, int(recv_displs[d][s]) * row_elems
            outs[d][ro:ro + k * row_elems] = np.asarray(send[s])[so:so + k * row_elems]
    return outs


__all__ = [
    "broadcast", "gather", "reduce", "scatter", "reduce_scatter", "all_reduce",
    "all_reduce_two_shot", "all_reduce_one_shot", "all_reduce_ring", "all_gather",
    "all_to_all", "all_to_all_v", "segment_elems", "SUM",
]
