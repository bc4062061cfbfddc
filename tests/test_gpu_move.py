"""GPU parity: bit copies through the C-ABI vs the oracle (bit-exact).

broadcast, gather (flat and last-dimension), scatter, all_gather,
all_to_all and all_to_all_v, with ragged sizes, unaligned buffers, in-place
forms and guard bands, plus the full workloads: int32 sampled_token_ids[256]
from rank 7, the fp32 [256, 16032] x 8 logits gather to rank 0, and the
8 x 16 MiB sequence-parallel all-gather.
"""
import numpy as np
import pytest
import torch

import movement_virtual_rank_b200 as M
import oracle
import workloads as W
from gpu_util import Guarded, from_dev, need_gpu, to_dev

pytestmark = pytest.mark.gpu


def rand(n, count, dtype, salt=0):
    if dtype == "int32":
        return W.ranks_values(W.W_MISC, n, count, "int32", salt=salt)
    return W.ranks_values(W.W_MISC, n, count, dtype, "normal", salt=salt)


@pytest.mark.parametrize("dtype", ["bf16", "fp32", "int32"])
@pytest.mark.parametrize("n", [1, 2, 5, 8])
@pytest.mark.parametrize("count", [1, 3, 256, 100003])
def test_broadcast(dtype, n, count):
    need_gpu()
    xs = rand(n, count, dtype, salt=count)
    for src in sorted({0, n - 1, n // 2}):
        bufs = [to_dev(x, dtype) for x in xs]
        M.coll_broadcast(bufs, src)
        torch.cuda.synchronize()
        want = oracle.broadcast(xs, src)
        for q in range(n):
            assert np.array_equal(from_dev(bufs[q], dtype), want[q]), (src, q)


def test_broadcast_sampled_token_ids():
    """PP broadcast of int32 sampled_token_ids[256] from the last stage (rank 7)."""
    need_gpu()
    xs = W.sampled_token_ids()
    bufs = [to_dev(x, "int32") for x in xs]
    M.coll_broadcast(bufs, 7)
    torch.cuda.synchronize()
    for q in range(8):
        assert np.array_equal(from_dev(bufs[q], "int32"), xs[7])


def test_broadcast_unaligned_guards():
    need_gpu()
    n, count = 4, 5003
    xs = rand(n, count, "bf16", salt=3)
    bufs = [Guarded(count, "bf16", offset=2 * r, fill=xs[r]) for r in range(n)]
    M.coll_broadcast([b.t for b in bufs], 1)
    torch.cuda.synchronize()
    for b in bufs:
        assert np.array_equal(b.host(), xs[1]) and b.guards_intact()


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("rows,cols", [(1, 1), (1, 1000), (3, 5), (17, 33), (64, 1000), (3, 4097)])
@pytest.mark.parametrize("n", [1, 3, 8])
def test_gather(dtype, rows, cols, n):
    """Flat and last-dimension gathers against the oracle; [3, 4097] rows
    move in 2- or 4-byte units, more than four per thread of a CTA."""
    need_gpu()
    xs = rand(n, rows * cols, dtype, salt=rows * 7 + cols)
    send = [to_dev(x, dtype).reshape(rows, cols) if rows > 1 else to_dev(x, dtype) for x in xs]
    for dst in sorted({0, n - 1}):
        canary = np.full(n * rows * cols, 0x5A5A if dtype == "bf16" else 1.25, dtype=np.uint16 if dtype == "bf16" else np.float32)
        out = to_dev(canary, dtype)
        M.coll_gather(send, out, dst, rows=rows)
        torch.cuda.synchronize()
        assert np.array_equal(from_dev(out, dtype), oracle.gather(xs, canary, rows=rows))


def test_gather_in_place_flat():
    need_gpu()
    n, c = 4, 999
    xs = rand(n, c, "fp32", salt=1)
    out = torch.zeros(n * c, dtype=torch.float32, device="cuda")
    out[2 * c:3 * c].copy_(to_dev(xs[2], "fp32"))
    send = [to_dev(x, "fp32") for x in xs]
    send[2] = out[2 * c:3 * c]
    M.coll_gather(send, out, 2)
    torch.cuda.synchronize()
    assert np.array_equal(from_dev(out, "fp32"), np.concatenate(xs))


def test_gather_logits_workload():
    """Vocab-parallel logits: 8 ranks x fp32 [256, 16032] N(0, 2) -> rank 0 [256, 128256]."""
    need_gpu()
    n, rows, cols = 8, 256, 16032
    xs = W.logits_shards(n, rows, cols)
    send = [to_dev(x, "fp32").reshape(rows, cols) for x in xs]
    out = torch.empty(rows, n * cols, dtype=torch.float32, device="cuda")
    M.coll_gather(send, out, 0)
    torch.cuda.synchronize()
    want = oracle.gather(xs, np.zeros(rows * n * cols, np.float32), rows=rows)
    assert np.array_equal(from_dev(out, "fp32").reshape(-1), want)


@pytest.mark.parametrize("n", [1, 2, 7, 8])
@pytest.mark.parametrize("count", [1, 5, 4096, 33333])
def test_scatter(n, count):
    need_gpu()
    full = rand(1, n * count, "bf16", salt=count)[0]
    src = to_dev(full, "bf16")
    recv = [torch.empty(count, dtype=torch.bfloat16, device="cuda") for _ in range(n)]
    M.coll_scatter(src, recv, n - 1)
    torch.cuda.synchronize()
    want = oracle.scatter(full, n)
    for r in range(n):
        assert np.array_equal(from_dev(recv[r], "bf16"), want[r])
    # gather(scatter(x)) == x on the device path too
    out = torch.empty(n * count, dtype=torch.bfloat16, device="cuda")
    M.coll_gather(recv, out, 0)
    torch.cuda.synchronize()
    assert np.array_equal(from_dev(out, "bf16"), full)


@pytest.mark.parametrize("dtype", ["bf16", "fp32", "int32"])
@pytest.mark.parametrize("n", [1, 2, 3, 8])
@pytest.mark.parametrize("count", [1, 9, 4096, 77777])
def test_all_gather(dtype, n, count):
    need_gpu()
    xs = rand(n, count, dtype, salt=count + n)
    send = [to_dev(x, dtype) for x in xs]
    recv = [torch.empty(n * count, dtype=send[0].dtype, device="cuda") for _ in range(n)]
    M.coll_all_gather(send, recv)
    torch.cuda.synchronize()
    want = oracle.all_gather(xs)
    for q in range(n):
        assert np.array_equal(from_dev(recv[q], dtype), want[q])


@pytest.mark.parametrize("op", ["all_gather", "broadcast"])
def test_bulk_fanout_partial_tile(op):
    """Fan-outs long enough for the bulk-copy kernel (one CTA per 2 tiles of
    8 KB) whose messages end 48 bytes into a tile: 8 sources of 4 MiB + 48 B
    (all_gather), or one source of 29 MiB + 48 B to 8 ranks (broadcast).
    Every output against the oracle, and guard bands past each buffer."""
    need_gpu()
    n = 8
    if op == "all_gather":
        count = (2 << 20) + 24
        xs = rand(n, count, "bf16", salt=41)
        send = [to_dev(x, "bf16") for x in xs]
        grecv = [Guarded(n * count, "bf16") for _ in range(n)]
        M.coll_all_gather(send, [b.t for b in grecv])
        torch.cuda.synchronize()
        want = oracle.all_gather(xs)
        for q in range(n):
            assert np.array_equal(grecv[q].host(), want[q]) and grecv[q].guards_intact(), q
    else:
        count = (29 << 19) + 24
        xs = rand(n, count, "bf16", salt=43)
        bufs = [Guarded(count, "bf16", fill=x) for x in xs]
        M.coll_broadcast([b.t for b in bufs], 5)
        torch.cuda.synchronize()
        want = oracle.broadcast(xs, 5)
        for q in range(n):
            assert np.array_equal(bufs[q].host(), want[q]) and bufs[q].guards_intact(), q


def test_all_gather_in_place_and_unaligned():
    need_gpu()
    n, count = 4, 12345
    xs = rand(n, count, "bf16", salt=9)
    recv = [to_dev(np.zeros(n * count, np.uint16), "bf16") for _ in range(n)]
    for r in range(n):
        recv[r][r * count:(r + 1) * count].copy_(to_dev(xs[r], "bf16"))
    send = [recv[r][r * count:(r + 1) * count] for r in range(n)]
    M.coll_all_gather(send, recv)
    torch.cuda.synchronize()
    for q in range(n):
        assert np.array_equal(from_dev(recv[q], "bf16"), np.concatenate(xs))
    gsend = [Guarded(count, "bf16", offset=2 + 2 * r, fill=xs[r]) for r in range(n)]
    grecv = [Guarded(n * count, "bf16", offset=6) for _ in range(n)]
    M.coll_all_gather([b.t for b in gsend], [b.t for b in grecv])
    torch.cuda.synchronize()
    for b in grecv:
        assert np.array_equal(b.host(), np.concatenate(xs)) and b.guards_intact()


def test_sp_all_gather_workload():
    """8 ranks x bf16 [1024, 8192] -> every rank [8192, 8192]: every element of
    every output against the oracle's all-gather."""
    need_gpu()
    n, rows, cols = 8, 1024, 8192
    xs = W.sp_allgather(n, rows, cols)
    c = rows * cols
    send = [to_dev(x, "bf16") for x in xs]
    recv = [torch.empty(n * c, dtype=torch.bfloat16, device="cuda") for _ in range(n)]
    M.coll_all_gather(send, recv)
    torch.cuda.synchronize()
    want = oracle.all_gather(xs)
    for q in range(n):
        assert np.array_equal(from_dev(recv[q], "bf16"), want[q]), q


@pytest.mark.parametrize("n", [1, 2, 3, 8])
@pytest.mark.parametrize("count", [1, 6, 1000])
def test_all_to_all(n, count):
    need_gpu()
    xs = rand(n, n * count, "bf16", salt=count)
    send = [to_dev(x, "bf16") for x in xs]
    recv = [torch.empty_like(t) for t in send]
    M.coll_all_to_all(send, recv)
    torch.cuda.synchronize()
    want = oracle.all_to_all(xs)
    for d in range(n):
        assert np.array_equal(from_dev(recv[d], "bf16"), want[d])


@pytest.mark.parametrize("n", [1, 2, 5, 8, 33])
@pytest.mark.parametrize("row", [1, 3, 8, 7168])
def test_all_to_all_v_roundtrip(n, row):
    """Ragged splits (zeros included) vs the oracle, then the transposed
    splits bring every row home (tutorial section 8.2)."""
    need_gpu()
    max_rows = 6 if row > 100 else 40
    sc = W.random_splits(n, max_rows, salt=n * 100 + row)
    sd = np.zeros_like(sc)
    sd[:, 1:] = np.cumsum(sc, axis=1)[:, :-1]
    rc = sc.T.copy()
    rd = np.zeros_like(rc)
    rd[:, 1:] = np.cumsum(rc, axis=1)[:, :-1]
    xs = [W.ranks_values(W.W_MISC, 1, max(1, int(sc[s].sum())) * row, "bf16", salt=s + 1)[0] for s in range(n)]
    send = [to_dev(x, "bf16") for x in xs]
    recv = [to_dev(np.full(max(1, int(rc[d].sum())) * row, 0x7777, np.uint16), "bf16") for d in range(n)]
    M.coll_all_to_all_v(send, recv, sc, sd, rd, row)
    torch.cuda.synchronize()
    want = oracle.all_to_all_v(xs, [from_dev(t, "bf16") * 0 + 0x7777 for t in recv], sc, sd, rd, row)
    got = [from_dev(t, "bf16") for t in recv]
    for d in range(n):
        assert np.array_equal(got[d], want[d]), d
    back = [torch.zeros_like(t) for t in send]
    M.coll_all_to_all_v(recv, back, rc, rd, sd, row)
    torch.cuda.synchronize()
    for s in range(n):
        k = int(sc[s].sum()) * row
        assert np.array_equal(from_dev(back[s], "bf16")[:k], xs[s][:k])


def test_all_to_all_v_many_launches():
    """64 ranks: 4096 blocks, more than one launch's job table."""
    need_gpu()
    n, row = 64, 4
    sc = W.random_splits(n, 3, salt=64)
    sd = np.zeros_like(sc)
    sd[:, 1:] = np.cumsum(sc, axis=1)[:, :-1]
    rc = sc.T.copy()
    rd = np.zeros_like(rc)
    rd[:, 1:] = np.cumsum(rc, axis=1)[:, :-1]
    xs = [np.arange(max(1, int(sc[s].sum())) * row, dtype=np.int32) + 1000000 * s for s in range(n)]
    send = [to_dev(x, "int32") for x in xs]
    recv = [torch.full((max(1, int(rc[d].sum())) * row,), -1, dtype=torch.int32, device="cuda") for d in range(n)]
    M.coll_all_to_all_v(send, recv, sc, sd, rd, row)
    torch.cuda.synchronize()
    want = oracle.all_to_all_v(xs, [np.full(t.numel(), -1, np.int32) for t in recv], sc, sd, rd, row)
    for d in range(n):
        assert np.array_equal(from_dev(recv[d], "int32"), want[d])


@pytest.mark.parametrize("count", [1 << 21, 2000008, 2000003])
@pytest.mark.parametrize("n", [2, 8])
def test_all_gather_bulk_copy_sizes(n, count):
    """Large fan-outs (at least 4 tiles of 8 KB per CTA, about 29 MB in all on
    148 SMs) take the bulk-copy (TMA) path: a whole number of tiles, a ragged
    last tile, and a length that is not a multiple of 16 bytes (which must
    take the element path instead).  The 2-rank cases stay below the
    threshold and check the element path at the same sizes."""
    need_gpu()
    xs = rand(n, count, "bf16", salt=count + 3 * n)
    send = [to_dev(x, "bf16") for x in xs]
    recv = [torch.full((n * count,), 3.0, dtype=torch.bfloat16, device="cuda") for _ in range(n)]
    M.coll_all_gather(send, recv)
    torch.cuda.synchronize()
    want = np.concatenate(xs)
    for q in range(n):
        assert np.array_equal(from_dev(recv[q], "bf16"), want)
    # in place
    recv2 = [torch.zeros(n * count, dtype=torch.bfloat16, device="cuda") for _ in range(n)]
    for r in range(n):
        recv2[r][r * count:(r + 1) * count].copy_(send[r])
    M.coll_all_gather([recv2[r][r * count:(r + 1) * count] for r in range(n)], recv2)
    torch.cuda.synchronize()
    for q in range(n):
        assert np.array_equal(from_dev(recv2[q], "bf16"), want)


@pytest.mark.parametrize("count", [1 << 23, (1 << 23) + 4, 3 * 1000003])
def test_broadcast_bulk_copy_sizes(count):
    need_gpu()
    n = 8
    xs = rand(n, count, "int32", salt=count)
    bufs = [to_dev(x, "int32") for x in xs]
    M.coll_broadcast(bufs, 5)
    torch.cuda.synchronize()
    for q in range(n):
        assert np.array_equal(from_dev(bufs[q], "int32"), xs[5])


def test_copy_jobs_bulk_copy_path():
    """Copy lists of 29 MB and more take the bulk-copy path: scatter of
    8 x 4 MiB, all-to-all of 8 x 8 MiB, and an all-to-all-v with ragged row
    counts, all checked on the device against their definitions."""
    need_gpu()
    n = 8
    c = 2 << 20  # bf16 elements per rank block (4 MiB)
    full = torch.randn(n * c, device="cuda").to(torch.bfloat16)
    recv = [torch.empty(c, dtype=torch.bfloat16, device="cuda") for _ in range(n)]
    M.coll_scatter(full, recv, 3)
    torch.cuda.synchronize()
    for r in range(n):
        assert torch.equal(recv[r].view(torch.int16), full[r * c:(r + 1) * c].view(torch.int16))
    blk = 1 << 19
    send = [torch.randn(n * blk, device="cuda").to(torch.bfloat16) for _ in range(n)]
    out = [torch.empty_like(t) for t in send]
    M.coll_all_to_all(send, out)
    torch.cuda.synchronize()
    for d in range(n):
        for s in range(n):
            assert torch.equal(out[d][s * blk:(s + 1) * blk].view(torch.int16),
                               send[s][d * blk:(d + 1) * blk].view(torch.int16))
    row = 1024
    sc = W.random_splits(n, 600, salt=99)
    sd = np.zeros_like(sc)
    sd[:, 1:] = np.cumsum(sc, axis=1)[:, :-1]
    rc = sc.T.copy()
    rd = np.zeros_like(rc)
    rd[:, 1:] = np.cumsum(rc, axis=1)[:, :-1]
    vs = [torch.randn(max(1, int(sc[s].sum())) * row, device="cuda").to(torch.bfloat16) for s in range(n)]
    vr = [torch.zeros(max(1, int(rc[d].sum())) * row, dtype=torch.bfloat16, device="cuda") for d in range(n)]
    assert int(sc.sum()) * row * 2 >= 29 << 20
    M.coll_all_to_all_v(vs, vr, sc, sd, rd, row)
    torch.cuda.synchronize()
    for s in range(n):
        for d in range(n):
            k = int(sc[s, d]) * row
            a, b = int(sd[s, d]) * row, int(rd[d, s]) * row
            assert torch.equal(vr[d][b:b + k].view(torch.int16), vs[s][a:a + k].view(torch.int16)), (s, d)
