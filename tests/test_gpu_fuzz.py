"""Seeded randomized parity: many small random configurations of every
reduction and movement entry point against the oracle, bit for bit.

Each case draws (from its own seed) the rank count, the element count (often
ragged), the dtype, the reduction op, whether the call is in place, and a
byte offset that makes some buffers unaligned.
"""
import numpy as np
import pytest
import torch

import movement_virtual_rank_b200 as M
import oracle
import workloads as W
from gpu_util import ESIZE, Guarded, need_gpu

pytestmark = pytest.mark.gpu

ALGOS = {M.ONESHOT: oracle.all_reduce_one_shot, M.TWOSHOT: oracle.all_reduce_two_shot,
         M.RING: oracle.all_reduce_ring, M.RING_LL: oracle.all_reduce_ring, M.RING_STEPS: oracle.all_reduce_ring,
         M.RING_CLUSTER: oracle.all_reduce_ring, M.TWOSHOT_LL: oracle.all_reduce_two_shot,
         M.RING_CTA: oracle.all_reduce_ring, M.RING_LANE: oracle.all_reduce_ring,
         M.TWOSHOT_LL128: oracle.all_reduce_two_shot}


def bits(a):
    a = np.asarray(a)
    return a.view(np.uint32) if a.dtype == np.float32 else a


def draw(seed):
    g = W.rng(W.W_MISC, 7, salt=seed)
    n = int(g.choice([1, 2, 3, 4, 5, 6, 7, 8, 9, 16]))
    count = int(g.choice([1, 2, 3, 7, 8, 15, 16, 17, 100, 1000, 4095, 4096, 4097, 33333, 100000]))
    dtype = str(g.choice(["bf16", "fp16", "fp32", "int32"]))
    op = int(g.integers(0, 4))
    off = int(g.choice([0, 0, 0, 1])) * ESIZE[dtype]  # some unaligned buffers
    if dtype == "int32":
        xs = [g.integers(-50, 50, count, dtype=np.int64).astype(np.int32) for _ in range(n)]
    else:
        xs = W.ranks_values(W.W_MISC, n, count, dtype, "uniform" if op == 3 else "normal", salt=seed)
    return g, n, count, dtype, op, off, xs


@pytest.mark.parametrize("seed", range(40))
def test_fuzz_all_reduce(seed):
    need_gpu()
    g, n, count, dtype, op, off, xs = draw(seed)
    algo = int(g.choice(list(ALGOS)))
    send = [Guarded(count, dtype, offset=off * (r % 2), fill=xs[r]) for r in range(n)]
    in_place = algo != M.ONESHOT and bool(g.integers(0, 2))
    recv = send if in_place else [Guarded(count, dtype, offset=off * ((r + 1) % 2)) for r in range(n)]
    ws = None
    if algo in (M.RING_CLUSTER, M.RING_CTA, M.RING_LANE):  # a RING-sized workspace: the fallback for unaligned buffers or N > 8
        need = M.coll_all_reduce_workspace_size(n, count, send[0].t.dtype, M.RING)
        ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    elif algo in (M.TWOSHOT_LL, M.TWOSHOT_LL128):
        need = M.coll_all_reduce_workspace_size(n, count, send[0].t.dtype, algo)
        ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    M.coll_all_reduce([b.t for b in send], [b.t for b in recv], op=op, algo=algo, workspace=ws)
    torch.cuda.synchronize()
    want = ALGOS[algo](xs, op, dtype)
    for q in range(n):
        assert np.array_equal(bits(recv[q].host()), bits(want[q])), (seed, n, count, dtype, op, algo, q)
    assert all(b.guards_intact() for b in send + recv)


@pytest.mark.parametrize("seed", range(40, 70))
def test_fuzz_reduce_scatter_and_reduce(seed):
    need_gpu()
    g, n, count, dtype, op, off, xs0 = draw(seed)
    per = max(1, count // n)
    if dtype == "int32":
        xs = [g.integers(-50, 50, per * n, dtype=np.int64).astype(np.int32) for _ in range(n)]
    else:
        xs = W.ranks_values(W.W_MISC, n, per * n, dtype, "uniform" if op == 3 else "normal", salt=seed + 1)
    send = [Guarded(per * n, dtype, offset=off * (r % 2), fill=xs[r]) for r in range(n)]
    recv = [Guarded(per, dtype, offset=off) for _ in range(n)]
    M.coll_reduce_scatter([b.t for b in send], [b.t for b in recv], op=op)
    dst = int(g.integers(0, n))
    red = Guarded(per * n, dtype, offset=off)
    M.coll_reduce([b.t for b in send], red.t, dst, op=op)
    torch.cuda.synchronize()
    want = oracle.reduce_scatter(xs, op, dtype)
    for r in range(n):
        assert np.array_equal(bits(recv[r].host()), bits(want[r])), (seed, r)
    assert np.array_equal(bits(red.host()), bits(oracle.reduce(xs, op, dtype)))
    assert all(b.guards_intact() for b in send + recv + [red])


@pytest.mark.parametrize("seed", range(70, 100))
def test_fuzz_movement(seed):
    need_gpu()
    g, n, count, dtype, op, off, xs = draw(seed)
    # all_gather
    send = [Guarded(count, dtype, offset=off * (r % 2), fill=xs[r]) for r in range(n)]
    recv = [Guarded(n * count, dtype, offset=off) for _ in range(n)]
    M.coll_all_gather([b.t for b in send], [b.t for b in recv])
    # broadcast from a random root
    src = int(g.integers(0, n))
    bc = [Guarded(count, dtype, offset=off * ((r + 1) % 2), fill=xs[r]) for r in range(n)]
    M.coll_broadcast([b.t for b in bc], src)
    # gather (flat) and scatter
    dst = int(g.integers(0, n))
    gat = Guarded(n * count, dtype, offset=off)
    M.coll_gather([b.t for b in send], gat.t, dst)
    full = np.concatenate(xs)
    sc_src = Guarded(n * count, dtype, offset=off, fill=full)
    sc = [Guarded(count, dtype, offset=off * (r % 2)) for r in range(n)]
    M.coll_scatter(sc_src.t, [b.t for b in sc], dst)
    torch.cuda.synchronize()
    for q in range(n):
        assert np.array_equal(bits(recv[q].host()), bits(full)), (seed, "all_gather", q)
        assert np.array_equal(bits(bc[q].host()), bits(xs[src])), (seed, "broadcast", q)
        assert np.array_equal(bits(sc[q].host()), bits(xs[q])), (seed, "scatter", q)
    assert np.array_equal(bits(gat.host()), bits(full))
    assert all(b.guards_intact() for b in send + recv + bc + sc + [gat, sc_src])
