"""GPU parity: the single-launch LL ring all-reduce (COLL_ALGO_RING_LL).

It follows the ring schedule, chunk order and rounding of the stream-ordered
ring, so its output is compared bit for bit with the oracle's ring; repeated
calls on one workspace check that the per-call flag epoch keeps earlier
lines from being taken for new ones.  The bounded wait is checked on its own
with coll_wait_flag on a flag that nothing sets: the kernel gives up, reports
COLL_DEV_TIMEOUT and the context stays usable.
"""
import time

import numpy as np
import pytest
import torch

import movement_virtual_rank_b200 as M
import oracle
import workloads as W
from gpu_util import from_dev, need_gpu, status_tensor, to_dev

pytestmark = pytest.mark.gpu


def bits(a):
    a = np.asarray(a)
    return a.view(np.uint32) if a.dtype == np.float32 else a


def run(xs, dtype, op, ws=None, in_place=False):
    send = [to_dev(x, dtype) for x in xs]
    recv = send if in_place else [torch.empty_like(t) for t in send]
    M.coll_all_reduce(send, recv, op=op, algo=M.RING_LL, workspace=ws)
    torch.cuda.synchronize()
    return [from_dev(t, dtype) for t in recv]


@pytest.mark.parametrize("n", [2, 3, 4, 8])
@pytest.mark.parametrize("count", [1, 9, 8 * 37 + 3, 65536 + 24, 300007, 1835008])
def test_ring_ll_bf16_sum(n, count):
    need_gpu()
    xs = W.ranks_values(W.W_MISC, n, count, "bf16", "normal", salt=count + 7 * n)
    want = oracle.all_reduce_ring(xs, 0, "bf16")
    got = run(xs, "bf16", 0)
    for q in range(n):
        assert np.array_equal(got[q], want[q]), q


@pytest.mark.parametrize("dtype", ["bf16", "fp16", "fp32", "int32"])
@pytest.mark.parametrize("op", [0, 1, 2, 3])
def test_ring_ll_dtypes_ops(dtype, op):
    need_gpu()
    n, count = 5, 12301
    if dtype == "int32":
        g = W.rng(W.W_MISC, 0, salt=op + 40)
        xs = [g.integers(-1000, 1000, count, dtype=np.int64).astype(np.int32) for _ in range(n)]
    else:
        xs = W.ranks_values(W.W_MISC, n, count, dtype, "uniform" if op == 3 else "normal", salt=op + 40)
    want = oracle.all_reduce_ring(xs, op, dtype)
    got = run(xs, dtype, op)
    for q in range(n):
        assert np.array_equal(bits(got[q]), bits(want[q])), q


def test_ring_ll_repeated_calls_one_workspace_and_in_place():
    """Twenty calls on one workspace: every call must use only its own lines."""
    need_gpu()
    n, count = 8, 200003
    need = M.coll_all_reduce_workspace_size(n, count, torch.bfloat16, M.RING_LL)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    for call in range(20):
        xs = W.ranks_values(W.W_MISC, n, count, "bf16", "normal", salt=500 + call)
        got = run(xs, "bf16", 0, ws=ws, in_place=(call % 2 == 1))
        want = oracle.all_reduce_ring(xs, 0, "bf16")
        for q in range(n):
            assert np.array_equal(got[q], want[q]), (call, q)
    st = ws[16:24].view(torch.int32)
    assert st.tolist() == [0, 0]


def test_ring_ll_tp_decode_workload():
    need_gpu()
    for tokens, hidden in W.tp_decode_shapes():
        xs = W.tp_decode(tokens, hidden)
        got = run(xs, "bf16", 0)
        want = oracle.all_reduce_ring(xs, 0, "bf16")
        for q in range(8):
            assert np.array_equal(got[q], want[q]), (tokens, hidden, q)


def test_ring_ll_unaligned_takes_the_ring_path():
    need_gpu()
    n, count = 4, 5001
    xs = W.ranks_values(W.W_MISC, n, count, "bf16", "normal", salt=77)
    raw = [torch.empty(count + 8, dtype=torch.bfloat16, device="cuda") for _ in range(n)]
    send = [raw[r][1:count + 1] for r in range(n)]
    for r in range(n):
        send[r].copy_(to_dev(xs[r], "bf16"))
    recv = [torch.empty(count + 8, dtype=torch.bfloat16, device="cuda")[3:count + 3] for _ in range(n)]
    M.coll_all_reduce(send, recv, algo=M.RING_LL)
    torch.cuda.synchronize()
    want = oracle.all_reduce_ring(xs, 0, "bf16")
    for q in range(n):
        assert np.array_equal(from_dev(recv[q], "bf16"), want[q])


def test_bounded_wait_times_out_and_context_survives():
    """A flag that nothing sets: the wait gives up after its budget, raises
    COLL_DEV_TIMEOUT, and later work on the same context is unaffected."""
    need_gpu()
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    st = status_tensor()
    t0 = time.perf_counter()
    M.coll_wait_flag(flag, 1, 20000, st)  # 20 ms budget
    torch.cuda.synchronize()
    dt = time.perf_counter() - t0
    assert st.tolist() == [M.DEV_TIMEOUT, 1]
    assert 0.015 < dt < 5.0
    # a flag that is already set returns at once with no status
    st.zero_()
    flag.fill_(7)
    M.coll_wait_flag(flag, 7, 20000, st)
    torch.cuda.synchronize()
    assert st.tolist() == [0, 0]
    # the context still works
    xs = W.ranks_values(W.W_MISC, 3, 999, "bf16", "normal", salt=1)
    got = run(xs, "bf16", 0)
    want = oracle.all_reduce_ring(xs, 0, "bf16")
    assert all(np.array_equal(g, w) for g, w in zip(got, want))


# ------------------------------------ cluster, CTA and lane rings ----
# RING_CLUSTER (ranks = CTAs of a cluster, hops over distributed shared
# memory), RING_CTA (ranks = warp groups of one CTA, hops in its shared
# memory) and RING_LANE (ranks = lanes of one warp, hops by warp shuffles)
# take the same tests.

ONE_LAUNCH = pytest.mark.parametrize("algo", [M.RING_CLUSTER, M.RING_CTA, M.RING_LANE],
                                     ids=["cluster", "cta", "lane"])


def run_cluster(xs, dtype, op, in_place=False, ws=None, algo=M.RING_CLUSTER):
    send = [to_dev(x, dtype) for x in xs]
    recv = send if in_place else [torch.empty_like(t) for t in send]
    M.coll_all_reduce(send, recv, op=op, algo=algo, workspace=ws)
    torch.cuda.synchronize()
    return [from_dev(t, dtype) for t in recv]


@ONE_LAUNCH
@pytest.mark.parametrize("n", [2, 3, 4, 5, 6, 7, 8])
@pytest.mark.parametrize("count", [1, 9, 8 * 37 + 3, 65536 + 24, 300007])
def test_ring_cluster_bf16_sum(algo, n, count):
    """Virtual ranks as the CTAs of a thread-block cluster, hops over
    distributed shared memory: bit-identical to the ring oracle."""
    need_gpu()
    xs = W.ranks_values(W.W_MISC, n, count, "bf16", "normal", salt=count + 11 * n)
    want = oracle.all_reduce_ring(xs, 0, "bf16")
    got = run_cluster(xs, "bf16", 0, in_place=(count % 2 == 1), algo=algo)
    for q in range(n):
        assert np.array_equal(got[q], want[q]), q


@pytest.mark.parametrize("dtype", ["bf16", "fp16", "fp32", "int32"])
@pytest.mark.parametrize("op", [0, 1, 2, 3])
@ONE_LAUNCH
def test_ring_cluster_dtypes_ops(algo, dtype, op):
    need_gpu()
    n, count = 7, 12301
    if dtype == "int32":
        g = W.rng(W.W_MISC, 0, salt=op + 90)
        xs = [g.integers(-1000, 1000, count, dtype=np.int64).astype(np.int32) for _ in range(n)]
    else:
        xs = W.ranks_values(W.W_MISC, n, count, dtype, "uniform" if op == 3 else "normal", salt=op + 90)
    want = oracle.all_reduce_ring(xs, op, dtype)
    ws = torch.zeros(64, dtype=torch.uint8, device="cuda")
    got = run_cluster(xs, dtype, op, ws=ws, algo=algo)
    for q in range(n):
        assert np.array_equal(bits(got[q]), bits(want[q])), q
    assert ws[16:24].view(torch.int32).tolist() == [0, 0]


@ONE_LAUNCH
def test_ring_cluster_tp_decode_workload(algo):
    need_gpu()
    for tokens, hidden in W.tp_decode_shapes():
        xs = W.tp_decode(tokens, hidden)
        got = run_cluster(xs, "bf16", 0, algo=algo)
        want = oracle.all_reduce_ring(xs, 0, "bf16")
        for q in range(8):
            assert np.array_equal(got[q], want[q]), (tokens, hidden, q)


@ONE_LAUNCH
def test_ring_cluster_fallbacks(algo):
    """Unaligned buffers or more than 8 ranks: with a RING workspace the call
    takes the RING path (same result); without one it is refused."""
    need_gpu()
    n, count = 4, 5001
    xs = W.ranks_values(W.W_MISC, n, count, "bf16", "normal", salt=78)
    raw = [torch.empty(count + 8, dtype=torch.bfloat16, device="cuda") for _ in range(n)]
    send = [raw[r][1:count + 1] for r in range(n)]
    for r in range(n):
        send[r].copy_(to_dev(xs[r], "bf16"))
    recv = [torch.empty(count + 8, dtype=torch.bfloat16, device="cuda")[3:count + 3] for _ in range(n)]
    with pytest.raises(M.CollError):
        M.coll_all_reduce(send, recv, algo=algo)
    ws = torch.zeros(M.coll_all_reduce_workspace_size(n, count, torch.bfloat16, M.RING), dtype=torch.uint8,
                     device="cuda")
    M.coll_all_reduce(send, recv, algo=algo, workspace=ws)
    torch.cuda.synchronize()
    want = oracle.all_reduce_ring(xs, 0, "bf16")
    for q in range(n):
        assert np.array_equal(from_dev(recv[q], "bf16"), want[q])
    xs9 = W.ranks_values(W.W_MISC, 9, 1000, "bf16", "normal", salt=79)
    ws9 = torch.zeros(M.coll_all_reduce_workspace_size(9, 1000, torch.bfloat16, M.RING), dtype=torch.uint8,
                      device="cuda")
    got = run_cluster(xs9, "bf16", 0, ws=ws9, algo=algo)
    want = oracle.all_reduce_ring(xs9, 0, "bf16")
    assert all(np.array_equal(g, w) for g, w in zip(got, want))


@pytest.mark.parametrize("n,count,dtype", [(2, 3_000_017, "bf16"), (5, 2_500_001, "bf16"), (8, 4_194_311, "bf16"),
                                           (3, 2_000_003, "fp32"), (8, 1_048_583, "int32"), (7, 999_999, "fp16"),
                                           (8, 3_000_000, "fp32"), (8, 2_500_002, "fp16"), (8, 5_000_011, "fp16")])
@ONE_LAUNCH
def test_ring_cluster_many_tiles(algo, n, count, dtype):
    """Messages of many tiles per CTA or cluster (the CTAs walk the tiles; at
    8 ranks the CTA ring then prefetches its inputs into registers across
    tile boundaries), with a ragged tail; odd counts run in place."""
    need_gpu()
    if dtype == "int32":
        g = W.rng(W.W_MISC, 0, salt=count)
        xs = [g.integers(-1000, 1000, count, dtype=np.int64).astype(np.int32) for _ in range(n)]
    else:
        xs = W.ranks_values(W.W_MISC, n, count, dtype, "normal", salt=count % 977)
    ws = torch.zeros(64, dtype=torch.uint8, device="cuda")
    got = run_cluster(xs, dtype, 0, in_place=(count % 2 == 1), ws=ws, algo=algo)
    want = oracle.all_reduce_ring(xs, 0, dtype)
    for q in range(n):
        assert np.array_equal(bits(got[q]), bits(want[q])), q
    assert ws[16:24].view(torch.int32).tolist() == [0, 0]


@ONE_LAUNCH
def test_ring_cluster_back_to_back(algo):
    """Consecutive calls on one stream (the next launch may start early and
    wait for this one): every result matches."""
    need_gpu()
    n, count = 8, 229_376 * 8
    xs = W.tp_decode(256, 7168)
    send = [to_dev(x, "bf16") for x in xs]
    outs = []
    for _ in range(3):
        recv = [torch.empty_like(t) for t in send]
        M.coll_all_reduce(send, recv, algo=algo)
        outs.append(recv)
    torch.cuda.synchronize()
    want = oracle.all_reduce_ring(xs, 0, "bf16")
    for recv in outs:
        for q in range(n):
            assert np.array_equal(from_dev(recv[q], "bf16"), want[q]), q


@pytest.mark.parametrize("tokens,hidden", [(1, 4096), (32, 7168), (160, 8192), (161, 8192), (256, 7168)])
def test_ring_forms_agree(tokens, hidden):
    """RING takes a one-launch form for aligned buffers (the lane ring up to
    16 KiB per rank at 8 ranks, the CTA ring above); every form (lane, CTA,
    cluster, stream-ordered steps) gives the same bits, and the workspace
    header's status pair stays clear."""
    need_gpu()
    xs = W.tp_decode(tokens, hidden)
    n, count = len(xs), tokens * hidden
    form = M.coll_all_reduce_form(n, count, torch.bfloat16, M.RING)
    assert form == (M.RING_LANE if 2 * count <= 16 << 10 else M.RING_CTA)
    want = oracle.all_reduce_ring(xs, 0, "bf16")
    for algo in (M.RING, M.RING_STEPS, M.RING_CLUSTER, M.RING_CTA, M.RING_LANE):
        send = [to_dev(x, "bf16") for x in xs]
        recv = [torch.empty_like(t) for t in send]
        ws = torch.zeros(M.coll_all_reduce_workspace_size(n, count, torch.bfloat16, M.RING), dtype=torch.uint8,
                         device="cuda")
        M.coll_all_reduce(send, recv, algo=algo, workspace=ws)
        torch.cuda.synchronize()
        for q in range(n):
            assert np.array_equal(from_dev(recv[q], "bf16"), want[q]), (algo, q)
        assert ws[16:24].view(torch.int32).tolist() == [0, 0]
