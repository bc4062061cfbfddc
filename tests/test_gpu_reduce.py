"""GPU parity: reductions through the C-ABI vs the oracle (bit-exact).

all_reduce (two-shot, one-shot, ring), reduce_scatter and reduce, over every
dtype and op, rank counts 1..8 (and a generic-path 13), sizes that span
several CTAs with ragged tails, in-place and unaligned forms, special values,
and the full workloads: 4 x 160 KB two-shot, and the TP-decode grid
(8 ranks, tokens 1..256 x hidden 4096/7168) for all three algorithms.
"""
import numpy as np
import pytest
import torch

import movement_virtual_rank_b200 as M
import oracle
import workloads as W
from gpu_util import ESIZE, Guarded, from_dev, need_gpu, to_dev

pytestmark = pytest.mark.gpu

ALGO_FN = {
    M.TWOSHOT: oracle.all_reduce_two_shot,
    M.ONESHOT: oracle.all_reduce_one_shot,
    M.RING: oracle.all_reduce_ring,
    M.RING_STEPS: oracle.all_reduce_ring,
}
OPNAME = {0: "sum", 1: "max", 2: "min", 3: "prod"}


def inputs(n, count, dtype, salt=0, dist="normal"):
    if dtype == "int32":
        g = W.rng(W.W_MISC, 0, salt=salt + 5)
        return [g.integers(-1000, 1000, count, dtype=np.int64).astype(np.int32) for _ in range(n)]
    if dtype == "fp32":
        return W.ranks_values(W.W_MISC, n, count, "fp32", dist, salt=salt)
    return W.ranks_values(W.W_MISC, n, count, dtype, dist, salt=salt)


def run_all_reduce(xs, dtype, op, algo, in_place=False):
    send = [to_dev(x, dtype) for x in xs]
    recv = send if in_place else [torch.empty_like(t) for t in send]
    M.coll_all_reduce(send, recv, op=op, algo=algo)
    torch.cuda.synchronize()
    return [from_dev(t, dtype) for t in recv]


def bits(a):
    a = np.asarray(a)
    return a.view(np.uint32) if a.dtype == np.float32 else a


def assert_ranks_equal(got, want, what=""):
    """Bit-for-bit equality (float32 arrays are compared as their bit patterns)."""
    for q, (g, w) in enumerate(zip(got, want)):
        g, w = bits(g), bits(w)
        if not np.array_equal(g, w):
            bad = np.nonzero(g != w)[0]
            raise AssertionError(f"{what} rank {q}: {bad.size} mismatches, first at {bad[:5]}: "
                                 f"got {g[bad[:5]]} want {w[bad[:5]]}")


@pytest.mark.parametrize("algo", [M.TWOSHOT, M.ONESHOT, M.RING, M.RING_STEPS])
@pytest.mark.parametrize("n", [1, 2, 3, 4, 5, 8])
@pytest.mark.parametrize("count", [1, 7, 8 * 37 + 3, 65536 + 24, 300007])
def test_all_reduce_bf16_sum(algo, n, count):
    need_gpu()
    xs = inputs(n, count, "bf16", salt=count + n)
    got = run_all_reduce(xs, "bf16", M.SUM, algo)
    assert_ranks_equal(got, ALGO_FN[algo](xs, 0, "bf16"), f"algo {algo}")


@pytest.mark.parametrize("dtype", ["bf16", "fp16", "fp32", "int32"])
@pytest.mark.parametrize("op", [0, 1, 2, 3])
@pytest.mark.parametrize("algo", [M.TWOSHOT, M.ONESHOT, M.RING, M.RING_STEPS])
@pytest.mark.parametrize("n", [3, 8, 13])
def test_all_reduce_dtypes_ops(dtype, op, algo, n):
    need_gpu()
    count = 4099 * 3
    xs = inputs(n, count, dtype, salt=7 * op + n, dist="uniform" if op == 3 else "normal")
    got = run_all_reduce(xs, dtype, op, algo)
    assert_ranks_equal(got, ALGO_FN[algo](xs, op, dtype), f"{dtype} {OPNAME[op]} algo {algo}")


@pytest.mark.parametrize("algo", [M.TWOSHOT, M.RING, M.RING_STEPS])
def test_all_reduce_in_place(algo):
    need_gpu()
    xs = inputs(8, 50001, "bf16", salt=3)
    got = run_all_reduce(xs, "bf16", M.SUM, algo, in_place=True)
    assert_ranks_equal(got, ALGO_FN[algo](xs, 0, "bf16"))


@pytest.mark.parametrize("algo", [M.TWOSHOT, M.ONESHOT, M.RING, M.RING_STEPS])
@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_all_reduce_unaligned_and_guards(algo, dtype):
    need_gpu()
    n, count = 5, 10007
    xs = inputs(n, count, dtype, salt=11)
    es = ESIZE[dtype]
    send = [Guarded(count, dtype, offset=es * (r + 1), fill=xs[r]) for r in range(n)]
    recv = [Guarded(count, dtype, offset=es * (r % 3)) for r in range(n)]
    M.coll_all_reduce([b.t for b in send], [b.t for b in recv], op=M.SUM, algo=algo)
    torch.cuda.synchronize()
    assert_ranks_equal([b.host() for b in recv], ALGO_FN[algo](xs, 0, dtype))
    assert all(b.guards_intact() for b in send + recv)
    assert_ranks_equal([b.host() for b in send], xs, "inputs modified")


def special_values(dtype):
    if dtype == "bf16":
        vals = [0x0000, 0x8000, 0x7F80, 0xFF80, 0x7FC1, 0x0001, 0x8001, 0x7F7F, 0xFF7F, 0x3F80, 0x0080]
        return np.array(vals, dtype=np.uint16)
    if dtype == "fp16":
        return np.array([0x0000, 0x8000, 0x7C00, 0xFC00, 0x7E01, 0x0001, 0x8001, 0x7BFF, 0xFBFF, 0x3C00],
                        dtype=np.uint16)
    return np.array([0.0, -0.0, np.inf, -np.inf, np.nan, 1e-45, -1e-45, 3.4e38, -3.4e38, 1.0], dtype=np.float32)


@pytest.mark.parametrize("dtype", ["bf16", "fp16", "fp32"])
@pytest.mark.parametrize("op", [0, 1, 2, 3])
def test_special_values(dtype, op):
    """Every ordered triple of special values (NaN, +-inf, +-0, subnormals,
    the largest finite values) across 3 ranks, vector and scalar paths."""
    need_gpu()
    v = special_values(dtype)
    k = v.size
    idx = np.array(np.meshgrid(np.arange(k), np.arange(k), np.arange(k), indexing="ij")).reshape(3, -1)
    xs = [v[idx[r]] for r in range(3)]
    for algo in (M.TWOSHOT, M.ONESHOT, M.RING, M.RING_STEPS):
        got = run_all_reduce(xs, dtype, op, algo)
        assert_ranks_equal(got, ALGO_FN[algo](xs, op, dtype), f"{dtype} {OPNAME[op]} algo {algo}")


def test_two_shot_160k_workload():
    """4 virtual ranks x 160 KB bf16 uniform[-1, 1], owner segments A..D."""
    need_gpu()
    xs = W.twoshot_160k()
    got = run_all_reduce(xs, "bf16", M.SUM, M.TWOSHOT)
    assert_ranks_equal(got, oracle.all_reduce_two_shot(xs, 0, "bf16"))


@pytest.mark.parametrize("tokens,hidden", W.tp_decode_shapes())
def test_tp_decode_workload(tokens, hidden):
    """8 ranks, bf16 [tokens, hidden] N(0,1): one-shot, two-shot and ring at
    the sizes the benchmark times, each bit-exact against its oracle; ring vs
    the rank-order reduction within 1 bf16 ulp."""
    need_gpu()
    xs = W.tp_decode(tokens, hidden)
    ref = oracle.all_reduce(xs, 0, "bf16")
    for algo in (M.ONESHOT, M.TWOSHOT, M.RING, M.RING_STEPS):
        got = run_all_reduce(xs, "bf16", M.SUM, algo)
        assert_ranks_equal(got, ALGO_FN[algo](xs, 0, "bf16"), f"algo {algo}")
        if algo == M.RING:
            assert int(oracle.bf16_ulp_diff(got[0], ref[0]).max()) <= 1


@pytest.mark.parametrize("dtype", ["bf16", "fp32", "int32"])
@pytest.mark.parametrize("op", [0, 1, 3])
@pytest.mark.parametrize("n", [1, 2, 8, 11])
def test_reduce_scatter(dtype, op, n):
    need_gpu()
    for per in (1, 8, 1000, 4096 * 3 + 5):
        xs = inputs(n, per * n, dtype, salt=per + op, dist="uniform" if op == 3 else "normal")
        send = [to_dev(x, dtype) for x in xs]
        recv = [torch.empty(per, dtype=send[0].dtype, device="cuda") for _ in range(n)]
        M.coll_reduce_scatter(send, recv, op=op)
        torch.cuda.synchronize()
        assert_ranks_equal([from_dev(t, dtype) for t in recv], oracle.reduce_scatter(xs, op, dtype), f"per {per}")


def test_reduce_scatter_in_place():
    need_gpu()
    n, per = 8, 12345
    xs = inputs(n, per * n, "bf16", salt=5)
    send = [to_dev(x, "bf16") for x in xs]
    recv = [send[r][r * per:(r + 1) * per] for r in range(n)]
    M.coll_reduce_scatter(send, recv)
    torch.cuda.synchronize()
    assert_ranks_equal([from_dev(t, "bf16") for t in recv], oracle.reduce_scatter(xs, 0, "bf16"))


@pytest.mark.parametrize("dtype", ["bf16", "fp16", "fp32", "int32"])
@pytest.mark.parametrize("op", [0, 1, 2, 3])
def test_reduce(dtype, op):
    need_gpu()
    n, count = 6, 77777
    xs = inputs(n, count, dtype, salt=op, dist="uniform")
    send = [to_dev(x, dtype) for x in xs]
    for dst in (0, n - 1):
        out = torch.empty_like(send[0])
        M.coll_reduce(send, out, dst, op=op)
        torch.cuda.synchronize()
        assert np.array_equal(bits(from_dev(out, dtype)), bits(oracle.reduce(xs, op, dtype)))
    # in place on the destination
    M.coll_reduce(send, send[2], 2, op=op)
    torch.cuda.synchronize()
    assert np.array_equal(bits(from_dev(send[2], dtype)), bits(oracle.reduce(xs, op, dtype)))


def test_sp_prefill_reduce_scatter_full_size():
    """8 ranks x bf16 [8192, 8192] -> [1024, 8192] blocks (the sequence-parallel
    prefill reduce-scatter), every element of every output block against the
    oracle.  The oracle runs on chunks of the block's element range (each
    element of a reduce-scatter depends only on the same element of every
    rank's input), so host memory stays bounded."""
    need_gpu()
    n, rows, cols = 8, 8192, 8192
    xs = W.sp_reduce_scatter(n, rows, cols)
    per = rows * cols // n
    send = [to_dev(x, "bf16") for x in xs]
    recv = [torch.empty(per, dtype=torch.bfloat16, device="cuda") for _ in range(n)]
    M.coll_reduce_scatter(send, recv)
    torch.cuda.synchronize()
    del send
    chunk = 1 << 20
    for lo in range(0, per, chunk):
        hi = min(per, lo + chunk)
        part = [np.concatenate([x[b * per + lo:b * per + hi] for b in range(n)]) for x in xs]
        want = oracle.reduce_scatter(part, 0, "bf16")
        for r in range(n):
            assert np.array_equal(from_dev(recv[r][lo:hi], "bf16"), want[r]), (r, lo)


@pytest.mark.parametrize("n,last", [(3, 256 << 10), (4, 64 << 10), (2, None), (8, None)])
@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_auto_both_sides_of_each_crossover(n, last, dtype):
    """AUTO at the measured crossovers: the form it reports on each side, and
    the result of the call against the oracle (both forms give the
    rank-order reduction), out of place and in place (always the two-shot)."""
    need_gpu()
    es = 2 if dtype == "bf16" else 4
    edge = last if last is not None else 64 << 10
    for nbytes in (edge, edge + 16):
        count = nbytes // es
        want_form = M.ONESHOT if last is not None and nbytes <= last else M.TWOSHOT
        tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
        assert M.coll_all_reduce_form(n, count, tdt, M.ALGO_AUTO) == want_form
        xs = inputs(n, count, dtype, salt=nbytes + n)
        want = oracle.all_reduce(xs, 0, dtype)
        send = [to_dev(x, dtype) for x in xs]
        recv = [torch.empty_like(t) for t in send]
        M.coll_all_reduce(send, recv, algo=M.ALGO_AUTO)
        M.coll_all_reduce(send, send, algo=M.ALGO_AUTO)  # in place
        torch.cuda.synchronize()
        for q in range(n):
            assert np.array_equal(bits(from_dev(recv[q], dtype)), bits(want[q])), (nbytes, q)
            assert np.array_equal(bits(from_dev(send[q], dtype)), bits(want[q])), (nbytes, q)
