"""GPU parity: RING_WIRE, the ring whose reduce-scatter hops carry the
partial rounded to the buffers' type, against the oracle's definition of
that variant (``oracle.all_reduce_ring_wire``), bit for bit.

The variant has its own result (an extra rounding per hop for bf16 / fp16
SUM and PROD); for fp32, int32, MAX and MIN it equals RING's, which the
oracle's pins establish and these tests check on the device as well.
"""
import numpy as np
import pytest
import torch

import movement_virtual_rank_b200 as M
import oracle
import workloads as W
from gpu_util import from_dev, need_gpu, to_dev

pytestmark = pytest.mark.gpu


def bits(a):
    a = np.asarray(a)
    return a.view(np.uint32) if a.dtype == np.float32 else a


def run(xs, dtype, op, in_place=False):
    send = [to_dev(x, dtype) for x in xs]
    recv = send if in_place else [torch.empty_like(t) for t in send]
    M.coll_all_reduce(send, recv, op=op, algo=M.RING_WIRE)
    torch.cuda.synchronize()
    return [from_dev(t, dtype) for t in recv]


def inputs(n, count, dtype, op, salt):
    if dtype == "int32":
        g = W.rng(W.W_MISC, 0, salt=salt)
        return [g.integers(-1000, 1000, count, dtype=np.int64).astype(np.int32) for _ in range(n)]
    return W.ranks_values(W.W_MISC, n, count, dtype, "uniform" if op == 3 else "normal", salt=salt)


@pytest.mark.parametrize("n", [2, 3, 4, 5, 6, 7, 8])
@pytest.mark.parametrize("count", [1, 9, 8 * 37 + 3, 65536 + 24, 300007])
def test_ring_wire_bf16_sum(n, count):
    need_gpu()
    xs = inputs(n, count, "bf16", 0, count + 13 * n)
    got = run(xs, "bf16", 0, in_place=(count % 2 == 1))
    want = oracle.all_reduce_ring_wire(xs, 0, "bf16")
    for q in range(n):
        assert np.array_equal(got[q], want[q]), q


@pytest.mark.parametrize("dtype", ["bf16", "fp16", "fp32", "int32"])
@pytest.mark.parametrize("op", [0, 1, 2, 3])
@pytest.mark.parametrize("n,count", [(7, 12301), (8, 4_194_311)])
def test_ring_wire_dtypes_ops(dtype, op, n, count):
    """Every dtype and op, at 7 ranks (the loops for any rank count) and at 8
    ranks across many tiles (the unrolled kernel with register prefetch)."""
    need_gpu()
    xs = inputs(n, count, dtype, op, op + 90 + n)
    got = run(xs, dtype, op, in_place=(op % 2 == 1))
    want = oracle.all_reduce_ring_wire(xs, op, dtype)
    for q in range(n):
        assert np.array_equal(bits(got[q]), bits(want[q])), q
    if dtype in ("fp32", "int32") or op in (1, 2):  # rounding to the storage type changes nothing
        ring = oracle.all_reduce_ring(xs, op, dtype)
        assert all(np.array_equal(bits(g), bits(r)) for g, r in zip(got, ring))


def test_ring_wire_tp_decode_workload():
    need_gpu()
    for tokens, hidden in W.tp_decode_shapes():
        xs = W.tp_decode(tokens, hidden)
        got = run(xs, "bf16", 0)
        want = oracle.all_reduce_ring_wire(xs, 0, "bf16")
        for q in range(8):
            assert np.array_equal(got[q], want[q]), (tokens, hidden, q)


def test_ring_wire_needs_aligned_buffers_and_at_most_8_ranks():
    need_gpu()
    n, count = 4, 5001
    raw = [torch.zeros(count + 8, dtype=torch.bfloat16, device="cuda") for _ in range(n)]
    send = [t[1:count + 1] for t in raw]
    recv = [torch.empty(count + 8, dtype=torch.bfloat16, device="cuda")[3:count + 3] for _ in range(n)]
    with pytest.raises(M.CollError):
        M.coll_all_reduce(send, recv, algo=M.RING_WIRE)
    xs = [torch.zeros(64, dtype=torch.bfloat16, device="cuda") for _ in range(9)]
    with pytest.raises(M.CollError):
        M.coll_all_reduce(xs, [torch.empty_like(t) for t in xs], algo=M.RING_WIRE)
