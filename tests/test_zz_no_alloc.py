"""The no-allocation ring all-reduce (coll_all_reduce_ring_noalloc).

Some callers cannot allocate device memory: a plug-in that only receives the
ranks' buffers from a framework owning all device memory, or a process whose
memory was fully reserved at start-up.  For them the library keeps the ring's
scratch in a fixed array of its own.  This file checks that entry point
through the C ABI, on two calls in a row, against the ordinary ring
all-reduce (which takes a workspace) and against the ring oracle, bit for bit
-- the tolerance every reduction test here uses -- including buffers that
start one element off a 16-byte boundary (the element-wise path); that a
call with no elements works as the warm-up; and that a size beyond the fixed
array is refused.  It is collected last, so a failure here leaves every
other test already run.
"""
import numpy as np
import pytest
import torch

import movement_virtual_rank_b200 as M
import oracle
import workloads as W
from gpu_util import TORCH, from_dev, need_gpu, to_dev

pytestmark = pytest.mark.gpu


def _ring_with_workspace(send):
    recv = [torch.empty_like(t) for t in send]
    M.coll_all_reduce(send, recv, algo=M.RING)
    return recv


def _offset_copies(xs, dtype, offset):
    """Device buffers holding xs, each starting `offset` elements past an
    allocation's (256-byte aligned) start."""
    out = []
    for x in xs:
        raw = torch.empty(x.size + offset + 8, dtype=TORCH[dtype], device="cuda")
        view = raw[offset:offset + x.size]
        view.copy_(to_dev(x, dtype))
        out.append(view)
    return out


def test_noalloc_warm_up_with_no_elements():
    """count == 0 through the C ABI: the call succeeds and enqueues nothing
    (it only looks up the fixed array, which is why it serves as a warm-up)."""
    need_gpu()
    import ctypes
    bufs = [torch.full((16,), 3, dtype=torch.bfloat16, device="cuda") for _ in range(3)]
    ptrs = (ctypes.c_void_p * 3)(*[b.data_ptr() for b in bufs])
    rc = M.lib().coll_all_reduce_ring_noalloc(ptrs, ptrs, 3, 0, M.BF16, M.SUM, None)
    torch.cuda.synchronize()
    assert rc == 0
    assert all(bool((b == 3).all()) for b in bufs)


@pytest.mark.parametrize("dtype,n,count,offset", [("bf16", 8, 256 * 7168, 0), ("bf16", 5, 30011, 0),
                                                  ("fp32", 3, 4099, 0), ("bf16", 4, 20001, 1),
                                                  ("fp32", 6, 7777, 1)])
def test_noalloc_matches_ring_and_oracle_twice(dtype, n, count, offset):
    need_gpu()
    for call in range(2):  # the second call reuses the array the first one left behind
        xs = W.ranks_values(W.W_MISC, n, count, dtype, "normal", salt=1000 * call + count)
        send = _offset_copies(xs, dtype, offset)
        want = oracle.all_reduce_ring(xs, 0, dtype)
        ring = [from_dev(t, dtype) for t in _ring_with_workspace(send)]
        recv = _offset_copies([np.full_like(x, 7) for x in xs], dtype, offset)
        M.coll_all_reduce_ring_noalloc(send, recv)
        torch.cuda.synchronize()
        for q in range(n):
            got = from_dev(recv[q], dtype)
            assert np.array_equal(got.view(np.uint8), ring[q].view(np.uint8)), (call, q)
            assert np.array_equal(got.view(np.uint8), want[q].view(np.uint8)), (call, q)


def test_noalloc_in_place_and_limit():
    need_gpu()
    n, count = 4, 1000
    xs = W.ranks_values(W.W_MISC, n, count, "bf16", "normal", salt=5)
    send = [to_dev(x, "bf16") for x in xs]
    want = oracle.all_reduce_ring(xs, 0, "bf16")
    M.coll_all_reduce_ring_noalloc(send, send)
    torch.cuda.synchronize()
    for q in range(n):
        assert np.array_equal(from_dev(send[q], "bf16"), want[q])
    big = [torch.zeros(M.RING_NOALLOC_MAX_COUNT + 1, dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    with pytest.raises(M.CollError) as e:
        M.coll_all_reduce_ring_noalloc(big, big)
    assert e.value.code == -5
