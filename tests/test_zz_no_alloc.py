"""The no-allocation ring all-reduce (coll_all_reduce_ring_noalloc).

Some callers cannot allocate device memory: a plug-in that only receives the
ranks' buffers from a framework owning all device memory, or a process whose
memory was fully reserved at start-up.  For them the library keeps the ring's
scratch in a fixed array of its own.  This file checks that entry point
through the C ABI against the ordinary ring all-reduce (which takes a
workspace), bit for bit -- the tolerance every reduction test here uses --
on two calls in a row, and that a size beyond the fixed array is refused.
It is collected last, so a failure here leaves every other test already run.
"""
import numpy as np
import pytest
import torch

import movement_virtual_rank_b200 as M
import workloads as W
from gpu_util import from_dev, need_gpu, to_dev

pytestmark = pytest.mark.gpu


def _ring_with_workspace(send):
    recv = [torch.empty_like(t) for t in send]
    M.coll_all_reduce(send, recv, algo=M.RING)
    return recv


@pytest.mark.parametrize("dtype,n,count", [("bf16", 8, 256 * 7168), ("bf16", 5, 30011), ("fp32", 3, 4099)])
def test_noalloc_matches_ring_twice(dtype, n, count):
    need_gpu()
    for call in range(2):  # the second call reuses the array the first one left behind
        xs = W.ranks_values(W.W_MISC, n, count, dtype, "normal", salt=1000 * call + count)
        send = [to_dev(x, dtype) for x in xs]
        want = [from_dev(t, dtype) for t in _ring_with_workspace(send)]
        recv = [torch.full_like(t, 7) for t in send]
        M.coll_all_reduce_ring_noalloc(send, recv)
        torch.cuda.synchronize()
        for q in range(n):
            got = from_dev(recv[q], dtype)
            assert np.array_equal(got.view(np.uint8), want[q].view(np.uint8)), (call, q)


def test_noalloc_in_place_and_limit():
    need_gpu()
    n, count = 4, 1000
    xs = W.ranks_values(W.W_MISC, n, count, "bf16", "normal", salt=5)
    send = [to_dev(x, "bf16") for x in xs]
    want = [from_dev(t, "bf16") for t in _ring_with_workspace(send)]
    M.coll_all_reduce_ring_noalloc(send, send)
    torch.cuda.synchronize()
    for q in range(n):
        assert np.array_equal(from_dev(send[q], "bf16"), want[q])
    big = [torch.zeros(M.RING_NOALLOC_MAX_COUNT + 1, dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    with pytest.raises(M.CollError) as e:
        M.coll_all_reduce_ring_noalloc(big, big)
    assert e.value.code == -5
