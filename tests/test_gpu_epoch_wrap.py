"""GPU: the call counter of the one-launch packet all-reduce forms (RING_LL,
TWOSHOT_LL, TWOSHOT_LL128) cannot wrap silently.

A line's flag carries the workspace's call counter in its upper bits (25 of
them for RING_LL, 30 for TWOSHOT_LL), so after that many calls the flags
would repeat those of the first call, and a FIFO line no call has rewritten
since could pass for a current one.  The kernels refuse instead: a call that
finds the counter used up does nothing but raise COLL_DEV_EPOCH_WRAP in the
workspace's status pair.  The test writes the counter (the u32 at byte 0 of
a zero-filled workspace) to two below the limit from the host, checks that
the next two calls are exact, that the third changes no output, leaves the
counter where it is and raises the code, and that a zero-filled workspace
serves again.  Nothing waits: the refusing kernel returns at once.
"""
import numpy as np
import pytest
import torch

import movement_virtual_rank_b200 as M
import oracle
import workloads as W
from gpu_util import from_dev, need_gpu, to_dev

pytestmark = pytest.mark.gpu

FORMS = [(M.RING_LL, M.RING_LL_CALLS_PER_FILL, oracle.all_reduce_ring),
         (M.TWOSHOT_LL, M.TWOSHOT_LL_CALLS_PER_FILL, oracle.all_reduce_two_shot),
         (M.TWOSHOT_LL128, M.TWOSHOT_LL_CALLS_PER_FILL, oracle.all_reduce_two_shot)]


@pytest.mark.parametrize("algo,limit,ref", FORMS, ids=["ring_ll", "twoshot_ll", "twoshot_ll128"])
@pytest.mark.parametrize("n,count", [(4, 5000), (8, 65536 + 24)])
def test_counter_stops_at_its_limit(algo, limit, ref, n, count):
    need_gpu()
    need = M.coll_all_reduce_workspace_size(n, count, torch.bfloat16, algo)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    hdr = ws[:4].view(torch.int32)
    hdr.fill_(limit - 2)  # the counter, two calls before its limit
    status = ws[16:24].view(torch.int32)
    for call in range(2):
        xs = W.ranks_values(W.W_MISC, n, count, "bf16", "normal", salt=31 * call + n)
        send = [to_dev(x, "bf16") for x in xs]
        recv = [torch.empty_like(t) for t in send]
        M.coll_all_reduce(send, recv, algo=algo, workspace=ws)
        torch.cuda.synchronize()
        want = ref(xs, 0, "bf16")
        for q in range(n):
            assert np.array_equal(from_dev(recv[q], "bf16"), want[q]), (call, q)
        assert status.tolist() == [0, 0]
    assert int(hdr.item()) == limit
    # the counter is used up: the call does nothing and says so
    xs = W.ranks_values(W.W_MISC, n, count, "bf16", "normal", salt=97)
    send = [to_dev(x, "bf16") for x in xs]
    recv = [torch.full_like(t, 5.0) for t in send]
    M.coll_all_reduce(send, recv, algo=algo, workspace=ws)
    torch.cuda.synchronize()
    assert status.tolist() == [M.DEV_EPOCH_WRAP, 1]
    assert int(hdr.item()) == limit
    for q in range(n):
        assert bool((recv[q] == 5.0).all()), q
    # a zero-filled workspace serves again
    ws.zero_()
    M.coll_all_reduce(send, recv, algo=algo, workspace=ws)
    torch.cuda.synchronize()
    want = ref(xs, 0, "bf16")
    for q in range(n):
        assert np.array_equal(from_dev(recv[q], "bf16"), want[q]), q
    assert status.tolist() == [0, 0]
    assert int(hdr.item()) == 1
