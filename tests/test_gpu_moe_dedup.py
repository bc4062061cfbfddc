"""GPU parity: the MoE route deduplicated per (token, destination rank).

coll_moe_route_dedup is compared exactly with the oracle's moe_route_dedup
(split matrix, displacements, every pair's receive row).  Dispatch with those
positions must leave exactly the oracle's receive buffers (a row reached by
two choices of a token is one row), and combine must give the oracle's
result, which equals the plain route's combine bit for bit when the expert
is the identity.
"""
import numpy as np
import pytest
import torch

import movement_virtual_rank_b200 as M
import oracle
import workloads as W
from gpu_util import from_dev, need_gpu, status_tensor, to_dev

pytestmark = pytest.mark.gpu


def route_on_device(ids, n_experts, dedup=True):
    n = len(ids)
    dids = [torch.from_numpy(np.ascontiguousarray(i)).cuda() for i in ids]
    sc = torch.empty(n * n, dtype=torch.int64, device="cuda")
    sd = torch.empty_like(sc)
    rd = torch.empty_like(sc)
    pos = [torch.empty(i.size, dtype=torch.int32, device="cuda") for i in ids]
    st = status_tensor()
    M.coll_moe_route(dids, n_experts, sc, sd, rd, pos, status=st, dedup=dedup)
    torch.cuda.synchronize()
    return dids, sc, sd, rd, pos, st


def check_route_dedup(ids, n_experts):
    n = len(ids)
    dids, sc, sd, rd, pos, st = route_on_device(ids, n_experts)
    wsc, wsd, wrd, wpos = oracle.moe_route_dedup(ids, n_experts)
    assert st.tolist() == [0, 0]
    assert np.array_equal(sc.cpu().numpy().reshape(n, n), wsc)
    assert np.array_equal(sd.cpu().numpy().reshape(n, n), wsd)
    assert np.array_equal(rd.cpu().numpy().reshape(n, n), wrd)
    for s in range(n):
        assert np.array_equal(pos[s].cpu().numpy(), wpos[s].astype(np.int32)), s
    return dids, pos, wsc, wpos


@pytest.mark.parametrize("n,tokens,topk,experts", [
    (1, 5, 1, 1), (2, 2, 1, 4), (2, 300, 2, 8), (4, 257, 4, 16), (8, 1000, 8, 64), (8, 512, 8, 1024),
    (3, 0, 2, 6), (5, 700, 3, 40), (8, 4096, 8, 256)])
def test_route_dedup(n, tokens, topk, experts):
    need_gpu()
    ids, _ = W.moe_routing(tokens, experts, topk, n)
    check_route_dedup(ids, experts)


def test_route_dedup_hand_example():
    need_gpu()
    ids = [np.array([[0, 1], [2, 0], [3, 2]], np.int32), np.array([[1, 3], [0, 1], [2, 3]], np.int32)]
    _, pos, wsc, _ = check_route_dedup(ids, 4)
    assert wsc.tolist() == [[2, 2], [2, 2]]
    assert pos[0].tolist() == [0, 0, 0, 1, 1, 1] and pos[1].tolist() == [2, 2, 3, 3, 3, 3]


def test_route_dedup_repeated_expert_is_reported():
    need_gpu()
    ids = [np.array([[0, 1], [1, 1], [2, 3]], np.int32), np.array([[0, 9], [2, 3], [1, 0]], np.int32)]
    st = route_on_device(ids, 4)[-1]
    assert st.tolist() == [M.DEV_BAD_ROUTE, 2]


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("n,tokens,topk,experts,hidden", [
    (2, 37, 2, 8, 8), (4, 300, 4, 16, 96), (8, 256, 8, 64, 200), (3, 50, 3, 9, 7), (4, 1024, 4, 16, 4096)])
def test_dispatch_combine_dedup(dtype, n, tokens, topk, experts, hidden):
    """The last case has enough rows for the bulk-copy dispatch."""
    need_gpu()
    ids, ws = W.moe_routing(tokens, experts, topk, n)
    xs = W.ranks_values(W.W_MISC, n, tokens * hidden, dtype, "normal", salt=hidden + 3)
    dids, pos, wsc, wpos = check_route_dedup(ids, experts)
    cap = int(wsc.sum(axis=0).max())
    xd = [to_dev(x, dtype) for x in xs]
    recv = [torch.zeros(cap * hidden, dtype=xd[0].dtype, device="cuda") for _ in range(n)]
    st = status_tensor()
    M.coll_moe_dispatch(xd, dids, pos, recv, experts, status=st)
    torch.cuda.synchronize()
    assert st.tolist() == [0, 0]
    want = oracle.moe_dispatch(xs, ids, wpos, [np.zeros(cap * hidden, dtype=xs[0].dtype) for _ in range(n)],
                               experts, hidden)
    for d in range(n):
        assert np.array_equal(from_dev(recv[d], dtype), want[d]), d
    wd = [torch.from_numpy(w).cuda() for w in ws]
    out = [torch.empty_like(x) for x in xd]
    M.coll_moe_combine(recv, dids, pos, wd, out, experts, status=st)
    torch.cuda.synchronize()
    assert st.tolist() == [0, 0]
    wc = oracle.moe_combine(want, ids, wpos, ws, experts, hidden, dtype)
    for s in range(n):
        assert np.array_equal(from_dev(out[s], dtype), wc[s]), s
    # the plain route through the same kernels: the same combined bits
    pdids, psc, _, _, ppos, _ = route_on_device(ids, experts, dedup=False)
    pcap = int(psc.cpu().numpy().reshape(n, n).sum(axis=0).max())
    precv = [torch.zeros(pcap * hidden, dtype=xd[0].dtype, device="cuda") for _ in range(n)]
    M.coll_moe_dispatch(xd, pdids, ppos, precv, experts)
    pout = [torch.empty_like(x) for x in xd]
    M.coll_moe_combine(precv, pdids, ppos, wd, pout, experts)
    torch.cuda.synchronize()
    for s in range(n):
        assert torch.equal(out[s].view(torch.uint8), pout[s].view(torch.uint8)), s


def test_moe_workload_dedup():
    """8 ranks x 4096 tokens x hidden 7168 bf16, 256 experts, top-8 Zipf
    routing: route exact; every received row against its source row on the
    device; combine equal to the plain route's combine on every element."""
    need_gpu()
    n, tokens, topk, experts, hidden = 8, 4096, 8, 256, 7168
    ids, ws = W.moe_routing(tokens, experts, topk, n)
    xs = W.moe_tokens(tokens, hidden, n)
    dids, pos, wsc, wpos = check_route_dedup(ids, experts)
    cap = int(wsc.sum(axis=0).max())
    xd = [to_dev(x, "bf16") for x in xs]
    recv = [torch.empty(cap * hidden, dtype=torch.bfloat16, device="cuda") for _ in range(n)]
    st = status_tensor()
    M.coll_moe_dispatch(xd, dids, pos, recv, experts, status=st)
    torch.cuda.synchronize()
    assert st.tolist() == [0, 0]
    epr = experts // n
    for s in range(n):
        d = ids[s].reshape(-1).astype(np.int64) // epr
        tok = np.repeat(np.arange(tokens), topk)
        src_rows = xd[s].view(tokens, hidden)
        for dd in range(n):
            m = d == dd
            got = recv[dd].view(cap, hidden)[torch.from_numpy(wpos[s][m]).cuda()]
            assert torch.equal(got.view(torch.int16), src_rows[torch.from_numpy(tok[m]).cuda()].view(torch.int16))
    wd = [torch.from_numpy(w).cuda() for w in ws]
    out = [torch.empty_like(x) for x in xd]
    M.coll_moe_combine(recv, dids, pos, wd, out, experts, status=st)
    del recv
    pdids, psc, _, _, ppos, _ = route_on_device(ids, experts, dedup=False)
    pcap = int(psc.cpu().numpy().reshape(n, n).sum(axis=0).max())
    precv = [torch.empty(pcap * hidden, dtype=torch.bfloat16, device="cuda") for _ in range(n)]
    M.coll_moe_dispatch(xd, pdids, ppos, precv, experts)
    pout = [torch.empty_like(x) for x in xd]
    M.coll_moe_combine(precv, pdids, ppos, wd, pout, experts)
    torch.cuda.synchronize()
    assert st.tolist() == [0, 0]
    for s in range(n):
        assert torch.equal(out[s].view(torch.int16), pout[s].view(torch.int16)), s
    # fewer rows moved than (token, expert) pairs
    assert int(wsc.sum()) < n * tokens * topk
