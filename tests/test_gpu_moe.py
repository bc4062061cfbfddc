"""GPU parity: MoE route / dispatch / combine vs the oracle.

Route outputs (split matrix, displacements, every pair's receive row) are
integers and compared exactly; dispatched rows are bit copies; combine is
bit-exact against the oracle's fp32 products-then-sums.  Small cases are
compared in full; the expert-parallel workload (8 ranks x 4096 tokens,
hidden 7168, 256 experts, top-8 Zipf-skewed routing) in full for route, on
every row's checksum and on sampled rows for dispatch, and on sampled
tokens for combine.
"""
import numpy as np
import pytest
import torch

import movement_virtual_rank_b200 as M
import oracle
import workloads as W
from gpu_util import from_dev, need_gpu, status_tensor, to_dev

pytestmark = pytest.mark.gpu


def route_on_device(ids, n_experts):
    n = len(ids)
    dids = [torch.from_numpy(np.ascontiguousarray(i)).cuda() for i in ids]
    sc = torch.empty(n * n, dtype=torch.int64, device="cuda")
    sd = torch.empty_like(sc)
    rd = torch.empty_like(sc)
    pos = [torch.empty(i.size, dtype=torch.int32, device="cuda") for i in ids]
    st = status_tensor()
    M.coll_moe_route(dids, n_experts, sc, sd, rd, pos, status=st)
    torch.cuda.synchronize()
    return dids, sc, sd, rd, pos, st


def check_route(ids, n_experts):
    n = len(ids)
    dids, sc, sd, rd, pos, st = route_on_device(ids, n_experts)
    wsc, wsd, wrd, wpos = oracle.moe_route(ids, n_experts)
    assert st.tolist() == [0, 0]
    assert np.array_equal(sc.cpu().numpy().reshape(n, n), wsc)
    assert np.array_equal(sd.cpu().numpy().reshape(n, n), wsd)
    assert np.array_equal(rd.cpu().numpy().reshape(n, n), wrd)
    for s in range(n):
        assert np.array_equal(pos[s].cpu().numpy(), wpos[s].astype(np.int32)), s
    return dids, pos, wsc, wpos


@pytest.mark.parametrize("n,tokens,topk,experts", [
    (1, 5, 1, 1), (2, 2, 1, 4), (2, 300, 2, 8), (4, 257, 4, 16), (8, 1000, 8, 64), (8, 512, 8, 1024),
    (3, 0, 2, 6), (5, 700, 3, 40)])
def test_route(n, tokens, topk, experts):
    need_gpu()
    ids, _ = W.moe_routing(tokens, experts, topk, n)
    check_route(ids, experts)


def test_route_tutorial_example():
    """Tutorial 8.4: rank 0 sends tA to expert 2, keeps tB (expert 0); rank 1
    sends tC to expert 1, keeps tD (expert 3)."""
    need_gpu()
    ids = [np.array([[2], [0]], np.int32), np.array([[1], [3]], np.int32)]
    dids, pos, wsc, wpos = check_route(ids, 4)
    # rows of width 2: rank 0 holds [tA, tB], rank 1 holds [tC, tD]
    x = [np.array([0x4000, 0x4001, 0x4100, 0x4101], np.uint16), np.array([0x4200, 0x4201, 0x4300, 0x4301], np.uint16)]
    xd = [to_dev(v, "bf16") for v in x]
    recv = [torch.zeros(4, dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    M.coll_moe_dispatch(xd, dids, pos, recv, 4)
    torch.cuda.synchronize()
    tA, tB, tC, tD = x[0][:2], x[0][2:], x[1][:2], x[1][2:]
    assert np.array_equal(from_dev(recv[0], "bf16"), np.concatenate([tB, tC]))
    assert np.array_equal(from_dev(recv[1], "bf16"), np.concatenate([tA, tD]))


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("n,tokens,topk,experts,hidden", [
    (2, 37, 2, 8, 8), (4, 300, 4, 16, 96), (8, 256, 8, 64, 200), (3, 50, 3, 9, 7)])
def test_dispatch_combine(dtype, n, tokens, topk, experts, hidden):
    need_gpu()
    ids, ws = W.moe_routing(tokens, experts, topk, n)
    xs = W.ranks_values(W.W_MISC, n, tokens * hidden, dtype, "normal", salt=hidden)
    dids, pos, wsc, wpos = check_route(ids, experts)
    cap = int(wsc.sum(axis=0).max())
    xd = [to_dev(x, dtype) for x in xs]
    recv = [torch.zeros(cap * hidden, dtype=xd[0].dtype, device="cuda") for _ in range(n)]
    st = status_tensor()
    M.coll_moe_dispatch(xd, dids, pos, recv, experts, status=st)
    torch.cuda.synchronize()
    assert st.tolist() == [0, 0]
    bufs = [np.zeros(cap * hidden, dtype=xs[0].dtype) for _ in range(n)]
    want = oracle.moe_dispatch(xs, ids, wpos, bufs, experts, hidden)
    got = [from_dev(t, dtype) for t in recv]
    for d in range(n):
        assert np.array_equal(got[d], want[d]), d
    # expert stand-in: scale each received row by 1 + (e mod 8)/8 (exact), so
    # that a row combined with the wrong expert's weight is caught
    scale = np.ones((n, cap), np.float32)
    epr = experts // n
    for s in range(n):
        for j, e in enumerate(ids[s].reshape(-1)):
            scale[int(e) // epr, int(wpos[s][j])] = 1 + (int(e) % 8) / 8
    ys = []
    for d in range(n):
        y = oracle.widen(want[d], dtype).reshape(cap, hidden) * scale[d][:, None]
        ys.append(oracle.narrow(y.reshape(-1).astype(np.float32), dtype))
    yd = [to_dev(y, dtype) for y in ys]
    wd = [torch.from_numpy(w).cuda() for w in ws]
    out = [torch.empty_like(x) for x in xd]
    M.coll_moe_combine(yd, dids, pos, wd, out, experts, status=st)
    torch.cuda.synchronize()
    assert st.tolist() == [0, 0]
    wc = oracle.moe_combine(ys, ids, wpos, ws, experts, hidden, dtype)
    for s in range(n):
        assert np.array_equal(from_dev(out[s], dtype), wc[s]), s


def test_bad_routes_and_overflow_are_reported():
    need_gpu()
    n, experts = 2, 4
    ids = [np.array([[0, 1], [1, 1], [2, 3]], np.int32), np.array([[0, 9], [2, 3], [1, 0]], np.int32)]
    _, _, _, _, _, st = route_on_device(ids, experts)
    assert st.tolist() == [M.DEV_BAD_ROUTE, 2]  # a repeated expert on rank 0, an id beyond range on rank 1
    good = [np.array([[0, 1], [2, 3]], np.int32), np.array([[0, 2], [1, 3]], np.int32)]
    dids, sc, sd, rd, pos, st = route_on_device(good, experts)
    x = [to_dev(np.arange(8, dtype=np.uint16), "bf16") for _ in range(n)]  # 2 tokens of hidden 4
    recv = [torch.zeros(8, dtype=torch.bfloat16, device="cuda") for _ in range(n)]  # 2 rows, 4 needed
    M.coll_moe_dispatch(x, dids, pos, recv, experts, status=st)
    torch.cuda.synchronize()
    assert st.tolist() == [M.DEV_SPLIT_OVERFLOW, 4]  # rows 2 and 3 of both destinations


def test_moe_workload():
    """8 ranks x 4096 tokens x hidden 7168 bf16, 256 experts, top-8 Zipf
    routing, at full size: every received row of the dispatch against the
    oracle's dispatch, and every combined token against the oracle's combine
    of the oracle's dispatch output (the identity expert), element by
    element."""
    need_gpu()
    n, tokens, topk, experts, hidden = 8, 4096, 8, 256, 7168
    ids, ws = W.moe_routing(tokens, experts, topk, n)
    xs = W.moe_tokens(tokens, hidden, n)
    dids, pos, wsc, wpos = check_route(ids, experts)
    per_dest = wsc.sum(axis=0)
    cap = int(per_dest.max())
    xd = [to_dev(x, "bf16") for x in xs]
    recv = [torch.empty(cap * hidden, dtype=torch.bfloat16, device="cuda") for _ in range(n)]
    st = status_tensor()
    M.coll_moe_dispatch(xd, dids, pos, recv, experts, status=st)
    torch.cuda.synchronize()
    assert st.tolist() == [0, 0]
    ys = oracle.moe_dispatch(xs, ids, wpos, [np.zeros(int(k) * hidden, np.uint16) for k in per_dest], experts,
                             hidden)
    for d in range(n):
        k = int(per_dest[d]) * hidden
        assert np.array_equal(from_dev(recv[d][:k], "bf16"), ys[d]), d
    wd = [torch.from_numpy(w).cuda() for w in ws]
    out = [torch.empty_like(x) for x in xd]
    M.coll_moe_combine(recv, dids, pos, wd, out, experts, status=st)
    torch.cuda.synchronize()
    assert st.tolist() == [0, 0]
    del xd, recv
    wc = oracle.moe_combine(ys, ids, wpos, ws, experts, hidden, "bf16")
    for s in range(n):
        assert np.array_equal(from_dev(out[s], "bf16"), wc[s]), s


@pytest.mark.parametrize("dtype,n,tokens,topk,experts,hidden", [
    ("bf16", 4, 1024, 4, 16, 4096), ("fp32", 3, 700, 3, 9, 4000)])
def test_dispatch_bulk_copy_path(dtype, n, tokens, topk, experts, hidden):
    """Enough rows per CTA for the bulk-copy dispatch: rows land exactly where
    the oracle puts them; a receive buffer a few rows short reports exactly
    the rows that do not fit and writes nothing outside it."""
    need_gpu()
    ids, ws = W.moe_routing(tokens, experts, topk, n)
    xs = W.ranks_values(W.W_MISC, n, tokens * hidden, dtype, "normal", salt=hidden + n)
    dids, pos, wsc, wpos = check_route(ids, experts)
    per_dest = wsc.sum(axis=0)
    cap = int(per_dest.max())
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
    short = cap - 5
    guard = [torch.full(((short + 2) * hidden,), 7.0, dtype=xd[0].dtype, device="cuda") for _ in range(n)]
    small = [g[:short * hidden] for g in guard]
    st.zero_()
    M.coll_moe_dispatch(xd, dids, pos, small, experts, status=st)
    torch.cuda.synchronize()
    lost = int(sum(max(0, int(c) - short) for c in per_dest))
    assert st.tolist() == [M.DEV_SPLIT_OVERFLOW, lost]
    fill = from_dev(torch.full(((short + 2) * hidden,), 7.0, dtype=xd[0].dtype, device="cuda"), dtype)
    for d in range(n):
        # rows the destination receives and that fit are written; every other
        # row of the buffer and its guard rows keep the fill value
        k = min(int(per_dest[d]), short) * hidden
        expect = fill.copy()
        expect[:k] = want[d][:k]
        assert np.array_equal(from_dev(guard[d], dtype), expect), d
