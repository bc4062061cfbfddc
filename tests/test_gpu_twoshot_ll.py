"""GPU parity: the fused single-launch packet two-shot all-reduce, with LL
lines (COLL_ALGO_TWOSHOT_LL) and with LL128 lines (COLL_ALGO_TWOSHOT_LL128).

Both keep the two-shot owner segments and arithmetic, so their output is
compared bit for bit with the oracle's two-shot.  Repeated calls on one
workspace check that the per-call flag epoch keeps an earlier call's lines
from being taken for new ones; a call started with the abort word already
set must still finish, and leave the header ready for the next call.
"""
import numpy as np
import pytest
import torch

import movement_virtual_rank_b200 as M
import oracle
import workloads as W
from gpu_util import Guarded, from_dev, need_gpu, to_dev

pytestmark = pytest.mark.gpu


def bits(a):
    a = np.asarray(a)
    return a.view(np.uint32) if a.dtype == np.float32 else a


FORMS = pytest.mark.parametrize("algo", [M.TWOSHOT_LL, M.TWOSHOT_LL128], ids=["ll", "ll128"])


def workspace(n, count, dtype, algo):
    tdt = {"bf16": torch.bfloat16, "fp16": torch.float16, "fp32": torch.float32, "int32": torch.int32}[dtype]
    need = M.coll_all_reduce_workspace_size(n, count, tdt, algo)
    return torch.zeros(need, dtype=torch.uint8, device="cuda")


def run(xs, dtype, op, ws, algo, in_place=False):
    send = [to_dev(x, dtype) for x in xs]
    recv = send if in_place else [torch.empty_like(t) for t in send]
    M.coll_all_reduce(send, recv, op=op, algo=algo, workspace=ws)
    torch.cuda.synchronize()
    return [from_dev(t, dtype) for t in recv]


@pytest.mark.parametrize("n", [2, 3, 4, 5, 8, 16])
@pytest.mark.parametrize("count", [1, 9, 8 * 37 + 3, 4096, 65536 + 24, 300007])
@FORMS
def test_twoshot_ll_bf16_sum(algo, n, count):
    need_gpu()
    xs = W.ranks_values(W.W_MISC, n, count, "bf16", "normal", salt=count + 13 * n)
    ws = workspace(n, count, "bf16", algo)
    got = run(xs, "bf16", 0, ws, algo, in_place=(count % 2 == 1))
    want = oracle.all_reduce_two_shot(xs, 0, "bf16")
    for q in range(n):
        assert np.array_equal(got[q], want[q]), q
    assert ws[16:24].view(torch.int32).tolist() == [0, 0]


@pytest.mark.parametrize("dtype", ["bf16", "fp16", "fp32", "int32"])
@pytest.mark.parametrize("op", [0, 1, 2, 3])
@FORMS
def test_twoshot_ll_dtypes_ops(algo, dtype, op):
    need_gpu()
    n, count = 7, 12301
    if dtype == "int32":
        g = W.rng(W.W_MISC, 0, salt=op + 140)
        xs = [g.integers(-1000, 1000, count, dtype=np.int64).astype(np.int32) for _ in range(n)]
    else:
        xs = W.ranks_values(W.W_MISC, n, count, dtype, "uniform" if op == 3 else "normal", salt=op + 140)
    ws = workspace(n, count, dtype, algo)
    got = run(xs, dtype, op, ws, algo)
    want = oracle.all_reduce_two_shot(xs, op, dtype)
    for q in range(n):
        assert np.array_equal(bits(got[q]), bits(want[q])), q


@pytest.mark.parametrize("tokens,hidden", W.tp_decode_shapes())
@FORMS
def test_twoshot_ll_tp_decode_workload(algo, tokens, hidden):
    need_gpu()
    xs = W.tp_decode(tokens, hidden)
    ws = workspace(8, tokens * hidden, "bf16", algo)
    got = run(xs, "bf16", 0, ws, algo)
    want = oracle.all_reduce_two_shot(xs, 0, "bf16")
    for q in range(8):
        assert np.array_equal(got[q], want[q]), q


@FORMS
def test_twoshot_ll_epochs(algo):
    """Five calls on one workspace with new data each time: every call's
    lines carry a new epoch, so none is taken from an earlier call."""
    need_gpu()
    n, count = 8, 20000
    ws = workspace(n, count, "bf16", algo)
    for k in range(5):
        xs = W.ranks_values(W.W_MISC, n, count, "bf16", "normal", salt=500 + k)
        got = run(xs, "bf16", 0, ws, algo)
        want = oracle.all_reduce_two_shot(xs, 0, "bf16")
        assert all(np.array_equal(g, w) for g, w in zip(got, want)), k
        assert ws[0:4].view(torch.int32).item() == k + 1  # the call counter
    assert ws[16:24].view(torch.int32).tolist() == [0, 0]


@FORMS
def test_twoshot_ll_abort_word_clears(algo):
    """A call that starts with the abort word set stops its waiting polls
    and finishes; it leaves the header clear, and the next call is exact."""
    need_gpu()
    n, count = 4, 50000
    ws = workspace(n, count, "bf16", algo)
    ws[8:12].view(torch.int32).fill_(1)  # abort word
    xs = W.ranks_values(W.W_MISC, n, count, "bf16", "normal", salt=600)
    run(xs, "bf16", 0, ws, algo)
    assert ws[8:12].view(torch.int32).item() == 0
    assert ws[0:4].view(torch.int32).item() == 1
    got = run(xs, "bf16", 0, ws, algo)
    want = oracle.all_reduce_two_shot(xs, 0, "bf16")
    assert all(np.array_equal(g, w) for g, w in zip(got, want))


@FORMS
def test_twoshot_ll_unaligned_takes_twoshot(algo):
    """Buffers off a 16-byte boundary run the plain two-shot kernel: same bits."""
    need_gpu()
    n, count = 3, 1001
    xs = W.ranks_values(W.W_MISC, n, count, "bf16", "normal", salt=601)
    assert M.coll_all_reduce_form(n, count, torch.bfloat16, algo, aligned=False) == M.TWOSHOT
    send = [Guarded(count, "bf16", offset=2, fill=xs[r]) for r in range(n)]
    recv = [Guarded(count, "bf16", offset=2) for _ in range(n)]
    M.coll_all_reduce([b.t for b in send], [b.t for b in recv], algo=algo,
                      workspace=workspace(n, count, "bf16", algo))
    torch.cuda.synchronize()
    want = oracle.all_reduce_two_shot(xs, 0, "bf16")
    for q in range(n):
        assert np.array_equal(recv[q].host(), want[q])
    assert all(b.guards_intact() for b in send + recv)
