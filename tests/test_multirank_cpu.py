"""The multi-process harness of bench.py on CPU (gloo, world size 2).

Every GPU runs an independent replica of the virtual-rank engine, so the only
cross-process steps are the harness's own: the barrier around the timed
region, the max over ranks of the device time, and the sum of work.  These
run here as two gloo ranks; a rank that never joins makes the others fail
with a timeout instead of hanging.
"""
import datetime
import os
import socket

import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q, mode):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench

    try:
        if mode == "absent" and rank == 1:
            return  # this rank never joins
        dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=5))
        r, w, local = bench.dist_env()
        assert (r, w, local) == (rank, world, rank)
        bench.barrier(w)
        mx = bench.max_over_ranks(1.5 + rank, w, "cpu")
        sm = bench.sum_over_ranks(10.0 * (rank + 1), w, "cpu")
        bench.barrier(w)
        q.put((rank, mx, sm))
        dist.destroy_process_group()
    except Exception as e:  # reported to the parent
        q.put((rank, "error", type(e).__name__))


def _run(mode):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_worker, args=(r, 2, port, q, mode)) for r in range(2)]
    for p in ps:
        p.start()
    for p in ps:
        p.join(timeout=120)
        if p.is_alive():
            p.kill()
    out = []
    while not q.empty():
        out.append(q.get())
    return sorted(out, key=lambda t: t[0])


def test_max_and_sum_over_two_ranks():
    res = _run("ok")
    assert res == [(0, 2.5, 30.0), (1, 2.5, 30.0)]


def test_missing_rank_times_out_not_hangs():
    res = _run("absent")
    assert len(res) == 1 and res[0][0] == 0 and res[0][1] == "error"
