"""Benchmark of the virtual-rank collectives on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload tp_decode|twoshot_160k|sp_prefill|moe|ll_sweep]

One "step" is one pass over every op of the chosen workload, each on its own
seeded synthetic inputs resident in HBM.  Before every op the L2 is flushed
(a memset of twice its size, outside the timed events); every op is timed
alone with CUDA events on the stream it runs on.  The step time is the sum of
the ops' times; ``value`` is the ops' algorithmic bytes (what each collective
must read plus write, once) over that time, summed over all GPUs, in GB/s.

Default workload (``tp_decode``): 8 virtual ranks, the TP-decode all-reduce
after RowParallelLinear (bf16 [tokens, hidden], tokens 1..256, hidden
4096/7168, N(0,1)) by one-shot, two-shot and ring, plus the broadcast of
int32 sampled_token_ids[256] from rank 7.

With --gpus N > 1 (torchrun, one process per GPU) every GPU runs its own
independent replica: the virtual ranks live inside one GPU, so there is no
exchange between GPUs (weak scaling; timing is the max over ranks).

``--impl reference`` times the CPU oracle (the plain definition of each op)
on this host's cores on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import contextlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

METRIC = "collective HBM GB/s (% of B200 peak) per op vs message size; µs/allreduce"


# ------------------------------------------------------------ workloads ----

class Op:
    """One timed collective call.

    run():    launches it (device buffers already filled)
    ref():    the oracle's version on the host inputs (CPU baseline)
    inputs:   [(device tensor, pinned host tensor)] for the end-to-end leg
    outputs:  [(device tensor, pinned host tensor)]
    """

    def __init__(self, name, run, alg_bytes, launches, inputs, outputs, meta, ref=None, kernel=None,
                 per_launch_bytes=None):
        self.name, self.run, self.alg_bytes, self.launches = name, run, alg_bytes, launches
        self.inputs, self.outputs, self.meta, self.ref = inputs, outputs, meta, ref
        self.kernel = kernel or name
        self.per_launch_bytes = per_launch_bytes if per_launch_bytes is not None else alg_bytes
        self.times = []
        self.e2e_times = []


def _pinned_like(t):
    import torch
    return torch.empty(t.shape, dtype=t.dtype, pin_memory=True)


def _dev(a: np.ndarray, dtype):
    import torch
    view = {torch.bfloat16: np.int16, torch.int32: np.int32, torch.float32: np.float32, torch.uint8: np.uint8}[dtype]
    tv = {torch.bfloat16: torch.int16}.get(dtype, dtype)
    return torch.from_numpy(np.ascontiguousarray(a).view(view).copy()).view(tv).view(dtype).cuda()


def build_tp_decode(M, oracle):
    import torch
    ops = []
    n = 8
    for tokens, hidden in W.tp_decode_shapes():
        xs = W.tp_decode(tokens, hidden, n)
        send = [_dev(x, torch.bfloat16) for x in xs]
        recv = [torch.empty_like(t) for t in send]
        ws = torch.empty(max(256, M.coll_all_reduce_workspace_size(n, tokens * hidden, torch.bfloat16, M.RING)),
                         dtype=torch.uint8, device="cuda")
        S = tokens * hidden * 2
        ins = [(t, _pinned_like(t)) for t in send]
        outs = [(t, _pinned_like(t)) for t in recv]
        for algo, aname, ref, launches in ((M.ONESHOT, "oneshot", oracle.all_reduce_one_shot, 1),
                                           (M.TWOSHOT, "twoshot", oracle.all_reduce_two_shot, 1),
                                           (M.RING, "ring", oracle.all_reduce_ring, 2 * (n - 1))):
            def run(send=send, recv=recv, algo=algo, ws=ws):
                M.coll_all_reduce(send, recv, algo=algo, workspace=ws)

            ops.append(Op(f"all_reduce/{aname}", run, 2 * n * S, launches, ins, outs,
                          {"op": "all_reduce", "algo": aname, "ranks": n, "shape": [tokens, hidden],
                           "bytes_per_rank": S},
                          ref=(lambda xs=xs, ref=ref: ref(xs, 0, "bf16")),
                          kernel=f"all_reduce/{aname}"))
    ids = W.sampled_token_ids(n)
    bufs = [_dev(x, torch.int32) for x in ids]

    def run_bc(bufs=bufs):
        M.coll_broadcast(bufs, 7)

    S = 256 * 4
    ops.append(Op("broadcast", run_bc, S * n, 1, [(t, _pinned_like(t)) for t in bufs],
                  [(t, _pinned_like(t)) for t in bufs],
                  {"op": "broadcast", "src": 7, "ranks": n, "dtype": "int32", "count": 256, "bytes_per_rank": S},
                  ref=lambda ids=ids: oracle.broadcast(ids, 7), kernel="broadcast"))
    cfg = {"workload": "tp_decode_allreduce_8vr", "virtual_ranks": n, "dtype": "bf16",
           "tokens": list(W.TP_DECODE_TOKENS), "hidden": list(W.TP_DECODE_HIDDEN),
           "algos": ["oneshot", "twoshot", "ring"], "plus": "broadcast int32[256] src=7",
           "values": "N(0,1) bf16 per rank, seeded"}
    return ops, cfg


def build_twoshot_160k(M, oracle):
    import torch
    n = 4
    xs = W.twoshot_160k(n)
    send = [_dev(x, torch.bfloat16) for x in xs]
    recv = [torch.empty_like(t) for t in send]
    S = xs[0].size * 2

    def run():
        M.coll_all_reduce(send, recv, algo=M.TWOSHOT)

    ops = [Op("all_reduce/twoshot", run, 2 * n * S, 1, [(t, _pinned_like(t)) for t in send],
              [(t, _pinned_like(t)) for t in recv],
              {"op": "all_reduce", "algo": "twoshot", "ranks": n, "bytes_per_rank": S},
              ref=lambda: oracle.all_reduce_two_shot(xs, 0, "bf16"), kernel="all_reduce/twoshot")]
    return ops, {"workload": "allreduce_twoshot_4vr_160KB", "virtual_ranks": n, "dtype": "bf16",
                 "values": "uniform[-1,1] bf16, seeded"}


def build_sp_prefill(M, oracle):
    import torch
    n = 8
    ag_in = W.sp_allgather(n)
    rs_in = W.sp_reduce_scatter(n)
    lg_in = W.logits_shards(n)
    ag_send = [_dev(x, torch.bfloat16) for x in ag_in]
    ag_recv = [torch.empty(n * x.size, dtype=torch.bfloat16, device="cuda") for x in ag_in]
    rs_send = [_dev(x, torch.bfloat16) for x in rs_in]
    rs_recv = [torch.empty(x.size // n, dtype=torch.bfloat16, device="cuda") for x in rs_in]
    lg_send = [_dev(x, torch.float32).reshape(256, 16032) for x in lg_in]
    lg_out = torch.empty(256, n * 16032, dtype=torch.float32, device="cuda")
    S_ag = ag_in[0].size * 2
    S_rs = rs_in[0].size * 2
    S_lg = lg_in[0].size * 4
    ops = [
        Op("all_gather", lambda: M.coll_all_gather(ag_send, ag_recv), n * S_ag + n * n * S_ag, 1,
           [(t, _pinned_like(t)) for t in ag_send], [(t, _pinned_like(t)) for t in ag_recv],
           {"op": "all_gather", "ranks": n, "bytes_per_rank": S_ag},
           ref=lambda: oracle.all_gather(ag_in), kernel="all_gather"),
        Op("reduce_scatter", lambda: M.coll_reduce_scatter(rs_send, rs_recv), n * S_rs + S_rs, 1,
           [(t, _pinned_like(t)) for t in rs_send], [(t, _pinned_like(t)) for t in rs_recv],
           {"op": "reduce_scatter", "ranks": n, "bytes_per_rank": S_rs},
           ref=lambda: oracle.reduce_scatter(rs_in, 0, "bf16"), kernel="reduce_scatter"),
        Op("gather", lambda: M.coll_gather(lg_send, lg_out, 0), 2 * n * S_lg, 1,
           [(t, _pinned_like(t)) for t in lg_send], [(lg_out, _pinned_like(lg_out))],
           {"op": "gather", "dst": 0, "ranks": n, "bytes_per_rank": S_lg, "dtype": "fp32"},
           ref=lambda: oracle.gather(lg_in, np.zeros(n * lg_in[0].size, np.float32), rows=256), kernel="gather"),
    ]
    return ops, {"workload": "sp_prefill_ag_rs_gather_8vr", "virtual_ranks": n,
                 "all_gather": "bf16 [1024,8192] -> [8192,8192]", "reduce_scatter": "bf16 [8192,8192] -> [1024,8192]",
                 "gather": "fp32 [256,16032] -> dst 0 [256,128256]"}


def build_moe(M, oracle):
    import torch
    n, tokens, topk, experts, hidden = 8, 4096, 8, 256, 7168
    ids, ws = W.moe_routing(tokens, experts, topk, n)
    xs = W.moe_tokens(tokens, hidden, n)
    dids = [torch.from_numpy(i).cuda() for i in ids]
    dw = [torch.from_numpy(w).cuda() for w in ws]
    x = [_dev(v, torch.bfloat16) for v in xs]
    sc = torch.empty(n * n, dtype=torch.int64, device="cuda")
    sd, rd = torch.empty_like(sc), torch.empty_like(sc)
    pos = [torch.empty(tokens * topk, dtype=torch.int32, device="cuda") for _ in range(n)]
    wsp = torch.empty(M.coll_moe_route_workspace_size(n, tokens, topk, experts), dtype=torch.uint8, device="cuda")
    M.coll_moe_route(dids, experts, sc, sd, rd, pos, workspace=wsp)
    torch.cuda.synchronize()
    cap = int(sc.view(n, n).sum(0).max().item())
    recv = [torch.empty(cap * hidden, dtype=torch.bfloat16, device="cuda") for _ in range(n)]
    out = [torch.empty_like(t) for t in x]
    row = hidden * 2
    pairs = n * tokens * topk
    ops = [
        Op("moe_route", lambda: M.coll_moe_route(dids, experts, sc, sd, rd, pos, workspace=wsp),
           pairs * 4 * 2, 3, [(t, _pinned_like(t)) for t in dids], [(t, _pinned_like(t)) for t in pos],
           {"op": "moe_route", "ranks": n, "tokens": tokens, "topk": topk, "experts": experts},
           ref=lambda: oracle.moe_route(ids, experts), kernel="moe_route"),
        Op("moe_dispatch", lambda: M.coll_moe_dispatch(x, dids, pos, recv, experts),
           n * tokens * row + pairs * row, 1, [(t, _pinned_like(t)) for t in x], [(t, _pinned_like(t)) for t in recv],
           {"op": "moe_dispatch", "ranks": n, "hidden": hidden, "rows_out": pairs}, kernel="moe_dispatch"),
        Op("moe_combine", lambda: M.coll_moe_combine(recv, dids, pos, dw, out, experts),
           pairs * row + pairs * 4 + n * tokens * row, 1, [(t, _pinned_like(t)) for t in recv],
           [(t, _pinned_like(t)) for t in out],
           {"op": "moe_combine", "ranks": n, "hidden": hidden}, kernel="moe_combine"),
    ]
    return ops, {"workload": "moe_dispatch_combine_8vr", "virtual_ranks": n, "tokens": tokens, "hidden": hidden,
                 "experts": experts, "topk": topk, "routing": "softmax(N(0,1)+log Zipf(1.1)) top-8, renormalised"}


def build_ll_sweep(M, oracle, sizes=None):
    import torch
    n = 8
    sizes = sizes or [1 << k for k in range(10, 29, 2)]
    ops = []
    for nbytes in sizes:
        count = nbytes // 2
        xs = W.ll_message(nbytes, n)
        send = [_dev(x, torch.bfloat16) for x in xs]
        recv = [torch.empty_like(t) for t in send]
        ops.append(Op(f"all_reduce/simple/{nbytes}", lambda s=send, r=recv: M.coll_all_reduce(s, r, algo=M.TWOSHOT),
                      2 * n * nbytes, 1, [], [], {"op": "all_reduce", "proto": "simple", "bytes_per_rank": nbytes},
                      kernel="all_reduce/twoshot"))
        for proto, pname in ((M.LL, "ll"), (M.LL128, "ll128")):
            pb = M.coll_packed_bytes(nbytes, proto)
            packed = [torch.empty(pb, dtype=torch.uint8, device="cuda") for _ in range(n)]
            for r in range(n):
                M.coll_ll_pack(send[r], packed[r], proto, 1)
            pout = [torch.empty(pb, dtype=torch.uint8, device="cuda") for _ in range(n)]
            ops.append(Op(f"all_reduce/{pname}/{nbytes}",
                          lambda p=packed, o=pout, c=count, pr=proto: M.coll_all_reduce_packed(p, o, c, torch.bfloat16, pr, 1),
                          2 * n * nbytes, 1, [], [],
                          {"op": "all_reduce_packed", "proto": pname, "bytes_per_rank": nbytes, "line_bytes": 2 * n * pb},
                          kernel=f"all_reduce/{pname}", per_launch_bytes=2 * n * pb))
    return ops, {"workload": "ll_ll128_allreduce_sweep_8vr", "virtual_ranks": n, "sizes": sizes}


WORKLOADS = {
    "tp_decode": build_tp_decode,
    "twoshot_160k": build_twoshot_160k,
    "sp_prefill": build_sp_prefill,
    "moe": build_moe,
    "ll_sweep": build_ll_sweep,
}


# ---------------------------------------------------------------- clocks ----

class Clocks:
    """nvidia-smi sampling during the timed region."""

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = os.path.join("/tmp", f"mvr_clocks_{os.getpid()}.csv")

    def __enter__(self):
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.f.close()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax = float(f[2])
            except ValueError:
                continue
            for nm, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        with contextlib.suppress(OSError):
            os.remove(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


# -------------------------------------------------------------- helpers ----

def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def lib_digest():
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "movement_virtual_rank_b200", "csrc")
    for fn in sorted(os.listdir(csrc)):
        with open(os.path.join(csrc, fn), "rb") as f:
            h.update(fn.encode() + f.read())
    return h.hexdigest()[:16]


def traffic_for(kernel: str, workload: str):
    """dram bytes per launch from a committed ncu summary, if taken on this exact source."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p))
    e = d.get(workload, {}).get(kernel)
    if e and e.get("source_digest") == lib_digest():
        return e.get("dram_bytes_per_launch")
    return None


def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)), int(os.environ.get("LOCAL_RANK", 0))


def max_over_ranks(value: float, world: int, device=None) -> float:
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(value: float, world: int, device=None) -> float:
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def cpu_cores_used() -> int:
    return 1  # numpy element-wise kernels run on the calling thread


def time_oracle(ops, min_s: float = 10.0, max_s: float = 30.0):
    """Run the oracle version of the step's ops, whole steps at a time, until
    about ``min_s`` seconds of CPU work (at most ``max_s``); returns
    (GB/s, sample description, seconds)."""
    refs = [op for op in ops if op.ref is not None]
    if not refs:
        return None, "no op of this workload has a CPU definition", 0.0
    secs, nbytes, passes, ops_done = 0.0, 0, 0, 0
    while secs < min_s:
        for op in refs:
            t0 = time.perf_counter()
            op.ref()
            secs += time.perf_counter() - t0
            nbytes += op.alg_bytes
            ops_done += 1
            if secs > max_s:
                break
        passes += 1
        if secs > max_s:
            break
    kinds = sorted(set(op.name.split("/")[0] for op in refs))
    sample = (f"{ops_done} oracle op calls = {ops_done / max(1, len(refs)):.2f} full steps of the same workload "
              f"({', '.join(kinds)}), full-size inputs")
    return (nbytes / secs / 1e9 if secs > 0 else None), sample, secs


def graph_latency(ops, stream, reps: int = 50, max_bytes_per_rank: int = 256 * 1024):
    """Latency floor of the small ops: ``reps`` back-to-back calls captured in
    one CUDA graph (no host launch cost, L2 warm), device time per call."""
    import torch
    out = {}
    for op in ops:
        if op.meta.get("bytes_per_rank", 1 << 62) > max_bytes_per_rank:
            continue
        g = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream()
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            op.run()  # warm the call path on the capture stream
        stream.wait_stream(side)
        torch.cuda.synchronize()
        with torch.cuda.graph(g):
            for _ in range(reps):
                op.run()
        for _ in range(3):
            g.replay()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        g.replay()
        b.record(stream)
        torch.cuda.synchronize()
        out[id(op)] = round(a.elapsed_time(b) * 1e3 / reps, 3)
        del g
    return out


# ------------------------------------------------------------------ main ----

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="tp_decode", choices=sorted(WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-graph", action="store_true")
    ap.add_argument("--lead-us", type=float, default=300.0, help="sleep before each timed op (outside the events)")
    args = ap.parse_args()
    rank, world, local = dist_env()

    if args.impl == "reference":
        return main_reference(args, rank, world)

    import torch
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    import movement_virtual_rank_b200 as M
    import oracle

    ops, cfg = WORKLOADS[args.workload](M, oracle)
    stream = torch.cuda.current_stream()
    l2 = torch.cuda.get_device_properties(local).L2_cache_size
    flush = torch.empty(2 * l2, dtype=torch.uint8, device="cuda")
    evs = {id(op): [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                    for _ in range(args.steps)] for op in ops}

    # Lead time: a bounded sleep kernel between the flush and the start event
    # keeps the GPU busy while the host enqueues the op, so the events time
    # the op's kernels back to back on the device, not the host's launch path
    # (that path is in the end-to-end number).
    lead_cycles = int(args.lead_us * 1e-6 * torch.cuda.get_device_properties(local).clock_rate * 1e3)

    def one_step(timed_index=None):
        for op in ops:
            flush.zero_()
            torch.cuda._sleep(lead_cycles)
            if timed_index is None:
                op.run()
            else:
                a, b = evs[id(op)][timed_index]
                a.record(stream)
                op.run()
                b.record(stream)

    with Clocks(local) as clk:
        time.sleep(0.5)  # let the sampler start
        for _ in range(max(args.warmup, 3)):
            one_step()
        torch.cuda.synchronize()
        barrier(world)
        torch.cuda.synchronize()
        wall0 = time.perf_counter()
        for k in range(args.steps):
            one_step(k)
        torch.cuda.synchronize()
        wall = time.perf_counter() - wall0
        barrier(world)
    clocks = clk.summary()
    graph_us = graph_latency(ops, stream) if not args.no_graph else {}
    for op in ops:
        op.times = [a.elapsed_time(b) * 1e-3 for a, b in evs[id(op)]]
    step_s = [sum(op.times[k] for op in ops) for k in range(args.steps)]
    total_s = sum(step_s)
    total_s_max = max_over_ranks(total_s, world, "cuda")
    bytes_step = sum(op.alg_bytes for op in ops)
    value = world * bytes_step * args.steps / total_s_max / 1e9
    hbm, hbm_src = peaks()

    # end-to-end leg: host->device of each op's inputs, the op, device->host of its outputs
    e2e = None
    if not args.no_e2e and all(op.inputs for op in ops):
        e_ev = {id(op): [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                         for _ in range(args.steps)] for op in ops}
        for k in range(-1, args.steps):
            for op in ops:
                if k >= 0:
                    e_ev[id(op)][k][0].record(stream)
                for dev_t, host_t in op.inputs:
                    dev_t.copy_(host_t, non_blocking=True)
                op.run()
                for dev_t, host_t in op.outputs:
                    host_t.copy_(dev_t, non_blocking=True)
                if k >= 0:
                    e_ev[id(op)][k][1].record(stream)
        torch.cuda.synchronize()
        e2e_s = sum(a.elapsed_time(b) * 1e-3 for op in ops for a, b in e_ev[id(op)])
        e2e_s = max_over_ranks(e2e_s, world, "cuda")
        h2d = sum(t.numel() * t.element_size() for op in ops for t, _ in op.inputs)
        d2h = sum(t.numel() * t.element_size() for op in ops for t, _ in op.outputs)
        e2e = {"value": round(world * bytes_step * args.steps / e2e_s / 1e9, 3), "unit": "GB/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "how": "per op: pinned host->device copy of its inputs, the C-ABI call, device->host copy of its "
                      "outputs, CUDA events around the three"}

    # per-op detail and the dominant kernel
    per_op = []
    by_kernel = {}
    for op in ops:
        med = statistics.median(op.times)
        gbs = op.alg_bytes / med / 1e9
        extra = {"graph_us": graph_us[id(op)]} if id(op) in graph_us else {}
        per_op.append({**op.meta, **extra, "us": round(med * 1e6, 3), "us_p10": round(np.percentile(op.times, 10) * 1e6, 3),
                       "us_p90": round(np.percentile(op.times, 90) * 1e6, 3), "gbs": round(gbs, 1),
                       "frac_measured_hbm": round(gbs / hbm, 4), "frac_8tbs": round(gbs / 8000, 4)})
        k = by_kernel.setdefault(op.kernel, {"time": 0.0, "bytes": 0, "launches": 0, "ops": 0})
        k["time"] += sum(op.times)
        k["bytes"] += op.per_launch_bytes * args.steps * (1 if op.launches == 1 else 0)
        k["launches"] += op.launches * args.steps
        k["ops"] += args.steps if op.launches == 1 else 0
    single = {k: v for k, v in by_kernel.items() if v["ops"]}
    dom = max(single, key=lambda k: single[k]["time"])
    d = single[dom]
    avg = d["time"] / d["ops"]
    achieved = d["bytes"] / d["ops"] / avg / 1e9
    roof = {"bound": "hbm", "kernel": dom, "achieved": round(achieved, 1), "peak": hbm, "unit": "GB/s",
            "frac": round(achieved / hbm, 4), "peak_source": f"{hbm_src} (MEASURED_PEAKS.json hbm_gbs, burst)",
            "share_of_step": round(d["time"] / total_s, 4),
            "traffic": traffic_for(dom, args.workload),
            "avg_launch_us": round(avg * 1e6, 3),
            "algorithmic_bytes_per_launch": round(d["bytes"] / d["ops"])}
    launches = sum(op.launches for op in ops) * args.steps

    cpu = None
    if rank == 0 and not args.no_cpu_baseline:
        v, sample, secs = time_oracle(ops)
        cpu = {"value": round(v, 4) if v else None, "unit": "GB/s", "cores": cpu_cores_used(), "kind": "oracle",
               "sample": sample, "seconds": round(secs, 2)}

    if rank == 0:
        line = {"metric": METRIC, "value": round(value, 3), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
                "warmup": max(args.warmup, 3), "ms_per_step": round(total_s_max / args.steps * 1e3, 4),
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
                "data": "synthetic", "impl": "ours",
                "config": {**cfg, "parallelism": f"replicas x{world} (virtual ranks inside each GPU)",
                           "l2": "flushed before every op (memset of 2x L2, outside the timed events)",
                           "timing": f"CUDA events around each op on its stream, after a {args.lead_us:.0f} us "
                                     "sleep kernel so the op's kernels run back to back"},
                "roofline": roof, "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches,
                "clocks": clocks, "wall_s_timed_region": round(wall, 3), "ops": per_op}
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


def main_reference(args, rank, world):
    """The oracle as it stands, on the host's cores (rank 0 only)."""
    if rank != 0:
        return
    import oracle

    ops, cfg = host_ops(args.workload, oracle)
    times = []
    nbytes = sum(op.alg_bytes for op in ops)
    for k in range(max(args.warmup, 0) + args.steps):
        t0 = time.perf_counter()
        for op in ops:
            op.ref()
        dt = time.perf_counter() - t0
        if k >= args.warmup:
            times.append(dt)
    total = sum(times)
    value = nbytes * len(times) / total / 1e9
    sample = f"every op of the workload with a CPU definition, full size, {len(times)} timed passes"
    line = {"metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(total / len(times) * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "impl": "reference",
            "config": cfg,
            "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": cpu_cores_used(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def host_ops(workload: str, oracle):
    """The workload's ops as oracle calls on host inputs (no GPU needed)."""
    ops = []
    if workload == "tp_decode":
        n = 8
        for tokens, hidden in W.tp_decode_shapes():
            xs = W.tp_decode(tokens, hidden, n)
            S = tokens * hidden * 2
            for aname, ref in (("oneshot", oracle.all_reduce_one_shot), ("twoshot", oracle.all_reduce_two_shot),
                               ("ring", oracle.all_reduce_ring)):
                ops.append(Op(f"all_reduce/{aname}", None, 2 * n * S, 0, [], [], {},
                              ref=(lambda xs=xs, ref=ref: ref(xs, 0, "bf16"))))
        ids = W.sampled_token_ids(n)
        ops.append(Op("broadcast", None, 256 * 4 * n, 0, [], [], {}, ref=lambda: oracle.broadcast(ids, 7)))
        cfg = {"workload": "tp_decode_allreduce_8vr", "virtual_ranks": n, "dtype": "bf16",
               "tokens": list(W.TP_DECODE_TOKENS), "hidden": list(W.TP_DECODE_HIDDEN),
               "algos": ["oneshot", "twoshot", "ring"], "plus": "broadcast int32[256] src=7"}
        return ops, cfg
    if workload == "twoshot_160k":
        xs = W.twoshot_160k(4)
        ops.append(Op("all_reduce/twoshot", None, 2 * 4 * xs[0].size * 2, 0, [], [], {},
                      ref=lambda: oracle.all_reduce_two_shot(xs, 0, "bf16")))
        return ops, {"workload": "allreduce_twoshot_4vr_160KB", "virtual_ranks": 4}
    raise SystemExit(f"--impl reference supports tp_decode and twoshot_160k, not {workload}")


if __name__ == "__main__":
    main()
