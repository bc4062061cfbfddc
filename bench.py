"""Benchmark of the virtual-rank collectives on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload full_step|tp_decode|twoshot_160k|sp_prefill|moe|
                               ll_sweep|single_image|ring_compare|movement]

One "step" is one call of every op of the chosen workload on seeded synthetic
inputs resident in HBM.  ``value`` is the ops' algorithmic bytes (what each
collective must read plus write, once) over the step's device time, summed
over all GPUs, in GB/s.

Default workload (``full_step``): every op of the hot path, 8 virtual ranks,
at the largest sizes the workloads give:
  * sequence-parallel prefill: all_gather bf16 [1024,8192] -> [8192,8192],
    reduce_scatter [8192,8192] -> [1024,8192], gather of fp32 [256,16032]
    logits shards to rank 0;
  * MoE: route, dispatch and combine of 4096 tokens per rank, hidden 7168
    bf16, 256 experts, top-8 Zipf-skewed routing;
  * all_reduce of bf16 uniform[-1,1] messages of 16 MiB and 256 MiB per rank:
    the Simple two-shot, and the LL and LL128 paths (encode every rank,
    packetised all-reduce, decode every rank);
  * the TP-decode all_reduce of bf16 [256,7168] by one-shot, two-shot and
    ring, and the broadcast of int32 sampled_token_ids[256] from rank 7;
  * reduce to rank 0 and scatter from rank 0, 16 MiB per rank.

How an op's device time is measured.  The op is replicated on R distinct
copies of its buffers (R = 1 for ops larger than L2, up to 256 for the
smallest) and the R calls are captured in one CUDA graph.  Each timed replay
is preceded (outside the events) by a read of a buffer twice the size of L2
and a bounded sleep kernel; CUDA events on the replay stream bracket the
replay, and the op's time is the replay time / R.  Each call touches its own
buffers once per replay, after the L2 has been flushed, so every call reads
inputs that are not in L2; the host's launch path is not in the number (it is
in the end-to-end leg).  The JSON also gives, per op, one call
timed alone between two events (``us_single``, which includes the ~2.5 us cost
of an event pair) and, for messages up to 256 KB per rank, the warm-L2
latency floor of back-to-back calls (``graph_us``).

With --gpus N > 1 (torchrun, one process per GPU) every GPU runs its own
independent replica: the virtual ranks live inside one GPU, so there is no
exchange between GPUs (weak scaling; timing is the max over ranks).

``--impl reference`` times the CPU oracle (the plain definition of each op)
on this host's cores on a bounded sample of the same workload: every op at
1/16 of its size (the first part of each rank's own seeded input, MoE the
first 1/16 of each rank's tokens), each op split into independent parts that
worker processes (one per core) run in parallel.
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
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

METRIC = "collective HBM GB/s (% of B200 peak) per op vs message size; µs/allreduce"


# ------------------------------------------------------------ workloads ----

class Op:
    """One collective call.

    bind(bufs) -> callable that launches the op on those device buffers
    bufs:       dict of name -> tensor or list of tensors (device)
    inputs / outputs: names in ``bufs`` copied host->device / device->host by
                the end-to-end leg (empty for the inner ops of a chain, whose
                inputs are the previous op's device outputs)
    ref():      the oracle's version of the op on the host inputs
    """

    def __init__(self, name, bind, bufs, alg_bytes, launches, meta, inputs=(), outputs=(), ref=None,
                 kernel=None, per_launch_bytes=None):
        self.name, self.bind, self.bufs = name, bind, bufs
        self.alg_bytes, self.launches, self.meta = alg_bytes, launches, meta
        self.inputs, self.outputs, self.ref = list(inputs), list(outputs), ref
        self.kernel = kernel or name
        self.per_launch_bytes = per_launch_bytes if per_launch_bytes is not None else alg_bytes
        self.run = bind(bufs)
        self.times, self.single = [], []

    def footprint(self) -> int:
        return sum(t.numel() * t.element_size() for t in _flat(self.bufs))

    def replicate(self):
        """A call of the same op on fresh device copies of its buffers."""
        copy = {k: ([t.clone() for t in v] if isinstance(v, list) else v.clone()) for k, v in self.bufs.items()}
        return self.bind(copy)


def _flat(bufs):
    for v in bufs.values():
        if isinstance(v, list):
            yield from v
        else:
            yield v


def _as_list(v):
    return v if isinstance(v, list) else [v]


def _dev(a: np.ndarray, dtype):
    import torch
    view = {torch.bfloat16: np.int16, torch.int32: np.int32, torch.float32: np.float32, torch.uint8: np.uint8}[dtype]
    return torch.from_numpy(np.ascontiguousarray(a).view(view).copy()).view(dtype).cuda()


FORM_NAMES = {1: "oneshot", 2: "twoshot", 4: "ring_ll", 5: "ring_cluster", 6: "ring_steps", 7: "twoshot_ll",
              8: "ring_cta", 9: "twoshot_ll128", 10: "ring_lane", 11: "ring_wire"}


def tp_decode_cfg(n):
    """The TP-decode workload's description, the same for both arms."""
    return {"workload": "tp_decode_allreduce_8vr", "virtual_ranks": n, "dtype": "bf16",
            "tokens": list(W.TP_DECODE_TOKENS), "hidden": list(W.TP_DECODE_HIDDEN),
            "algos": ["oneshot", "twoshot", "ring"], "plus": "broadcast int32[256] src=7",
            "values": "N(0,1) bf16 per rank, seeded"}


def twoshot_160k_cfg(n):
    return {"workload": "allreduce_twoshot_4vr_160KB", "virtual_ranks": n, "dtype": "bf16",
            "values": "uniform[-1,1] bf16, seeded"}


FULL_STEP_AR_BYTES = (16 << 20, 256 << 20)  # all-reduce bytes per rank: the >= 16 MiB end of the LL sweep
FULL_STEP_MOVE_BYTES = 16 << 20             # reduce / scatter bytes per rank


def full_step_cfg(n=8):
    """The default workload's description, the same for both arms."""
    return {"workload": "all_hot_path_ops_largest_configs_8vr", "virtual_ranks": n,
            "sp_prefill": {"all_gather": "bf16 [1024,8192] -> [8192,8192]",
                           "reduce_scatter": "bf16 [8192,8192] -> [1024,8192]",
                           "gather": "fp32 [256,16032] -> dst 0 [256,128256]"},
            "moe": {"tokens": 4096, "hidden": 7168, "experts": 256, "topk": 8,
                    "routing": "softmax(N(0,1)+log Zipf(1.1)) top-8, renormalised",
                    "ops": ["route", "dispatch", "combine"]},
            "all_reduce": {"bytes_per_rank": list(FULL_STEP_AR_BYTES), "values": "uniform[-1,1] bf16",
                           "paths": ["simple two-shot", "LL: pack, packetised all-reduce, unpack",
                                     "LL128: pack, packetised all-reduce, unpack"]},
            "tp_decode": {"shape": [256, 7168], "algos": ["oneshot", "twoshot", "ring"],
                          "plus": "broadcast int32[256] src=7"},
            "movement": {"bytes_per_rank": FULL_STEP_MOVE_BYTES, "ops": ["reduce to rank 0", "scatter from rank 0"]}}


def build_tp_decode(M, oracle):
    import torch
    ops = []
    n = 8
    for tokens, hidden in W.tp_decode_shapes():
        xs = W.tp_decode(tokens, hidden, n)
        S = tokens * hidden * 2
        send = [_dev(x, torch.bfloat16) for x in xs]
        for algo, aname, ref in ((M.ONESHOT, "oneshot", oracle.all_reduce_one_shot),
                                 (M.TWOSHOT, "twoshot", oracle.all_reduce_two_shot),
                                 (M.RING, "ring", oracle.all_reduce_ring)):
            form = M.coll_all_reduce_form(n, tokens * hidden, torch.bfloat16, algo)
            launches = 2 * (n - 1) if form == M.RING_STEPS else 1
            bufs = {"send": send, "recv": [torch.empty_like(t) for t in send]}
            if algo in (M.RING, M.RING_LL):
                need = M.coll_all_reduce_workspace_size(n, tokens * hidden, torch.bfloat16, algo)
                bufs["ws"] = torch.zeros(need, dtype=torch.uint8, device="cuda")

            def bind(b, algo=algo):
                ws = b.get("ws")
                return lambda: M.coll_all_reduce(b["send"], b["recv"], algo=algo, workspace=ws)

            ops.append(Op(f"all_reduce/{aname}", bind, bufs, 2 * n * S, launches,
                          {"op": "all_reduce", "algo": aname, "ranks": n, "shape": [tokens, hidden],
                           "bytes_per_rank": S, "form": FORM_NAMES[form]},
                          inputs=["send"], outputs=["recv"],
                          ref=(lambda xs=xs, ref=ref: ref(xs, 0, "bf16")), kernel=f"all_reduce/{aname}"))
    ids = W.sampled_token_ids(n)
    S = 256 * 4
    ops.append(Op("broadcast", lambda b: (lambda: M.coll_broadcast(b["bufs"], 7)),
                  {"bufs": [_dev(x, torch.int32) for x in ids]}, S * n, 1,
                  {"op": "broadcast", "src": 7, "ranks": n, "dtype": "int32", "count": 256, "bytes_per_rank": S},
                  inputs=["bufs"], outputs=["bufs"], ref=lambda ids=ids: oracle.broadcast(ids, 7), kernel="broadcast"))
    cfg = tp_decode_cfg(n)
    return ops, cfg


def build_twoshot_160k(M, oracle):
    import torch
    n = 4
    xs = W.twoshot_160k(n)
    S = xs[0].size * 2
    send = [_dev(x, torch.bfloat16) for x in xs]
    ops = [Op("all_reduce/twoshot", lambda b: (lambda: M.coll_all_reduce(b["send"], b["recv"], algo=M.TWOSHOT)),
              {"send": send, "recv": [torch.empty_like(t) for t in send]}, 2 * n * S, 1,
              {"op": "all_reduce", "algo": "twoshot", "ranks": n, "bytes_per_rank": S},
              inputs=["send"], outputs=["recv"], ref=lambda: oracle.all_reduce_two_shot(xs, 0, "bf16"),
              kernel="all_reduce/twoshot")]
    return ops, twoshot_160k_cfg(n)


def build_sp_prefill(M, oracle):
    import torch
    n = 8
    ag_in = W.sp_allgather(n)
    rs_in = W.sp_reduce_scatter(n)
    lg_in = W.logits_shards(n)
    S_ag, S_rs, S_lg = ag_in[0].size * 2, rs_in[0].size * 2, lg_in[0].size * 4
    ops = [
        Op("all_gather", lambda b: (lambda: M.coll_all_gather(b["send"], b["recv"])),
           {"send": [_dev(x, torch.bfloat16) for x in ag_in],
            "recv": [torch.empty(n * x.size, dtype=torch.bfloat16, device="cuda") for x in ag_in]},
           n * S_ag + n * n * S_ag, 1, {"op": "all_gather", "ranks": n, "bytes_per_rank": S_ag},
           inputs=["send"], outputs=["recv"], ref=lambda: oracle.all_gather(ag_in), kernel="all_gather"),
        Op("reduce_scatter", lambda b: (lambda: M.coll_reduce_scatter(b["send"], b["recv"])),
           {"send": [_dev(x, torch.bfloat16) for x in rs_in],
            "recv": [torch.empty(x.size // n, dtype=torch.bfloat16, device="cuda") for x in rs_in]},
           n * S_rs + S_rs, 1, {"op": "reduce_scatter", "ranks": n, "bytes_per_rank": S_rs},
           inputs=["send"], outputs=["recv"], ref=lambda: oracle.reduce_scatter(rs_in, 0, "bf16"),
           kernel="reduce_scatter"),
        Op("gather", lambda b: (lambda: M.coll_gather(b["send"], b["out"], 0)),
           {"send": [_dev(x, torch.float32).reshape(256, 16032) for x in lg_in],
            "out": torch.empty(256, n * 16032, dtype=torch.float32, device="cuda")},
           2 * n * S_lg, 1, {"op": "gather", "dst": 0, "ranks": n, "bytes_per_rank": S_lg, "dtype": "fp32"},
           inputs=["send"], outputs=["out"],
           ref=lambda: oracle.gather(lg_in, np.zeros(n * lg_in[0].size, np.float32), rows=256), kernel="gather"),
    ]
    return ops, {"workload": "sp_prefill_ag_rs_gather_8vr", "virtual_ranks": n,
                 "all_gather": "bf16 [1024,8192] -> [8192,8192]", "reduce_scatter": "bf16 [8192,8192] -> [1024,8192]",
                 "gather": "fp32 [256,16032] -> dst 0 [256,128256]"}


MOE_TOKENS = 4096  # tokens per rank of the MoE workload (and of the all-to-all-v split matrix); --moe-tokens


def moe_ops(M, oracle, dedup: bool = True, chain: bool = False):
    """The MoE workload's ops (8 virtual ranks x MOE_TOKENS tokens, hidden
    7168 bf16, 256 experts, top-8): route, dispatch and combine, plus, with
    ``dedup``, the same three on the route deduplicated per (token,
    destination rank).  ``chain``: the end-to-end leg uploads only what a
    caller holds on the host (expert ids, token rows, weights) and downloads
    only the combined tokens."""
    import torch
    n, tokens, topk, experts, hidden = 8, MOE_TOKENS, 8, 256, 7168
    ids, ws = W.moe_routing(tokens, experts, topk, n)
    xs = W.moe_tokens(tokens, hidden, n)
    dids = [torch.from_numpy(i).cuda() for i in ids]
    x = [_dev(v, torch.bfloat16) for v in xs]
    del xs
    split = {"sc": torch.empty(n * n, dtype=torch.int64, device="cuda")}
    split["sd"], split["rd"] = torch.empty_like(split["sc"]), torch.empty_like(split["sc"])
    pos = [torch.empty(tokens * topk, dtype=torch.int32, device="cuda") for _ in range(n)]
    wsp = torch.empty(M.coll_moe_route_workspace_size(n, tokens, topk, experts), dtype=torch.uint8, device="cuda")
    M.coll_moe_route(dids, experts, split["sc"], split["sd"], split["rd"], pos, workspace=wsp)
    torch.cuda.synchronize()
    cap = int(split["sc"].view(n, n).sum(0).max().item())
    recv = [torch.empty(cap * hidden, dtype=torch.bfloat16, device="cuda") for _ in range(n)]
    dw = [torch.from_numpy(w).cuda() for w in ws]
    row = hidden * 2
    pairs = n * tokens * topk

    def io_of(inp, out):
        if not chain:
            return [inp], [out]
        return ([inp] if inp else []), ([out] if out else [])

    ops = []
    i, o = io_of("ids", None if chain else "pos")
    ops.append(Op("moe_route",
                  lambda b: (lambda: M.coll_moe_route(b["ids"], experts, b["sc"], b["sd"], b["rd"], b["pos"],
                                                      workspace=b["ws"])),
                  {"ids": dids, "pos": pos, "ws": wsp, **split}, pairs * 4 * 2, 3,
                  {"op": "moe_route", "ranks": n, "tokens": tokens, "topk": topk, "experts": experts},
                  inputs=i, outputs=o, ref=lambda: oracle.moe_route(ids, experts), kernel="moe_route"))
    i, o = io_of("x", None if chain else "recv")
    ops.append(Op("moe_dispatch", lambda b: (lambda: M.coll_moe_dispatch(b["x"], b["ids"], b["pos"], b["recv"],
                                                                         experts)),
                  {"x": x, "ids": dids, "pos": pos, "recv": recv}, n * tokens * row + pairs * row, 1,
                  {"op": "moe_dispatch", "ranks": n, "hidden": hidden, "rows_out": pairs},
                  inputs=i, outputs=o, kernel="moe_dispatch"))
    i, o = io_of("w" if chain else "y", "out")
    ops.append(Op("moe_combine",
                  lambda b: (lambda: M.coll_moe_combine(b["y"], b["ids"], b["pos"], b["w"], b["out"], experts)),
                  {"y": recv, "ids": dids, "pos": pos, "w": dw,
                   "out": [torch.empty_like(t) for t in x]}, pairs * row + pairs * 4 + n * tokens * row, 1,
                  {"op": "moe_combine", "ranks": n, "hidden": hidden},
                  inputs=i, outputs=o, kernel="moe_combine"))
    if not dedup:
        return ops
    # the route deduplicated per (token, destination rank): one row per pair reached
    dsplit = {k: torch.empty_like(v) for k, v in split.items()}
    dpos = [torch.empty_like(p) for p in pos]
    M.coll_moe_route_dedup(dids, experts, dsplit["sc"], dsplit["sd"], dsplit["rd"], dpos, workspace=wsp)
    torch.cuda.synchronize()
    uniq = int(dsplit["sc"].sum().item())
    dcap = int(dsplit["sc"].view(n, n).sum(0).max().item())
    drecv = [torch.empty(dcap * hidden, dtype=torch.bfloat16, device="cuda") for _ in range(n)]
    ops += [
        Op("moe_route_dedup",
           lambda b: (lambda: M.coll_moe_route_dedup(b["ids"], experts, b["sc"], b["sd"], b["rd"], b["pos"],
                                                     workspace=b["ws"])),
           {"ids": dids, "pos": dpos, "ws": wsp, **dsplit}, pairs * 4 * 2, 3,
           {"op": "moe_route_dedup", "ranks": n, "tokens": tokens, "topk": topk, "experts": experts},
           inputs=["ids"], outputs=["pos"], ref=lambda: oracle.moe_route_dedup(ids, experts), kernel="moe_route"),
        Op("moe_dispatch_dedup",
           lambda b: (lambda: M.coll_moe_dispatch(b["x"], b["ids"], b["pos"], b["recv"], experts)),
           {"x": x, "ids": dids, "pos": dpos, "recv": drecv}, n * tokens * row + uniq * row, 1,
           {"op": "moe_dispatch_dedup", "ranks": n, "hidden": hidden, "rows_out": uniq},
           inputs=["x"], outputs=["recv"], kernel="moe_dispatch_dedup"),
        Op("moe_combine_dedup",
           lambda b: (lambda: M.coll_moe_combine(b["y"], b["ids"], b["pos"], b["w"], b["out"], experts)),
           {"y": drecv, "ids": dids, "pos": dpos, "w": dw,
            "out": [torch.empty_like(t) for t in x]}, uniq * row + pairs * 4 + n * tokens * row, 1,
           {"op": "moe_combine_dedup", "ranks": n, "hidden": hidden, "rows_in": uniq},
           inputs=["y"], outputs=["out"], kernel="moe_combine_dedup"),
    ]
    return ops


def build_moe(M, oracle):
    return moe_ops(M, oracle, dedup=True), {
        "workload": "moe_dispatch_combine_8vr", "virtual_ranks": 8, "tokens": MOE_TOKENS, "hidden": 7168,
        "experts": 256, "topk": 8, "routing": "softmax(N(0,1)+log Zipf(1.1)) top-8, renormalised"}


LL_SIZES = None  # bytes per rank of the LL sweep (default 1 KB .. 256 MB, powers of 4); --ll-sizes


def build_ll_sweep(M, oracle, sizes=None):
    import torch
    n = 8
    sizes = sizes or LL_SIZES or [1 << k for k in range(10, 29, 2)]
    ops = []
    for nbytes in sizes:
        count = nbytes // 2
        xs = W.ll_message(nbytes, n)
        send = [_dev(x, torch.bfloat16) for x in xs]
        ops.append(Op(f"all_reduce/simple/{nbytes}",
                      lambda b: (lambda: M.coll_all_reduce(b["send"], b["recv"], algo=M.TWOSHOT)),
                      {"send": send, "recv": [torch.empty_like(t) for t in send]}, 2 * n * nbytes, 1,
                      {"op": "all_reduce", "proto": "simple", "bytes_per_rank": nbytes},
                      inputs=["send"], outputs=["recv"], kernel="all_reduce/simple"))
        for proto, pname in ((M.LL, "ll"), (M.LL128, "ll128")):
            pb = M.coll_packed_bytes(nbytes, proto)
            packed = [torch.empty(pb, dtype=torch.uint8, device="cuda") for _ in range(n)]
            for r in range(n):
                M.coll_ll_pack(send[r], packed[r], proto, 1)

            def bind(b, count=count, proto=proto):
                return lambda: M.coll_all_reduce_packed(b["pin"], b["pout"], count, torch.bfloat16, proto, 1)

            ops.append(Op(f"all_reduce/{pname}/{nbytes}", bind,
                          {"pin": packed, "pout": [torch.empty(pb, dtype=torch.uint8, device="cuda") for _ in range(n)]},
                          2 * n * nbytes, 1,
                          {"op": "all_reduce_packed", "proto": pname, "bytes_per_rank": nbytes,
                           "line_bytes": 2 * n * pb},
                          inputs=["pin"], outputs=["pout"], kernel=f"all_reduce/{pname}", per_launch_bytes=2 * n * pb))
    return ops, {"workload": "ll_ll128_allreduce_sweep_8vr", "virtual_ranks": n, "sizes": sizes}


def build_ring_compare(M, oracle):
    """Ring and packet all-reduce latency on the TP-decode shapes (8 virtual
    ranks, bf16): the ring as one launch per step (RING_STEPS), as one
    cooperative launch with LL packets between ranks (RING_LL) and as one
    launch of 8-CTA clusters with the hops over distributed shared memory
    (RING_CLUSTER) and as one launch whose CTAs hold all 8 ranks as warp
    groups, the hops in shared memory (RING_CTA) and as one launch whose warps hold all 8 ranks as lanes,
    the hops by warp shuffles (RING_LANE); the two-shot with LL / LL128 packets fused into one cooperative
    launch (TWOSHOT_LL, TWOSHOT_LL128); and the stream-ordered packet path of the LL sweep
    (LL pack of every rank, packetised two-shot, unpack of every rank: three launches)."""
    import torch
    n = 8
    ops = []
    for tokens, hidden in W.tp_decode_shapes():
        xs = W.tp_decode(tokens, hidden, n)
        count = tokens * hidden
        S = count * 2
        send = [_dev(x, torch.bfloat16) for x in xs]
        for algo, aname, launches in ((M.RING_STEPS, "ring_steps", 2 * (n - 1)), (M.RING_LL, "ring_ll", 1),
                                      (M.RING_CLUSTER, "ring_cluster", 1), (M.RING_CTA, "ring_cta", 1),
                                      (M.RING_LANE, "ring_lane", 1), (M.RING_WIRE, "ring_wire", 1),
                                      (M.TWOSHOT_LL, "twoshot_ll", 1), (M.TWOSHOT_LL128, "twoshot_ll128", 1)):
            need = max(64, M.coll_all_reduce_workspace_size(n, count, torch.bfloat16, algo))
            ops.append(Op(f"all_reduce/{aname}",
                          lambda b, algo=algo: (lambda: M.coll_all_reduce(b["send"], b["recv"], algo=algo,
                                                                           workspace=b["ws"])),
                          {"send": send, "recv": [torch.empty_like(t) for t in send],
                           "ws": torch.zeros(need, dtype=torch.uint8, device="cuda")},
                          2 * n * S, launches, {"op": "all_reduce", "algo": aname, "shape": [tokens, hidden],
                                                "bytes_per_rank": S},
                          inputs=["send"], outputs=["recv"], kernel=f"all_reduce/{aname}"))
        pb = M.coll_packed_bytes(S, M.LL)

        def bind_ll(b, count=count):
            def run():
                M.coll_ll_pack_ranks(b["send"], b["pin"], M.LL, 1)
                M.coll_all_reduce_packed(b["pin"], b["pout"], count, torch.bfloat16, M.LL, 1)
                M.coll_ll_unpack_ranks(b["pout"], b["recv"], M.LL, 1)
            return run

        ops.append(Op("all_reduce/ll_pack_ar_unpack", bind_ll,
                      {"send": send, "recv": [torch.empty_like(t) for t in send],
                       "pin": [torch.empty(pb, dtype=torch.uint8, device="cuda") for _ in range(n)],
                       "pout": [torch.empty(pb, dtype=torch.uint8, device="cuda") for _ in range(n)]},
                      2 * n * S, 3, {"op": "all_reduce", "algo": "ll_pack_ar_unpack",
                                             "shape": [tokens, hidden], "bytes_per_rank": S},
                      inputs=["send"], outputs=["recv"], kernel="all_reduce/ll_pack_ar_unpack"))
    return ops, {"workload": "ring_compare_8vr", "virtual_ranks": n, "shapes": W.tp_decode_shapes(),
                 "variants": ["ring_steps (launch per step)", "ring_ll (one launch, LL packets)",
                              "ring_cluster (one launch, cluster DSMEM hops)",
                              "ring_cta (one launch, ranks as warp groups, shared-memory hops)",
                              "ring_lane (one launch, ranks as lanes, warp-shuffle hops)",
                              "ring_wire (the CTA ring with partials rounded to bf16 at every hop: a different result)",
                              "twoshot_ll (one launch, LL packets, fused)",
                              "twoshot_ll128 (one launch, LL128 packets, fused)",
                              "LL pack + packetised two-shot + unpack (stream-ordered, 3 launches)"]}


def build_movement(M, oracle):
    """The remaining single-call collectives at 16 MiB per rank (8 virtual
    ranks, bf16): reduce to rank 0, scatter from rank 0, all-to-all with equal
    blocks, all-to-all-v with the MoE workload's skewed split matrix (one
    7168-wide row per routed token), and LL / LL128 pack and unpack."""
    import torch
    n = 8
    S = 16 << 20
    c = S // 2
    xs = W.ranks_values(W.W_MISC, n, c, "bf16", "normal", salt=16)
    send = [_dev(x, torch.bfloat16) for x in xs]
    ops = [
        Op("reduce", lambda b: (lambda: M.coll_reduce(b["send"], b["out"], 0)),
           {"send": send, "out": torch.empty(c, dtype=torch.bfloat16, device="cuda")}, n * S + S, 1,
           {"op": "reduce", "dst": 0, "bytes_per_rank": S}, inputs=["send"], outputs=["out"],
           ref=lambda: oracle.reduce(xs, 0, "bf16"), kernel="reduce"),
        Op("scatter", lambda b: (lambda: M.coll_scatter(b["src"], b["recv"], 0)),
           {"src": torch.cat(send), "recv": [torch.empty(c, dtype=torch.bfloat16, device="cuda") for _ in range(n)]},
           2 * n * S, 1, {"op": "scatter", "src": 0, "bytes_per_rank": S}, inputs=["src"], outputs=["recv"],
           kernel="scatter"),
        Op("all_to_all", lambda b: (lambda: M.coll_all_to_all(b["send"], b["recv"])),
           {"send": send, "recv": [torch.empty_like(t) for t in send]}, 2 * n * S, 1,
           {"op": "all_to_all", "bytes_per_rank": S}, inputs=["send"], outputs=["recv"],
           ref=lambda: oracle.all_to_all(xs), kernel="all_to_all"),
    ]
    # all-to-all-v: the MoE workload's split matrix
    ids, _ = W.moe_routing(MOE_TOKENS, 256, 8, n)
    sc, sd, rd, _pos = oracle.moe_route(ids, 256)
    row = 7168
    cap_s = [int(sc[s].sum()) for s in range(n)]
    cap_r = [int(sc[:, d].sum()) for d in range(n)]
    moved = int(sc.sum()) * row * 2
    ops.append(Op("all_to_all_v",
                  lambda b: (lambda: M.coll_all_to_all_v(b["send"], b["recv"], sc, sd, rd, row)),
                  {"send": [torch.randn(k * row, device="cuda").to(torch.bfloat16) for k in cap_s],
                   "recv": [torch.empty(k * row, dtype=torch.bfloat16, device="cuda") for k in cap_r]},
                  2 * moved, 1, {"op": "all_to_all_v", "rows": int(sc.sum()), "row_elems": row,
                                 "splits": f"MoE workload routing ({MOE_TOKENS} tokens per rank, Zipf 1.1, top-8, "
                                           "256 experts)"},
                  inputs=["send"], outputs=["recv"], kernel="all_to_all_v"))
    for proto, pname in ((M.LL, "ll"), (M.LL128, "ll128")):
        pb = M.coll_packed_bytes(S, proto)
        packed = torch.empty(pb, dtype=torch.uint8, device="cuda")
        M.coll_ll_pack(send[0], packed, proto, 3)
        ops.append(Op(f"{pname}_pack", lambda b, proto=proto: (lambda: M.coll_ll_pack(b["src"], b["packed"], proto, 3)),
                      {"src": send[0], "packed": torch.empty(pb, dtype=torch.uint8, device="cuda")}, S + pb, 1,
                      {"op": f"{pname}_pack", "bytes": S, "packed_bytes": pb}, inputs=["src"], outputs=["packed"],
                      kernel=f"{pname}_pack"))
        ops.append(Op(f"{pname}_unpack",
                      lambda b, proto=proto: (lambda: M.coll_ll_unpack(b["packed"], b["dst"], proto, 3)),
                      {"packed": packed, "dst": torch.empty(c, dtype=torch.bfloat16, device="cuda")}, S + pb, 1,
                      {"op": f"{pname}_unpack", "bytes": S, "packed_bytes": pb}, inputs=["packed"], outputs=["dst"],
                      kernel=f"{pname}_unpack"))
    return ops, {"workload": "movement_16MiB_8vr", "virtual_ranks": n, "bytes_per_rank": S,
                 "ops": ["reduce", "scatter", "all_to_all", "all_to_all_v", "ll/ll128 pack", "ll/ll128 unpack"]}


def build_single_image(M, oracle):
    """Single-image embedding sync (sglang PR 33307 summary): the owner's
    [n_tok, hidden] bf16 rows reach every rank by a padded all-gather (old
    path) or a broadcast (new path); 8 virtual ranks, owner 5."""
    import torch
    from movement_virtual_rank_b200 import single_image as SI
    n, owner, hidden = 8, 5, 7168
    g = SI.VirtualGroup(n)
    ops = []
    for n_tok in (256, 1024, 4096):
        S = n_tok * hidden * 2
        rows = W.ranks_values(W.W_MISC, 1, n_tok * hidden, "bf16", salt=n_tok)[0]
        truth = _dev(rows, torch.bfloat16).reshape(n_tok, hidden)
        padded = [torch.zeros(n_tok, hidden, dtype=torch.bfloat16, device="cuda") for _ in range(n)]
        padded[owner].copy_(truth)
        ops.append(Op(f"single_image/padded_all_gather/{n_tok}",
                      lambda b: (lambda: SI.sync_single_image_padded_all_gather(g, b["padded"], b["gathered"], owner,
                                                                                 n_tok)),
                      {"padded": padded,
                       "gathered": [torch.empty(n * n_tok, hidden, dtype=torch.bfloat16, device="cuda")
                                    for _ in range(n)]},
                      n * S + n * n * S, 1, {"op": "single_image_padded_all_gather", "n_tok": n_tok,
                                             "hidden": hidden, "bytes_per_rank": S},
                      inputs=["padded"], outputs=["gathered"], kernel="single_image/padded_all_gather"))
        bufs = [torch.empty(n_tok, hidden, dtype=torch.bfloat16, device="cuda") for _ in range(n)]
        bufs[owner].copy_(truth)
        ops.append(Op(f"single_image/broadcast/{n_tok}",
                      lambda b: (lambda: SI.sync_single_image_broadcast(g, b["bufs"], owner)),
                      {"bufs": bufs}, n * S, 1,
                      {"op": "single_image_broadcast", "n_tok": n_tok, "hidden": hidden, "bytes_per_rank": S},
                      inputs=["bufs"], outputs=["bufs"], kernel="single_image/broadcast"))
    return ops, {"workload": "single_image_sync_8vr", "virtual_ranks": n, "owner": owner, "hidden": hidden,
                 "n_tok": [256, 1024, 4096], "paths": ["padded all_gather (old)", "broadcast (new)"]}


def _protocol_ops(M, nbytes, n=8):
    """All-reduce of a bf16 uniform[-1,1] message of ``nbytes`` per rank by
    the Simple two-shot and by the LL and LL128 paths (every rank encodes its
    message, the packetised all-reduce sums the packets and re-encodes the
    result, every rank decodes it).  The three share the input buffers; the
    end-to-end leg uploads the message and downloads the decoded sum."""
    import torch
    count = nbytes // 2
    xs = W.ll_message(nbytes, n)
    send = [_dev(x, torch.bfloat16) for x in xs]
    del xs
    tag = f"{nbytes >> 20}MiB"
    ops = [Op(f"all_reduce/twoshot/{tag}",
              lambda b: (lambda: M.coll_all_reduce(b["send"], b["recv"], algo=M.TWOSHOT)),
              {"send": send, "recv": [torch.empty_like(t) for t in send]}, 2 * n * nbytes, 1,
              {"op": "all_reduce", "algo": "twoshot", "proto": "simple", "ranks": n, "bytes_per_rank": nbytes},
              inputs=["send"], outputs=["recv"], kernel="all_reduce/twoshot")]
    for proto, pname in ((M.LL, "ll"), (M.LL128, "ll128")):
        pb = M.coll_packed_bytes(nbytes, proto)
        pin = [torch.empty(pb, dtype=torch.uint8, device="cuda") for _ in range(n)]
        pout = [torch.empty(pb, dtype=torch.uint8, device="cuda") for _ in range(n)]
        recv = [torch.empty_like(t) for t in send]

        def pack(b, proto=proto):
            return lambda: M.coll_ll_pack_ranks(b["send"], b["pin"], proto, 1)

        def reduce_packed(b, proto=proto):
            return lambda: M.coll_all_reduce_packed(b["pin"], b["pout"], count, torch.bfloat16, proto, 1)

        def unpack(b, proto=proto):
            return lambda: M.coll_ll_unpack_ranks(b["pout"], b["recv"], proto, 1)

        ops += [
            Op(f"{pname}_pack/{tag}", pack, {"send": send, "pin": pin}, n * (nbytes + pb), 1,
               {"op": f"{pname}_pack", "ranks": n, "bytes_per_rank": nbytes, "packed_bytes_per_rank": pb},
               inputs=["send"], kernel=f"{pname}_pack"),
            Op(f"all_reduce/{pname}/{tag}", reduce_packed, {"pin": pin, "pout": pout}, 2 * n * nbytes, 1,
               {"op": "all_reduce_packed", "proto": pname, "ranks": n, "bytes_per_rank": nbytes,
                "line_bytes": 2 * n * pb, "note": "gbs counts payload bytes; the roofline counts line bytes"},
               kernel=f"all_reduce/{pname}", per_launch_bytes=2 * n * pb),
            Op(f"{pname}_unpack/{tag}", unpack, {"pout": pout, "recv": recv}, n * (pb + nbytes), 1,
               {"op": f"{pname}_unpack", "ranks": n, "bytes_per_rank": nbytes, "packed_bytes_per_rank": pb},
               outputs=["recv"], kernel=f"{pname}_unpack"),
        ]
    return ops


def build_full_step(M, oracle):
    """Every op of the hot path at the largest sizes (see the module docstring)."""
    import torch
    n = 8
    sp, _ = build_sp_prefill(M, oracle)
    for op in sp:
        op.ref = None
    ops = list(sp)
    ops += moe_ops(M, oracle, dedup=False, chain=True)
    for op in ops:
        op.ref = None
    for nbytes in FULL_STEP_AR_BYTES:
        ops += _protocol_ops(M, nbytes, n)
    # the TP-decode all-reduce at its largest shape, by the three algorithms
    tokens, hidden = 256, 7168
    S = tokens * hidden * 2
    send = [_dev(x, torch.bfloat16) for x in W.tp_decode(tokens, hidden, n)]
    for algo, aname in ((M.ONESHOT, "oneshot"), (M.TWOSHOT, "twoshot"), (M.RING, "ring")):
        form = M.coll_all_reduce_form(n, tokens * hidden, torch.bfloat16, algo)
        bufs = {"send": send, "recv": [torch.empty_like(t) for t in send]}
        if algo == M.RING:
            need = M.coll_all_reduce_workspace_size(n, tokens * hidden, torch.bfloat16, algo)
            bufs["ws"] = torch.zeros(need, dtype=torch.uint8, device="cuda")

        def bind(b, algo=algo):
            ws = b.get("ws")
            return lambda: M.coll_all_reduce(b["send"], b["recv"], algo=algo, workspace=ws)

        ops.append(Op(f"all_reduce/{aname}/{tokens}x{hidden}", bind, bufs, 2 * n * S,
                      2 * (n - 1) if form == M.RING_STEPS else 1,
                      {"op": "all_reduce", "algo": aname, "ranks": n, "shape": [tokens, hidden], "bytes_per_rank": S,
                       "form": FORM_NAMES[form]},
                      inputs=["send"], outputs=["recv"],
                      kernel="all_reduce/twoshot" if algo == M.TWOSHOT else f"all_reduce/{aname}"))
    ids = W.sampled_token_ids(n)
    ops.append(Op("broadcast", lambda b: (lambda: M.coll_broadcast(b["bufs"], 7)),
                  {"bufs": [_dev(x, torch.int32) for x in ids]}, 256 * 4 * n, 1,
                  {"op": "broadcast", "src": 7, "ranks": n, "dtype": "int32", "count": 256, "bytes_per_rank": 1024},
                  inputs=["bufs"], outputs=["bufs"], kernel="broadcast"))
    # reduce and scatter (no workload fixes their size): 16 MiB per rank
    S = FULL_STEP_MOVE_BYTES
    c = S // 2
    xs = [_dev(x, torch.bfloat16) for x in W.ranks_values(W.W_MISC, n, c, "bf16", "normal", salt=16)]
    ops.append(Op("reduce", lambda b: (lambda: M.coll_reduce(b["send"], b["out"], 0)),
                  {"send": xs, "out": torch.empty(c, dtype=torch.bfloat16, device="cuda")}, n * S + S, 1,
                  {"op": "reduce", "dst": 0, "ranks": n, "bytes_per_rank": S}, inputs=["send"], outputs=["out"],
                  kernel="reduce"))
    ops.append(Op("scatter", lambda b: (lambda: M.coll_scatter(b["src"], b["recv"], 0)),
                  {"src": torch.cat(xs), "recv": [torch.empty(c, dtype=torch.bfloat16, device="cuda")
                                                  for _ in range(n)]},
                  2 * n * S, 1, {"op": "scatter", "src": 0, "ranks": n, "bytes_per_rank": S},
                  inputs=["src"], outputs=["recv"], kernel="scatter"))
    return ops, full_step_cfg(n)


FORMS_RANKS = (2, 3, 4, 8)
FORMS_BYTES = tuple(1 << k for k in range(10, 29, 2))  # 1 KiB .. 256 MiB per rank


def build_allreduce_forms(M, oracle):
    """Every one-launch all-reduce form (one-shot, two-shot, the lane, CTA
    and cluster rings, the fused LL / LL128 two-shots and the LL ring) on bf16 messages of 1 KiB
    .. 256 MiB per rank at 2, 3, 4 and 8 virtual ranks: the measurements the
    AUTO choice rests on.  The LL forms move 4x the payload through L2 and
    stop at 16 MiB (two-shot) and 4 MiB (ring) per rank.  Inputs are seeded
    normal values drawn on the device (timing only)."""
    import torch
    g = torch.Generator(device="cuda")
    g.manual_seed(W.SEED_BASE + 77)
    ops = []
    forms = ((M.ONESHOT, "oneshot", None), (M.TWOSHOT, "twoshot", None), (M.RING_LANE, "ring_lane", None),
             (M.RING_CTA, "ring_cta", None),
             (M.RING_CLUSTER, "ring_cluster", None), (M.TWOSHOT_LL, "twoshot_ll", 16 << 20),
             (M.TWOSHOT_LL128, "twoshot_ll128", 64 << 20), (M.RING_LL, "ring_ll", 4 << 20))
    for n in FORMS_RANKS:
        for nbytes in FORMS_BYTES:
            count = nbytes // 2
            send = [torch.randn(count, generator=g, device="cuda").to(torch.bfloat16) for _ in range(n)]
            recv = [torch.empty_like(t) for t in send]
            for algo, aname, cap in forms:
                if cap is not None and nbytes > cap:
                    continue
                bufs = {"send": send, "recv": recv}
                need = M.coll_all_reduce_workspace_size(n, count, torch.bfloat16, algo)
                if need:
                    bufs["ws"] = torch.zeros(need, dtype=torch.uint8, device="cuda")

                def bind(b, algo=algo):
                    ws = b.get("ws")
                    return lambda: M.coll_all_reduce(b["send"], b["recv"], algo=algo, workspace=ws)

                ops.append(Op(f"all_reduce/{aname}/{n}x{nbytes}", bind, bufs, 2 * n * nbytes, 1,
                              {"op": "all_reduce", "algo": aname, "ranks": n, "bytes_per_rank": nbytes},
                              kernel=f"all_reduce/{aname}"))
    return ops, {"workload": "allreduce_forms_sweep", "virtual_ranks": list(FORMS_RANKS),
                 "bytes_per_rank": list(FORMS_BYTES), "dtype": "bf16",
                 "forms": ["oneshot", "twoshot", "ring_lane", "ring_cta", "ring_cluster", "twoshot_ll <= 16 MiB",
                           "twoshot_ll128 <= 64 MiB", "ring_ll <= 4 MiB"]}


def build_hbm_ceilings(M, oracle):
    """Context for the movement kernels' fractions: what this GPU's HBM does
    for a write-only stream (a fill), a read-only one (a sum) and a copy, on
    4 GiB, and for a 1 -> 8 fan-out and an 8 -> 1 fan-in of 128 MiB, with
    torch's own kernels.  The collectives here mostly write far
    more than they read (all_gather and dispatch write 8 bytes per byte read),
    so the copy figure that the roofline uses is not their only ceiling."""
    import torch
    n = 1 << 30  # 4 GiB of fp32
    a = torch.ones(n, device="cuda")
    b = torch.empty(n, device="cuda")
    nb = 4 * n
    small = 128 << 20  # bytes
    s_small = torch.ones(small // 2, dtype=torch.bfloat16, device="cuda")
    d_big = torch.empty(8, small // 2, dtype=torch.bfloat16, device="cuda")
    return [
        Op("write_only_fill", lambda bf: (lambda: bf["b"].fill_(2.0)), {"b": b}, nb, 0,
           {"op": "fill (torch)", "bytes": nb}, kernel="write_only_fill"),
        Op("read_only_sum", lambda bf: (lambda: bf["a"].sum()), {"a": a}, nb, 0,
           {"op": "sum (torch)", "bytes": nb}, kernel="read_only_sum"),
        # an element-wise kernel: a captured copy_ of one dtype becomes a
        # copy-engine transfer, which is not what the kernels here compete with
        Op("copy", lambda bf: (lambda: torch.mul(bf["a"], 1.0, out=bf["b"])), {"a": a, "b": b}, 2 * nb, 0,
           {"op": "copy (torch elementwise)", "bytes": 2 * nb}, kernel="copy"),
        # the all_gather / dispatch mix (one byte read, eight written) and the
        # combine / reduce_scatter mix (eight read, one written), at the
        # default step's all_gather size: 128 MiB <-> 8 x 128 MiB of bf16
        Op("fan_out_1to8", lambda bf: (lambda: bf["d"].copy_(bf["s"].expand(8, -1))),
           {"s": s_small, "d": d_big}, small + 8 * small, 0,
           {"op": "1 -> 8 broadcast copy (torch elementwise)", "bytes": 9 * small}, kernel="fan_out_1to8"),
        Op("fan_in_8to1", lambda bf: (lambda: torch.sum(bf["d"], 0, out=bf["s"])),
           {"s": s_small, "d": d_big}, small + 8 * small, 0,
           {"op": "8 -> 1 sum (torch)", "bytes": 9 * small}, kernel="fan_in_8to1"),
    ], {"workload": "hbm_ceilings_4GiB", "note": "torch kernels, context only"}


WORKLOADS = {
    "full_step": build_full_step,
    "hbm_ceilings": build_hbm_ceilings,
    "allreduce_forms": build_allreduce_forms,
    "single_image": build_single_image,
    "ring_compare": build_ring_compare,
    "movement": build_movement,
    "tp_decode": build_tp_decode,
    "twoshot_160k": build_twoshot_160k,
    "sp_prefill": build_sp_prefill,
    "moe": build_moe,
    "ll_sweep": build_ll_sweep,
}


# ---------------------------------------------------- the oracle on the host ----
#
# The CPU baseline and the reference arm run the oracle, as it stands, on a
# sample of a workload: each op is split into independent parts (element
# ranges, rows, or groups of tokens, each a smaller instance of the same op on
# the same kind of inputs) that worker processes, one per core, run at once.
# The parts' inputs are written once into a file that every worker maps, so a
# step moves no input between processes; what a step times is the oracle's
# own work on every part of every op.

ORACLE_SAMPLE = 16  # the oracle's sample is 1/ORACLE_SAMPLE of every op of a workload


class HostOp:
    """One op of a workload for the CPU oracle.  ``kind`` names a task in
    HOST_TASKS; ``pieces`` are its independent parts, each a dict of arrays
    (with the part's own parameters in ``params``); ``alg_bytes`` is what the
    whole (sampled) op must read plus write."""

    def __init__(self, name, kind, pieces, alg_bytes, **params):
        self.name, self.kind, self.alg_bytes, self.params = name, kind, alg_bytes, params
        self.pieces = [p for p in pieces if p is not None]


HOST_TASKS = {}  # kind -> fn(oracle module, the piece's arrays, params) -> the oracle's result


def _host_task(kind):
    def deco(fn):
        HOST_TASKS[kind] = fn
        return fn
    return deco


@_host_task("broadcast")
def _t_broadcast(o, a, prm):
    return o.broadcast(list(a["x"]), prm["src"])


@_host_task("gather")
def _t_gather(o, a, prm):
    return o.gather(list(a["x"]), a["dst"], rows=int(a["x"].shape[1] // prm["cols"]))


@_host_task("reduce")
def _t_reduce(o, a, prm):
    return o.reduce(list(a["x"]), 0, prm["dtype"])


@_host_task("scatter")
def _t_scatter(o, a, prm):
    return o.scatter(a["src"], prm["n"])


@_host_task("reduce_scatter")
def _t_reduce_scatter(o, a, prm):
    return o.reduce_scatter(list(a["x"]), 0, prm["dtype"])


@_host_task("all_gather")
def _t_all_gather(o, a, prm):
    return o.all_gather(list(a["x"]))


@_host_task("all_reduce")
def _t_all_reduce(o, a, prm):
    fn = {"oneshot": o.all_reduce_one_shot, "twoshot": o.all_reduce_two_shot, "ring": o.all_reduce_ring}[prm["algo"]]
    return fn(list(a["x"]), 0, prm["dtype"])


@_host_task("pack")
def _t_pack(o, a, prm):
    return [o.pack(x, prm["proto"], 1) for x in a["x"]]


@_host_task("all_reduce_packed")
def _t_all_reduce_packed(o, a, prm):
    p = a["p"]
    return o.all_reduce_packed(list(p), int(a["count"][0]), "bf16", 0, prm["proto"], 1)


@_host_task("unpack")
def _t_unpack(o, a, prm):
    nbytes = int(a["count"][0]) * 2
    return [o.unpack(p, nbytes, prm["proto"], 1) for p in a["p"]]


@_host_task("moe_route")
def _t_moe_route(o, a, prm):
    return o.moe_route(list(a["ids"]), prm["experts"])


@_host_task("moe_dispatch")
def _t_moe_dispatch(o, a, prm):
    n = a["ids"].shape[0]
    return o.moe_dispatch(list(a["x"]), list(a["ids"]), list(a["pos"]), [a[f"recv{d}"] for d in range(n)],
                          prm["experts"], prm["hidden"])


@_host_task("moe_combine")
def _t_moe_combine(o, a, prm):
    n = a["ids"].shape[0]
    return o.moe_combine([a[f"y{d}"] for d in range(n)], list(a["ids"]), list(a["pos"]), list(a["w"]),
                         prm["experts"], prm["hidden"], "bf16")


def _split(total: int, parts: int, align: int = 1):
    """[lo, hi) ranges cutting [0, total) into at most ``parts`` pieces whose
    starts are multiples of ``align``."""
    step = max(align, -(-total // max(1, parts) // align) * align) if total else align
    return [(lo, min(total, lo + step)) for lo in range(0, total, step)]


def _stack(xs):
    return np.ascontiguousarray(np.stack([np.asarray(x) for x in xs]))


def host_ar_pieces(oracle, xs, parts, name, algo, alg_per_elem, align=8, whole=False):
    n, e = len(xs), xs[0].size
    x = _stack(xs)
    rng_ = [(0, e)] if whole else _split(e, parts, align)
    return HostOp(name, "all_reduce", [{"x": np.ascontiguousarray(x[:, lo:hi])} for lo, hi in rng_],
                  alg_per_elem * e, algo=algo, dtype="bf16")


def host_full_step(oracle, parts: int, frac: int = ORACLE_SAMPLE):
    """The default workload for the oracle: every op at 1/frac of its size,
    on the first part of each rank's own input stream (MoE: the first
    tokens of each rank), each op cut into about ``parts`` pieces."""
    n = 8
    ops = []
    # sequence-parallel prefill
    rows = 1024 // frac
    x = _stack(W.sp_allgather(n, rows=rows))
    e = x.shape[1]
    ops.append(HostOp("all_gather", "all_gather", [{"x": np.ascontiguousarray(x[:, lo:hi])}
                                                   for lo, hi in _split(e, parts, 8)], (n + n * n) * e * 2))
    rows = 8192 // frac
    x = _stack(W.sp_reduce_scatter(n, rows=rows)).reshape(n, n, -1)  # [rank, output block, element]
    e = x.shape[2]
    ops.append(HostOp("reduce_scatter", "reduce_scatter",
                      [{"x": np.ascontiguousarray(x[:, :, lo:hi]).reshape(n, -1)} for lo, hi in _split(e, parts, 8)],
                      (n * n * e + n * e) * 2, dtype="bf16"))
    rows, cols = 256 // frac, 16032
    x = _stack(W.logits_shards(n, rows=rows)).reshape(n, rows, cols)
    ops.append(HostOp("gather", "gather",
                      [{"x": np.ascontiguousarray(x[:, lo:hi]).reshape(n, -1),
                        "dst": np.zeros((hi - lo) * n * cols, np.float32)} for lo, hi in _split(rows, parts)],
                      2 * n * rows * cols * 4, cols=cols))
    # MoE: each piece is the route, dispatch and combine of a group of tokens
    tokens, topk, experts, hidden = 4096 // frac, 8, 256, 7168
    ids, ws = W.moe_routing(tokens, experts, topk, n)
    xt = _stack(W.moe_tokens(tokens, hidden, n)).reshape(n, tokens, hidden)
    route, disp, comb = [], [], []
    for lo, hi in _split(tokens, parts):
        pid = np.ascontiguousarray(np.stack([i[lo:hi] for i in ids]))
        pw = np.ascontiguousarray(np.stack([w[lo:hi] for w in ws]))
        px = np.ascontiguousarray(xt[:, lo:hi]).reshape(n, -1)
        sc, _sd, _rd, pos = oracle.moe_route(list(pid), experts)
        recv0 = [np.zeros(int(sc[:, d].sum()) * hidden, np.uint16) for d in range(n)]
        y = oracle.moe_dispatch(list(px), list(pid), pos, recv0, experts, hidden)
        ppos = np.ascontiguousarray(np.stack(pos))
        route.append({"ids": pid})
        disp.append({"ids": pid, "x": px, "pos": ppos, **{f"recv{d}": recv0[d] for d in range(n)}})
        comb.append({"ids": pid, "w": pw, "pos": ppos, **{f"y{d}": y[d] for d in range(n)}})
    pairs, row = n * tokens * topk, hidden * 2
    ops.append(HostOp("moe_route", "moe_route", route, pairs * 4 * 2, experts=experts))
    ops.append(HostOp("moe_dispatch", "moe_dispatch", disp, n * tokens * row + pairs * row, experts=experts,
                      hidden=hidden))
    ops.append(HostOp("moe_combine", "moe_combine", comb, pairs * row + pairs * 4 + n * tokens * row,
                      experts=experts, hidden=hidden))
    # all-reduce of the 16 MiB and 256 MiB messages: Simple, LL, LL128
    for nbytes in FULL_STEP_AR_BYTES:
        count = nbytes // 2 // frac
        xs = W.ll_message(nbytes, n, elems=count)
        tag = f"{nbytes >> 20}MiB"
        ops.append(host_ar_pieces(oracle, xs, parts, f"all_reduce/twoshot/{tag}", "twoshot", 2 * n * 2, align=960))
        x = _stack(xs)
        for proto, pname in ((oracle.LL, "ll"), (oracle.LL128, "ll128")):
            pk, ar, up = [], [], []
            for lo, hi in _split(count, parts, 960):  # 1920 bytes: whole 16-byte groups and whole LL128 lines
                part = np.ascontiguousarray(x[:, lo:hi])
                packed = np.ascontiguousarray(np.stack([oracle.pack(v, proto, 1) for v in part]))
                cnt = np.array([hi - lo], np.int64)
                pk.append({"x": part})
                ar.append({"p": packed, "count": cnt})
                up.append({"p": packed, "count": cnt})
            pb = oracle.packed_bytes(count * 2, proto)
            ops.append(HostOp(f"{pname}_pack/{tag}", "pack", pk, n * (count * 2 + pb), proto=proto))
            ops.append(HostOp(f"all_reduce/{pname}/{tag}", "all_reduce_packed", ar, 2 * n * count * 2, proto=proto))
            ops.append(HostOp(f"{pname}_unpack/{tag}", "unpack", up, n * (count * 2 + pb), proto=proto))
    # TP decode at [256, 7168]: one-shot, two-shot, ring; the broadcast
    e = 256 * 7168 // frac
    xs = W.tp_decode(256, 7168, n, elems=e)
    ops.append(host_ar_pieces(oracle, xs, parts, "all_reduce/oneshot/256x7168", "oneshot", 2 * n * 2))
    ops.append(host_ar_pieces(oracle, xs, parts, "all_reduce/twoshot/256x7168", "twoshot", 2 * n * 2))
    # the ring's chunks (hence its order of addition) follow from the whole
    # message, so it runs as one piece
    ops.append(host_ar_pieces(oracle, xs, parts, "all_reduce/ring/256x7168", "ring", 2 * n * 2, whole=True))
    ops.append(HostOp("broadcast", "broadcast", [{"x": _stack(W.sampled_token_ids(n))}], 256 * 4 * n, src=7))
    # reduce and scatter
    c = FULL_STEP_MOVE_BYTES // 2 // frac
    x = _stack(W.ranks_values(W.W_MISC, n, c, "bf16", "normal", salt=16))
    ops.append(HostOp("reduce", "reduce", [{"x": np.ascontiguousarray(x[:, lo:hi])} for lo, hi in _split(c, parts, 8)],
                      (n * c + c) * 2, dtype="bf16"))
    ops.append(HostOp("scatter", "scatter",
                      [{"src": np.ascontiguousarray(x[:, lo:hi]).reshape(-1)} for lo, hi in _split(c, parts, 8)],
                      2 * n * c * 2, n=n))
    desc = (f"every op of the workload at 1/{frac} of its size (the first 1/{frac} of each rank's own seeded input; "
            f"MoE: the first {tokens} tokens of each rank), each op cut into up to {parts} independent pieces")
    return ops, full_step_cfg(n), desc


def host_tp_decode(oracle, parts: int):
    n = 8
    ops = []
    for tokens, hidden in W.tp_decode_shapes():
        xs = W.tp_decode(tokens, hidden, n)
        for algo in ("oneshot", "twoshot"):
            ops.append(host_ar_pieces(oracle, xs, parts, f"all_reduce/{algo}/{tokens}x{hidden}", algo, 2 * n * 2))
        ops.append(host_ar_pieces(oracle, xs, parts, f"all_reduce/ring/{tokens}x{hidden}", "ring", 2 * n * 2,
                                  whole=True))
    ops.append(HostOp("broadcast", "broadcast", [{"x": _stack(W.sampled_token_ids(n))}], 256 * 4 * n, src=7))
    return ops, tp_decode_cfg(n), "every op of the workload at full size, one-shot and two-shot cut into pieces"


def host_twoshot_160k(oracle, parts: int):
    xs = W.twoshot_160k(4)
    ops = [host_ar_pieces(oracle, xs, parts, "all_reduce/twoshot", "twoshot", 2 * 4 * 2)]
    return ops, twoshot_160k_cfg(4), "the workload at full size, cut into pieces"


HOST_WORKLOADS = {"full_step": host_full_step, "tp_decode": host_tp_decode, "twoshot_160k": host_twoshot_160k}

_WORKER = {}


def _worker_init(path, manifest):
    import oracle
    mm = np.memmap(path, dtype=np.uint8, mode="c")
    views = {}
    for key, arrays in manifest.items():
        views[key] = {nm: np.ndarray(shape, dtype=np.dtype(dt), buffer=mm, offset=off)
                      for nm, (off, dt, shape) in arrays.items()}
    _WORKER.update(oracle=oracle, mm=mm, views=views)


def _worker_run(task):
    i, p, kind, params = task
    HOST_TASKS[kind](_WORKER["oracle"], _WORKER["views"][(i, p)], params)  # the result stays in the worker
    return i


class OracleRunner:
    """The host ops of a workload on ``workers`` processes (spawned, so that
    it is safe after CUDA has been used in the parent)."""

    def __init__(self, ops, workers: int):
        import multiprocessing as mp
        import oracle
        self.ops, self.oracle = ops, oracle
        self.bytes_per_step = sum(op.alg_bytes for op in ops)
        self.tasks = [(i, p, op.kind, op.params) for i, op in enumerate(ops) for p in range(len(op.pieces))]
        # biggest pieces first, so that the last ones to start are short
        size = {(i, p): sum(a.nbytes for a in ops[i].pieces[p].values()) for i, p, _, _ in self.tasks}
        self.tasks.sort(key=lambda t: -size[(t[0], t[1])])
        fd, self.path = tempfile.mkstemp(prefix="mvr_oracle_", suffix=".bin")
        manifest, off = {}, 0
        with os.fdopen(fd, "wb") as f:
            for i, op in enumerate(ops):
                for p, arrays in enumerate(op.pieces):
                    entry = {}
                    for nm, a in arrays.items():
                        a = np.ascontiguousarray(a)
                        pad = (-off) % 64
                        f.write(b"\0" * pad)
                        off += pad
                        entry[nm] = (off, a.dtype.str, a.shape)
                        f.write(a.tobytes())
                        off += a.nbytes
                    manifest[(i, p)] = entry
            f.write(b"\0" * 64)
        self.workers = workers
        self.pool = mp.get_context("spawn").Pool(workers, initializer=_worker_init, initargs=(self.path, manifest))

    def step(self) -> float:
        t0 = time.perf_counter()
        for _ in self.pool.imap_unordered(_worker_run, self.tasks, chunksize=1):
            pass
        return time.perf_counter() - t0

    def single_thread_step(self) -> float:
        """The same tasks one after another in this process, on one core."""
        t0 = time.perf_counter()
        for i, p, kind, params in self.tasks:
            HOST_TASKS[kind](self.oracle, self.ops[i].pieces[p], params)
        return time.perf_counter() - t0

    def close(self):
        self.pool.terminate()
        self.pool.join()
        with contextlib.suppress(OSError):
            os.remove(self.path)


def oracle_workers() -> int:
    """One worker per core this process may run on (at most 64)."""
    return max(1, min(64, len(os.sched_getaffinity(0))))


def host_workload(workload: str, oracle, parts: int):
    if workload not in HOST_WORKLOADS:
        raise SystemExit(f"--impl reference supports {', '.join(sorted(HOST_WORKLOADS))}, not {workload}")
    return HOST_WORKLOADS[workload](oracle, parts)


def time_oracle(workload: str, min_s: float = 10.0, max_s: float = 30.0):
    """The CPU baseline of the GPU arm: whole sampled steps of the workload
    on all cores until about ``min_s`` seconds (at most ``max_s``), then one
    step on one core.  Returns the cpu_baseline object, or None when the
    workload has no oracle step."""
    import oracle
    if workload not in HOST_WORKLOADS:
        return None
    workers = oracle_workers()
    ops, _cfg, desc = host_workload(workload, oracle, workers)
    run = OracleRunner(ops, workers)
    try:
        run.step()  # warm-up: workers map their inputs
        secs, steps = 0.0, 0
        while secs < min_s and secs < max_s:
            secs += run.step()
            steps += 1
        single = run.single_thread_step()
    finally:
        run.close()
    return {"value": round(run.bytes_per_step * steps / secs / 1e9, 4), "unit": "GB/s", "cores": workers,
            "cpu_model": cpu_model(), "kind": "oracle", "sample": f"{steps} steps of {desc}",
            "seconds": round(secs, 2), "single_thread_value": round(run.bytes_per_step / single / 1e9, 4),
            "single_thread_seconds_per_step": round(single, 3)}


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


def sources_digest(files) -> str:
    import hashlib
    h = hashlib.sha256()
    for fn in sorted(files):
        with open(os.path.join(ROOT, fn), "rb") as f:
            h.update(fn.encode() + f.read())
    return h.hexdigest()[:16]


def traffic_for(kernel: str, workload: str):
    """DRAM bytes per call from profiles/traffic.json, if the counters were
    taken on the kernel's current source (its files' digest still matches)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p))
    e = d.get(workload, {}).get(kernel)
    if e and e.get("digest") == sources_digest(e.get("sources", [])):
        return e.get("dram_bytes_per_call")
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


def cpu_model() -> str:
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def empty_kernel_graph_us(stream, reps: int = 50) -> float:
    """Context for the latency floors: device time per launch of an empty
    (zero-cycle sleep) kernel, ``reps`` of them back to back in one CUDA graph."""
    import torch
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for _ in range(reps):
            torch.cuda._sleep(0)
    for _ in range(3):
        g.replay()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    g.replay()
    b.record(stream)
    torch.cuda.synchronize()
    us = a.elapsed_time(b) * 1e3 / reps
    del g
    return round(us, 3)


def graph_latency(ops, stream, reps: int = 50, max_bytes_per_rank: int = 256 * 1024):
    """Latency floor of the small ops: ``reps`` back-to-back calls on the same
    buffers captured in one CUDA graph (L2 warm), device time per call."""
    import torch
    out = {}
    for op in ops:
        if op.meta.get("bytes_per_rank", 1 << 62) > max_bytes_per_rank:
            continue
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
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
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="full_step", choices=sorted(WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-graph", action="store_true")
    ap.add_argument("--lead-us", type=float, default=300.0, help="sleep before each timed replay (outside the events)")
    ap.add_argument("--cold-factor", type=float, default=2.5, help="replicas x footprint >= this x L2")
    ap.add_argument("--max-replicas", type=int, default=256)
    ap.add_argument("--moe-tokens", type=int, default=4096,
                    help="tokens per rank of the MoE workload and of the all-to-all-v splits (smaller for ncu captures)")
    ap.add_argument("--ll-sizes", default=None,
                    help="comma-separated bytes per rank for the LL sweep (smaller for ncu captures)")
    ap.add_argument("--filter", default=None,
                    help="time only the ops whose 'name shape' (e.g. 'all_reduce/ring 256x7168') matches this regex")
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

    global MOE_TOKENS, LL_SIZES
    MOE_TOKENS = args.moe_tokens
    LL_SIZES = [int(x) for x in args.ll_sizes.split(",")] if args.ll_sizes else None
    ops, cfg = WORKLOADS[args.workload](M, oracle)
    if args.filter:
        import re
        pat = re.compile(args.filter)
        ops = [op for op in ops if pat.search(f"{op.name} {'x'.join(map(str, op.meta.get('shape', [])))}")]
        if not ops:
            raise SystemExit(f"--filter {args.filter!r} matches no op of workload {args.workload}")
        cfg = {**cfg, "filter": args.filter}
    prop = torch.cuda.get_device_properties(local)
    l2 = prop.L2_cache_size
    flush = torch.empty(2 * l2 // 4, dtype=torch.int32, device="cuda")
    lead_cycles = int(args.lead_us * 1e-6 * prop.clock_rate * 1e3)
    stream = torch.cuda.Stream()

    # R cold replicas per op, captured in one graph
    graphs = {}
    for op in ops:
        fp = max(1, op.footprint())
        reps = int(min(args.max_replicas, max(1, math.ceil(args.cold_factor * l2 / fp))))
        runs = [op.run] + [op.replicate() for _ in range(reps - 1)]
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(stream):
            for r in runs:  # run every replica once outside capture
                r()
        stream.synchronize()
        with torch.cuda.graph(g, stream=stream):
            for r in runs:
                r()
        graphs[id(op)] = (g, reps, runs)
    torch.cuda.synchronize()

    evs = {id(op): [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                    for _ in range(args.steps)] for op in ops}

    def one_step(k=None):
        with torch.cuda.stream(stream):
            for op in ops:
                g, reps, _ = graphs[id(op)]
                flush.sum()
                torch.cuda._sleep(lead_cycles)
                if k is None:
                    g.replay()
                else:
                    a, b = evs[id(op)][k]
                    a.record(stream)
                    g.replay()
                    b.record(stream)

    with Clocks(local) as clk:
        time.sleep(0.5)  # let the sampler start
        for _ in range(max(args.warmup, 3)):
            one_step()
        torch.cuda.synchronize()
        barrier(world)
        wall0 = time.perf_counter()
        for k in range(args.steps):
            one_step(k)
        torch.cuda.synchronize()
        wall = time.perf_counter() - wall0
        barrier(world)
    clocks = clk.summary()
    for op in ops:
        reps = graphs[id(op)][1]
        op.times = [a.elapsed_time(b) * 1e-3 / reps for a, b in evs[id(op)]]

    # one call alone between two events (includes the event pair's own cost)
    for op in ops:
        pairs = []
        with torch.cuda.stream(stream):
            for _ in range(5):
                flush.sum()
                torch.cuda._sleep(lead_cycles)
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                op.run()
                b.record(stream)
                pairs.append((a, b))
        stream.synchronize()
        op.single = [a.elapsed_time(b) * 1e-3 for a, b in pairs[1:]]
    graph_us = {}
    empty_us = None
    if not args.no_graph:
        with torch.cuda.stream(stream):
            graph_us = graph_latency(ops, stream)
            if graph_us:
                empty_us = empty_kernel_graph_us(stream)

    step_s = [sum(op.times[k] for op in ops) for k in range(args.steps)]
    total_s = sum(step_s)
    total_s_max = max_over_ranks(total_s, world, "cuda")
    bytes_step = sum(op.alg_bytes for op in ops)
    value = world * bytes_step * args.steps / total_s_max / 1e9
    hbm, hbm_src = peaks()

    # end-to-end: host->device of each op's inputs (pinned), the call through
    # the Python binding, device->host of its outputs.  Three streams: copies
    # in, calls, copies out.  An op's upload waits for the previous call (ops
    # of one shape share input buffers) and, when its inputs are the previous
    # op's outputs, for their download; so the upload of one op overlaps the
    # download of the one before (PCIe is full duplex).  Events bracket whole
    # steps.
    e2e = None
    if not args.no_e2e and any(op.inputs for op in ops) and any(op.outputs for op in ops):
        host_in = {}  # one pinned source per device input buffer, shared by the ops that upload it

        def pinned_in(t):
            if t.data_ptr() not in host_in:
                h = torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
                h.copy_(t)
                host_in[t.data_ptr()] = h
            return host_in[t.data_ptr()]

        pinned = {id(op): ([(t, pinned_in(t)) for nm in op.inputs for t in _as_list(op.bufs[nm])],
                           [(t, torch.empty(t.shape, dtype=t.dtype, pin_memory=True))
                            for nm in op.outputs for t in _as_list(op.bufs[nm])]) for op in ops}

        def spans(ts):
            return [(t.data_ptr(), t.data_ptr() + t.numel() * t.element_size()) for t in ts]

        def overlap(a, b):
            return any(x0 < y1 and y0 < x1 for x0, x1 in a for y0, y1 in b)

        in_spans = {id(op): spans([d for d, _ in pinned[id(op)][0]]) for op in ops}
        out_spans = {id(op): spans([d for d, _ in pinned[id(op)][1]]) for op in ops}
        s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        prev = None  # (op, call done, download done)
        for k in range(-1, args.steps):
            if k == 0:
                if prev is not None:
                    stream.wait_event(prev[2])
                t0.record(stream)
                s_in.wait_event(t0)
            for op in ops:
                ins, outs = pinned[id(op)]
                if prev is not None:
                    s_in.wait_event(prev[1])
                    if overlap(in_spans[id(op)], out_spans[id(prev[0])]):
                        s_in.wait_event(prev[2])
                with torch.cuda.stream(s_in):
                    for d, h in ins:
                        d.copy_(h, non_blocking=True)
                ev_in = torch.cuda.Event()
                ev_in.record(s_in)
                stream.wait_event(ev_in)
                if prev is not None and overlap(out_spans[id(op)], out_spans[id(prev[0])]):
                    stream.wait_event(prev[2])  # the previous download still reads these buffers
                with torch.cuda.stream(stream):
                    op.run()
                ev_run = torch.cuda.Event()
                ev_run.record(stream)
                s_out.wait_event(ev_run)
                with torch.cuda.stream(s_out):
                    for d, h in outs:
                        h.copy_(d, non_blocking=True)
                ev_out = torch.cuda.Event()
                ev_out.record(s_out)
                prev = (op, ev_run, ev_out)
        stream.wait_event(prev[2])
        t1.record(stream)
        torch.cuda.synchronize()
        e2e_s = max_over_ranks(t0.elapsed_time(t1) * 1e-3, world, "cuda")
        h2d = sum(d.numel() * d.element_size() for op in ops for d, _ in pinned[id(op)][0])
        d2h = sum(d.numel() * d.element_size() for op in ops for d, _ in pinned[id(op)][1])
        e2e = {"value": round(world * bytes_step * args.steps / e2e_s / 1e9, 3), "unit": "GB/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "how": "per op: pinned host->device copy of its inputs, the call through the Python binding of the "
                      "C ABI, device->host copy of its outputs, on three streams (an upload overlaps the previous "
                      "op's download); in a chain of ops (encode, packetised sum, decode; MoE route, dispatch, "
                      "combine) only what a caller holds on the host goes up and only the chain's result comes "
                      "down; CUDA events around the timed steps"}

    per_op, by_kernel = [], {}
    for op in ops:
        med = statistics.median(op.times)
        gbs = op.alg_bytes / med / 1e9
        extra = {"graph_us": graph_us[id(op)]} if id(op) in graph_us else {}
        per_op.append({**op.meta, "us": round(med * 1e6, 3),
                       "us_p10": round(float(np.percentile(op.times, 10)) * 1e6, 3),
                       "us_p90": round(float(np.percentile(op.times, 90)) * 1e6, 3),
                       "us_single": round(statistics.median(op.single) * 1e6, 3), **extra,
                       "replicas": graphs[id(op)][1], "gbs": round(gbs, 1),
                       "frac_measured_hbm": round(gbs / hbm, 4), "frac_8tbs": round(gbs / 8000, 4)})
        k = by_kernel.setdefault(op.kernel, {"time": 0.0, "bytes": 0, "calls": 0, "launches": 0})
        k["time"] += sum(op.times)
        k["bytes"] += op.per_launch_bytes * args.steps
        k["calls"] += args.steps
        k["launches"] += op.launches * args.steps
    dom = max(by_kernel, key=lambda k: by_kernel[k]["time"])
    d = by_kernel[dom]
    avg_call = d["time"] / d["calls"]
    achieved = d["bytes"] / d["calls"] / avg_call / 1e9
    launches_per_call = d["launches"] / d["calls"]  # an op whose form depends on size averages over its shapes
    roof = {"bound": "hbm", "kernel": dom, "launches_per_call": round(launches_per_call, 3),
            "achieved": round(achieved, 1),
            "peak": hbm, "unit": "GB/s", "frac": round(achieved / hbm, 4),
            "peak_source": f"{hbm_src} (MEASURED_PEAKS.json hbm_gbs, burst)",
            "share_of_step": round(d["time"] / total_s, 4), "traffic": traffic_for(dom, args.workload),
            "avg_call_us": round(avg_call * 1e6, 3),
            "avg_launch_us": round(avg_call * 1e6 / launches_per_call, 3) if launches_per_call else None,
            "algorithmic_bytes_per_call": round(d["bytes"] / d["calls"]),
            "note": "achieved = the op's algorithmic bytes / its device time; for a multi-launch op both are "
                    "spread evenly over its launches, so per launch the ratio is the same"}
    launches = sum(op.launches * graphs[id(op)][1] for op in ops) * args.steps

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = time_oracle(args.workload)

    if rank == 0:
        line = {"metric": METRIC, "value": round(value, 3), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
                "warmup": max(args.warmup, 3), "ms_per_step": round(total_s_max / args.steps * 1e3, 4),
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
                "data": "synthetic", "impl": "ours",
                "config": {**cfg, "parallelism": f"replicas x{world} (virtual ranks inside each GPU)",
                           "l2": "flushed: a read of 2 x L2 before each replay; each of the R calls in a replay "
                                 "uses its own buffers once",
                           "timing": "CUDA events around a CUDA-graph replay of the R calls, after a "
                                     f"{args.lead_us:.0f} us sleep kernel; op time = replay time / R"},
                "roofline": roof, "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches,
                "clocks": clocks, "wall_s_timed_region": round(wall, 3),
                "latency_floor_context": {"empty_kernel_graph_us": empty_us,
                                          "note": "graph_us of an op (<= 256 KB per rank) is its warm back-to-back "
                                                  "latency in a CUDA graph; an empty kernel launched the same way "
                                                  "costs empty_kernel_graph_us"},
                "ops": per_op}
        print(json.dumps(line), flush=True)
    graphs.clear()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


def main_reference(args, rank, world):
    """The oracle as it stands, on the host's cores (rank 0 only), on a
    bounded sample of the same workload."""
    if rank != 0:
        return
    import oracle

    workers = oracle_workers()
    ops, cfg, desc = host_workload(args.workload, oracle, workers)
    run = OracleRunner(ops, workers)
    try:
        for _ in range(max(args.warmup, 0)):
            run.step()
        times = [run.step() for _ in range(args.steps)]
        single = run.single_thread_step()
    finally:
        run.close()
    total = sum(times)
    value = run.bytes_per_step * len(times) / total / 1e9
    line = {"metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(total / len(times) * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "impl": "reference",
            "config": cfg,
            "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": workers, "cpu_model": cpu_model(),
                             "kind": "oracle", "sample": f"each step: {desc}",
                             "single_thread_value": round(run.bytes_per_step / single / 1e9, 4),
                             "single_thread_seconds_per_step": round(single, 3)},
            "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
