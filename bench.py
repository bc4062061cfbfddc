"""Benchmark of the virtual-rank collectives on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload tp_decode|twoshot_160k|sp_prefill|moe|ll_sweep|
                               single_image|ring_compare|movement]

One "step" is one call of every op of the chosen workload on seeded synthetic
inputs resident in HBM.  ``value`` is the ops' algorithmic bytes (what each
collective must read plus write, once) over the step's device time, summed
over all GPUs, in GB/s.

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

Default workload (``tp_decode``): 8 virtual ranks, the TP-decode all-reduce
after RowParallelLinear (bf16 [tokens, hidden], tokens 1..256, hidden
4096/7168, N(0,1)) by one-shot, two-shot and ring, plus the broadcast of
int32 sampled_token_ids[256] from rank 7.

With --gpus N > 1 (torchrun, one process per GPU) every GPU runs its own
independent replica: the virtual ranks live inside one GPU, so there is no
exchange between GPUs (weak scaling; timing is the max over ranks).

``--impl reference`` times the CPU oracle (the plain definition of each op)
on this host's cores on the same workload.
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
    """One collective call.

    bind(bufs) -> callable that launches the op on those device buffers
    bufs:       dict of name -> tensor or list of tensors (device)
    inputs / outputs: names in ``bufs`` copied host->device / device->host by
                the end-to-end leg
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
              8: "ring_cta"}


def tp_decode_cfg(n):
    """The TP-decode workload's description, the same for both arms."""
    return {"workload": "tp_decode_allreduce_8vr", "virtual_ranks": n, "dtype": "bf16",
            "tokens": list(W.TP_DECODE_TOKENS), "hidden": list(W.TP_DECODE_HIDDEN),
            "algos": ["oneshot", "twoshot", "ring"], "plus": "broadcast int32[256] src=7",
            "values": "N(0,1) bf16 per rank, seeded"}


def twoshot_160k_cfg(n):
    return {"workload": "allreduce_twoshot_4vr_160KB", "virtual_ranks": n, "dtype": "bf16",
            "values": "uniform[-1,1] bf16, seeded"}


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


def build_moe(M, oracle):
    import torch
    n, tokens, topk, experts, hidden = 8, MOE_TOKENS, 8, 256, 7168
    ids, ws = W.moe_routing(tokens, experts, topk, n)
    xs = W.moe_tokens(tokens, hidden, n)
    dids = [torch.from_numpy(i).cuda() for i in ids]
    x = [_dev(v, torch.bfloat16) for v in xs]
    split = {"sc": torch.empty(n * n, dtype=torch.int64, device="cuda")}
    split["sd"], split["rd"] = torch.empty_like(split["sc"]), torch.empty_like(split["sc"])
    pos = [torch.empty(tokens * topk, dtype=torch.int32, device="cuda") for _ in range(n)]
    wsp = torch.empty(M.coll_moe_route_workspace_size(n, tokens, topk, experts), dtype=torch.uint8, device="cuda")
    M.coll_moe_route(dids, experts, split["sc"], split["sd"], split["rd"], pos, workspace=wsp)
    torch.cuda.synchronize()
    cap = int(split["sc"].view(n, n).sum(0).max().item())
    recv = [torch.empty(cap * hidden, dtype=torch.bfloat16, device="cuda") for _ in range(n)]
    row = hidden * 2
    pairs = n * tokens * topk
    ops = [
        Op("moe_route",
           lambda b: (lambda: M.coll_moe_route(b["ids"], experts, b["sc"], b["sd"], b["rd"], b["pos"],
                                               workspace=b["ws"])),
           {"ids": dids, "pos": pos, "ws": wsp, **split}, pairs * 4 * 2, 3,
           {"op": "moe_route", "ranks": n, "tokens": tokens, "topk": topk, "experts": experts},
           inputs=["ids"], outputs=["pos"], ref=lambda: oracle.moe_route(ids, experts), kernel="moe_route"),
        Op("moe_dispatch", lambda b: (lambda: M.coll_moe_dispatch(b["x"], b["ids"], b["pos"], b["recv"], experts)),
           {"x": x, "ids": dids, "pos": pos, "recv": recv}, n * tokens * row + pairs * row, 1,
           {"op": "moe_dispatch", "ranks": n, "hidden": hidden, "rows_out": pairs},
           inputs=["x"], outputs=["recv"], kernel="moe_dispatch"),
        Op("moe_combine",
           lambda b: (lambda: M.coll_moe_combine(b["y"], b["ids"], b["pos"], b["w"], b["out"], experts)),
           {"y": recv, "ids": dids, "pos": pos, "w": [torch.from_numpy(w).cuda() for w in ws],
            "out": [torch.empty_like(t) for t in x]}, pairs * row + pairs * 4 + n * tokens * row, 1,
           {"op": "moe_combine", "ranks": n, "hidden": hidden},
           inputs=["y"], outputs=["out"], kernel="moe_combine"),
    ]
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
           {"y": drecv, "ids": dids, "pos": dpos, "w": [torch.from_numpy(w).cuda() for w in ws],
            "out": [torch.empty_like(t) for t in x]}, uniq * row + pairs * 4 + n * tokens * row, 1,
           {"op": "moe_combine_dedup", "ranks": n, "hidden": hidden, "rows_in": uniq},
           inputs=["y"], outputs=["out"], kernel="moe_combine_dedup"),
    ]
    return ops, {"workload": "moe_dispatch_combine_8vr", "virtual_ranks": n, "tokens": tokens, "hidden": hidden,
                 "experts": experts, "topk": topk, "routing": "softmax(N(0,1)+log Zipf(1.1)) top-8, renormalised"}


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
    groups, the hops in shared memory (RING_CTA); the two-shot with LL packets fused into one cooperative
    launch (TWOSHOT_LL); and the stream-ordered packet path of the LL sweep
    (per-rank LL pack, packetised two-shot, per-rank unpack)."""
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
                                      (M.TWOSHOT_LL, "twoshot_ll", 1)):
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
                for r in range(n):
                    M.coll_ll_pack(b["send"][r], b["pin"][r], M.LL, 1)
                M.coll_all_reduce_packed(b["pin"], b["pout"], count, torch.bfloat16, M.LL, 1)
                for r in range(n):
                    M.coll_ll_unpack(b["pout"][r], b["recv"][r], M.LL, 1)
            return run

        ops.append(Op("all_reduce/ll_pack_ar_unpack", bind_ll,
                      {"send": send, "recv": [torch.empty_like(t) for t in send],
                       "pin": [torch.empty(pb, dtype=torch.uint8, device="cuda") for _ in range(n)],
                       "pout": [torch.empty(pb, dtype=torch.uint8, device="cuda") for _ in range(n)]},
                      2 * n * S, 2 * n + 1, {"op": "all_reduce", "algo": "ll_pack_ar_unpack",
                                             "shape": [tokens, hidden], "bytes_per_rank": S},
                      inputs=["send"], outputs=["recv"], kernel="all_reduce/ll_pack_ar_unpack"))
    return ops, {"workload": "ring_compare_8vr", "virtual_ranks": n, "shapes": W.tp_decode_shapes(),
                 "variants": ["ring_steps (launch per step)", "ring_ll (one launch, LL packets)",
                              "ring_cluster (one launch, cluster DSMEM hops)",
                              "ring_cta (one launch, ranks as warp groups, shared-memory hops)",
                              "twoshot_ll (one launch, LL packets, fused)",
                              "LL pack + packetised two-shot + unpack (stream-ordered)"]}


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


WORKLOADS = {
    "single_image": build_single_image,
    "ring_compare": build_ring_compare,
    "movement": build_movement,
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


def cpu_cores_used() -> int:
    return 1  # numpy element-wise kernels run on the calling thread


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


def time_oracle(ops, min_s: float = 10.0, max_s: float = 30.0):
    """Run the oracle version of the step's ops, whole steps at a time, until
    about ``min_s`` seconds of CPU work (at most ``max_s``); returns
    (GB/s, sample description, seconds)."""
    refs = [op for op in ops if op.ref is not None]
    if not refs:
        return None, "no op of this workload has a CPU definition", 0.0
    secs, nbytes, ops_done = 0.0, 0, 0
    while secs < min_s:
        for op in refs:
            t0 = time.perf_counter()
            op.ref()
            secs += time.perf_counter() - t0
            nbytes += op.alg_bytes
            ops_done += 1
            if secs > max_s:
                break
        if secs > max_s:
            break
    kinds = sorted(set(op.name.split("/")[0] for op in refs))
    sample = (f"{ops_done} oracle op calls = {ops_done / max(1, len(refs)):.2f} full steps of the same workload "
              f"({', '.join(kinds)}), full-size inputs")
    return (nbytes / secs / 1e9 if secs > 0 else None), sample, secs


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
    ap.add_argument("--workload", default="tp_decode", choices=sorted(WORKLOADS))
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
    if not args.no_e2e and all(op.inputs and op.outputs for op in ops):
        pinned = {id(op): ([(t, torch.empty(t.shape, dtype=t.dtype, pin_memory=True))
                            for nm in op.inputs for t in _as_list(op.bufs[nm])],
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
                      "op's download); CUDA events around the timed steps"}

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
            "avg_launch_us": round(avg_call * 1e6 / launches_per_call, 3),
            "algorithmic_bytes_per_call": round(d["bytes"] / d["calls"]),
            "note": "achieved = the op's algorithmic bytes / its device time; for a multi-launch op both are "
                    "spread evenly over its launches, so per launch the ratio is the same"}
    launches = sum(op.launches * graphs[id(op)][1] for op in ops) * args.steps

    cpu = None
    if rank == 0 and not args.no_cpu_baseline:
        v, sample, secs = time_oracle(ops)
        cpu = {"value": round(v, 4) if v else None, "unit": "GB/s", "cores": cpu_cores_used(), "cpu_model": cpu_model(),
               "kind": "oracle",
               "sample": sample, "seconds": round(secs, 2)}

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
    """The oracle as it stands, on the host's cores (rank 0 only)."""
    if rank != 0:
        return
    import oracle

    ops, cfg = host_ops(args.workload, oracle)
    times = []
    nbytes = sum(alg for alg, _ in ops)
    for k in range(max(args.warmup, 0) + args.steps):
        t0 = time.perf_counter()
        for _, ref in ops:
            ref()
        dt = time.perf_counter() - t0
        if k >= args.warmup:
            times.append(dt)
    total = sum(times)
    value = nbytes * len(times) / total / 1e9
    sample = f"every op of the workload, full size, {len(times)} timed passes on one core"
    line = {"metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(total / len(times) * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "impl": "reference",
            "config": cfg,
            "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": cpu_cores_used(), "cpu_model": cpu_model(),
                             "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def host_ops(workload: str, oracle):
    """The workload's ops as (algorithmic bytes, oracle call) on host inputs (no GPU)."""
    ops = []
    if workload == "tp_decode":
        n = 8
        for tokens, hidden in W.tp_decode_shapes():
            xs = W.tp_decode(tokens, hidden, n)
            S = tokens * hidden * 2
            for ref in (oracle.all_reduce_one_shot, oracle.all_reduce_two_shot, oracle.all_reduce_ring):
                ops.append((2 * n * S, lambda xs=xs, ref=ref: ref(xs, 0, "bf16")))
        ids = W.sampled_token_ids(n)
        ops.append((256 * 4 * n, lambda: oracle.broadcast(ids, 7)))
        cfg = tp_decode_cfg(n)
        return ops, cfg
    if workload == "twoshot_160k":
        xs = W.twoshot_160k(4)
        ops.append((2 * 4 * xs[0].size * 2, lambda: oracle.all_reduce_two_shot(xs, 0, "bf16")))
        return ops, twoshot_160k_cfg(4)
    raise SystemExit(f"--impl reference supports tp_decode and twoshot_160k, not {workload}")


if __name__ == "__main__":
    main()
