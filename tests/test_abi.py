"""The C-ABI library on the CPU: it loads, exports every entry point that
include/coll.h declares, and rejects bad arguments on the host before any
launch.  No kernel runs here (these tests are skipped where a GPU is
visible, because they pass made-up pointer values that must never reach a
kernel)."""
import ctypes
import os
import re

import numpy as np
import pytest
import torch

import movement_virtual_rank_b200 as M
import oracle
from conftest import ROOT

HEADER = os.path.join(ROOT, "include", "coll.h")
no_gpu = pytest.mark.skipif(torch.cuda.is_available(), reason="host-only argument checks use fake pointers")


def declared():
    txt = open(HEADER).read()
    return sorted(set(re.findall(r"^COLL_API\s+[\w\s\*]+?\b(coll_\w+)\s*\(", txt, flags=re.M)))


def test_header_declarations_are_exported():
    names = declared()
    assert len(names) >= 20
    L = M.lib()
    for n in names:
        assert hasattr(L, n), n
    # the binding covers exactly the declared entry points
    assert sorted(M.symbols()) == names


def test_exports_match_nm():
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", M.LIB_PATH], capture_output=True, text=True).stdout
    exported = {l.split()[-1] for l in out.splitlines() if " T " in l}
    assert set(declared()) <= exported
    assert {e for e in exported if e.startswith("coll_")} == set(declared())


def _header_value(name: str) -> int:
    """The value of a #define in coll.h (integer expressions of literals, shifts
    and other defines)."""
    txt = open(HEADER).read()
    m = re.search(rf"^#define\s+{name}\s+(.+?)(?:/\*.*)?$", txt, flags=re.M)
    assert m, name
    expr = re.sub(r"\b(COLL_\w+)\b", lambda k: str(_header_value(k.group(1))), m.group(1))
    expr = re.sub(r"(\d+)u\b", r"\1", expr)
    return int(eval(expr, {"__builtins__": {}}))  # digits, parentheses, shifts and divisions only


def test_binding_constants_match_header():
    """The Python binding's copies of the header's numbers are the header's."""
    assert M.RING_NOALLOC_MAX_COUNT == _header_value("COLL_RING_NOALLOC_MAX_COUNT")
    assert M.RING_LL_CALLS_PER_FILL == _header_value("COLL_RING_LL_CALLS_PER_FILL")
    assert M.TWOSHOT_LL_CALLS_PER_FILL == _header_value("COLL_TWOSHOT_LL_CALLS_PER_FILL")
    assert M.MAX_RANKS == _header_value("COLL_MAX_RANKS")
    for py, c in (("DEV_OK", "COLL_DEV_OK"), ("DEV_FLAG_MISMATCH", "COLL_DEV_FLAG_MISMATCH"),
                  ("DEV_TIMEOUT", "COLL_DEV_TIMEOUT"), ("DEV_SPLIT_OVERFLOW", "COLL_DEV_SPLIT_OVERFLOW"),
                  ("DEV_BAD_ROUTE", "COLL_DEV_BAD_ROUTE"), ("DEV_EPOCH_WRAP", "COLL_DEV_EPOCH_WRAP")):
        assert getattr(M, py) == _header_value(c), py


# AUTO's measured crossovers (bytes per rank): (ranks, last bytes of the one-shot or None)
AUTO_ONESHOT_UP_TO = {2: None, 3: 256 << 10, 4: 64 << 10, 5: None, 8: None, 16: None}


def test_auto_form_follows_the_measured_crossovers():
    L = M.lib()
    for n, last in AUTO_ONESHOT_UP_TO.items():
        for dt, es in ((M.BF16, 2), (M.FP32, 4), (M.INT32, 4)):
            for nbytes in (16, 1 << 10, 64 << 10, 256 << 10, 1 << 20, 256 << 20):
                for b in (nbytes - es, nbytes, nbytes + es):
                    want = M.ONESHOT if last is not None and b <= last else M.TWOSHOT
                    for aligned in (0, 1):
                        assert L.coll_all_reduce_form(n, b // es, dt, M.ALGO_AUTO, aligned) == want, (n, b, dt)


def test_version_and_strerror():
    assert M.coll_version() == 10000
    for code in (0, -1, -2, -3, -4, -5):
        assert M.coll_strerror(code)
    assert M.coll_strerror(-99) == "unknown status"


def test_packed_bytes_matches_oracle():
    for nbytes in (0, 1, 3, 4, 5, 119, 120, 121, 1 << 20, (1 << 28) + 7):
        for proto in (M.LL, M.LL128):
            assert M.coll_packed_bytes(nbytes, proto) == oracle.packed_bytes(nbytes, proto)
        assert M.coll_packed_bytes(nbytes, M.SIMPLE) == nbytes


def test_workspace_sizes():
    L = M.lib()
    assert L.coll_all_reduce_workspace_size(8, 1000, M.BF16, M.TWOSHOT) == 0
    ws = L.coll_all_reduce_workspace_size(8, 1000, M.BF16, M.RING)
    assert ws >= 4000 and ws % 256 == 0
    # TWOSHOT_LL128: header + two FIFOs of N x N segments in groups of 4 lines (480 payload B in 512 B)
    seg = -(-(-(-1000 // 8)) // 8) * 8
    assert L.coll_all_reduce_workspace_size(8, 1000, M.BF16, M.TWOSHOT_LL128) == 256 + 2 * 64 * -(-seg * 2 // 480) * 512
    assert L.coll_moe_route_workspace_size(8, 4096, 8, 256) > 0
    assert L.coll_moe_route_workspace_size(8, 4096, 8, 250) == 0  # experts not divisible by ranks
    assert L.coll_moe_route_workspace_size(8, 4096, 8, 2048) == 0  # too many experts


# RING's one-launch form by rank count: the largest bytes per rank at which
# the lane ring (RING_LANE) was measured fastest (None: every size); above
# it the CTA ring (RING_CTA)
RING_LANE_UP_TO = {2: None, 3: 256 << 10, 4: 256 << 10, 5: 16 << 10, 6: 16 << 10, 7: 16 << 10, 8: 16 << 10}


def test_ring_form_by_ranks_and_size():
    """RING picks RING_LANE or RING_CTA on the measured crossovers (host logic)."""
    L = M.lib()
    for n, up_to in RING_LANE_UP_TO.items():
        for nbytes in (16, 1 << 10, 16 << 10, (16 << 10) + 16, 256 << 10, (256 << 10) + 16, 1 << 20, 256 << 20):
            want = M.RING_LANE if up_to is None or nbytes <= up_to else M.RING_CTA
            assert L.coll_all_reduce_form(n, nbytes // 2, M.BF16, M.RING, 1) == want, (n, nbytes)
            assert L.coll_all_reduce_form(n, nbytes // 2, M.BF16, M.RING, 0) == M.RING_STEPS, (n, nbytes)


def test_all_reduce_form():
    """Which form coll_all_reduce runs (host logic only, no device call)."""
    L = M.lib()
    assert L.coll_all_reduce_form(8, 1000, M.BF16, M.RING, 1) == M.RING_LANE  # 2000 B per rank
    assert L.coll_all_reduce_form(8, 256 * 7168, M.BF16, M.RING, 1) == M.RING_CTA
    assert L.coll_all_reduce_form(8, 1 << 30, M.FP32, M.RING, 1) == M.RING_CTA
    assert L.coll_all_reduce_form(8, 1000, M.BF16, M.RING, 0) == M.RING_STEPS  # unaligned
    assert L.coll_all_reduce_form(9, 1000, M.BF16, M.RING, 1) == M.RING_STEPS  # more ranks than a CTA holds
    assert L.coll_all_reduce_form(2, 1000, M.BF16, M.RING, 1) == M.RING_LANE
    assert L.coll_all_reduce_form(2, 1 << 30, M.FP32, M.RING, 1) == M.RING_LANE
    assert L.coll_all_reduce_form(8, 5 << 20, M.BF16, M.RING_CLUSTER, 1) == M.RING_CLUSTER
    assert L.coll_all_reduce_form(8, 1000, M.BF16, M.RING_CLUSTER, 0) == M.RING_STEPS
    assert L.coll_all_reduce_form(8, 1000, M.BF16, M.RING_LL, 1) == M.RING_LL
    assert L.coll_all_reduce_form(8, 1000, M.BF16, M.RING_LL, 0) == M.RING_STEPS
    assert L.coll_all_reduce_form(8, 1000, M.BF16, M.ALGO_AUTO, 1) == M.TWOSHOT
    assert L.coll_all_reduce_form(8, 1000, M.BF16, M.ONESHOT, 1) == M.ONESHOT
    assert L.coll_all_reduce_form(8, 1000, M.BF16, M.RING_STEPS, 1) == M.RING_STEPS
    assert L.coll_all_reduce_form(8, 1000, M.BF16, M.TWOSHOT_LL, 1) == M.TWOSHOT_LL
    assert L.coll_all_reduce_form(8, 1000, M.BF16, M.TWOSHOT_LL, 0) == M.TWOSHOT
    assert L.coll_all_reduce_form(0, 1000, M.BF16, M.RING, 1) == -1
    assert L.coll_all_reduce_form(8, 1000, 9, M.RING, 1) == -1
    assert L.coll_all_reduce_form(8, 1000, M.BF16, M.RING_CTA, 1) == M.RING_CTA
    assert L.coll_all_reduce_form(8, 1000, M.BF16, M.RING_CTA, 0) == M.RING_STEPS
    assert L.coll_all_reduce_form(9, 1000, M.BF16, M.RING_CTA, 1) == M.RING_STEPS
    assert L.coll_all_reduce_form(8, 1000, M.BF16, M.TWOSHOT_LL128, 1) == M.TWOSHOT_LL128
    assert L.coll_all_reduce_form(8, 1000, M.BF16, M.TWOSHOT_LL128, 0) == M.TWOSHOT
    assert L.coll_all_reduce_form(8, 1000, M.BF16, M.RING_LANE, 1) == M.RING_LANE
    assert L.coll_all_reduce_form(8, 1000, M.BF16, M.RING_LANE, 0) == M.RING_STEPS
    assert L.coll_all_reduce_form(9, 1000, M.BF16, M.RING_LANE, 1) == M.RING_STEPS
    assert L.coll_all_reduce_form(3, 1000, M.BF16, M.RING_LANE, 1) == M.RING_LANE
    assert L.coll_all_reduce_form(8, 1000, M.BF16, M.RING_WIRE, 1) == M.RING_WIRE
    assert L.coll_all_reduce_form(2, 1 << 30, M.FP32, M.RING_WIRE, 1) == M.RING_WIRE
    assert L.coll_all_reduce_form(8, 1000, M.BF16, M.RING_WIRE, 0) == -2  # no stream-ordered form
    assert L.coll_all_reduce_form(9, 1000, M.BF16, M.RING_WIRE, 1) == -2
    assert L.coll_all_reduce_form(8, 1000, M.BF16, 12, 1) == -2
    # RING and RING_STEPS: a 256-byte header, then 4 bytes of partial per element
    for algo in (M.RING, M.RING_STEPS):
        assert L.coll_all_reduce_workspace_size(8, 1000, M.BF16, algo) == 256 + 4096
    # TWOSHOT_LL: two LL FIFOs of N x N segments (seg = 128 elements here), 8 bytes per 4
    assert L.coll_all_reduce_workspace_size(8, 1000, M.BF16, M.TWOSHOT_LL) == 256 + 2 * 2 * 64 * 128 * 2


def _arr(vals):
    a = (ctypes.c_void_p * len(vals))(*vals)
    return ctypes.cast(a, ctypes.POINTER(ctypes.c_void_p)), a


BASE = 0x7F0000000000  # made-up, 256-byte aligned addresses; never dereferenced


@no_gpu
def test_invalid_arguments_rejected_on_host():
    L = M.lib()
    p, _k = _arr([BASE + i * 0x100000 for i in range(4)])
    q, _k2 = _arr([BASE + 0x10000000 + i * 0x100000 for i in range(4)])
    null, _k3 = _arr([BASE, 0, BASE + 0x200000, BASE + 0x300000])
    # rank counts, null pointers, out-of-range roots
    assert L.coll_all_reduce(p, q, 0, 16, M.BF16, M.SUM, M.TWOSHOT, None, 0, None) == -1
    assert L.coll_all_reduce(p, q, 65, 16, M.BF16, M.SUM, M.TWOSHOT, None, 0, None) == -1
    assert L.coll_all_reduce(null, q, 4, 16, M.BF16, M.SUM, M.TWOSHOT, None, 0, None) == -1
    assert L.coll_broadcast(p, 4, 16, M.BF16, 4, None) == -1
    assert L.coll_broadcast(p, 4, 16, M.BF16, -1, None) == -1
    assert L.coll_gather(p, BASE + 0x40000000, 4, 0, 16, M.FP32, 0, None) == -1
    assert L.coll_reduce(p, BASE + 0x40000000, 4, 16, M.BF16, M.SUM, 7, None) == -1
    # unsupported dtype / op / algo
    assert L.coll_all_reduce(p, q, 4, 16, 9, M.SUM, M.TWOSHOT, None, 0, None) == -2
    assert L.coll_all_reduce(p, q, 4, 16, M.BF16, 9, M.TWOSHOT, None, 0, None) == -2
    assert L.coll_all_reduce(p, q, 4, 16, M.BF16, M.SUM, 12, None, 0, None) == -2
    assert L.coll_moe_combine(p, p, p, p, q, 4, 8, 2, 8, 16, M.INT32, 100, None, None) == -2
    # ring without workspace
    assert L.coll_all_reduce(p, q, 4, 16, M.BF16, M.SUM, M.RING, None, 0, None) == -5
    assert L.coll_all_reduce(p, q, 4, 16, M.BF16, M.SUM, M.RING, BASE + 0x50000000, 8, None) == -5
    assert L.coll_all_reduce(p, q, 4, 16, M.BF16, M.SUM, M.RING_STEPS, None, 0, None) == -5
    # CTA ring: no one-launch form (9 ranks, or unaligned buffers) and no RING workspace for the
    # stream-ordered fallback; a status workspace that is misaligned or inside a rank's buffer
    p9, _k6 = _arr([BASE + i * 0x100000 for i in range(9)])
    q9, _k7 = _arr([BASE + 0x10000000 + i * 0x100000 for i in range(9)])
    pu, _k8 = _arr([BASE + 2 + i * 0x100000 for i in range(4)])
    assert L.coll_all_reduce(p9, q9, 9, 16, M.BF16, M.SUM, M.RING_CTA, None, 0, None) == -2
    assert L.coll_all_reduce(pu, q, 4, 16, M.BF16, M.SUM, M.RING_CTA, None, 0, None) == -2
    assert L.coll_all_reduce(p, q, 4, 16, M.BF16, M.SUM, M.RING_CTA, BASE + 0x50000008, 64, None) == -5
    assert L.coll_all_reduce(p, q, 4, 1 << 16, M.BF16, M.SUM, M.RING_CTA, BASE + 0x100, 64, None) == -3
    assert L.coll_all_reduce(p9, q9, 9, 16, M.BF16, M.SUM, M.RING_LANE, None, 0, None) == -2
    assert L.coll_all_reduce(pu, q, 4, 16, M.BF16, M.SUM, M.RING_LANE, None, 0, None) == -2
    assert L.coll_all_reduce(p9, q9, 9, 16, M.BF16, M.SUM, M.RING_WIRE, None, 0, None) == -2
    assert L.coll_all_reduce(pu, q, 4, 16, M.BF16, M.SUM, M.RING_WIRE, None, 0, None) == -2
    assert L.coll_all_reduce(p, q, 4, 16, M.BF16, M.SUM, M.RING_LANE, BASE + 0x50000008, 64, None) == -5
    # fused LL two-shot: workspace missing, too small, or not 256-byte aligned
    need = L.coll_all_reduce_workspace_size(4, 16, M.BF16, M.TWOSHOT_LL)
    assert L.coll_all_reduce(p, q, 4, 16, M.BF16, M.SUM, M.TWOSHOT_LL, None, 0, None) == -5
    assert L.coll_all_reduce(p, q, 4, 16, M.BF16, M.SUM, M.TWOSHOT_LL, BASE + 0x50000000, need - 1, None) == -5
    assert L.coll_all_reduce(p, q, 4, 16, M.BF16, M.SUM, M.TWOSHOT_LL, BASE + 0x50000010, need, None) == -5
    # a workspace inside a rank's buffer
    assert L.coll_all_reduce(p, q, 4, 1 << 16, M.BF16, M.SUM, M.TWOSHOT_LL, BASE + 0x100, 1 << 24, None) == -3
    # the deduplicated MoE route validates like the plain one
    assert L.coll_moe_route_dedup(p, 4, 16, 0, 8, BASE, BASE, BASE, q, None, BASE, 1 << 20, None) == -1
    assert L.coll_moe_route_dedup(p, 4, 16, 2, 8, BASE, BASE, BASE, q, None, BASE + 8, 1 << 20, None) == -5
    # packets: step 0, LL step with zero low word, misaligned packet buffer
    assert L.coll_ll_pack(BASE, BASE + 0x100000, 64, M.LL, 0, None) == -1
    assert L.coll_ll_pack(BASE, BASE + 0x100000, 64, M.LL, 1 << 32, None) == -1
    assert L.coll_ll_pack(BASE, BASE + 0x100008, 64, M.LL128, 1, None) == -1
    assert L.coll_ll_unpack(BASE, BASE + 0x100000, 64, M.LL, 0, None, None) == -1
    assert L.coll_ll_pack(BASE, BASE + 0x100000, 64, 7, 1, None) == -2
    assert L.coll_all_reduce_packed(p, q, 4, 16, M.BF16, M.SUM, M.LL128, 0, None, None) == -1
    # the N-rank codecs: the same checks per rank, plus overlap between ranks
    assert L.coll_ll_pack_ranks(p, q, 4, 64, M.LL, 0, None) == -1
    assert L.coll_ll_pack_ranks(p, q, 0, 64, M.LL, 1, None) == -1
    assert L.coll_ll_pack_ranks(p, q, 4, 64, 7, 1, None) == -2
    assert L.coll_ll_unpack_ranks(q, p, 4, 64, M.LL128, 0, None, None) == -1
    q8, _k8 = _arr([BASE + 0x10000000 + i * 0x100000 + (8 if i == 2 else 0) for i in range(4)])
    assert L.coll_ll_pack_ranks(p, q8, 4, 64, M.LL, 1, None) == -1  # a packet buffer not 16-byte aligned
    qo, _ko = _arr([BASE + 0x10000000 + i * 0x40 for i in range(4)])  # packets 64 B apart, 128 B long
    assert L.coll_ll_pack_ranks(p, qo, 4, 64, M.LL, 1, None) == -3
    assert L.coll_ll_pack_ranks(p, p, 4, 64, M.LL, 1, None) == -3  # message and packet buffer overlap
    po, _kpo = _arr([BASE + i * 0x20 for i in range(4)])  # decoded messages 32 B apart, 64 B long
    assert L.coll_ll_unpack_ranks(q, po, 4, 64, M.LL, 1, None, None) == -3
    # MoE shapes
    assert L.coll_moe_route(p, 4, 16, 0, 8, BASE, BASE, BASE, q, None, BASE, 1 << 20, None) == -1
    assert L.coll_moe_route(p, 4, 16, 2, 6, BASE, BASE, BASE, q, None, BASE, 1 << 20, None) == -1
    assert L.coll_moe_route(p, 4, 16, 2, 8, BASE, BASE, BASE, q, None, BASE, 16, None) == -5
    assert L.coll_moe_route(p, 4, 16, 2, 8, BASE, BASE, BASE, q, None, BASE + 8, 1 << 20, None) == -5
    # all-to-all-v: negative counts, overflowing a stated capacity
    n = 2
    cnt = np.array([1, 1, 1, 1], np.int64)
    neg = np.array([1, -1, 1, 1], np.int64)
    dsp = np.array([0, 1, 0, 1], np.int64)
    cap = np.array([1, 1], np.int64)
    P = ctypes.POINTER(ctypes.c_int64)
    pp, _k4 = _arr([BASE, BASE + 0x1000])
    qq, _k5 = _arr([BASE + 0x10000, BASE + 0x11000])
    f = L.coll_all_to_all_v
    assert f(pp, qq, n, neg.ctypes.data_as(P), dsp.ctypes.data_as(P), dsp.ctypes.data_as(P), None, None, 4, M.BF16, None) == -1
    assert f(pp, qq, n, cnt.ctypes.data_as(P), dsp.ctypes.data_as(P), dsp.ctypes.data_as(P), cap.ctypes.data_as(P), None, 4, M.BF16, None) == -1
    # two sources landing on the same receive rows
    same = np.array([0, 0, 0, 0], np.int64)
    assert f(pp, qq, n, cnt.ctypes.data_as(P), dsp.ctypes.data_as(P), same.ctypes.data_as(P), None, None, 4, M.BF16, None) == -3


@no_gpu
def test_alias_rules_on_host():
    L = M.lib()
    n, count = 4, 1024
    b = 2 * count
    send, _k1 = _arr([BASE + i * 0x100000 for i in range(n)])
    # outputs overlapping each other
    bad, _k2 = _arr([BASE + 0x10000000, BASE + 0x10000000 + b // 2, BASE + 0x10100000, BASE + 0x10200000])
    assert L.coll_all_reduce(send, bad, n, count, M.BF16, M.SUM, M.TWOSHOT, None, 0, None) == -3
    # an output overlapping another rank's input
    cross, _k3 = _arr([BASE + 0x100000, BASE + 0x20000000, BASE + 0x20100000, BASE + 0x20200000])
    assert L.coll_all_reduce(send, cross, n, count, M.BF16, M.SUM, M.TWOSHOT, None, 0, None) == -3
    # in place is an error for one-shot
    assert L.coll_all_reduce(send, send, n, count, M.BF16, M.SUM, M.ONESHOT, None, 0, None) == -3
    # broadcast buffers must be disjoint
    ov, _k4 = _arr([BASE, BASE + 16, BASE + 0x100000, BASE + 0x200000])
    assert L.coll_broadcast(ov, n, count, M.BF16, 0, None) == -3
    # reduce-scatter output inside another rank's input
    rs_out, _k5 = _arr([BASE + 0x100000 + 8, BASE + 0x30000000, BASE + 0x30100000, BASE + 0x30200000])
    assert L.coll_reduce_scatter(send, rs_out, n, count // n, M.BF16, M.SUM, None) == -3
    # all-to-all input and output overlap
    assert L.coll_all_to_all(send, send, n, count // n, M.BF16, None) == -3


@no_gpu
def test_zero_counts_are_noops_on_host():
    L = M.lib()
    p, _k = _arr([BASE + i * 0x100000 for i in range(4)])
    q, _k2 = _arr([BASE + 0x10000000 + i * 0x100000 for i in range(4)])
    assert L.coll_all_reduce(p, q, 4, 0, M.BF16, M.SUM, M.RING, None, 0, None) == 0
    assert L.coll_broadcast(p, 4, 0, M.INT32, 1, None) == 0
    assert L.coll_all_gather(p, q, 4, 0, M.BF16, None) == 0
    assert L.coll_ll_pack(BASE, BASE + 0x100000, 0, M.LL, 1, None) == 0
    assert L.coll_ll_pack_ranks(p, q, 4, 0, M.LL128, 1, None) == 0
    assert L.coll_ll_unpack_ranks(q, p, 4, 0, M.LL, 1, None, None) == 0
    # a single rank in place does nothing
    assert L.coll_all_reduce(p, p, 1, 100, M.BF16, M.SUM, M.TWOSHOT, None, 0, None) == 0
    assert L.coll_broadcast(p, 1, 100, M.BF16, 0, None) == 0


def test_binding_rejects_cpu_tensors():
    x = [torch.zeros(8, dtype=torch.bfloat16) for _ in range(2)]
    with pytest.raises(ValueError):
        M.coll_all_reduce(x, x)
    with pytest.raises(ValueError):
        M.coll_broadcast(x, 0)
