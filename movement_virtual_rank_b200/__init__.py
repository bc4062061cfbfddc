"""Virtual-rank collectives on one B200: Python binding of ``libmvrcoll.so``.

Each of N virtual ranks is a torch CUDA tensor; every function here has the
name of the C entry point it calls (``include/coll.h``) and only marshals
arguments: it checks devices, dtypes and contiguity, turns the tensors into
device pointers and calls the library through ctypes.  Every step of every
collective runs in the library's CUDA kernels.  There is no fallback: if the
shared library has not been built, the first call raises ImportError.

    python -m movement_virtual_rank_b200.build     # builds libmvrcoll.so in-tree
"""
from __future__ import annotations

import ctypes
import os

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmvrcoll.so")

BF16, FP16, FP32, INT32 = 0, 1, 2, 3
SUM, MAX, MIN, PROD = 0, 1, 2, 3
(ALGO_AUTO, ONESHOT, TWOSHOT, RING, RING_LL, RING_CLUSTER, RING_STEPS, TWOSHOT_LL, RING_CTA, TWOSHOT_LL128,
 RING_LANE, RING_WIRE) = range(12)
SIMPLE, LL, LL128 = 0, 1, 2
DEV_OK, DEV_FLAG_MISMATCH, DEV_TIMEOUT, DEV_SPLIT_OVERFLOW, DEV_BAD_ROUTE, DEV_EPOCH_WRAP = 0, 1, 2, 3, 4, 5
RING_LL_CALLS_PER_FILL, TWOSHOT_LL_CALLS_PER_FILL = 1 << 25, 1 << 30  # calls one zero-filled workspace serves
MAX_RANKS = 64

_DTYPES = {torch.bfloat16: BF16, torch.float16: FP16, torch.float32: FP32, torch.int32: INT32}
_ESIZE = {BF16: 2, FP16: 2, FP32: 4, INT32: 4}
OPS = {"sum": SUM, "max": MAX, "min": MIN, "prod": PROD}
ALGOS = {"auto": ALGO_AUTO, "oneshot": ONESHOT, "twoshot": TWOSHOT, "ring": RING, "ring_ll": RING_LL,
         "ring_cluster": RING_CLUSTER, "ring_steps": RING_STEPS, "twoshot_ll": TWOSHOT_LL,
         "ring_cta": RING_CTA, "twoshot_ll128": TWOSHOT_LL128,
         "ring_lane": RING_LANE, "ring_wire": RING_WIRE}
PROTOS = {"simple": SIMPLE, "ll": LL, "ll128": LL128}


class CollError(RuntimeError):
    def __init__(self, fn: str, code: int, msg: str):
        super().__init__(f"{fn} failed: {msg} (status {code})")
        self.code = code


_lib = None
_VP = ctypes.c_void_p
_SZ = ctypes.c_size_t
_I = ctypes.c_int
_U64 = ctypes.c_uint64
_I64 = ctypes.c_int64
_PP = ctypes.POINTER(ctypes.c_void_p)
_PI64 = ctypes.POINTER(ctypes.c_int64)

_SIGS = {
    "coll_broadcast": (_I, [_PP, _I, _SZ, _I, _I, _VP]),
    "coll_gather": (_I, [_PP, _VP, _I, _SZ, _SZ, _I, _I, _VP]),
    "coll_reduce": (_I, [_PP, _VP, _I, _SZ, _I, _I, _I, _VP]),
    "coll_scatter": (_I, [_VP, _PP, _I, _SZ, _I, _I, _VP]),
    "coll_reduce_scatter": (_I, [_PP, _PP, _I, _SZ, _I, _I, _VP]),
    "coll_all_reduce": (_I, [_PP, _PP, _I, _SZ, _I, _I, _I, _VP, _SZ, _VP]),
    "coll_all_reduce_workspace_size": (_SZ, [_I, _SZ, _I, _I]),
    "coll_all_reduce_form": (_I, [_I, _SZ, _I, _I, _I]),
    "coll_all_gather": (_I, [_PP, _PP, _I, _SZ, _I, _VP]),
    "coll_all_to_all": (_I, [_PP, _PP, _I, _SZ, _I, _VP]),
    "coll_all_to_all_v": (_I, [_PP, _PP, _I, _PI64, _PI64, _PI64, _PI64, _PI64, _SZ, _I, _VP]),
    "coll_packed_bytes": (_SZ, [_SZ, _I]),
    "coll_ll_pack": (_I, [_VP, _VP, _SZ, _I, _U64, _VP]),
    "coll_ll_unpack": (_I, [_VP, _VP, _SZ, _I, _U64, _VP, _VP]),
    "coll_ll_pack_ranks": (_I, [_PP, _PP, _I, _SZ, _I, _U64, _VP]),
    "coll_ll_unpack_ranks": (_I, [_PP, _PP, _I, _SZ, _I, _U64, _VP, _VP]),
    "coll_all_reduce_packed": (_I, [_PP, _PP, _I, _SZ, _I, _I, _I, _U64, _VP, _VP]),
    "coll_moe_route": (_I, [_PP, _I, _I, _I, _I, _VP, _VP, _VP, _PP, _VP, _VP, _SZ, _VP]),
    "coll_moe_route_dedup": (_I, [_PP, _I, _I, _I, _I, _VP, _VP, _VP, _PP, _VP, _VP, _SZ, _VP]),
    "coll_moe_route_workspace_size": (_SZ, [_I, _I, _I, _I]),
    "coll_moe_dispatch": (_I, [_PP, _PP, _PP, _PP, _I, _I, _I, _I, _SZ, _I, _I64, _VP, _VP]),
    "coll_moe_combine": (_I, [_PP, _PP, _PP, _PP, _PP, _I, _I, _I, _I, _SZ, _I, _I64, _VP, _VP]),
    "coll_all_reduce_ring_noalloc": (_I, [_PP, _PP, _I, _SZ, _I, _I, _VP]),
    "coll_wait_flag": (_I, [_VP, ctypes.c_uint32, ctypes.c_uint32, _VP, _VP]),
    "coll_strerror": (ctypes.c_char_p, [_I]),
    "coll_version": (_I, []),
}


def lib():
    """The loaded shared library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                f"{LIB_PATH} is missing: build it with `python -m movement_virtual_rank_b200.build` "
                "(there is no fallback implementation)")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def symbols() -> list[str]:
    return sorted(_SIGS)


# ------------------------------------------------------------ marshalling ----

def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _check(fn: str, rc: int):
    if rc != 0:
        raise CollError(fn, rc, lib().coll_strerror(rc).decode())


def _cuda(t: torch.Tensor, what: str):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{what} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{what} must be contiguous")
    return t


def _ranks(ts, what: str, dtype=None):
    ts = list(ts)
    if not 1 <= len(ts) <= MAX_RANKS:
        raise ValueError(f"{what}: 1..{MAX_RANKS} ranks required, got {len(ts)}")
    dev = None
    for i, t in enumerate(ts):
        _cuda(t, f"{what}[{i}]")
        if dtype is not None and t.dtype != dtype:
            raise ValueError(f"{what}[{i}] has dtype {t.dtype}, expected {dtype}")
        dev = dev or t.device
        if t.device != dev:
            raise ValueError(f"{what}: all ranks must be on one device")
    return ts


def _ptrs(ts):
    arr = (ctypes.c_void_p * len(ts))(*[t.data_ptr() for t in ts])
    return ctypes.cast(arr, _PP), arr


def _dt(t: torch.Tensor) -> int:
    try:
        return _DTYPES[t.dtype]
    except KeyError:
        raise ValueError(f"unsupported dtype {t.dtype}") from None


def _op(op) -> int:
    return OPS[op] if isinstance(op, str) else int(op)


def _i64(a, n: int):
    a = np.ascontiguousarray(np.asarray(a, dtype=np.int64).reshape(-1))
    if a.size != n:
        raise ValueError(f"expected {n} entries, got {a.size}")
    return a, a.ctypes.data_as(_PI64)


def _same_numel(ts, what):
    n0 = ts[0].numel()
    for i, t in enumerate(ts):
        if t.numel() != n0:
            raise ValueError(f"{what}[{i}] has {t.numel()} elements, expected {n0}")
    return n0


# ------------------------------------------------------------- collectives ----

def coll_broadcast(bufs, src: int, stream=None):
    bufs = _ranks(bufs, "bufs", bufs[0].dtype)
    n = _same_numel(bufs, "bufs")
    p, _keep = _ptrs(bufs)
    with torch.cuda.device(bufs[0].device):
        _check("coll_broadcast", lib().coll_broadcast(p, len(bufs), n, _dt(bufs[0]), src, _stream(stream)))


def coll_gather(send, recv_dst: torch.Tensor, dst: int, rows: int | None = None, stream=None):
    send = _ranks(send, "send", send[0].dtype)
    _cuda(recv_dst, "recv_dst")
    n = _same_numel(send, "send")
    if rows is None:
        rows = int(np.prod(send[0].shape[:-1])) if send[0].dim() >= 2 else 1
    if rows <= 0 or n % rows:
        raise ValueError("rows must divide the per-rank element count")
    if recv_dst.numel() != n * len(send) or recv_dst.dtype != send[0].dtype:
        raise ValueError("recv_dst must hold N blocks of the send dtype")
    p, _keep = _ptrs(send)
    with torch.cuda.device(recv_dst.device):
        _check("coll_gather", lib().coll_gather(p, recv_dst.data_ptr(), len(send), rows, n // rows,
                                                _dt(recv_dst), dst, _stream(stream)))


def coll_reduce(send, recv_dst: torch.Tensor, dst: int, op="sum", stream=None):
    send = _ranks(send, "send", send[0].dtype)
    _cuda(recv_dst, "recv_dst")
    n = _same_numel(send, "send")
    if recv_dst.numel() != n or recv_dst.dtype != send[0].dtype:
        raise ValueError("recv_dst must match the send buffers")
    p, _keep = _ptrs(send)
    with torch.cuda.device(recv_dst.device):
        _check("coll_reduce", lib().coll_reduce(p, recv_dst.data_ptr(), len(send), n, _dt(recv_dst), _op(op),
                                                dst, _stream(stream)))


def coll_scatter(send_src: torch.Tensor, recv, src: int, stream=None):
    recv = _ranks(recv, "recv", send_src.dtype)
    _cuda(send_src, "send_src")
    n = _same_numel(recv, "recv")
    if send_src.numel() != n * len(recv):
        raise ValueError("send_src must hold N blocks")
    p, _keep = _ptrs(recv)
    with torch.cuda.device(send_src.device):
        _check("coll_scatter", lib().coll_scatter(send_src.data_ptr(), p, len(recv), n, _dt(send_src), src,
                                                  _stream(stream)))


def coll_reduce_scatter(send, recv, op="sum", stream=None):
    send = _ranks(send, "send", send[0].dtype)
    recv = _ranks(recv, "recv", send[0].dtype)
    if len(send) != len(recv):
        raise ValueError("send and recv must list the same ranks")
    _same_numel(send, "send")
    c = _same_numel(recv, "recv")
    if send[0].numel() != c * len(send):
        raise ValueError("every send buffer must hold N output blocks")
    ps, _k1 = _ptrs(send)
    pr, _k2 = _ptrs(recv)
    with torch.cuda.device(send[0].device):
        _check("coll_reduce_scatter", lib().coll_reduce_scatter(ps, pr, len(send), c, _dt(send[0]), _op(op),
                                                                _stream(stream)))


def coll_all_reduce_workspace_size(nranks: int, count: int, dtype: torch.dtype, algo=TWOSHOT) -> int:
    algo = ALGOS[algo] if isinstance(algo, str) else int(algo)
    return int(lib().coll_all_reduce_workspace_size(nranks, count, _DTYPES[dtype], algo))


def coll_all_reduce_form(nranks: int, count: int, dtype: torch.dtype, algo=TWOSHOT, aligned: bool = True) -> int:
    """The form coll_all_reduce() runs: ONESHOT, TWOSHOT, TWOSHOT_LL, TWOSHOT_LL128,
    RING_LL, RING_CLUSTER, RING_CTA, RING_LANE, RING_WIRE (one launch each) or
    RING_STEPS (2(N-1) launches)."""
    algo = ALGOS[algo] if isinstance(algo, str) else int(algo)
    rc = int(lib().coll_all_reduce_form(nranks, count, _DTYPES[dtype], algo, 1 if aligned else 0))
    if rc < 0:
        _check("coll_all_reduce_form", rc)
    return rc


def coll_all_reduce(send, recv, op="sum", algo=TWOSHOT, workspace: torch.Tensor | None = None, stream=None):
    """``workspace``: a CUDA tensor passed through to the library when given.
    RING, RING_STEPS, RING_LL, TWOSHOT_LL and TWOSHOT_LL128 need one of at least
    coll_all_reduce_workspace_size() bytes (zero-filled before its first
    RING_LL / TWOSHOT_LL / TWOSHOT_LL128 use) and get a zeroed one allocated here when it
    is omitted;
    RING_CLUSTER uses one, when given, for its status pair and its fallback
    to RING_STEPS; RING_CTA and RING_LANE only for that fallback; RING_WIRE
    ignores it (it has no fallback: unaligned buffers or more than 8 ranks
    raise)."""
    algo = ALGOS[algo] if isinstance(algo, str) else int(algo)
    send = _ranks(send, "send", send[0].dtype)
    recv = _ranks(recv, "recv", send[0].dtype)
    if len(send) != len(recv):
        raise ValueError("send and recv must list the same ranks")
    n = _same_numel(send, "send")
    if _same_numel(recv, "recv") != n:
        raise ValueError("send and recv sizes differ")
    ws_ptr, ws_bytes = None, 0
    if workspace is None and algo in (RING, RING_LL, RING_STEPS, TWOSHOT_LL, TWOSHOT_LL128):
        need = coll_all_reduce_workspace_size(len(send), n, send[0].dtype, algo)
        workspace = torch.zeros(max(need, 256), dtype=torch.uint8, device=send[0].device)
    if workspace is not None:
        ws_ptr, ws_bytes = workspace.data_ptr(), workspace.numel() * workspace.element_size()
    ps, _k1 = _ptrs(send)
    pr, _k2 = _ptrs(recv)
    with torch.cuda.device(send[0].device):
        _check("coll_all_reduce", lib().coll_all_reduce(ps, pr, len(send), n, _dt(send[0]), _op(op), algo,
                                                        ws_ptr, ws_bytes, _stream(stream)))


RING_NOALLOC_MAX_COUNT = (8 << 20) // 4


def coll_all_reduce_ring_noalloc(send, recv, op="sum", stream=None):
    """Ring all-reduce that takes no workspace and allocates nothing, for
    callers that may not allocate device memory: its partial sums live in a
    fixed 8 MiB array inside the library (at most RING_NOALLOC_MAX_COUNT
    elements per rank).  Same result as coll_all_reduce(..., algo=RING).
    Calls that overlap on the GPU share that array and race.  The first call
    on a device looks up the array (and, under lazy module loading, is when
    the driver places it): a call with empty tensors is a warm-up."""
    send = _ranks(send, "send", send[0].dtype)
    recv = _ranks(recv, "recv", send[0].dtype)
    if len(send) != len(recv):
        raise ValueError("send and recv must list the same ranks")
    n = _same_numel(send, "send")
    if _same_numel(recv, "recv") != n:
        raise ValueError("send and recv sizes differ")
    ps, _k1 = _ptrs(send)
    pr, _k2 = _ptrs(recv)
    with torch.cuda.device(send[0].device):
        _check("coll_all_reduce_ring_noalloc",
               lib().coll_all_reduce_ring_noalloc(ps, pr, len(send), n, _dt(send[0]), _op(op), _stream(stream)))


def coll_all_gather(send, recv, stream=None):
    send = _ranks(send, "send", send[0].dtype)
    recv = _ranks(recv, "recv", send[0].dtype)
    n = _same_numel(send, "send")
    if _same_numel(recv, "recv") != n * len(send):
        raise ValueError("every recv buffer must hold N send blocks")
    ps, _k1 = _ptrs(send)
    pr, _k2 = _ptrs(recv)
    with torch.cuda.device(send[0].device):
        _check("coll_all_gather", lib().coll_all_gather(ps, pr, len(send), n, _dt(send[0]), _stream(stream)))


def coll_all_to_all(send, recv, stream=None):
    send = _ranks(send, "send", send[0].dtype)
    recv = _ranks(recv, "recv", send[0].dtype)
    n = _same_numel(send, "send")
    if _same_numel(recv, "recv") != n or n % len(send):
        raise ValueError("send/recv must hold N equal blocks")
    ps, _k1 = _ptrs(send)
    pr, _k2 = _ptrs(recv)
    with torch.cuda.device(send[0].device):
        _check("coll_all_to_all", lib().coll_all_to_all(ps, pr, len(send), n // len(send), _dt(send[0]),
                                                        _stream(stream)))


def coll_all_to_all_v(send, recv, send_counts, send_displs, recv_displs, row_elems: int,
                      check_capacity: bool = True, stream=None):
    """Counts and displacements are host [N, N] arrays in rows:
    send_counts[s][d], send_displs[s][d], recv_displs[d][s]."""
    send = _ranks(send, "send", send[0].dtype)
    recv = _ranks(recv, "recv", send[0].dtype)
    n = len(send)
    if len(recv) != n:
        raise ValueError("send and recv must list the same ranks")
    sc, psc = _i64(send_counts, n * n)
    sd, psd = _i64(send_displs, n * n)
    rd, prd = _i64(recv_displs, n * n)
    pcap_s = pcap_r = None
    if check_capacity:
        scap, pcap_s = _i64([t.numel() // row_elems for t in send], n)
        rcap, pcap_r = _i64([t.numel() // row_elems for t in recv], n)
    ps, _k1 = _ptrs(send)
    pr, _k2 = _ptrs(recv)
    with torch.cuda.device(send[0].device):
        _check("coll_all_to_all_v", lib().coll_all_to_all_v(ps, pr, n, psc, psd, prd, pcap_s, pcap_r, row_elems,
                                                            _dt(send[0]), _stream(stream)))


# ----------------------------------------------------------------- packets ----

def coll_packed_bytes(nbytes: int, proto) -> int:
    proto = PROTOS[proto] if isinstance(proto, str) else int(proto)
    return int(lib().coll_packed_bytes(nbytes, proto))


def _nbytes(t: torch.Tensor) -> int:
    return t.numel() * t.element_size()


def coll_ll_pack(src: torch.Tensor, packed: torch.Tensor, proto, step: int, nbytes: int | None = None,
                 stream=None):
    proto = PROTOS[proto] if isinstance(proto, str) else int(proto)
    _cuda(src, "src")
    _cuda(packed, "packed")
    nbytes = _nbytes(src) if nbytes is None else nbytes
    if _nbytes(packed) < coll_packed_bytes(nbytes, proto):
        raise ValueError("packed buffer too small")
    with torch.cuda.device(src.device):
        _check("coll_ll_pack", lib().coll_ll_pack(src.data_ptr(), packed.data_ptr(), nbytes, proto, step,
                                                  _stream(stream)))


def coll_ll_unpack(packed: torch.Tensor, dst: torch.Tensor, proto, step: int, status: torch.Tensor | None = None,
                   nbytes: int | None = None, stream=None):
    proto = PROTOS[proto] if isinstance(proto, str) else int(proto)
    _cuda(packed, "packed")
    _cuda(dst, "dst")
    nbytes = _nbytes(dst) if nbytes is None else nbytes
    if _nbytes(packed) < coll_packed_bytes(nbytes, proto):
        raise ValueError("packed buffer too small")
    st = None if status is None else _cuda(status, "status").data_ptr()
    with torch.cuda.device(dst.device):
        _check("coll_ll_unpack", lib().coll_ll_unpack(packed.data_ptr(), dst.data_ptr(), nbytes, proto, step, st,
                                                      _stream(stream)))


def coll_ll_pack_ranks(src, packed, proto, step: int, nbytes: int | None = None, stream=None):
    """Encode every rank's message (``src[r]`` into ``packed[r]``) in one launch."""
    proto = PROTOS[proto] if isinstance(proto, str) else int(proto)
    src = _ranks(src, "src")
    packed = _ranks(packed, "packed")
    if len(src) != len(packed):
        raise ValueError("src and packed must list the same ranks")
    nbytes = _nbytes(src[0]) if nbytes is None else nbytes
    for t in src:
        if _nbytes(t) < nbytes:
            raise ValueError("src buffer too small")
    for t in packed:
        if _nbytes(t) < coll_packed_bytes(nbytes, proto):
            raise ValueError("packed buffer too small")
    (ps, _ks), (pp, _kp) = _ptrs(src), _ptrs(packed)
    with torch.cuda.device(src[0].device):
        _check("coll_ll_pack_ranks", lib().coll_ll_pack_ranks(ps, pp, len(src), nbytes, proto, step, _stream(stream)))


def coll_ll_unpack_ranks(packed, dst, proto, step: int, status: torch.Tensor | None = None,
                         nbytes: int | None = None, stream=None):
    """Decode every rank's packets (``packed[r]`` into ``dst[r]``) in one launch."""
    proto = PROTOS[proto] if isinstance(proto, str) else int(proto)
    packed = _ranks(packed, "packed")
    dst = _ranks(dst, "dst")
    if len(packed) != len(dst):
        raise ValueError("packed and dst must list the same ranks")
    nbytes = _nbytes(dst[0]) if nbytes is None else nbytes
    for t in dst:
        if _nbytes(t) < nbytes:
            raise ValueError("dst buffer too small")
    for t in packed:
        if _nbytes(t) < coll_packed_bytes(nbytes, proto):
            raise ValueError("packed buffer too small")
    st = None if status is None else _cuda(status, "status").data_ptr()
    (pp, _kp), (pd, _kd) = _ptrs(packed), _ptrs(dst)
    with torch.cuda.device(dst[0].device):
        _check("coll_ll_unpack_ranks", lib().coll_ll_unpack_ranks(pp, pd, len(dst), nbytes, proto, step, st,
                                                                  _stream(stream)))


def coll_all_reduce_packed(packed_in, packed_out, count: int, dtype: torch.dtype, proto, step: int, op="sum",
                           status: torch.Tensor | None = None, stream=None):
    proto = PROTOS[proto] if isinstance(proto, str) else int(proto)
    packed_in = _ranks(packed_in, "packed_in")
    packed_out = _ranks(packed_out, "packed_out")
    need = coll_packed_bytes(count * _ESIZE[_DTYPES[dtype]], proto)
    for t in packed_in + packed_out:
        if _nbytes(t) < need:
            raise ValueError("packed buffer too small")
    st = None if status is None else _cuda(status, "status").data_ptr()
    pi, _k1 = _ptrs(packed_in)
    po, _k2 = _ptrs(packed_out)
    with torch.cuda.device(packed_in[0].device):
        _check("coll_all_reduce_packed", lib().coll_all_reduce_packed(pi, po, len(packed_in), count, _DTYPES[dtype],
                                                                      _op(op), proto, step, st, _stream(stream)))


# --------------------------------------------------------------------- MoE ----

def coll_moe_route_workspace_size(nranks: int, tokens: int, topk: int, n_experts: int) -> int:
    return int(lib().coll_moe_route_workspace_size(nranks, tokens, topk, n_experts))


def coll_moe_route(topk_ids, n_experts: int, send_counts: torch.Tensor, send_displs: torch.Tensor,
                   recv_displs: torch.Tensor, pos, status: torch.Tensor | None = None,
                   workspace: torch.Tensor | None = None, stream=None, dedup: bool = False):
    """topk_ids: per rank int32 [tokens, topk]; outputs: int64 [N*N] tensors and
    per-rank int32 [tokens*topk] positions.  ``workspace`` is allocated here when omitted.
    ``dedup`` calls coll_moe_route_dedup (one row per (token, destination rank))."""
    topk_ids = _ranks(topk_ids, "topk_ids", torch.int32)
    pos = _ranks(pos, "pos", torch.int32)
    n = len(topk_ids)
    tokens, topk = topk_ids[0].shape
    for t in (send_counts, send_displs, recv_displs):
        _cuda(t, "split matrix")
        if t.dtype != torch.int64 or t.numel() != n * n:
            raise ValueError("split matrices must be int64 [N*N]")
    need = coll_moe_route_workspace_size(n, tokens, topk, n_experts)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=topk_ids[0].device)
    st = None if status is None else _cuda(status, "status").data_ptr()
    pi, _k1 = _ptrs(topk_ids)
    pp, _k2 = _ptrs(pos)
    with torch.cuda.device(topk_ids[0].device):
        fn = "coll_moe_route_dedup" if dedup else "coll_moe_route"
        _check(fn, getattr(lib(), fn)(
            pi, n, tokens, topk, n_experts, send_counts.data_ptr(), send_displs.data_ptr(), recv_displs.data_ptr(),
            pp, st, workspace.data_ptr(), _nbytes(workspace), _stream(stream)))


def coll_moe_route_dedup(topk_ids, n_experts: int, send_counts: torch.Tensor, send_displs: torch.Tensor,
                         recv_displs: torch.Tensor, pos, status: torch.Tensor | None = None,
                         workspace: torch.Tensor | None = None, stream=None):
    """The route with one row per (token, destination rank); see coll_moe_route."""
    coll_moe_route(topk_ids, n_experts, send_counts, send_displs, recv_displs, pos, status, workspace, stream,
                   dedup=True)


def coll_moe_dispatch(x, topk_ids, pos, recv, n_experts: int, status: torch.Tensor | None = None, stream=None):
    """x: per rank [tokens, hidden]; recv: per rank [capacity, hidden] (one capacity for all)."""
    x = _ranks(x, "x", x[0].dtype)
    recv = _ranks(recv, "recv", x[0].dtype)
    topk_ids = _ranks(topk_ids, "topk_ids", torch.int32)
    pos = _ranks(pos, "pos", torch.int32)
    n = len(x)
    tokens, topk = topk_ids[0].shape
    hidden = x[0].numel() // max(tokens, 1)
    cap = min(t.numel() for t in recv) // max(hidden, 1)
    st = None if status is None else _cuda(status, "status").data_ptr()
    px, _a = _ptrs(x)
    pi, _b = _ptrs(topk_ids)
    pp, _c = _ptrs(pos)
    pr, _d = _ptrs(recv)
    with torch.cuda.device(x[0].device):
        _check("coll_moe_dispatch", lib().coll_moe_dispatch(px, pi, pp, pr, n, tokens, topk, n_experts, hidden,
                                                            _dt(x[0]), cap, st, _stream(stream)))


def coll_moe_combine(y, topk_ids, pos, topk_w, out, n_experts: int, status: torch.Tensor | None = None,
                     stream=None):
    """y: per rank [capacity, hidden] expert outputs; topk_w: per rank fp32 [tokens, topk];
    out: per rank [tokens, hidden]."""
    y = _ranks(y, "y", y[0].dtype)
    out = _ranks(out, "out", y[0].dtype)
    topk_ids = _ranks(topk_ids, "topk_ids", torch.int32)
    pos = _ranks(pos, "pos", torch.int32)
    topk_w = _ranks(topk_w, "topk_w", torch.float32)
    n = len(y)
    tokens, topk = topk_ids[0].shape
    hidden = out[0].numel() // max(tokens, 1)
    cap = min(t.numel() for t in y) // max(hidden, 1)
    st = None if status is None else _cuda(status, "status").data_ptr()
    py, _a = _ptrs(y)
    pi, _b = _ptrs(topk_ids)
    pp, _c = _ptrs(pos)
    pw, _d = _ptrs(topk_w)
    po, _e = _ptrs(out)
    with torch.cuda.device(y[0].device):
        _check("coll_moe_combine", lib().coll_moe_combine(py, pi, pp, pw, po, n, tokens, topk, n_experts, hidden,
                                                          _dt(y[0]), cap, st, _stream(stream)))


def coll_wait_flag(flag: torch.Tensor, expect: int, budget_us: int, status: torch.Tensor, stream=None):
    """Bounded wait on a device word (flag: int32/uint32 CUDA tensor, first element)."""
    _cuda(flag, "flag")
    _cuda(status, "status")
    with torch.cuda.device(flag.device):
        _check("coll_wait_flag", lib().coll_wait_flag(flag.data_ptr(), expect & 0xFFFFFFFF, budget_us,
                                                      status.data_ptr(), _stream(stream)))


def coll_strerror(code: int) -> str:
    return lib().coll_strerror(code).decode()


def coll_version() -> int:
    return int(lib().coll_version())

