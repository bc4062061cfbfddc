"""LL and LL128 packet layouts and the packetised all-reduce.

Test infrastructure only (see ``oracle/__init__.py``).

"From NCCL Ring LL to PCIe IPC AllReduce" (hjcheng0602.cn), section
"Traditional LL Protocols": an LL line is [4 B data | 4 B flag] (so at most
half the bytes are payload); an LL128 line is [120 B data | 8 B flag].  Section
"Pro5000 ?": the LL receiver keeps re-reading 16-byte groups until BOTH flags in
the group equal the current step, and only then uses the data read with them.

Readings taken:

* LL line: little-endian u32 data word at byte 0, u32 flag = (u32)step at
  byte 4.  A message whose length is not a multiple of 4 has its last data
  word zero-padded.  Packed size = 8 * ceil(bytes / 4).
* LL128 line: bytes [120 L, 120 L + 120) of the message at line bytes 0..119
  (zero-padded at the end of the message), little-endian u64 flag = step at
  bytes 120..127.  Packed size = 128 * ceil(bytes / 120).  (NCCL's real LL128
  layout spreads the flag over a warp; the page does not describe that, so it
  is not used.)
* step >= 1, and for LL (u32)step != 0: zero-filled memory must never pass.
* unpack writes exactly ``bytes`` bytes whatever the flags say and counts the
  lines whose flag is not ``step``.
* packetised all-reduce: the N packed inputs are decoded (flags counted over
  every rank's lines), reduced in rank order, and the result re-encoded with
  flag = step into every rank's packed output.
"""
from __future__ import annotations

import numpy as np

from .numerics import reduce_ranks

SIMPLE, LL, LL128 = 0, 1, 2


def _ceil(a: int, b: int) -> int:
    return -(-a // b)


def packed_bytes(nbytes: int, proto: int) -> int:
    if proto == SIMPLE:
        return nbytes
    if proto == LL:
        return 8 * _ceil(nbytes, 4)
    if proto == LL128:
        return 128 * _ceil(nbytes, 120)
    raise ValueError(proto)


def _check_step(proto: int, step: int):
    assert step >= 1
    if proto == LL:
        assert step & 0xFFFFFFFF != 0


def pack(msg: np.ndarray, proto: int, step: int) -> np.ndarray:
    """Encode the bytes of ``msg`` (any dtype, viewed as uint8) into lines."""
    _check_step(proto, step)
    b = np.ascontiguousarray(msg).view(np.uint8).reshape(-1)
    nbytes = b.size
    if proto == LL:
        nlines = _ceil(nbytes, 4)
        data = np.zeros(nlines * 4, dtype=np.uint8)
        data[:nbytes] = b
        lines = np.empty((nlines, 2), dtype="<u4")
        lines[:, 0] = data.view("<u4")
        lines[:, 1] = step & 0xFFFFFFFF
        return lines.view(np.uint8).reshape(-1)
    if proto == LL128:
        nlines = _ceil(nbytes, 120)
        out = np.zeros((nlines, 128), dtype=np.uint8)
        data = np.zeros(nlines * 120, dtype=np.uint8)
        data[:nbytes] = b
        out[:, :120] = data.reshape(nlines, 120)
        out[:, 120:] = np.full(nlines, step, dtype="<u8").view(np.uint8).reshape(nlines, 8)
        return out.reshape(-1)
    raise ValueError(proto)


def unpack(packed: np.ndarray, nbytes: int, proto: int, step: int):
    """Decode; returns (message bytes as uint8[nbytes], number of bad-flag lines)."""
    _check_step(proto, step)
    p = np.ascontiguousarray(packed).view(np.uint8).reshape(-1)
    assert p.size == packed_bytes(nbytes, proto)
    if proto == LL:
        lines = p.view("<u4").reshape(-1, 2)
        bad = int(np.count_nonzero(lines[:, 1] != (step & 0xFFFFFFFF)))
        data = np.ascontiguousarray(lines[:, 0]).view(np.uint8)
        return data[:nbytes].copy(), bad
    if proto == LL128:
        lines = p.reshape(-1, 128)
        flags = np.ascontiguousarray(lines[:, 120:]).view("<u8").reshape(-1)
        bad = int(np.count_nonzero(flags != np.uint64(step)))
        data = np.ascontiguousarray(lines[:, :120]).reshape(-1)
        return data[:nbytes].copy(), bad
    raise ValueError(proto)


def all_reduce_packed(packed_in, count: int, dtype: str, op: int, proto: int, step: int):
    """Packetised all-reduce: returns (packed outputs per rank, bad-flag lines)."""
    from .numerics import ESIZE, NP_STORAGE

    nbytes = count * ESIZE[dtype]
    decoded, bad = [], 0
    for p in packed_in:
        data, b = unpack(p, nbytes, proto, step)
        bad += b
        decoded.append(data.view(NP_STORAGE[dtype]))
    full = reduce_ranks(decoded, op, dtype)
    enc = pack(full, proto, step)
    return [enc.copy() for _ in packed_in], bad
