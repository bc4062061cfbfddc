"""Element types and the per-element reduction of the oracle.

Test infrastructure only (see ``oracle/__init__.py``).

Readings taken (the pages fix none of these; the workloads do):

* Summation: "fp32 accumulate in rank order" of the TP-decode and two-shot
  workloads.  ``acc = widen(x_0)``, then ``acc = acc + widen(x_r)`` for
  r = 1 .. N-1, each addition an IEEE binary32 round-to-nearest-even add
  (numpy float32 arithmetic), then ONE rounding to the storage type.
  Starting from x_0 rather than +0 keeps -0 when every input is -0.
* Rounding to bf16 / fp16: round to nearest, ties to even (IEEE 754
  roundTiesToEven); overflow goes to +-inf.  A NaN result of any float type
  becomes the canonical quiet NaN (bf16 0x7FC0, fp16 0x7E00, fp32
  0x7FC00000), sign and payload dropped: IEEE leaves NaN payloads to the
  implementation, and x86 and the GPU pick different ones.
* MAX / MIN (the tutorial's section 3.1 lists SUM, MAX, MIN, PROD): the
  running value is replaced only by a strictly greater (smaller) value, so
  between equal values (+0 / -0) the earlier rank wins; a NaN, once met,
  stays.  Widening is exact, so the narrowed result is the winning input's
  own bits, except that a NaN comes out as the canonical NaN.
* PROD: fp32 products in rank order, one rounding at the end.
* int32: SUM and PROD wrap modulo 2^32, MAX and MIN are exact.
"""
from __future__ import annotations

import numpy as np

DTYPES = ("bf16", "fp16", "fp32", "int32")
SUM, MAX, MIN, PROD = 0, 1, 2, 3
OPS = (SUM, MAX, MIN, PROD)

ESIZE = {"bf16": 2, "fp16": 2, "fp32": 4, "int32": 4}
NP_STORAGE = {"bf16": np.uint16, "fp16": np.uint16, "fp32": np.float32, "int32": np.int32}


# ---------------------------------------------------------------- bf16 ----

def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """bf16 is the top half of a binary32 word: widening is exact."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def f32_to_bf16_bits(f: np.ndarray) -> np.ndarray:
    """binary32 -> bfloat16 with round-to-nearest-even, written from the rule.

    Keep the top 16 bits; the dropped low 16 bits decide: above one half of
    the last kept place -> round up, below -> truncate, exactly one half ->
    round to the even (last kept bit 0) neighbour.  A carry out of the kept
    significand moves into the exponent, which is how IEEE encodings round up
    to the next binade and, from the largest finite value, to infinity.
    """
    u = np.ascontiguousarray(f, dtype=np.float32).view(np.uint32)
    keep = u >> np.uint32(16)
    drop = u & np.uint32(0xFFFF)
    half = np.uint32(0x8000)
    up = (drop > half) | ((drop == half) & ((keep & np.uint32(1)) == 1))
    out = (keep + up.astype(np.uint32)).astype(np.uint16)
    nan = (u & np.uint32(0x7FFFFFFF)) > np.uint32(0x7F800000)
    out[nan] = 0x7FC0
    return out


def bf16_ulp_diff(a_bits: np.ndarray, b_bits: np.ndarray) -> np.ndarray:
    """Distance in units of the last place between two bf16 arrays (finite)."""

    def ordered(x):
        x = np.asarray(x, dtype=np.uint16).astype(np.int32)
        mag = x & 0x7FFF
        return np.where(x & 0x8000, -mag, mag)

    return np.abs(ordered(a_bits) - ordered(b_bits))


# ---------------------------------------------------------------- fp16 ----

def f16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return np.asarray(b, dtype=np.uint16).view(np.float16).astype(np.float32)


def f32_to_f16_bits(f: np.ndarray) -> np.ndarray:
    """binary32 -> binary16, round-to-nearest-even (numpy's conversion), NaN canonical."""
    f = np.ascontiguousarray(f, dtype=np.float32)
    with np.errstate(over="ignore", invalid="ignore"):
        out = f.astype(np.float16).view(np.uint16).copy()
    out[np.isnan(f)] = 0x7E00
    return out


# ------------------------------------------------------------- generic ----

def widen(x: np.ndarray, dtype: str) -> np.ndarray:
    """Storage -> arithmetic type (fp32 for the float types, int32 for int32)."""
    if dtype == "bf16":
        return bf16_bits_to_f32(x)
    if dtype == "fp16":
        return f16_bits_to_f32(x)
    if dtype == "fp32":
        return np.asarray(x, dtype=np.float32)
    if dtype == "int32":
        return np.asarray(x, dtype=np.int32)
    raise ValueError(dtype)


def narrow(acc: np.ndarray, dtype: str) -> np.ndarray:
    """Arithmetic type -> storage, the single rounding of a reduction."""
    if dtype == "bf16":
        return f32_to_bf16_bits(acc)
    if dtype == "fp16":
        return f32_to_f16_bits(acc)
    if dtype == "fp32":
        out = np.array(acc, dtype=np.float32, copy=True)
        out.view(np.uint32)[np.isnan(out)] = 0x7FC00000
        return out
    if dtype == "int32":
        return np.asarray(acc, dtype=np.int32)
    raise ValueError(dtype)


def combine(acc: np.ndarray, v: np.ndarray, op: int, dtype: str) -> np.ndarray:
    """One accumulation step ``acc <- acc (op) v`` in the arithmetic type."""
    with np.errstate(over="ignore", invalid="ignore"):
        if op == SUM:
            return acc + v
        if op == PROD:
            return acc * v
        if op in (MAX, MIN):
            better = (v > acc) if op == MAX else (v < acc)
            if dtype != "int32":
                better = ~np.isnan(acc) & (np.isnan(v) | better)
            return np.where(better, v, acc)
    raise ValueError(op)


def reduce_ranks(xs, op: int, dtype: str, order=None) -> np.ndarray:
    """Elementwise reduction of the ranks' arrays ``xs`` (storage type).

    ``order`` is the rank order of the accumulation (default 0 .. N-1).
    The result is rounded once, to the storage type.
    """
    order = list(range(len(xs))) if order is None else list(order)
    acc = widen(xs[order[0]], dtype).copy()
    for r in order[1:]:
        acc = combine(acc, widen(xs[r], dtype), op, dtype)
    return narrow(acc, dtype)
