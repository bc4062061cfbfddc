"""Planted mistakes in the oracle (CPU only): each mutant below is a plausible
slip -- a dropped term, a wrong sign, order or index, a transposed operand, a
missing rounding rule -- and at least one pin must reject it.  This is how the
pins themselves are checked: the oracle is only trusted because a wrong oracle
would fail them.
"""
import numpy as np
import pytest

import oracle
import oracle_pins as P
from oracle import collectives as C
from oracle import moe as M
from oracle import numerics as NUM
from oracle import packets as PK

MODULES = (oracle, C, M, NUM, PK)


def _patch(monkeypatch, name, fn):
    hit = False
    for mod in MODULES:
        if hasattr(mod, name):
            monkeypatch.setattr(mod, name, fn)
            hit = True
    assert hit, name


_orig_narrow = NUM.narrow
_orig_combine = NUM.combine
_orig_widen = NUM.widen


def m_truncate_bf16(mp):
    _patch(mp, "f32_to_bf16_bits", lambda f: (np.ascontiguousarray(f, np.float32).view(np.uint32) >> 16).astype(np.uint16))


def m_round_half_up_bf16(mp):
    def f(x):
        u = np.ascontiguousarray(x, np.float32).view(np.uint32)
        return ((u + np.uint32(0x8000)) >> 16).astype(np.uint16)
    _patch(mp, "f32_to_bf16_bits", f)


def m_drop_last_rank(mp):
    orig = NUM.reduce_ranks

    def f(xs, op, dtype, order=None):
        return orig(xs[:-1] if len(xs) > 1 else xs, op, dtype, None if order is None else [o for o in order if o < len(xs) - 1] or None)
    _patch(mp, "reduce_ranks", f)


def m_reverse_order(mp):
    orig = NUM.reduce_ranks

    def f(xs, op, dtype, order=None):
        order = list(range(len(xs))) if order is None else list(order)
        return orig(xs, op, dtype, order[::-1])
    _patch(mp, "reduce_ranks", f)


def m_wrong_sign(mp):
    def f(acc, v, op, dtype):
        return acc - v if op == 0 else _orig_combine(acc, v, op, dtype)
    _patch(mp, "combine", f)


def m_round_every_step(mp):
    def f(xs, op, dtype, order=None):
        order = list(range(len(xs))) if order is None else list(order)
        acc = xs[order[0]]
        for r in order[1:]:
            acc = _orig_narrow(_orig_combine(_orig_widen(acc, dtype), _orig_widen(xs[r], dtype), op, dtype), dtype)
        return _orig_narrow(_orig_widen(acc, dtype), dtype)
    _patch(mp, "reduce_ranks", f)


def m_max_ties_to_later(mp):
    def f(acc, v, op, dtype):
        if op in (1, 2):
            better = (v >= acc) if op == 1 else (v <= acc)
            return np.where(better, v, acc)
        return _orig_combine(acc, v, op, dtype)
    _patch(mp, "combine", f)


def m_allgather_reversed(mp):
    _patch(mp, "all_gather", lambda xs: [np.concatenate([np.asarray(x) for x in xs[::-1]]) for _ in xs])


def m_reduce_scatter_block_swap(mp):
    orig = C.reduce_scatter
    _patch(mp, "reduce_scatter", lambda xs, op, dtype: orig(xs, op, dtype)[::-1])


def m_gather_first_dim(mp):
    def f(xs, dst_buf, rows=1):
        return np.concatenate([np.asarray(x) for x in xs])
    _patch(mp, "gather", f)


def m_a2a_transposed(mp):
    def f(xs):
        n = len(xs)
        c = xs[0].size // n
        return [np.concatenate([np.asarray(xs[d])[s * c:(s + 1) * c] for s in range(n)]) for d in range(n)]
    _patch(mp, "all_to_all", f)


def m_a2av_displ_transposed(mp):
    orig = C.all_to_all_v
    _patch(mp, "all_to_all_v", lambda send, bufs, sc, sd, rd, row: orig(send, bufs, sc, sd, np.asarray(rd).T, row))


def m_route_token_major(mp):
    orig = M.moe_route

    def f(topk_ids, n_experts):
        sc, sd, rd, pos = orig(topk_ids, n_experts)
        n = len(topk_ids)
        epr = n_experts // n
        new = []
        for s in range(n):
            e = np.asarray(topk_ids[s]).reshape(-1)
            d = e // epr
            p = np.empty_like(pos[s])
            for dd in range(n):
                idx = np.nonzero(d == dd)[0]  # token-major order
                p[idx] = rd[dd, s] + np.arange(idx.size)
            new.append(p)
        return sc, sd, rd, new
    _patch(mp, "moe_route", f)


def m_dedup_route_is_pair_route(mp):
    _patch(mp, "moe_route_dedup", lambda topk_ids, n_experts: M.moe_route(topk_ids, n_experts))


def m_dedup_route_expert_order(mp):
    """Dedup rows, but ordered inside a destination by the token's smallest
    expert there, then token."""
    orig = M.moe_route_dedup

    def f(topk_ids, n_experts):
        sc, sd, rd, pos = orig(topk_ids, n_experts)
        n = len(topk_ids)
        epr = n_experts // n
        new = []
        for s in range(n):
            ids2 = np.asarray(topk_ids[s])
            t_, k_ = ids2.shape
            p = np.empty_like(pos[s])
            for d in range(n):
                reach = [t for t in range(t_) if (ids2[t] // epr == d).any()]
                key = sorted(reach, key=lambda t: (int(ids2[t][ids2[t] // epr == d].min()), t))
                for r, t in enumerate(key):
                    for k in range(k_):
                        if ids2[t, k] // epr == d:
                            p[t * k_ + k] = rd[d, s] + r
            new.append(p)
        return sc, sd, rd, new
    _patch(mp, "moe_route_dedup", f)


def m_combine_f64(mp):
    def f(ys, topk_ids, pos, topk_w, n_experts, hidden, dtype):
        n = len(topk_ids)
        epr = n_experts // n
        outs = []
        for s in range(n):
            ids2 = np.asarray(topk_ids[s])
            t_, k_ = ids2.shape
            acc = np.zeros((t_, hidden))
            for k in range(k_):
                for t in range(t_):
                    d = int(ids2[t, k]) // epr
                    p = int(pos[s][t * k_ + k])
                    acc[t] += float(topk_w[s][t, k]) * _orig_widen(np.asarray(ys[d])[p * hidden:(p + 1) * hidden], dtype)
            outs.append(_orig_narrow(acc.astype(np.float32).reshape(-1), dtype))
        return outs
    _patch(mp, "moe_combine", f)


def m_ll_flag_first(mp):
    orig = PK.pack

    def f(msg, proto, step):
        p = orig(msg, proto, step)
        if proto == PK.LL:
            p = p.view("<u4").reshape(-1, 2)[:, ::-1].copy().view(np.uint8).reshape(-1)
        return p
    _patch(mp, "pack", f)


def m_ll128_flag_at_front(mp):
    orig = PK.pack

    def f(msg, proto, step):
        p = orig(msg, proto, step)
        if proto == PK.LL128:
            p = np.roll(p.reshape(-1, 128), 8, axis=1).reshape(-1)
        return p
    _patch(mp, "pack", f)


def m_unpack_ignores_flags(mp):
    orig = PK.unpack
    _patch(mp, "unpack", lambda packed, nbytes, proto, step: (orig(packed, nbytes, proto, step)[0], 0))


def m_ring_starts_at_owner(mp):
    def f(xs, op, dtype, trace=None):
        n = len(xs)
        count = xs[0].size
        seg = C.segment_elems(count, n, dtype)
        outs = [np.empty_like(np.asarray(xs[0])) for _ in range(n)]
        for c in range(n):
            lo, hi = min(c * seg, count), min((c + 1) * seg, count)
            done = NUM.reduce_ranks([np.asarray(x)[lo:hi] for x in xs], op, dtype, order=[(c + k) % n for k in range(n)])
            for q in range(n):
                outs[q][lo:hi] = done
        return outs
    _patch(mp, "all_reduce_ring", f)


def m_ring_partials_in_storage_type(mp):
    """the ring rounds its partials to the storage type at every hop (a
    bf16 wire type) instead of carrying fp32 to the owner"""
    def f(acc, v, op, dtype):
        r = _orig_combine(acc, v, op, dtype)
        return _orig_widen(_orig_narrow(r, dtype), dtype) if dtype in ("bf16", "fp16") else r
    mp.setattr(C, "combine", f)


def m_ring_wire_without_hop_rounding(mp):
    """the storage-type ring carries fp32 partials after all (rounds once)"""
    _patch(mp, "all_reduce_ring_wire", lambda xs, op, dtype: C.all_reduce_ring(xs, op, dtype))


def m_ring_wire_rank_order(mp):
    """the storage-type ring rounds at every step but adds in rank order 0..N-1"""
    def f(xs, op, dtype):
        n = len(xs)
        acc = np.array(np.asarray(xs[0]), copy=True)
        for r in range(1, n):
            acc = NUM.narrow(NUM.combine(NUM.widen(acc, dtype), NUM.widen(np.asarray(xs[r]), dtype), op, dtype), dtype)
        return [np.array(acc, copy=True) for _ in range(n)]
    _patch(mp, "all_reduce_ring_wire", f)


def m_segment_unaligned(mp):
    _patch(mp, "segment_elems", lambda count, n, dtype: -(-count // n) + 1)


def m_ulp_diff_no_sign_fold(mp):
    """the ulp distance compares magnitudes only (the sign bit dropped)"""
    _patch(mp, "bf16_ulp_diff", lambda a, b: np.abs((np.asarray(a, np.uint16).astype(np.int32) & 0x7FFF)
                                                    - (np.asarray(b, np.uint16).astype(np.int32) & 0x7FFF)))


def m_ulp_diff_raw_bits(mp):
    """the ulp distance subtracts the raw 16-bit patterns"""
    _patch(mp, "bf16_ulp_diff", lambda a, b: np.abs(np.asarray(a, np.uint16).astype(np.int32)
                                                    - np.asarray(b, np.uint16).astype(np.int32)))


MUTANTS = [v for k, v in sorted(globals().items()) if k.startswith("m_")]


@pytest.mark.parametrize("mutant", MUTANTS, ids=lambda f: f.__name__)
def test_some_pin_rejects(mutant, monkeypatch):
    mutant(monkeypatch)
    caught = []
    for pin in P.ALL_PINS:
        try:
            pin()
        except Exception as e:  # AssertionError, or a crash caused by the mutant
            caught.append(pin.__name__)
    assert caught, f"no pin rejects {mutant.__name__}"
