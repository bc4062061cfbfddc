"""Pins for the oracle: each ``pin_*`` raises AssertionError when the oracle
disagrees with something other than itself -- a worked example from the pages
(tests/golden), a library conversion, fp64 / exact-rational brute force, or an
identity the pages state.  ``test_oracle_pins.py`` runs them all;
``test_oracle_mutations.py`` plants mistakes in the oracle and checks that at
least one pin catches each.
"""
from __future__ import annotations

import collections
import fractions
import math
import struct

import numpy as np
import torch

import oracle
import workloads as W
from oracle import numerics as NUM
from conftest import read_golden

SUM, MAX, MIN, PROD = 0, 1, 2, 3


def bf16(vals) -> np.ndarray:
    """Exact float values -> bf16 bits via torch (library conversion)."""
    t = torch.tensor(np.asarray(vals, dtype=np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16).copy()


def bf16_to_float(bits) -> np.ndarray:
    t = torch.from_numpy(np.asarray(bits, dtype=np.uint16).view(np.int16).copy())
    return t.view(torch.bfloat16).to(torch.float64).numpy()


# ------------------------------------------------------------ rounding ----

def pin_bf16_rne_vs_torch():
    # every bf16 upper half combined with the low halves that decide rounding
    hi = np.arange(1 << 16, dtype=np.uint32)
    lows = np.array([0, 1, 0x7FFF, 0x8000, 0x8001, 0xFFFF, 0x4000, 0xC000], dtype=np.uint32)
    u = (hi[:, None] << 16 | lows[None, :]).reshape(-1)
    f = u.view(np.float32)
    got = NUM.f32_to_bf16_bits(f)
    ref = torch.from_numpy(f.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    nan = np.isnan(f)
    assert np.array_equal(got[~nan], ref[~nan]), "bf16 RNE differs from torch"
    assert np.all(got[nan] == 0x7FC0)


def pin_bf16_ulp_diff_brute_force():
    """bf16_ulp_diff against a count of representable values: every finite
    bf16 value, widened by torch to float64, sorted into one ladder (+0 and -0
    are one rung); the distance of two values is how many rungs apart they
    sit.  Random pairs, neighbours, sign flips, and the edges: the zeros, the
    subnormals either side of zero, the largest finite values."""
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    vals = bf16_to_float(bits)
    finite = np.isfinite(vals)
    ladder = np.unique(vals[finite])
    assert ladder.size == 2 * (0x7F80 - 1) + 1  # 0x0001..0x7F7F each side, and one zero

    def rungs(a, b):
        ia = np.searchsorted(ladder, bf16_to_float(a))
        ib = np.searchsorted(ladder, bf16_to_float(b))
        return np.abs(ia - ib)

    fin = bits[finite]
    g = np.random.default_rng(5)
    a = g.choice(fin, 40000)
    b = np.concatenate([g.choice(fin, 20000), a[20000:]])
    near = a[20000:30000].astype(np.int32) + g.integers(-3, 4, 10000)
    near = np.clip(near, 0, 0xFFFF).astype(np.uint16)
    near = np.where(np.isfinite(bf16_to_float(near)), near, a[20000:30000])
    b[20000:30000] = near
    b[30000:] = a[30000:] ^ np.uint16(0x8000)  # the same magnitude, the other sign
    edges = [(0x0000, 0x8000, 0), (0x0000, 0x0001, 1), (0x8000, 0x0001, 1), (0x8001, 0x0001, 2),
             (0x8002, 0x0003, 5), (0x007F, 0x0080, 1), (0x3F7F, 0x3F80, 1), (0x7F7E, 0x7F7F, 1),
             (0xFF7F, 0x7F7F, 2 * 0x7F7F), (0xBF80, 0x3F80, 2 * 0x3F80)]
    ea = np.array([e[0] for e in edges], np.uint16)
    eb = np.array([e[1] for e in edges], np.uint16)
    assert np.array_equal(rungs(ea, eb), [e[2] for e in edges])  # the ladder itself, by hand
    a, b = np.concatenate([a, ea]), np.concatenate([b, eb])
    assert np.array_equal(oracle.bf16_ulp_diff(a, b), rungs(a, b))
    assert np.array_equal(oracle.bf16_ulp_diff(b, a), rungs(a, b))


def pin_bf16_hand_cases():
    one = 1.0
    cases = {
        one: 0x3F80,
        one + 2.0 ** -8: 0x3F80,          # exactly half an ulp above 1: ties to even (1.0)
        one + 3 * 2.0 ** -8: 0x3F82,      # half way between 1+2^-7 (odd) and 1+2^-6 (even)
        one + 2.0 ** -8 + 2.0 ** -20: 0x3F81,  # just above half: rounds up
        -0.0: 0x8000,
        float(np.finfo(np.float32).max): 0x7F80,  # rounds up past the largest bf16 -> inf
        float("inf"): 0x7F80,
        -float("inf"): 0xFF80,
        2.0 ** -133: 0x0001,              # smallest bf16 subnormal
    }
    for x, want in cases.items():
        got = int(NUM.f32_to_bf16_bits(np.array([x], dtype=np.float32))[0])
        assert got == want, (x, hex(got), hex(want))
    assert int(NUM.f32_to_bf16_bits(np.array([np.nan], dtype=np.float32))[0]) == 0x7FC0
    # widening is exact
    b = np.arange(1 << 16, dtype=np.uint16)
    fin = (b & 0x7F80) != 0x7F80
    assert np.array_equal(NUM.bf16_bits_to_f32(b)[fin].astype(np.float64), bf16_to_float(b)[fin])


def pin_fp16_vs_torch():
    g = W.rng(W.W_MISC, 0, salt=11)
    f = np.concatenate([
        g.standard_normal(200000).astype(np.float32) * 1000,
        g.standard_normal(200000).astype(np.float32) * 1e-5,
        np.array([65504, 65520, 65519.99, 1e-8, -0.0, np.inf], dtype=np.float32),
    ])
    got = NUM.f32_to_f16_bits(f)
    ref = torch.from_numpy(f).to(torch.float16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, ref)


# ---------------------------------------------------------- reductions ----

def _random_ranks(n, c, seed, scale_spread=False):
    g = W.rng(W.W_MISC, n, salt=seed)
    vals = g.standard_normal((n, c))
    if scale_spread:
        vals *= 2.0 ** g.integers(-20, 20, size=(n, c))
    return [bf16(vals[r]) for r in range(n)]


def pin_sum_vs_fp64():
    """|oracle - exact| <= 2^-8 * sum|x| per element; equality with the
    correctly rounded exact sum wherever fp32 accumulation was exact."""
    for n in (1, 2, 3, 4, 7, 8):
        for spread in (False, True):
            xs = _random_ranks(n, 4096, 100 + n, spread)
            got = bf16_to_float(oracle.reduce_ranks(xs, SUM, "bf16"))
            vals = np.stack([bf16_to_float(x) for x in xs])
            exact = vals.sum(axis=0)  # fp64, exact for these magnitudes
            tol = 2.0 ** -8 * np.abs(vals).sum(axis=0)
            assert np.all(np.abs(got - exact) <= tol + 1e-300), n
            f32 = np.zeros(vals.shape[1], dtype=np.float32) + vals[0].astype(np.float32)
            for r in range(1, n):
                f32 = (f32 + vals[r].astype(np.float32)).astype(np.float32)
            ok = f32.astype(np.float64) == exact
            ref = bf16(exact.astype(np.float32))
            assert np.array_equal(oracle.reduce_ranks(xs, SUM, "bf16")[ok], ref[ok])


def pin_sum_order_and_single_rounding():
    # fp32 storage: 1 + 2^-24 rounds back to 1 (tie to even) twice in rank order
    xs = [np.array([1.0], np.float32), np.array([2.0 ** -24], np.float32), np.array([2.0 ** -24], np.float32)]
    assert float(oracle.reduce_ranks(xs, SUM, "fp32")[0]) == 1.0
    # ... and 1 + 2^-23 in the rotated order 1, 2, 0 (exact, no tie)
    assert float(oracle.reduce_ranks(xs, SUM, "fp32", order=[1, 2, 0])[0]) == 1.0 + 2.0 ** -23
    # bf16: fp32 accumulation then one rounding: 1 + 3*2^-8 -> tie -> 1 + 2^-6.
    xs = [bf16([1.0]), bf16([2.0 ** -8]), bf16([2.0 ** -8]), bf16([2.0 ** -8])]
    assert int(oracle.reduce_ranks(xs, SUM, "bf16")[0]) == 0x3F82
    # -0 is kept when every input is -0; one +0 makes it +0
    assert int(oracle.reduce_ranks([bf16([-0.0])] * 3, SUM, "bf16")[0]) == 0x8000
    assert int(oracle.reduce_ranks([bf16([-0.0]), bf16([0.0])], SUM, "bf16")[0]) == 0x0000
    # overflow to inf, inf - inf = NaN (canonical)
    big = bf16([3.0e38])
    assert int(oracle.reduce_ranks([big, big], SUM, "bf16")[0]) == 0x7F80
    inf, ninf = bf16([np.inf]), bf16([-np.inf])
    assert int(oracle.reduce_ranks([inf, ninf], SUM, "bf16")[0]) == 0x7FC0
    # fp32 storage: every NaN result is the canonical quiet NaN 0x7FC00000
    f_inf, f_ninf = np.array([np.inf], np.float32), np.array([-np.inf], np.float32)
    assert int(oracle.reduce_ranks([f_inf, f_ninf], SUM, "fp32").view(np.uint32)[0]) == 0x7FC00000
    neg_nan = np.array([0xFFC12345], np.uint32).view(np.float32)
    assert int(oracle.reduce_ranks([neg_nan, f_inf], MAX, "fp32").view(np.uint32)[0]) == 0x7FC00000


def pin_maxmin():
    xs = _random_ranks(5, 3000, 7)
    vals = np.stack([bf16_to_float(x) for x in xs])
    assert np.array_equal(bf16_to_float(oracle.reduce_ranks(xs, MAX, "bf16")), vals.max(axis=0))
    assert np.array_equal(bf16_to_float(oracle.reduce_ranks(xs, MIN, "bf16")), vals.min(axis=0))
    # ties between -0 and +0: the earlier rank wins
    pz, nz = bf16([0.0]), bf16([-0.0])
    assert int(oracle.reduce_ranks([nz, pz], MAX, "bf16")[0]) == 0x8000
    assert int(oracle.reduce_ranks([pz, nz], MAX, "bf16")[0]) == 0x0000
    assert int(oracle.reduce_ranks([pz, nz], MIN, "bf16")[0]) == 0x0000
    # NaN propagates wherever it sits
    nan = np.array([0x7FC1], dtype=np.uint16)
    for pos in range(3):
        xs3 = [bf16([1.0]), bf16([5.0]), bf16([2.0])]
        xs3[pos] = nan
        assert int(oracle.reduce_ranks(xs3, MAX, "bf16")[0]) == 0x7FC0
        assert int(oracle.reduce_ranks(xs3, MIN, "bf16")[0]) == 0x7FC0
    # int32 exact
    g = W.rng(W.W_MISC, 3, salt=5)
    ints = [g.integers(-2 ** 31, 2 ** 31, 1000, dtype=np.int64).astype(np.int32) for _ in range(4)]
    assert np.array_equal(oracle.reduce_ranks(ints, MAX, "int32"), np.max(np.stack(ints), axis=0))
    assert np.array_equal(oracle.reduce_ranks(ints, MIN, "int32"), np.min(np.stack(ints), axis=0))


def pin_prod_and_int32_wrap():
    g = W.rng(W.W_MISC, 4, salt=9)
    xs = [bf16(g.uniform(0.5, 2.0, 2000)) for _ in range(6)]
    got = bf16_to_float(oracle.reduce_ranks(xs, PROD, "bf16"))
    exact = np.prod(np.stack([bf16_to_float(x) for x in xs]), axis=0)
    assert np.all(np.abs(got - exact) <= 2.0 ** -8 * np.abs(exact) * (1 + 6 * 2.0 ** -23))
    ints = [g.integers(-2 ** 31, 2 ** 31, 500, dtype=np.int64).astype(np.int32) for _ in range(5)]
    s = [0] * 500
    p = [1] * 500
    for x in ints:
        for i, v in enumerate(x.tolist()):
            s[i] = (s[i] + v) % (1 << 32)
            p[i] = (p[i] * v) % (1 << 32)
    to_i32 = lambda a: np.array([v - (1 << 32) if v >= (1 << 31) else v for v in a], dtype=np.int64)
    assert np.array_equal(oracle.reduce_ranks(ints, SUM, "int32").astype(np.int64), to_i32(s))
    assert np.array_equal(oracle.reduce_ranks(ints, PROD, "int32").astype(np.int64), to_i32(p))


# ------------------------------------------------------ worked examples ----

def _symbols(tokens, table):
    return np.array([table[t] for t in tokens], dtype=np.int32)


def pin_golden_allgather():
    gd = read_golden("allgather_tutorial_7_3.txt")
    n = int(gd["ranks"][0])
    syms = sorted({t for k in gd for v in gd[k] for t in v.split() if t.startswith("t")})
    table = {s: 1000 + i for i, s in enumerate(syms)}
    ins = {int(v.split()[0]): v.split()[1:] for v in [f"{i} {x}" for i, x in enumerate(gd["in 0"] + gd["in 1"])]}
    xs = [_symbols(gd[f"in {r}"][0].split(), table) for r in range(n)]
    outs = oracle.all_gather(xs)
    for r in range(n):
        assert np.array_equal(outs[r], _symbols(gd[f"out {r}"][0].split(), table))
    del ins


def _bind_sum_example(gd, seed):
    n = int(gd["ranks"][0])
    g = W.rng(W.W_MISC, 50, salt=seed)
    ins = [gd[f"in {r}"][0].split() for r in range(n)]
    val = {}
    for toks in ins:
        for t in toks:
            val[t] = float(g.integers(-64, 64))  # small integers: every sum is exact in bf16
    for line in gd["sum"]:
        lhs, rhs = [p.strip() for p in line.split("=")]
        val[lhs] = sum(val[t.strip()] for t in rhs.split("+"))
    xs = [bf16([val[t] for t in toks]) for toks in ins]
    return n, val, xs


def pin_golden_reduce_scatter():
    gd = read_golden("reduce_scatter_tutorial_5_3.txt")
    n, val, xs = _bind_sum_example(gd, 1)
    outs = oracle.reduce_scatter(xs, SUM, "bf16")
    for r in range(n):
        want = bf16([val[t] for t in gd[f"out {r}"][0].split()])
        assert np.array_equal(outs[r], want), (r, outs[r], want)


def pin_golden_all_reduce():
    gd = read_golden("allreduce_tutorial_6_3.txt")
    n, val, xs = _bind_sum_example(gd, 2)
    for fn in (oracle.all_reduce, oracle.all_reduce_two_shot, oracle.all_reduce_one_shot, oracle.all_reduce_ring):
        outs = fn(xs, SUM, "bf16")
        for r in range(n):
            want = bf16([val[t] for t in gd[f"out {r}"][0].split()])
            assert np.array_equal(outs[r], want), fn.__name__


def pin_golden_all_to_all():
    gd = read_golden("all_to_all_tutorial_8_1.txt")
    n = int(gd["ranks"][0])
    table = {f"{s}>{d}": 100 * s + d + 1 for s in range(n) for d in range(n)}
    xs = [_symbols(gd[f"in {r}"][0].split(), table) for r in range(n)]
    outs = oracle.all_to_all(xs)
    for d in range(n):
        assert np.array_equal(outs[d], _symbols(gd[f"out {d}"][0].split(), table))
    # the same exchange through all_to_all_v with unit splits
    cnt = np.ones((n, n), dtype=np.int64)
    sd = np.tile(np.arange(n), (n, 1))
    outs_v = oracle.all_to_all_v(xs, [np.zeros(n, np.int32)] * n, cnt, sd, sd, 1)
    for d in range(n):
        assert np.array_equal(outs_v[d], outs[d])


def pin_golden_moe():
    gd = read_golden("moe_tutorial_8_4.txt")
    n, e = int(gd["ranks"][0]), int(gd["experts"][0])
    names, topk = [], []
    for r in range(n):
        pairs = [p.split(":") for p in gd[f"route {r}"][0].split()]
        names.append([p[0] for p in pairs])
        topk.append(np.array([[int(p[1])] for p in pairs], dtype=np.int32))
    table = {nm: 10 * (i + 1) for i, nm in enumerate(sorted(sum(names, [])))}
    hidden = 3
    xs = [bf16(np.repeat([table[nm] for nm in names[r]], hidden).astype(float)) for r in range(n)]
    sc, sd, rd, pos = oracle.moe_route(topk, e)
    recv = [np.zeros(int(sc[:, d].sum()) * hidden, np.uint16) for d in range(n)]
    recv = oracle.moe_dispatch(xs, topk, pos, recv, e, hidden)
    for d in range(n):
        want = bf16(np.repeat([table[nm] for nm in gd[f"recv {d}"][0].split()], hidden).astype(float))
        assert np.array_equal(recv[d], want), (d, recv[d], want)
    # combine with weight 1 returns every token to its owner unchanged
    w = [np.ones((len(names[r]), 1), np.float32) for r in range(n)]
    back = oracle.moe_combine(recv, topk, pos, w, e, hidden, "bf16")
    for r in range(n):
        assert np.array_equal(back[r], xs[r])


def pin_golden_two_shot_segments():
    gd = read_golden("twoshot_ringll_160k.txt")
    n = int(gd["ranks"][0])
    count = int(gd["bytes"][0]) // 2
    xs = W.twoshot_160k(n, count)
    trace = []
    outs = oracle.all_reduce_two_shot(xs, SUM, "bf16", trace=trace)
    want = []
    for line in gd["segment A"] + gd["segment B"] + gd["segment C"] + gd["segment D"]:
        f = line.split()
        want.append((int(f[1]), int(f[3]), int(f[4])))
    assert sorted(trace) == sorted(want), (trace, want)
    ref = oracle.all_reduce(xs, SUM, "bf16")
    for q in range(n):
        assert np.array_equal(outs[q], ref[q])


# ----------------------------------------------------------- invariants ----

def pin_movement_identities():
    for n in (1, 2, 3, 8):
        c = 37
        xs = [W.ranks_values(W.W_MISC, n, c, "int32")[r] + r for r in range(n)]
        # broadcast: every rank equals the root, bit for bit
        for src in range(n):
            outs = oracle.broadcast(xs, src)
            assert all(np.array_equal(o, xs[src]) for o in outs)
        # gather(scatter(x)) == x ; all_gather on every rank == gather on dst
        full = np.concatenate(xs)
        sc = oracle.scatter(full, n)
        assert np.array_equal(oracle.gather(sc, np.zeros_like(full)), full)
        ag = oracle.all_gather(xs)
        for q in range(n):
            assert np.array_equal(ag[q], oracle.gather(xs, np.zeros_like(full)))
        # brute force, element by element
        for q in range(n):
            for r in range(n):
                for i in range(c):
                    assert ag[q][r * c + i] == xs[r][i]
        # last-dimension gather: out[row, r*cols + j] = in[r][row, j]
        rows, cols = 3, 5
        ys = [np.arange(rows * cols, dtype=np.int32) + 100 * r for r in range(n)]
        got = oracle.gather(ys, np.zeros(n * rows * cols, np.int32), rows=rows).reshape(rows, n * cols)
        for r in range(n):
            for row in range(rows):
                for j in range(cols):
                    assert got[row, r * cols + j] == ys[r][row * cols + j]


def pin_reduction_identities():
    for n in (2, 3, 4, 8):
        c = 8 * n * 5 + 3 * 8 * n  # divisible by n
        xs = _random_ranks(n, c, 200 + n)
        ar = oracle.all_reduce(xs, SUM, "bf16")
        rs = oracle.reduce_scatter(xs, SUM, "bf16")
        ag = oracle.all_gather(rs)
        one = oracle.all_reduce_one_shot(xs, SUM, "bf16")
        two = oracle.all_reduce_two_shot(xs, SUM, "bf16")
        for q in range(n):
            assert np.array_equal(ar[q], ag[q])  # AllReduce == ReduceScatter + AllGather (tutorial 6.1)
            assert np.array_equal(ar[q], one[q]) and np.array_equal(ar[q], two[q])
        for dst in range(n):
            assert np.array_equal(oracle.reduce(xs, SUM, "bf16"), ar[dst])  # Reduce == AllReduce on dst
        ring = oracle.all_reduce_ring(xs, SUM, "bf16")
        for q in range(n):
            assert int(oracle.bf16_ulp_diff(ring[q], ar[q]).max()) <= 1


def pin_ring_schedule():
    n = 5
    xs = _random_ranks(n, 83, 9)
    trace = []
    oracle.all_reduce_ring(xs, SUM, "bf16", trace=trace)
    rs = [t for t in trace if t[0] == "rs"]
    ag = [t for t in trace if t[0] == "ag"]
    assert len(rs) == n * (n - 1) and len(ag) == n * (n - 1)  # 2(N-1) steps of N transfers
    for _, k, c, frm, to in rs:
        assert to == (frm + 1) % n  # ring neighbour
    for c in range(n):
        visited = [(c + 1) % n] + [t[4] for t in rs if t[2] == c]
        assert sorted(visited) == list(range(n)) and visited[-1] == c  # every rank once, complete on c
    # every (step, rank) sends exactly one chunk
    for k in range(1, n):
        assert sorted(t[3] for t in rs if t[1] == k) == list(range(n))
    # the ring's accumulation order is visible in fp32: chunk c sums c+1, ..., c
    vals = [np.array([1.0, 2.0 ** -24, 2.0 ** -24, 0.0, 0.0], np.float32)[[r]] for r in range(n)]
    # N=5, count 1: only chunk 0 holds data; order 1,2,3,4,0: 2^-24 + 2^-24 + 0 + 0 + 1 = 1 + 2^-23
    out = oracle.all_reduce_ring(vals, SUM, "fp32")
    assert float(out[0][0]) == 1.0 + 2.0 ** -23
    assert float(oracle.all_reduce(vals, SUM, "fp32")[0][0]) == 1.0


def pin_ring_wire_hand_example():
    """The per-hop-rounding ring on one bf16 element, worked by hand.  With 3
    ranks and 1 element only chunk 0 holds data, accumulated in the ring
    order: rank 1's value, then rank 2's, then rank 0's.  bf16 keeps 8
    significant bits, so next to 1 the spacing is 2^-7 and 1 + 2^-8 is a tie
    that rounds to even, to 1.  With t = 2^-8, ranks (x0, x1, x2):
      (t, 1, t): 1 + t -> 1, then 1 + t -> 1; the fp32-partial ring keeps
                 1 + 2t = 1 + 2^-7 exactly and rounds once to it;
      (t, t, 1): t + 1 -> 1, then 1 + t -> 1 (rank order would give
                 t + t = 2^-7 exactly, then 1 + 2^-7);
      (1, t, t): t + t = 2^-7 exactly, then 2^-7 + 1 = 1 + 2^-7, which bf16
                 holds: both rings agree."""
    t = 2.0 ** -8
    cases = [((t, 1.0, t), 1.0, 1.0 + 2.0 ** -7),   # x0, x1, x2 -> wire, fp32 ring
             ((t, t, 1.0), 1.0, 1.0 + 2.0 ** -7),
             ((1.0, t, t), 1.0 + 2.0 ** -7, 1.0 + 2.0 ** -7)]
    for vals, want_wire, want_ring in cases:
        xs = [bf16([v]) for v in vals]
        wire = oracle.all_reduce_ring_wire(xs, SUM, "bf16")
        ring = oracle.all_reduce_ring(xs, SUM, "bf16")
        for q in range(3):
            assert float(bf16_to_float(wire[q])[0]) == want_wire, (vals, q)
            assert float(bf16_to_float(ring[q])[0]) == want_ring, (vals, q)


def _bf16_rne_fraction(q: fractions.Fraction) -> fractions.Fraction:
    """A rational rounded to the nearest bf16 value, ties to even (finite,
    normal range), from the definition: 8 significant bits."""
    if q == 0:
        return fractions.Fraction(0)
    sign = -1 if q < 0 else 1
    a = abs(q)
    e = math.floor(math.log2(a))
    if fractions.Fraction(2) ** e > a:
        e -= 1
    elif fractions.Fraction(2) ** (e + 1) <= a:
        e += 1
    ulp = fractions.Fraction(2) ** (e - 7)
    m = a / ulp  # in [128, 256)
    lo = math.floor(m)
    rem = m - lo
    if rem > fractions.Fraction(1, 2) or (rem == fractions.Fraction(1, 2) and lo % 2 == 1):
        lo += 1
    return sign * lo * ulp


def pin_ring_wire_exact_rational():
    """Random bf16 inputs on 2..8 ranks: every element equals the chunk's
    ring-order sum with a round to bf16 after every addition, computed in
    exact rationals (no float arithmetic in the reference)."""
    g = W.rng(W.W_MISC, 11, salt=3)
    for n in range(2, 9):
        count = 40
        xs = [bf16(g.uniform(-4, 4, count).astype(np.float32)) for _ in range(n)]
        got = oracle.all_reduce_ring_wire(xs, SUM, "bf16")
        seg = oracle.segment_elems(count, n, "bf16")
        vals = [[fractions.Fraction(float(v)) for v in bf16_to_float(x)] for x in xs]
        for e in range(count):
            c = e // seg
            acc = vals[(c + 1) % n][e]
            for k in range(1, n):
                acc = _bf16_rne_fraction(acc + vals[(c + 1 + k) % n][e])
            for q in range(n):
                assert fractions.Fraction(float(bf16_to_float(got[q][e:e + 1])[0])) == acc, (n, e, q)


def pin_ring_wire_reduces_to_ring():
    """Where rounding to the storage type changes nothing the two rings
    agree bit for bit: fp32 and int32 (storage = arithmetic type), MAX / MIN
    (the winner's own bits), and 2 ranks (one addition, one rounding)."""
    for dtype in ("fp32", "int32"):
        for op in (SUM, PROD, MAX, MIN):
            for n in (2, 3, 5, 8):
                if dtype == "int32":
                    g = W.rng(W.W_MISC, 12, salt=n + 10 * op)
                    xs = [g.integers(-1000, 1000, 333, dtype=np.int64).astype(np.int32) for _ in range(n)]
                else:
                    xs = W.ranks_values(W.W_MISC, n, 333, dtype, "uniform" if op == PROD else "normal", salt=n + op)
                a = oracle.all_reduce_ring_wire(xs, op, dtype)
                b = oracle.all_reduce_ring(xs, op, dtype)
                for q in range(n):
                    assert np.array_equal(np.asarray(a[q]).view(np.uint32), np.asarray(b[q]).view(np.uint32))
    for dtype in ("bf16", "fp16"):
        for op in (MAX, MIN):
            xs = W.ranks_values(W.W_MISC, 6, 1001, dtype, "normal", salt=op)
            assert all(np.array_equal(a, b) for a, b in zip(oracle.all_reduce_ring_wire(xs, op, dtype),
                                                            oracle.all_reduce_ring(xs, op, dtype)))
        for op in (SUM, PROD):
            xs = W.ranks_values(W.W_MISC, 2, 1001, dtype, "uniform", salt=op + 7)
            assert all(np.array_equal(a, b) for a, b in zip(oracle.all_reduce_ring_wire(xs, op, dtype),
                                                            oracle.all_reduce_ring(xs, op, dtype)))


def pin_all_to_all_v_roundtrip():
    for n in (1, 2, 5, 8):
        row = 3
        sc = W.random_splits(n, 6, salt=n)
        sd = np.zeros_like(sc)
        sd[:, 1:] = np.cumsum(sc, axis=1)[:, :-1]
        rc = sc.T.copy()  # recv_counts[d][s]
        rd = np.zeros_like(rc)
        rd[:, 1:] = np.cumsum(rc, axis=1)[:, :-1]
        g = W.rng(W.W_MISC, n, salt=77)
        xs = [g.integers(0, 1 << 30, int(sc[s].sum()) * row).astype(np.int32) for s in range(n)]
        bufs = [np.full(int(rc[d].sum()) * row, -1, np.int32) for d in range(n)]
        out = oracle.all_to_all_v(xs, bufs, sc, sd, rd, row)
        # brute force element by element
        for s in range(n):
            for d in range(n):
                for j in range(int(sc[s, d]) * row):
                    assert out[d][rd[d, s] * row + j] == xs[s][sd[s, d] * row + j]
        # transposed splits send everything home
        back = oracle.all_to_all_v(out, [np.zeros_like(x) for x in xs], rc, rd, sd, row)
        for s in range(n):
            assert np.array_equal(back[s], xs[s])
    # world size 1 is a copy
    x = np.arange(10, dtype=np.int32)
    assert np.array_equal(oracle.all_to_all([x])[0], x)


# ------------------------------------------------------------------ MoE ----

def pin_moe_route_counts_and_layout():
    n, t, k, e = 4, 64, 4, 16
    ids, ws = W.moe_routing(t, e, k, n)
    sc, sd, rd, pos = oracle.moe_route(ids, e)
    assert sc.sum() == n * t * k
    epr = e // n
    for s in range(n):
        cnt = collections.Counter(int(v) // epr for v in ids[s].reshape(-1))
        for d in range(n):
            assert sc[s, d] == cnt.get(d, 0)
    # positions: a bijection onto each destination's rows, blocks by source
    for d in range(n):
        got = []
        for s in range(n):
            mask = (ids[s].reshape(-1) // epr) == d
            p = pos[s][mask]
            assert p.size == sc[s, d]
            if p.size:
                assert p.min() == rd[d, s] and p.max() == rd[d, s] + sc[s, d] - 1
            got.extend(p.tolist())
        assert sorted(got) == list(range(int(sc[:, d].sum())))
    # order within a (source, destination) block: expert ascending, then token
    for s in range(n):
        flat = ids[s].reshape(-1)
        keyed = sorted(range(flat.size), key=lambda j: (int(flat[j]), j // k))
        p_sorted = [int(pos[s][j]) for j in keyed]
        for d in range(n):
            seq = [p for j, p in zip(keyed, p_sorted) if int(flat[j]) // epr == d]
            assert seq == sorted(seq) and (not seq or seq == list(range(seq[0], seq[0] + len(seq))))


def pin_moe_route_dedup_hand_example():
    """Two ranks, experts 0,1 on rank 0 and 2,3 on rank 1 (the tutorial's
    placement), three tokens, top-2; worked by hand."""
    ids = [np.array([[0, 1], [2, 0], [3, 2]], np.int32),   # rank 0: t0 -> {0}, t1 -> {1, 0}, t2 -> {1}
           np.array([[1, 3], [0, 1], [2, 3]], np.int32)]   # rank 1: t0 -> {0, 1}, t1 -> {0}, t2 -> {1}
    sc, sd, rd, pos = oracle.moe_route_dedup(ids, 4)
    assert sc.tolist() == [[2, 2], [2, 2]]
    assert sd.tolist() == [[0, 2], [0, 2]]
    assert rd.tolist() == [[0, 2], [0, 2]]
    assert pos[0].tolist() == [0, 0, 0, 1, 1, 1]
    assert pos[1].tolist() == [2, 2, 3, 3, 3, 3]


def pin_moe_route_dedup_layout():
    n, t, k, e = 4, 64, 4, 16
    ids, _ = W.moe_routing(t, e, k, n)
    sc, sd, rd, pos = oracle.moe_route_dedup(ids, e)
    epr = e // n
    for d in range(n):
        got = []
        for s in range(n):
            d2 = ids[s] // epr
            reach = [tt for tt in range(t) if (d2[tt] == d).any()]
            assert sc[s, d] == len(reach)
            rows = [int(pos[s][tt * k + kk]) for tt in reach for kk in range(k) if d2[tt, kk] == d]
            per_tok = [{int(pos[s][tt * k + kk]) for kk in range(k) if d2[tt, kk] == d} for tt in reach]
            assert all(len(v) == 1 for v in per_tok)  # one row per (token, destination)
            firsts = [min(v) for v in per_tok]
            assert firsts == list(range(rd[d, s], rd[d, s] + len(reach)))  # token order, source block
            got.extend(firsts)
            assert set(rows) == set(firsts)
        assert sorted(got) == list(range(int(sc[:, d].sum())))
    # fewer rows than (token, expert) pairs whenever two experts of a token share a rank
    assert sc.sum() < n * t * k


def pin_moe_route_dedup_reduces_to_route():
    """With one expert per rank no token reaches a rank twice, and the two
    routes (expert order inside a destination = token order) coincide."""
    n, t, k = 8, 40, 3
    ids, _ = W.moe_routing(t, n, k, n)
    a = oracle.moe_route(ids, n)
    b = oracle.moe_route_dedup(ids, n)
    for x, y in zip(a[:3], b[:3]):
        assert np.array_equal(x, y)
    for s in range(n):
        assert np.array_equal(a[3][s], b[3][s])


def pin_moe_dedup_combine_equals_route_combine():
    """Identity expert: dispatch then combine gives the same bits with either
    route, since every choice reads a copy of its own token's row."""
    n, t, k, e, h = 4, 24, 4, 16, 8
    ids, ws = W.moe_routing(t, e, k, n)
    xs = [W.ranks_values(W.W_MISC, n, t * h, "bf16", salt=9)[r] for r in range(n)]
    outs = []
    for route in (oracle.moe_route, oracle.moe_route_dedup):
        sc, sd, rd, pos = route(ids, e)
        bufs = [np.zeros(int(sc[:, d].sum()) * h, np.uint16) for d in range(n)]
        ys = oracle.moe_dispatch(xs, ids, pos, bufs, e, h)
        outs.append(oracle.moe_combine(ys, ids, pos, ws, e, h, "bf16"))
    for s in range(n):
        assert np.array_equal(outs[0][s], outs[1][s])


def pin_moe_dispatch_is_permute_then_all_to_all_v():
    n, t, k, e, h = 4, 48, 4, 16, 8
    ids, ws = W.moe_routing(t, e, k, n)
    xs = [W.ranks_values(W.W_MISC, n, t * h, "bf16", salt=3)[r] for r in range(n)]
    sc, sd, rd, pos = oracle.moe_route(ids, e)
    bufs = [np.zeros(int(sc[:, d].sum()) * h, np.uint16) for d in range(n)]
    direct = oracle.moe_dispatch(xs, ids, pos, bufs, e, h)
    send = oracle.moe_permute_send(xs, ids, e, h)
    via = oracle.all_to_all_v(send, bufs, sc, sd, rd, h)
    for d in range(n):
        assert np.array_equal(direct[d], via[d])


def _fl32(q: fractions.Fraction) -> fractions.Fraction:
    """Round an exact rational to the nearest binary32 (ties to even)."""
    if q == 0:
        return fractions.Fraction(0)
    x = float(q)  # correctly rounded to binary64 by Python
    f = struct.unpack("<f", struct.pack("<f", x))[0]
    # fix double rounding: compare distances exactly
    cands = {f, float(np.nextafter(np.float32(f), np.float32(np.inf))), float(np.nextafter(np.float32(f), np.float32(-np.inf)))}
    best = min(cands, key=lambda c: (abs(fractions.Fraction(c) - q),
                                     struct.unpack("<I", struct.pack("<f", c))[0] & 1))
    return fractions.Fraction(best)


def pin_moe_combine_exact_rational():
    n, t, k, e, h = 2, 6, 3, 8, 4
    ids, ws = W.moe_routing(t, e, k, n)
    xs = [W.ranks_values(W.W_MISC, n, t * h, "bf16", salt=4)[r] for r in range(n)]
    sc, sd, rd, pos = oracle.moe_route(ids, e)
    bufs = [np.zeros(int(sc[:, d].sum()) * h, np.uint16) for d in range(n)]
    ys = oracle.moe_dispatch(xs, ids, pos, bufs, e, h)
    got = oracle.moe_combine(ys, ids, pos, ws, e, h, "bf16")
    for s in range(n):
        xv = bf16_to_float(xs[s]).reshape(t, h)
        for tt in range(t):
            for j in range(h):
                acc = None
                for kk in range(k):
                    prod = _fl32(fractions.Fraction(float(ws[s][tt, kk])) * fractions.Fraction(xv[tt, j]))
                    acc = prod if acc is None else _fl32(acc + prod)
                want = int(bf16([float(acc)])[0])
                assert int(got[s][tt * h + j]) == want
        # identity expert + renormalised weights: back to x within 2 ulps
        assert int(oracle.bf16_ulp_diff(got[s], xs[s]).max()) <= 2
    # Hand-derived cases (one rank, one token, hidden 1, experts 0..3 on rank 0).
    one_tok = [np.array([[0, 1, 2]], np.int32)]
    pos1 = [np.array([0, 1, 2])]
    # (a) fp32 after every step: (1+2^-8) + 2^-24 is a binary32 tie -> stays
    #     1+2^-8, twice; 1+2^-8 is a bf16 tie -> even -> 1.0 (0x3F80).  Summing
    #     in float64 would give 1+2^-8+2^-23 -> 0x3F81.
    w = [np.array([[1 + 2.0 ** -8, 2.0 ** -24, 2.0 ** -24]], np.float32)]
    y = [bf16([1.0, 1.0, 1.0])]
    assert int(oracle.moe_combine(y, one_tok, pos1, w, 4, 1, "bf16")[0][0]) == 0x3F80
    # (b) products rounded before the add (no fused multiply-add):
    #     w1*y1 = (1+2^-23)(1+2^-7) = 1+2^-7+2^-23+2^-30 -> fl32 drops 2^-30, so
    #     -(1+2^-7+2^-23) + fl32(w1*y1) = 0 exactly (a fused add would leave 2^-30).
    two_tok = [np.array([[0, 1]], np.int32)]
    w = [np.array([[-(1 + 2.0 ** -7 + 2.0 ** -23), 1 + 2.0 ** -23]], np.float32)]
    y = [bf16([1.0, 1 + 2.0 ** -7])]
    assert int(oracle.moe_combine(y, two_tok, [np.array([0, 1])], w, 4, 1, "bf16")[0][0]) == 0x0000


# -------------------------------------------------------------- packets ----

def _hexbytes(s):
    return np.array([int(b, 16) for b in s.split()], dtype=np.uint8)


def pin_golden_ll_layout():
    gd = read_golden("ll_line_layout.txt")
    msg = _hexbytes(gd["message"][0])
    step = int(gd["step"][0], 0)
    packed = oracle.pack(msg, oracle.LL, step)
    assert np.array_equal(packed, _hexbytes(gd["packed"][0]))
    data, bad = oracle.unpack(packed, msg.size, oracle.LL, step)
    assert np.array_equal(data, msg) and bad == 0
    gd = read_golden("ll128_line_layout.txt")
    step = int(gd["step"][0], 0)
    m = int(gd["message_len"][0])
    msg = (np.arange(m) % 251 + 1).astype(np.uint8)
    packed = oracle.pack(msg, oracle.LL128, step).reshape(-1, 128)
    flag = _hexbytes(gd["line 0 flag"][0])
    assert packed.shape == (2, 128)
    assert np.array_equal(packed[0, :120], msg[:120]) and np.array_equal(packed[0, 120:], flag)
    assert np.array_equal(packed[1, :5], msg[120:]) and not packed[1, 5:120].any()
    assert np.array_equal(packed[1, 120:], _hexbytes(gd["line 1 flag"][0]))


def pin_packet_roundtrip_and_flags():
    g = W.rng(W.W_MISC, 1, salt=21)
    for proto in (oracle.LL, oracle.LL128):
        for nbytes in (0, 1, 3, 4, 5, 8, 119, 120, 121, 239, 240, 1000, 4097):
            msg = g.integers(0, 256, nbytes).astype(np.uint8)
            step = int(g.integers(1, 1 << 31))
            p = oracle.pack(msg, proto, step)
            assert p.size == oracle.packed_bytes(nbytes, proto)
            assert p.size == (8 * math.ceil(nbytes / 4) if proto == oracle.LL else 128 * math.ceil(nbytes / 120))
            back, bad = oracle.unpack(p, nbytes, proto, step)
            assert bad == 0 and np.array_equal(back, msg)
            # every line's flag is the step
            if proto == oracle.LL:
                assert np.all(p.view("<u4").reshape(-1, 2)[:, 1] == step)
            else:
                assert np.all(np.ascontiguousarray(p.reshape(-1, 128)[:, 120:]).view("<u8") == step)
            # a wrong step fails every line; corrupting k lines counts k
            nl = p.size // (8 if proto == oracle.LL else 128)
            assert oracle.unpack(p, nbytes, proto, step + 1)[1] == nl
            if nl:
                q = p.copy()
                lines = sorted(set(g.integers(0, nl, 3).tolist()))
                for L in lines:
                    off = 8 * L + 4 if proto == oracle.LL else 128 * L + 120
                    q[off] ^= 0x5A
                assert oracle.unpack(q, nbytes, proto, step)[1] == len(lines)


def pin_packed_all_reduce():
    n = 4
    for proto in (oracle.LL, oracle.LL128):
        for count in (1, 2, 59, 60, 61, 600):
            xs = W.ranks_values(W.W_MISC, n, count, "bf16", "uniform", salt=count)
            step = 5
            packed = [oracle.pack(x, proto, step) for x in xs]
            outs, bad = oracle.all_reduce_packed(packed, count, "bf16", SUM, proto, step)
            assert bad == 0
            ref = oracle.all_reduce(xs, SUM, "bf16")
            for q in range(n):
                data, b = oracle.unpack(outs[q], count * 2, proto, step)
                assert b == 0 and np.array_equal(data.view(np.uint16), ref[q])


ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]
