"""Randomized properties of the oracle (CPU only), checked with hypothesis.

Each property is an identity that holds whatever the inputs, stated without
the oracle's own arithmetic:

* the owner segments of the two-shot scheme cannot change a per-element
  result, so the two-shot equals the rank-order reduction bit for bit, and a
  reduce-scatter's blocks laid end to end equal the reduce;
* the ring's rotated order can change a floating-point sum only by rounding,
  but integer sums (mod 2^32) and MAX / MIN of distinct finite values are
  order-free, so there the ring equals the rank-order reduction exactly;
* where every fp32 partial is exact, the bf16 ring sum is the exact sum
  rounded once (to nearest even, as torch rounds it), whatever the order;
  elsewhere its error stays within 2^-8 (half a bf16 ulp, relative) of the
  sum of the magnitudes, plus the fp32 partials' own error;
* movement composes: gather then scatter returns every rank's block, and an
  all-to-all-v followed by the transposed one returns every rank's rows;
* unpack(pack(message)) is the message with no flag mismatch, for LL and LL128;
* with an identity expert, the deduplicated MoE route combines to the same
  bits as the per-(token, expert) route.
"""
import numpy as np
import torch
from hypothesis import given, settings, strategies as st

import oracle
import workloads as W

SET = settings(max_examples=25, deadline=None, derandomize=True)


def values(g, n, count, dtype, op):
    if dtype == "int32":
        return [g.integers(-2**31, 2**31, count, dtype=np.int64).astype(np.int32) for _ in range(n)]
    f = g.uniform(-1, 1, (n, count)) if op == 3 else g.standard_normal((n, count)) * 4
    out = []
    for r in range(n):
        if dtype == "fp32":
            out.append(f[r].astype(np.float32))
        else:
            out.append(oracle.narrow(f[r].astype(np.float32), dtype))
    return out


def bits(a):
    a = np.asarray(a)
    return a.view(np.uint32) if a.dtype == np.float32 else a


@SET
@given(n=st.integers(1, 9), count=st.integers(1, 400), dtype=st.sampled_from(["bf16", "fp16", "fp32", "int32"]),
       op=st.integers(0, 3), seed=st.integers(0, 10**6))
def test_two_shot_equals_rank_order(n, count, dtype, op, seed):
    xs = values(np.random.default_rng(seed), n, count, dtype, op)
    ref = oracle.all_reduce(xs, op, dtype)
    for q, y in enumerate(oracle.all_reduce_two_shot(xs, op, dtype)):
        assert np.array_equal(bits(y), bits(ref[q]))
    assert np.array_equal(bits(oracle.reduce(xs, op, dtype)), bits(ref[0]))


@SET
@given(n=st.integers(1, 9), per=st.integers(1, 60), dtype=st.sampled_from(["bf16", "fp32", "int32"]),
       op=st.integers(0, 3), seed=st.integers(0, 10**6))
def test_reduce_scatter_blocks_make_the_reduce(n, per, dtype, op, seed):
    xs = values(np.random.default_rng(seed), n, n * per, dtype, op)
    rs = oracle.reduce_scatter(xs, op, dtype)
    assert np.array_equal(bits(np.concatenate(rs)), bits(oracle.reduce(xs, op, dtype)))


@SET
@given(n=st.integers(2, 9), count=st.integers(1, 300), op=st.sampled_from([0, 3]), seed=st.integers(0, 10**6))
def test_ring_integer_sum_and_product_are_order_free(n, count, op, seed):
    xs = values(np.random.default_rng(seed), n, count, "int32", op)
    ref = oracle.all_reduce(xs, op, "int32")
    for q, y in enumerate(oracle.all_reduce_ring(xs, op, "int32")):
        assert np.array_equal(y, ref[q])


@SET
@given(n=st.integers(2, 9), count=st.integers(1, 300), op=st.sampled_from([1, 2]), seed=st.integers(0, 10**6))
def test_ring_max_min_of_distinct_values_are_order_free(n, count, op, seed):
    g = np.random.default_rng(seed)
    # distinct, nonzero, finite fp32 values: no ties, no signed zeros, no NaN
    pool = g.permutation(np.arange(1, n * count + 1, dtype=np.int64)) * g.choice([-1, 1], n * count)
    xs = [(pool[r * count:(r + 1) * count] * 0.5).astype(np.float32) for r in range(n)]
    ref = oracle.all_reduce(xs, op, "fp32")
    for q, y in enumerate(oracle.all_reduce_ring(xs, op, "fp32")):
        assert np.array_equal(bits(y), bits(ref[q]))


def bf16_bits_of(x64):
    """torch's round-to-nearest-even of fp64 values that fp32 holds exactly"""
    t = torch.from_numpy(np.asarray(x64, np.float64).astype(np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def bf16_value(bits):
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


@SET
@given(n=st.integers(2, 9), count=st.integers(1, 300), seed=st.integers(0, 10**6))
def test_ring_bf16_sum_of_exact_partials_is_the_rounded_exact_sum(n, count, seed):
    g = np.random.default_rng(seed)
    # k * 2^-e with |k| < 256 and 0 <= e <= 8: exact in bf16 (8 significant
    # bits), while any partial sum of up to 9 of them lies on the 2^-8 grid
    # below 2^12 and so is exact in fp32 (20 bits) but usually needs more
    # bits than bf16 has: only the final rounding may act
    v = g.integers(-255, 256, (n, count)) * 2.0 ** -g.integers(0, 9, (n, count))
    xs = [bf16_bits_of(x) for x in v]
    assert all(np.array_equal(bf16_value(x), w) for x, w in zip(xs, v))
    want = bf16_bits_of(v.sum(axis=0))
    for y in oracle.all_reduce_ring(xs, 0, "bf16"):
        assert np.array_equal(y, want)


@SET
@given(n=st.integers(2, 9), count=st.integers(1, 300), seed=st.integers(0, 10**6))
def test_ring_bf16_sum_error_is_bounded_by_the_magnitudes(n, count, seed):
    g = np.random.default_rng(seed)
    xs = [bf16_bits_of(g.standard_normal(count) * 4) for _ in range(n)]
    vals = np.stack([bf16_value(x) for x in xs])
    exact = vals.sum(axis=0)  # fp64: exact for these magnitudes
    # one final rounding (<= 2^-8 relative) and n - 1 fp32 additions (<= 2^-24 each)
    tol = (2.0 ** -8 + (n - 1) * 2.0 ** -24) * np.abs(vals).sum(axis=0) + 2.0 ** -133
    for y in oracle.all_reduce_ring(xs, 0, "bf16"):
        assert np.all(np.abs(bf16_value(y) - exact) <= tol)


@SET
@given(n=st.integers(1, 9), count=st.integers(1, 200), dst=st.integers(0, 8), seed=st.integers(0, 10**6))
def test_gather_then_scatter_is_identity(n, count, dst, seed):
    dst %= n
    g = np.random.default_rng(seed)
    xs = [g.integers(0, 2**16, count, dtype=np.int64).astype(np.uint16) for _ in range(n)]
    full = oracle.gather(xs, np.zeros(n * count, np.uint16))
    assert np.array_equal(full, np.concatenate(xs))
    back = oracle.scatter(full, n)
    for r in range(n):
        assert np.array_equal(back[r], xs[r])
    for q, y in enumerate(oracle.all_gather(xs)):
        assert np.array_equal(y, full)


@SET
@given(n=st.integers(1, 6), max_rows=st.integers(0, 12), row=st.integers(1, 5), seed=st.integers(0, 10**6))
def test_all_to_all_v_transposed_round_trip(n, max_rows, row, seed):
    g = np.random.default_rng(seed)
    sc = g.integers(0, max_rows + 1, (n, n)).astype(np.int64)
    sd = np.zeros_like(sc)
    sd[:, 1:] = np.cumsum(sc, axis=1)[:, :-1]
    rc = sc.T.copy()
    rd = np.zeros_like(sc)
    rd[:, 1:] = np.cumsum(rc, axis=1)[:, :-1]
    xs = [g.integers(0, 2**16, int(sc[s].sum()) * row, dtype=np.int64).astype(np.uint16) for s in range(n)]
    bufs = [np.zeros(int(rc[d].sum()) * row, np.uint16) for d in range(n)]
    there = oracle.all_to_all_v(xs, bufs, sc, sd, rd, row)
    back = oracle.all_to_all_v(there, [np.zeros_like(x) for x in xs], rc, rd, sd, row)
    for s in range(n):
        assert np.array_equal(back[s], xs[s])


@SET
@given(nbytes=st.integers(0, 2000), step=st.integers(1, 2**40), ll128=st.booleans(), seed=st.integers(0, 10**6))
def test_unpack_of_pack_is_the_message(nbytes, step, ll128, seed):
    proto = oracle.LL128 if ll128 else oracle.LL
    if proto == oracle.LL and step % 2**32 == 0:
        step += 1
    msg = np.random.default_rng(seed).integers(0, 256, nbytes, dtype=np.int64).astype(np.uint8)
    packed = oracle.pack(msg, proto, step)
    assert packed.size == oracle.packed_bytes(nbytes, proto)
    data, bad = oracle.unpack(packed, nbytes, proto, step)
    assert np.array_equal(data, msg) and bad == 0


@settings(max_examples=10, deadline=None, derandomize=True)
@given(n=st.sampled_from([2, 4]), tokens=st.integers(1, 20), topk=st.integers(1, 4), epr=st.integers(1, 4),
       seed=st.integers(0, 10**6))
def test_dedup_route_combines_like_the_plain_route(n, tokens, topk, epr, seed):
    experts = n * epr
    topk = min(topk, experts)
    ids, ws = W.moe_routing(tokens, experts, topk, n)
    h = 3
    g = np.random.default_rng(seed)
    xs = [oracle.narrow(g.standard_normal(tokens * h).astype(np.float32), "bf16") for _ in range(n)]
    outs = []
    for route in (oracle.moe_route, oracle.moe_route_dedup):
        sc, sd, rd, pos = route(ids, experts)
        bufs = [np.zeros(int(sc[:, d].sum()) * h, np.uint16) for d in range(n)]
        ys = oracle.moe_dispatch(xs, ids, pos, bufs, experts, h)
        outs.append(oracle.moe_combine(ys, ids, pos, ws, experts, h, "bf16"))
    for s in range(n):
        assert np.array_equal(outs[0][s], outs[1][s])
