"""GPU parity: LL / LL128 codecs and the packetised all-reduce vs the oracle.

Packed bytes are compared bit for bit with the oracle's encoding; decode
round-trips; corrupted flags are counted exactly in the device status (a
host-made corruption: no kernel waits, so nothing can hang); the
packetised all-reduce matches the oracle's and, once decoded, the Simple
two-shot all-reduce.
"""
import numpy as np
import pytest
import torch

import movement_virtual_rank_b200 as M
import oracle
import workloads as W
from gpu_util import need_gpu, status_tensor, to_dev

pytestmark = pytest.mark.gpu
SIZES = [1, 2, 3, 4, 5, 15, 16, 17, 31, 32, 33, 119, 120, 121, 239, 240, 241, 1000, 4097, 65536 + 12, 1 << 20]


def u8(nbytes, salt):
    return W.rng(W.W_MISC, 2, salt=salt).integers(0, 256, nbytes).astype(np.uint8)


@pytest.mark.parametrize("proto", [M.LL, M.LL128])
@pytest.mark.parametrize("nbytes", SIZES)
@pytest.mark.parametrize("src_off", [0, 1, 8])
def test_pack_unpack(proto, nbytes, src_off):
    need_gpu()
    msg = u8(nbytes, nbytes + src_off)
    step = 0x1234_5678 + nbytes if proto == M.LL else (0xABCD << 40) + nbytes
    raw = torch.zeros(nbytes + 64, dtype=torch.uint8, device="cuda")
    src = raw[src_off:src_off + nbytes]
    src.copy_(torch.from_numpy(msg).cuda())
    pb = M.coll_packed_bytes(nbytes, proto)
    packed = torch.full((pb + 32,), 0xEE, dtype=torch.uint8, device="cuda")
    M.coll_ll_pack(src, packed[:pb], proto, step)
    torch.cuda.synchronize()
    assert np.array_equal(packed[:pb].cpu().numpy(), oracle.pack(msg, proto, step))
    assert (packed[pb:] == 0xEE).all()
    out_raw = torch.full((nbytes + 64,), 0x33, dtype=torch.uint8, device="cuda")
    dst = out_raw[src_off + 3:src_off + 3 + nbytes]
    st = status_tensor()
    M.coll_ll_unpack(packed[:pb], dst, proto, step, status=st)
    torch.cuda.synchronize()
    assert np.array_equal(dst.cpu().numpy(), msg)
    o = out_raw.cpu().numpy()
    assert (o[:src_off + 3] == 0x33).all() and (o[src_off + 3 + nbytes:] == 0x33).all()
    assert st.tolist() == [0, 0]


@pytest.mark.parametrize("proto", [M.LL, M.LL128])
def test_unpack_counts_bad_flags(proto):
    """Lines whose flag differs from the step (a stale or torn packet) are
    counted exactly; the kernel returns normally."""
    need_gpu()
    nbytes = 100003
    msg = u8(nbytes, 1)
    step = 41
    packed_np = oracle.pack(msg, proto, step)
    line = 8 if proto == M.LL else 128
    flag_at = 4 if proto == M.LL else 120
    nlines = packed_np.size // line
    g = W.rng(W.W_MISC, 3, salt=proto)
    lines = np.unique(g.integers(0, nlines, 57))
    bad = packed_np.copy()
    for L in lines:
        bad[L * line + flag_at] ^= 0x40
    packed = torch.from_numpy(bad).cuda()
    dst = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    st = status_tensor()
    M.coll_ll_unpack(packed, dst, proto, step, status=st)
    torch.cuda.synchronize()
    _, want_bad = oracle.unpack(bad, nbytes, proto, step)
    assert want_bad == lines.size
    assert st.tolist() == [M.DEV_FLAG_MISMATCH, lines.size]
    assert np.array_equal(dst.cpu().numpy(), msg)  # data is still delivered
    # a stale step fails every line
    st.zero_()
    M.coll_ll_unpack(torch.from_numpy(packed_np).cuda(), dst, proto, step + 1, status=st)
    torch.cuda.synchronize()
    assert st.tolist() == [M.DEV_FLAG_MISMATCH, nlines]


@pytest.mark.parametrize("proto", [M.LL, M.LL128])
@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("n", [1, 2, 3, 8])
@pytest.mark.parametrize("count", [1, 2, 3, 59, 60, 61, 1000, 30001])
def test_all_reduce_packed(proto, dtype, n, count):
    need_gpu()
    xs = W.ranks_values(W.W_LL_SWEEP, n, count, dtype, "uniform", salt=count)
    step = 7
    esize = 2 if dtype == "bf16" else 4
    pin = [oracle.pack(x, proto, step) for x in xs]
    want, want_bad = oracle.all_reduce_packed(pin, count, dtype, 0, proto, step)
    dev_in = [torch.from_numpy(p).cuda() for p in pin]
    dev_out = [torch.full_like(p, 0x99) for p in dev_in]
    st = status_tensor()
    M.coll_all_reduce_packed(dev_in, dev_out, count, torch.bfloat16 if dtype == "bf16" else torch.float32,
                             proto, step, status=st)
    torch.cuda.synchronize()
    assert st.tolist() == [0, 0] and want_bad == 0
    for q in range(n):
        assert np.array_equal(dev_out[q].cpu().numpy(), want[q]), q
    # decoded, it equals the Simple (two-shot) all-reduce
    simple = oracle.all_reduce_two_shot(xs, 0, dtype)
    data, _ = oracle.unpack(want[0], count * esize, proto, step)
    assert np.array_equal(data.view(simple[0].dtype), simple[0])


@pytest.mark.parametrize("proto", [M.LL, M.LL128])
def test_all_reduce_packed_in_place_and_bad_flags(proto):
    need_gpu()
    n, count = 4, 5000
    xs = W.ranks_values(W.W_LL_SWEEP, n, count, "bf16", "uniform", salt=3)
    step = 3
    pin = [oracle.pack(x, proto, step) for x in xs]
    line = 8 if proto == M.LL else 128
    flag_at = 4 if proto == M.LL else 120
    pin[2][5 * line + flag_at] ^= 1  # one stale line on rank 2
    want, want_bad = oracle.all_reduce_packed(pin, count, "bf16", 0, proto, step)
    dev = [torch.from_numpy(p).cuda() for p in pin]
    st = status_tensor()
    M.coll_all_reduce_packed(dev, dev, count, torch.bfloat16, proto, step, status=st)
    torch.cuda.synchronize()
    assert want_bad == 1 and st.tolist() == [M.DEV_FLAG_MISMATCH, 1]
    for q in range(n):
        assert np.array_equal(dev[q].cpu().numpy(), want[q])


@pytest.mark.parametrize("log2", [10, 16, 20, 24, 28])
def test_ll_sweep_sizes(log2):
    """The LL / LL128 sweep sizes (8 ranks, 1 KB .. 256 MB per rank): every
    packed output compared on the device with the packed Simple result, and
    every line of it against the oracle's packetised all-reduce.  The oracle
    runs on chunks of whole lines (each line of the result depends only on
    the same line of every rank's packets), so host memory stays bounded.
    Every rank's Simple output equals rank 0's, and the one-launch codecs for
    all ranks give the one-rank calls' bytes, encoding and decoding."""
    need_gpu()
    n, nbytes = 8, 1 << log2
    count = nbytes // 2
    xs = W.ll_message(nbytes, n)
    send = [to_dev(x, "bf16") for x in xs]
    simple = [torch.empty_like(t) for t in send]
    M.coll_all_reduce(send, simple, algo=M.TWOSHOT)
    for q in range(1, n):
        assert torch.equal(simple[q].view(torch.int16), simple[0].view(torch.int16)), q
    for proto in (M.LL, M.LL128):
        step = log2 + 1
        pb = M.coll_packed_bytes(nbytes, proto)
        packed = [torch.empty(pb, dtype=torch.uint8, device="cuda") for _ in range(n)]
        for r in range(n):
            M.coll_ll_pack(send[r], packed[r], proto, step)
        together = [torch.empty(pb, dtype=torch.uint8, device="cuda") for _ in range(n)]
        M.coll_ll_pack_ranks(send, together, proto, step)
        torch.cuda.synchronize()
        for r in range(n):
            assert torch.equal(together[r], packed[r]), r
        del together
        out = [torch.empty(pb, dtype=torch.uint8, device="cuda") for _ in range(n)]
        st = status_tensor()
        M.coll_all_reduce_packed(packed, out, count, torch.bfloat16, proto, step, status=st)
        ref = torch.empty(pb, dtype=torch.uint8, device="cuda")
        M.coll_ll_pack(simple[0], ref, proto, step)
        dec = torch.empty_like(send[0])
        M.coll_ll_unpack(out[3], dec, proto, step, status=st)
        torch.cuda.synchronize()
        assert st.tolist() == [0, 0]
        for q in range(n):
            assert torch.equal(out[q], ref)
        assert torch.equal(dec.view(torch.int16), simple[0].view(torch.int16))
        decs = [torch.empty_like(send[0]) for _ in range(n)]
        M.coll_ll_unpack_ranks(out, decs, proto, step, status=st)
        torch.cuda.synchronize()
        assert st.tolist() == [0, 0]
        for q in range(n):
            assert torch.equal(decs[q].view(torch.int16), simple[0].view(torch.int16)), q
        del packed, ref, dec, decs
        line = 8 if proto == M.LL else 128
        per = 2 if proto == M.LL else 60  # bf16 elements of payload per line
        nl = pb // line
        chunk = (1 << 24) // per  # lines: 16 Mi payload elements per oracle call
        for l0 in range(0, nl, chunk):
            l1 = min(nl, l0 + chunk)
            lo, hi = l0 * per, min(count, l1 * per)
            pin = [oracle.pack(x[lo:hi], proto, step) for x in xs]
            want, bad = oracle.all_reduce_packed(pin, hi - lo, "bf16", 0, proto, step)
            assert bad == 0
            got = out[0][l0 * line:l1 * line].cpu().numpy()
            assert np.array_equal(got, want[0]), (proto, l0)
        del out


@pytest.mark.parametrize("proto", [M.LL, M.LL128])
@pytest.mark.parametrize("nbytes", [16 << 20, (16 << 20) + 4, (16 << 20) + 120 * 7 + 3, 10_000_000, 3 * (1 << 22) + 1000,
                                    (20 << 20) + 4])
def test_pack_unpack_bulk_path(proto, nbytes):
    """Long aligned messages take the bulk-copy codec for whole tiles and the
    element kernels for the tail: the packet bytes are the oracle's, the
    round trip is exact, and bytes past either buffer stay untouched.  One
    rank's LL pack takes the resident grid up to 8 tiles per resident CTA
    (the sizes up to 16 MiB + 843 B) and the in-order grid above (20 MiB)."""
    need_gpu()
    msg = u8(nbytes, nbytes % 1000 + 5)
    step = 0x0BAD_CAFE if proto == M.LL else (0x5A5A << 36) + 3
    src = torch.from_numpy(msg).cuda()
    pb = M.coll_packed_bytes(nbytes, proto)
    packed = torch.full((pb + 256,), 0xEE, dtype=torch.uint8, device="cuda")
    M.coll_ll_pack(src, packed[:pb], proto, step)
    torch.cuda.synchronize()
    assert np.array_equal(packed[:pb].cpu().numpy(), oracle.pack(msg, proto, step))
    assert (packed[pb:] == 0xEE).all()
    out = torch.full((nbytes + 256,), 0x33, dtype=torch.uint8, device="cuda")
    st = status_tensor()
    M.coll_ll_unpack(packed[:pb], out[:nbytes], proto, step, status=st)
    torch.cuda.synchronize()
    assert torch.equal(out[:nbytes], src)
    assert (out[nbytes:] == 0x33).all()
    assert st.tolist() == [0, 0]


@pytest.mark.parametrize("proto", [M.LL, M.LL128])
def test_unpack_counts_bad_flags_bulk_path(proto):
    """Corrupted flags spread over the bulk-copy tiles and the tail are
    counted exactly."""
    need_gpu()
    nbytes = (16 << 20) + 1000
    msg = u8(nbytes, 77)
    step = 9
    pk = oracle.pack(msg, proto, step)
    line = 8 if proto == M.LL else 128
    flag_at = 4 if proto == M.LL else 120
    nlines = pk.size // line
    g = W.rng(W.W_MISC, 3, salt=78)
    bad_lines = np.unique(np.concatenate([g.choice(nlines, 300, replace=False), [0, nlines - 1, nlines - 2]]))
    for L in bad_lines:
        pk[L * line + flag_at] ^= 0x40
    packed = torch.from_numpy(pk).cuda()
    out = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    st = status_tensor()
    M.coll_ll_unpack(packed, out, proto, step, status=st)
    torch.cuda.synchronize()
    assert st.tolist() == [M.DEV_FLAG_MISMATCH, int(bad_lines.size)]
    assert torch.equal(out, torch.from_numpy(msg).cuda())  # the data are written all the same


@pytest.mark.parametrize("proto", [M.LL, M.LL128])
@pytest.mark.parametrize("n,nbytes", [(1, 1000), (3, 1), (3, 121), (8, 4097), (8, 65536 + 12), (5, (1 << 20) + 7),
                                      (8, (2 << 20) + 12), (8, 16 << 20), (8, (16 << 20) + 120 * 3 + 5), (2, 10_000_000),
                                      (2, (64 << 20) + 4097)])
@pytest.mark.parametrize("unaligned_rank", [None, 1])
def test_pack_unpack_ranks(proto, n, nbytes, unaligned_rank):
    """All ranks' messages in one launch (a CTA row per rank): every rank's
    packets are the oracle's encoding of its own message, the round trip is
    exact, and no byte outside a buffer is touched.  One rank's message at an
    odd offset sends every rank down the unaligned code."""
    need_gpu()
    if unaligned_rank is not None and unaligned_rank >= n:
        pytest.skip("fewer ranks")
    step = 0x2468_1357 + n if proto == M.LL else (0x77 << 48) + nbytes
    pb = M.coll_packed_bytes(nbytes, proto)
    msgs = [u8(nbytes, 31 * r + nbytes % 997) for r in range(n)]
    offs = [1 if r == unaligned_rank else 0 for r in range(n)]
    raws = [torch.zeros(nbytes + 64, dtype=torch.uint8, device="cuda") for _ in range(n)]
    src = [raws[r][offs[r]:offs[r] + nbytes] for r in range(n)]
    for r in range(n):
        src[r].copy_(torch.from_numpy(msgs[r]).cuda())
    pk_raw = [torch.full((pb + 64,), 0xEE, dtype=torch.uint8, device="cuda") for _ in range(n)]
    packed = [t[:pb] for t in pk_raw]
    M.coll_ll_pack_ranks(src, packed, proto, step)
    torch.cuda.synchronize()
    for r in range(n):
        assert np.array_equal(packed[r].cpu().numpy(), oracle.pack(msgs[r], proto, step)), r
        assert (pk_raw[r][pb:] == 0xEE).all(), r
    out_raw = [torch.full((nbytes + 64,), 0x33, dtype=torch.uint8, device="cuda") for _ in range(n)]
    dst = [out_raw[r][offs[r] + 3:offs[r] + 3 + nbytes] for r in range(n)]
    st = status_tensor()
    M.coll_ll_unpack_ranks(packed, dst, proto, step, status=st)
    torch.cuda.synchronize()
    for r in range(n):
        assert np.array_equal(dst[r].cpu().numpy(), msgs[r]), r
        o = out_raw[r].cpu().numpy()
        assert (o[:offs[r] + 3] == 0x33).all() and (o[offs[r] + 3 + nbytes:] == 0x33).all(), r
    assert st.tolist() == [0, 0]


@pytest.mark.parametrize("proto", [M.LL, M.LL128])
def test_unpack_ranks_counts_bad_flags(proto):
    """Corrupted flags in several ranks' packets are counted exactly, summed
    over the ranks, and every rank's data is still written."""
    need_gpu()
    n, nbytes, step = 4, (1 << 20) + 333, 5
    line = 8 if proto == M.LL else 128
    flag_at = 4 if proto == M.LL else 120
    msgs = [u8(nbytes, 500 + r) for r in range(n)]
    total = 0
    packed = []
    for r in range(n):
        pk = oracle.pack(msgs[r], proto, step)
        if r in (1, 3):
            g = W.rng(W.W_MISC, 4, salt=r)
            lines = np.unique(g.integers(0, pk.size // line, 40 + r))
            for L in lines:
                pk[L * line + flag_at] ^= 0x10
            total += lines.size
        packed.append(torch.from_numpy(pk).cuda())
    dst = [torch.empty(nbytes, dtype=torch.uint8, device="cuda") for _ in range(n)]
    st = status_tensor()
    M.coll_ll_unpack_ranks(packed, dst, proto, step, status=st)
    torch.cuda.synchronize()
    assert st.tolist() == [M.DEV_FLAG_MISMATCH, total]
    for r in range(n):
        assert np.array_equal(dst[r].cpu().numpy(), msgs[r]), r
