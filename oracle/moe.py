"""MoE expert-parallel dispatch / combine over virtual ranks.

Test infrastructure only (see ``oracle/__init__.py``).

Follows the vLLM collectives tutorial (gsyq.cn/news/307221), section 8.4
("MoE Dispatch / Combine"): with experts split evenly over the EP ranks
(rank 0 holds experts 0,1 and rank 1 holds 2,3 in its example), dispatch sends
every token to the rank that holds each expert it was routed to; combine sends
the expert outputs back by original token ownership.  Section 8.2 says the
per-peer lengths then differ, i.e. an all-to-all-v.

Readings taken (the pages are silent on these):

* Expert e lives on rank e // (E / N).
* One dispatched row per (token, chosen expert) pair; a token routed to two
  experts on the same rank is sent twice (no per-rank de-duplication).
* Send order on source s: by destination rank, then expert id ascending, then
  token index ascending (destination-major equals expert-major because
  experts are assigned to ranks in contiguous blocks).  Receive order on
  destination d: by source rank ascending (tutorial 8.1, "[from 0, from 1,
  ...]"), then the sender's order.
* A token's K expert ids are distinct and lie in [0, E).
* The expert between dispatch and combine is the identity (expert compute is
  out of scope); tests may scale rows per expert to catch mix-ups.
* combine: ``acc = fl32(w_0 * y_0)``, then ``acc = fl32(acc + fl32(w_k * y_k))``
  for k = 1 .. K-1 (k ascending, products and sums each rounded to binary32,
  no fused multiply-add), then one rounding to the storage type.
"""
from __future__ import annotations

import numpy as np

from .numerics import narrow, widen


def moe_route(topk_ids, n_experts: int):
    """Split matrix and row positions of every (token, k) pair.

    Returns (send_counts[N,N], send_displs[N,N], recv_displs[N,N] (indexed
    [d][s]), pos: list of int64 [T*K] arrays -- the row of pair (t, k) in the
    receive buffer of rank topk_ids[t,k] // (E/N)).
    """
    n = len(topk_ids)
    assert n_experts % n == 0
    epr = n_experts // n
    send_counts = np.zeros((n, n), dtype=np.int64)
    for s in range(n):
        ids = np.asarray(topk_ids[s]).reshape(-1)
        assert ids.size == 0 or (ids.min() >= 0 and ids.max() < n_experts)
        cnt = np.bincount(ids, minlength=n_experts)
        for d in range(n):
            send_counts[s, d] = cnt[d * epr:(d + 1) * epr].sum()
    send_displs = np.zeros((n, n), dtype=np.int64)
    for s in range(n):
        for d in range(1, n):
            send_displs[s, d] = send_displs[s, d - 1] + send_counts[s, d - 1]
    recv_displs = np.zeros((n, n), dtype=np.int64)  # [d][s]
    for d in range(n):
        for s in range(1, n):
            recv_displs[d, s] = recv_displs[d, s - 1] + send_counts[s - 1, d]
    pos = []
    for s in range(n):
        ids2 = np.asarray(topk_ids[s])
        t_, k_ = ids2.shape
        for t in range(t_):
            assert len(set(ids2[t].tolist())) == k_, "a token's experts must be distinct"
        e = ids2.reshape(-1).astype(np.int64)
        tok = np.repeat(np.arange(t_, dtype=np.int64), k_)
        order = np.lexsort((tok, e))  # primary key: expert, then token
        send_pos = np.empty(e.size, dtype=np.int64)
        send_pos[order] = np.arange(e.size, dtype=np.int64)
        d = e // epr
        pos.append(recv_displs[d, s] + send_pos - send_displs[s, d])
    return send_counts, send_displs, recv_displs, pos


def moe_route_dedup(topk_ids, n_experts: int):
    """Route with one dispatched row per (token, destination rank).

    The tutorial (section 8.5.1) only names dispatch designs that send a
    token once per rank it must reach; the readings taken here:

    * ``send_counts[s][d]`` is the number of tokens of source s with at least
      one chosen expert on rank d.
    * Send order on source s: by destination rank, then token ascending;
      receive order on d: by source rank ascending, then the sender's order.
    * ``pos[s][t*K + k]`` is the row of (t, rank of expert k) in that rank's
      receive buffer, the same row for every k whose experts share a rank.

    Same return values as ``moe_route``; ``moe_dispatch`` and ``moe_combine``
    take the positions unchanged (a row reached twice is written twice with
    the same bytes, and read once per choice).
    """
    n = len(topk_ids)
    assert n_experts % n == 0
    epr = n_experts // n
    send_counts = np.zeros((n, n), dtype=np.int64)
    dest = []
    for s in range(n):
        ids2 = np.asarray(topk_ids[s])
        assert ids2.size == 0 or (ids2.min() >= 0 and ids2.max() < n_experts)
        for t in range(ids2.shape[0]):
            assert len(set(ids2[t].tolist())) == ids2.shape[1], "a token's experts must be distinct"
        d2 = ids2.astype(np.int64) // epr  # [T, K] destination rank of every choice
        dest.append(d2)
        for d in range(n):
            send_counts[s, d] = int((d2 == d).any(axis=1).sum())
    send_displs = np.zeros((n, n), dtype=np.int64)
    for s in range(n):
        for d in range(1, n):
            send_displs[s, d] = send_displs[s, d - 1] + send_counts[s, d - 1]
    recv_displs = np.zeros((n, n), dtype=np.int64)  # [d][s]
    for d in range(n):
        for s in range(1, n):
            recv_displs[d, s] = recv_displs[d, s - 1] + send_counts[s - 1, d]
    pos = []
    for s in range(n):
        d2 = dest[s]
        t_, k_ = d2.shape
        p = np.empty(t_ * k_, dtype=np.int64)
        for d in range(n):
            reach = (d2 == d).any(axis=1)               # tokens of s that go to d
            rank = np.cumsum(reach) - 1                 # their order among them
            for t in np.nonzero(reach)[0]:
                for k in range(k_):
                    if d2[t, k] == d:
                        p[t * k_ + k] = recv_displs[d, s] + rank[t]
        pos.append(p)
    return send_counts, send_displs, recv_displs, pos


def moe_permute_send(xs, topk_ids, n_experts: int, hidden: int):
    """The sender-side layout: rank s's rows in send order (dest, expert, token)."""
    out = []
    for s in range(len(xs)):
        ids2 = np.asarray(topk_ids[s])
        t_, k_ = ids2.shape
        e = ids2.reshape(-1)
        tok = np.repeat(np.arange(t_), k_)
        order = np.lexsort((tok, e))
        x = np.asarray(xs[s]).reshape(t_, hidden)
        out.append(x[tok[order]].reshape(-1))
    return out


def moe_dispatch(xs, topk_ids, pos, recv_bufs, n_experts: int, hidden: int):
    """recv[d][pos(s,t,k)] = x[s][t] for every source s, token t and choice k."""
    n = len(xs)
    epr = n_experts // n
    outs = [np.array(b, copy=True) for b in recv_bufs]
    for s in range(n):
        ids2 = np.asarray(topk_ids[s])
        t_, k_ = ids2.shape
        x = np.asarray(xs[s]).reshape(t_, hidden)
        for j in range(t_ * k_):
            t, d = j // k_, int(ids2.reshape(-1)[j]) // epr
            p = int(pos[s][j])
            outs[d][p * hidden:(p + 1) * hidden] = x[t]
    return outs


def moe_combine(ys, topk_ids, pos, topk_w, n_experts: int, hidden: int, dtype: str, tokens=None):
    """out[s][t] = round( sum_k w[s][t][k] * y[d_k][pos(s,t,k)] ), k ascending.

    ``tokens`` (optional, per source a list of token indices) restricts the
    computation to those tokens; the result then holds their rows in order.
    """
    n = len(topk_ids)
    epr = n_experts // n
    outs = []
    for s in range(n):
        ids2 = np.asarray(topk_ids[s])
        w = np.asarray(topk_w[s], dtype=np.float32)
        t_, k_ = ids2.shape
        sel = list(range(t_)) if tokens is None else list(tokens[s])
        acc = np.zeros((len(sel), hidden), dtype=np.float32)
        for k in range(k_):
            rows = np.empty((len(sel), hidden), dtype=np.float32)
            for i, t in enumerate(sel):
                d = int(ids2[t, k]) // epr
                p = int(pos[s][t * k_ + k])
                rows[i] = widen(np.asarray(ys[d])[p * hidden:(p + 1) * hidden], dtype)
            prod = (w[sel, k:k + 1] * rows).astype(np.float32)
            acc = prod if k == 0 else (acc + prod).astype(np.float32)
        outs.append(narrow(acc.reshape(-1), dtype))
    return outs
