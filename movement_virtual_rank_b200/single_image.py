"""Single-image embedding sync on virtual ranks: padded all-gather vs broadcast.

sglang PR 33307 summary (prhub), "motivation" and "key code": when a request
carries a single image, only one rank (the owner) holds its embedding rows.
The old path pads every rank's rows to ``max_len``, all-gathers N x max_len
rows and keeps the owner's first ``n_tok``; the new path broadcasts the
owner's ``n_tok`` rows, one copy instead of N.  Both leave bit-identical rows
on every rank.

``VirtualGroup`` presents the virtual ranks of this GPU with the two
collective calls the sync needs; tests substitute a fake group (the page's
own unit-test pattern) to check which call is made.
"""
from __future__ import annotations

import torch

from . import coll_all_gather, coll_broadcast


class VirtualGroup:
    """The N virtual ranks of one GPU as a group with broadcast / all_gather."""

    def __init__(self, nranks: int):
        self.size = nranks

    def broadcast(self, bufs, src: int):
        coll_broadcast(bufs, src)
        return bufs

    def all_gather(self, send, recv):
        coll_all_gather(send, recv)
        return recv


def sync_single_image_broadcast(group, bufs, owner: int):
    """New path: ``bufs[r]`` are [n_tok, hidden] tensors, ``bufs[owner]`` holds
    the owner's rows; after the call every rank's buffer holds them."""
    group.broadcast(bufs, owner)
    return bufs


def sync_single_image_padded_all_gather(group, padded, gathered, owner: int, n_tok: int):
    """Old path: ``padded[r]`` are [max_len, hidden] (only the owner's first
    ``n_tok`` rows matter), ``gathered[r]`` are [N * max_len, hidden]; every
    rank keeps rows owner * max_len .. + n_tok of its gathered buffer."""
    group.all_gather(padded, gathered)
    max_len = padded[0].shape[0]
    return [g[owner * max_len: owner * max_len + n_tok] for g in gathered]


def sync_single_image(group, per_rank_rows, owner: int, n_tok: int, hidden: int, dtype=torch.bfloat16):
    """The dispatch of the page's fast path: with one image, broadcast from its
    owner into fresh [n_tok, hidden] buffers on the other ranks."""
    bufs = []
    for r in range(group.size):
        if r == owner:
            bufs.append(per_rank_rows[r].contiguous())
        else:
            bufs.append(torch.empty((n_tok, hidden), dtype=dtype, device=per_rank_rows[owner].device))
    return sync_single_image_broadcast(group, bufs, owner)
