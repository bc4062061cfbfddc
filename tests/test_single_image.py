"""Single-image embedding sync (sglang PR 33307 summary): the broadcast path
must be taken for one image, from its owner, and both paths must leave
bit-identical rows on every rank.

The CPU test uses the page's own pattern: a fake group whose all_gather
fails the test if reached and whose broadcast records its source.
"""
import numpy as np
import pytest
import torch

import workloads as W
from movement_virtual_rank_b200 import single_image as SI


def test_single_image_takes_broadcast_from_owner():
    calls = []

    class FakeGroup:
        size = 2

        def all_gather(self, send, recv):
            raise AssertionError("a single image must not reach the all-gather")

        def broadcast(self, bufs, src):
            calls.append(src)
            for b in bufs:
                b.copy_(bufs[src])
            return bufs

    rows = [torch.zeros(0, 2), torch.randn(4, 2, generator=torch.Generator().manual_seed(1))]
    out = SI.sync_single_image(FakeGroup(), rows, owner=1, n_tok=4, hidden=2, dtype=torch.float32)
    assert calls == [1]
    for o in out:
        assert torch.equal(o, rows[1])


@pytest.mark.gpu
@pytest.mark.parametrize("n_tok,hidden", [(1, 8), (37, 7168), (1024, 7168)])
def test_padded_all_gather_and_broadcast_agree_bitwise(n_tok, hidden):
    """8 virtual ranks, owner 5: path A (pad to max_len, all-gather, slice the
    owner's rows) == path B (broadcast from the owner) == the owner's rows."""
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    n, owner, max_len = 8, 5, n_tok + 3
    truth = W.ranks_values(W.W_MISC, 1, n_tok * hidden, "bf16", salt=n_tok)[0].view(np.int16)
    truth_t = torch.from_numpy(truth.copy()).view(torch.bfloat16).reshape(n_tok, hidden).cuda()
    g = SI.VirtualGroup(n)
    padded = [torch.full((max_len, hidden), 9.0, dtype=torch.bfloat16, device="cuda") for _ in range(n)]
    padded[owner][:n_tok].copy_(truth_t)
    gathered = [torch.empty(n * max_len, hidden, dtype=torch.bfloat16, device="cuda") for _ in range(n)]
    a = SI.sync_single_image_padded_all_gather(g, padded, gathered, owner, n_tok)
    rows = [torch.empty(0, hidden, dtype=torch.bfloat16, device="cuda") for _ in range(n)]
    rows[owner] = truth_t
    b = SI.sync_single_image(g, rows, owner, n_tok, hidden)
    torch.cuda.synchronize()
    for r in range(n):
        assert torch.equal(a[r].view(torch.int16), truth_t.view(torch.int16))
        assert torch.equal(b[r].view(torch.int16), truth_t.view(torch.int16))
