"""CPU oracle for the virtual-rank collectives -- TEST INFRASTRUCTURE ONLY.

A plain, slow, loop-by-loop restatement of what the collectives compute, in
numpy, written from the pages' definitions:

* the eight collectives of the vLLM collectives tutorial (gsyq.cn/news/307221,
  sections 1.1 Broadcast ... 8.2 All-to-All / All-to-Allv), with the MoE
  dispatch/combine example of its section 8.4;
* the two-shot (owner reduces its segment, then sends it to everyone), the
  one-shot and the ring all-reduce of "From NCCL Ring LL to PCIe IPC
  AllReduce" (section "Pro5000 ?") and of the TP communication essay
  (52jiny.com thread-1337, section on how communication erodes scaling);
* the LL [4 B data | 4 B flag] and LL128 [120 B data | 8 B flag] packet
  layouts of "From NCCL Ring LL ..." (section "Traditional LL Protocols").

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU baseline
(and its ``--impl reference`` arm) may import this package.  It shares no code
with the CUDA library under ``movement_virtual_rank_b200/``; the only module
both sides use is ``workloads`` (seeded random inputs, no collective
arithmetic).

Every function is pinned by ``tests/test_oracle_*.py`` against something other
than itself (worked examples from the pages, fp64 / exact-rational brute
force, library conversions, algebraic invariants).  See each module's header
for the readings taken where the pages are silent.
"""
from .numerics import (  # noqa: F401
    DTYPES, OPS, SUM, MAX, MIN, PROD,
    bf16_bits_to_f32, f32_to_bf16_bits, f16_bits_to_f32, f32_to_f16_bits,
    widen, narrow, reduce_ranks, bf16_ulp_diff,
)
from .collectives import (  # noqa: F401
    broadcast, gather, reduce, scatter, reduce_scatter, all_reduce,
    all_reduce_one_shot, all_reduce_two_shot, all_reduce_ring, all_reduce_ring_wire, all_gather,
    all_to_all, all_to_all_v, segment_elems,
)
from .moe import moe_route, moe_route_dedup, moe_dispatch, moe_combine, moe_permute_send  # noqa: F401
from .packets import (  # noqa: F401
    LL, LL128, packed_bytes, pack, unpack, all_reduce_packed,
)
