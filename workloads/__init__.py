"""Seeded synthetic inputs for the virtual-rank collectives.

This module is shared by the oracle side (``oracle/``, the tests) and the
device side (``bench.py``, the GPU tests).  It holds only random-number
recipes, shapes and dtype packing; it contains none of the collectives'
arithmetic (no reduction, no concatenation, no routing scan, no packet
encoding), so neither side can inherit a mistake from the other through it.

Conventions
-----------
* One ``numpy.random.Generator(PCG64(seed))`` per (workload, rank), seed
  ``20261202 + 1000 * workload + rank``.  Rank ``r`` of a workload therefore
  gets the same values whatever the number of ranks or the order of calls.
* ``bf16`` arrays are carried as ``uint16`` bit patterns; the fp32 -> bf16 step
  of the input recipe is torch's CPU conversion (round to nearest even), a
  library routine, so the recipe itself does no rounding arithmetic.
* ``fp16`` arrays are carried as ``uint16`` bit patterns too.
* Sizes follow the workloads the pages describe:
  - TP decode all_reduce after RowParallelLinear (collectives tutorial
    gsyq.cn/news/307221, section 6.3/6.4.1) on [tokens, hidden] activations;
  - the 160 KB, 4-GPU, A/B/C/D example of "From NCCL Ring LL to PCIe IPC
    AllReduce" (section "Pro5000 ?");
  - the sequence-parallel AllGather -> local -> ReduceScatter chain
    (tutorial sections 5.3 and 7.3) and the vocab logits gather to rank 0
    (tutorial section 2.2.1);
  - MoE dispatch/combine over expert-parallel ranks (tutorial section 8.4);
  - LL / LL128 packets ("From NCCL Ring LL ...", "Traditional LL Protocols").
"""
from __future__ import annotations

import concurrent.futures as _cf
import math

import numpy as np

SEED_BASE = 20261202

# Workload ids (used only to derive seeds).
W_TWOSHOT_160K = 1
W_TP_DECODE = 2
W_SP_PREFILL = 3
W_MOE = 4
W_LL_SWEEP = 5
W_MISC = 9  # unit tests and fuzzing

TP_DECODE_TOKENS = (1, 8, 32, 128, 256)
TP_DECODE_HIDDEN = (4096, 7168)
VOCAB = 128256  # vocab of the sampled-token-id broadcast


def rng(workload: int, rank: int, salt: int = 0) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(SEED_BASE + 1000 * workload + rank + 7919 * salt))


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns through torch's CPU conversion (input recipe only)."""
    import torch

    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16).copy()


def f32_to_f16_bits(a: np.ndarray) -> np.ndarray:
    import torch

    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t.to(torch.float16).view(torch.int16).numpy().view(np.uint16).copy()


def _normal(g: np.random.Generator, n: int, std: float = 1.0) -> np.ndarray:
    a = g.standard_normal(n, dtype=np.float32)
    if std != 1.0:
        a *= np.float32(std)
    return a


def _uniform(g: np.random.Generator, n: int) -> np.ndarray:
    return g.uniform(-1.0, 1.0, n).astype(np.float32)


def _per_rank(fn, nranks: int, parallel: bool):
    if not parallel or nranks == 1:
        return [fn(r) for r in range(nranks)]
    with _cf.ThreadPoolExecutor(max_workers=min(nranks, 8)) as ex:
        return list(ex.map(fn, range(nranks)))


def ranks_values(workload: int, nranks: int, count: int, dtype: str = "bf16",
                 dist: str = "normal", std: float = 1.0, salt: int = 0,
                 parallel: bool = True) -> list[np.ndarray]:
    """Per-rank 1-D inputs of ``count`` elements.

    dtype: "bf16" / "fp16" (uint16 bits), "fp32" (float32), "int32".
    dist:  "normal" (mean 0, standard deviation ``std``), "uniform" ([-1, 1]),
           "randint" (int32 in [0, VOCAB)).
    """

    def one(r: int) -> np.ndarray:
        g = rng(workload, r, salt)
        if dtype == "int32":
            return g.integers(0, VOCAB, count, dtype=np.int32)
        a = _normal(g, count, std) if dist == "normal" else _uniform(g, count)
        if dtype == "bf16":
            return f32_to_bf16_bits(a)
        if dtype == "fp16":
            return f32_to_f16_bits(a)
        if dtype == "fp32":
            return a
        raise ValueError(dtype)

    return _per_rank(one, nranks, parallel and count >= (1 << 20))


# --------------------------------------------------------------------------
# The five workloads.
# --------------------------------------------------------------------------

def twoshot_160k(nranks: int = 4, count: int = 81920) -> list[np.ndarray]:
    """all_reduce input: 4 ranks x 160 KB of bf16, uniform[-1, 1]."""
    return ranks_values(W_TWOSHOT_160K, nranks, count, "bf16", "uniform")


def tp_decode_shapes() -> list[tuple[int, int]]:
    return [(t, h) for h in TP_DECODE_HIDDEN for t in TP_DECODE_TOKENS]


def tp_decode(tokens: int, hidden: int, nranks: int = 8, elems: int | None = None) -> list[np.ndarray]:
    """Per-rank RowParallelLinear partial outputs, bf16 [tokens, hidden], N(0,1).

    ``elems`` (optional) returns only the first ``elems`` values of each
    rank's input: a prefix sample of the same workload."""
    salt = tokens * 100003 + hidden
    return ranks_values(W_TP_DECODE, nranks, tokens * hidden if elems is None else elems, "bf16", "normal",
                        salt=salt)


def sampled_token_ids(nranks: int = 8, count: int = 256) -> list[np.ndarray]:
    """int32 sampled_token_ids on every rank (only the source's values matter)."""
    return ranks_values(W_TP_DECODE, nranks, count, "int32", salt=1)


def sp_allgather(nranks: int = 8, rows: int = 1024, cols: int = 8192) -> list[np.ndarray]:
    return ranks_values(W_SP_PREFILL, nranks, rows * cols, "bf16", "normal", salt=1)


def sp_reduce_scatter(nranks: int = 8, rows: int = 8192, cols: int = 8192) -> list[np.ndarray]:
    return ranks_values(W_SP_PREFILL, nranks, rows * cols, "bf16", "normal", salt=2)


def logits_shards(nranks: int = 8, rows: int = 256, cols: int = 16032) -> list[np.ndarray]:
    """fp32 vocab-parallel logits shards, N(0, 2) read as standard deviation 2."""
    return ranks_values(W_SP_PREFILL, nranks, rows * cols, "fp32", "normal", std=2.0, salt=3)


def ll_message(nbytes: int, nranks: int = 8, elems: int | None = None) -> list[np.ndarray]:
    """bf16 uniform[-1, 1] payloads of ``nbytes`` bytes (uint16 bits); with
    ``elems``, only the first ``elems`` values of each (a prefix sample)."""
    return ranks_values(W_LL_SWEEP, nranks, nbytes // 2 if elems is None else elems, "bf16", "uniform",
                        salt=nbytes.bit_length())


# --------------------------------------------------------------------------
# MoE routing inputs.  The collective path starts at (topk_ids, topk_w); the
# softmax / top-k below only manufacture those inputs, in float64 on the host.
# --------------------------------------------------------------------------

def zipf_expert_bias(n_experts: int, s: float = 1.1) -> np.ndarray:
    """log p_e with p_e proportional to rank_e^-s and rank_e a seeded permutation."""
    g = rng(W_MOE, 999)
    ranks = g.permutation(n_experts) + 1
    p = ranks.astype(np.float64) ** (-s)
    p /= p.sum()
    return np.log(p)


def moe_routing(tokens: int, n_experts: int, topk: int, nranks: int,
                renormalize: bool = True, zipf_s: float = 1.1):
    """Per-rank (topk_ids int32 [T,K], topk_w float32 [T,K]).

    logits = N(0,1) + log Zipf bias; probabilities by softmax; the K largest
    probabilities (ties to the lower expert id) listed in descending order;
    weights renormalised over the K chosen (``renormalize``).
    """
    bias = zipf_expert_bias(n_experts, zipf_s)
    ids, ws = [], []
    for r in range(nranks):
        g = rng(W_MOE, r, salt=1)
        logits = g.standard_normal((tokens, n_experts)) + bias[None, :]
        logits -= logits.max(axis=1, keepdims=True)
        p = np.exp(logits)
        p /= p.sum(axis=1, keepdims=True)
        # stable sort on -p: equal probabilities keep ascending expert id
        order = np.argsort(-p, axis=1, kind="stable")[:, :topk]
        pk = np.take_along_axis(p, order, axis=1)
        if renormalize:
            pk = pk / pk.sum(axis=1, keepdims=True)
        ids.append(order.astype(np.int32))
        ws.append(pk.astype(np.float32))
    return ids, ws


def moe_tokens(tokens: int, hidden: int, nranks: int) -> list[np.ndarray]:
    """bf16 [tokens, hidden] N(0,1) token activations per rank (flattened)."""
    return ranks_values(W_MOE, nranks, tokens * hidden, "bf16", "normal", salt=2)


def random_splits(nranks: int, max_rows: int, workload: int = W_MISC, salt: int = 0) -> np.ndarray:
    """A ragged [N, N] send-count matrix (rows s -> d), zeros included."""
    g = rng(workload, 0, salt=salt + 17)
    m = g.integers(0, max_rows + 1, size=(nranks, nranks))
    m[g.random((nranks, nranks)) < 0.15] = 0
    return m.astype(np.int64)


def ceil_div(a: int, b: int) -> int:
    return -(-a // b)


__all__ = [n for n in dir() if not n.startswith("_") and n not in ("np", "math")]
