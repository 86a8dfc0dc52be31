"""Tensor-parallel layout of the fused op's weights (host-side index logic).

TensorRT-LLM 深度工程实践, §4.1 Tensor Parallelism: the QKV and gate/up
projections are split by columns (each rank computes some output features for
every token), the output and down projections by rows (each rank holds a slice
of K and produces a partial sum that the ranks all-reduce). For the fused op:

* QKV: rank r of g takes query heads [r Hq/g, (r+1) Hq/g) and KV heads
  [r Hkv/g, (r+1) Hkv/g) -- whole heads, so its q/k/v outputs are its heads'
  outputs and attention needs no exchange. Every rank recomputes the norm of the
  full rows (cheap), so the fused op runs unchanged on the rank's W rows.
* SwiGLU: rank r takes gate rows [r I/g, (r+1) I/g) and the matching up rows
  I + the same range, so SiLU(gate) * up stays within the rank.
* Row-parallel partner (o_proj / down): rank r takes W columns (the K range)
  [r K/g, (r+1) K/g) and the matching slice of its input; the partial outputs
  are summed by fnl_tp_allreduce into the next fused op's x.
"""
from __future__ import annotations


def _span(n: int, rank: int, world: int, what: str) -> range:
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} of world {world}")
    if n % world:
        raise ValueError(f"{what} ({n}) is not divisible by the tensor-parallel size {world}")
    per = n // world
    return range(rank * per, (rank + 1) * per)


def qkv_rows(Hq: int, Hkv: int, D: int, rank: int, world: int) -> list:
    """Indices of the W rows (output features) of rank `rank`: its query heads,
    then its key heads, then its value heads, each head's D rows contiguous (the
    fused op's [Q | K | V] column order, reading R7)."""
    rows = []
    for h in _span(Hq, rank, world, "Hq"):
        rows.extend(range(h * D, (h + 1) * D))
    for h in _span(Hkv, rank, world, "Hkv"):
        rows.extend(range((Hq + h) * D, (Hq + h + 1) * D))
    for h in _span(Hkv, rank, world, "Hkv"):
        rows.extend(range((Hq + Hkv + h) * D, (Hq + Hkv + h + 1) * D))
    return rows


def swiglu_rows(I: int, rank: int, world: int) -> list:
    """Indices of the W rows of rank `rank` in the [gate; up] layout: its gate
    rows, then the matching up rows (so the rank's W is again [gate; up])."""
    span = _span(I, rank, world, "I")
    return list(span) + [I + j for j in span]


def row_split(K: int, rank: int, world: int) -> slice:
    """The K range of rank `rank` for a row-parallel projection (its slice of
    W's columns and of the input's features)."""
    span = _span(K, rank, world, "K")
    return slice(span.start, span.stop)
