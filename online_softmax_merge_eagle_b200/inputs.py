"""Seeded synthetic inputs shared by the tests, the smoke check and the benchmark.

This module holds no attention arithmetic: it only draws random tensors and
document lengths, so that the CUDA path and the CPU oracle see the same data.

Recipe (stated once, used everywhere):
  * q, cache_k, cache_v, grad_out ~ N(0, 1), drawn in that order in fp32 from
    ``torch.Generator().manual_seed(seed)`` on the CPU, then rounded to the
    compute dtype (bf16 by round-to-nearest-even).  The oracle consumes the
    same rounded values widened to fp64.
  * packed documents: lengths from ``numpy.random.default_rng(seed).integers
    (lo, hi + 1)`` drawn until they reach the total, the last one truncated.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch


@dataclass(frozen=True)
class Workload:
    """One synthetic workload: shapes, dtype and mask structure."""
    name: str
    B: int
    Tq: int
    H: int
    D: int
    num_blocks: int
    dtype: torch.dtype
    Tk: int | None = None          # block-0 key length (defaults to Tq)
    q_pos_offset: int = 0
    k_pos_offset: int = 0
    doc_lengths: tuple[int, ...] | None = None
    backward: bool = True
    chunks: int = 0                # >0: block 0 processed as this many chunks (zig-zag pairs)
    single_launch: bool = False    # chunked forward: one launch per emulated rank
    seed: int = 0
    notes: str = ""

    @property
    def tk(self) -> int:
        return self.Tq if self.Tk is None else self.Tk

    @property
    def scale(self) -> float:
        return self.D ** -0.5


def doc_lengths(total: int, lo: int, hi: int, seed: int = 0) -> tuple[int, ...]:
    """Document lengths ~ Uniform[lo, hi] (integers), drawn until they sum to
    ``total``; the last document is truncated to fit."""
    rng = np.random.default_rng(seed)
    out: list[int] = []
    acc = 0
    while acc < total:
        n = int(rng.integers(lo, hi + 1))
        n = min(n, total - acc)
        out.append(n)
        acc += n
    return tuple(out)


def doc_lengths_multiple(total: int, lo: int, hi: int, multiple: int,
                         seed: int = 0) -> tuple[int, ...]:
    """doc_lengths(total, lo, hi, seed) with every length rounded down to a
    multiple of ``multiple`` (zero-length documents dropped) and the remainder
    added to the last document; ``total`` must be a multiple of ``multiple``."""
    assert total % multiple == 0
    out = [n // multiple * multiple for n in doc_lengths(total, lo, hi, seed)]
    out = [n for n in out if n > 0]
    out[-1] += total - sum(out)
    return tuple(out)


def cu_seqlens(lengths) -> np.ndarray:
    """int32 [num_docs + 1] prefix sums of document lengths."""
    return np.concatenate([[0], np.cumsum(np.asarray(lengths, dtype=np.int64))]).astype(np.int32)


WORKLOADS: dict[str, Workload] = {
    "tiny_fp32": Workload("tiny_fp32", B=1, Tq=256, H=4, D=64, num_blocks=2, dtype=torch.float32,
                          notes="single document, scale 1/8"),
    "dense_bf16": Workload("dense_bf16", B=2, Tq=8192, H=32, D=128, num_blocks=8,
                           dtype=torch.bfloat16, notes="single document per batch row"),
    "dense_bf16_h8": Workload("dense_bf16_h8", B=1, Tq=8192, H=8, D=128, num_blocks=8,
                              dtype=torch.bfloat16,
                              notes="dense_bf16 with B=1, H=8 (one eighth): the ncu capture size"),
    "varlen_bf16": Workload("varlen_bf16", B=1, Tq=32768, H=32, D=128, num_blocks=4,
                            dtype=torch.bfloat16, doc_lengths=doc_lengths(32768, 256, 8192, 0),
                            notes="packed documents, Uniform[256, 8192] lengths, seed 0"),
    "chunked_bf16": Workload("chunked_bf16", B=1, Tq=131072, H=8, D=128, num_blocks=4,
                             dtype=torch.bfloat16, backward=False, chunks=16,
                             notes="block 0 as 16 zig-zag chunks (emulated cp=8), merged"),
    "chunked_single_bf16": Workload("chunked_single_bf16", B=1, Tq=131072, H=8, D=128,
                                    num_blocks=4, dtype=torch.bfloat16, backward=False, chunks=16,
                                    single_launch=True,
                                    notes="chunked_bf16 with one forward launch per emulated rank"),
    "chunked_bwd_bf16": Workload("chunked_bwd_bf16", B=1, Tq=131072, H=8, D=128, num_blocks=4,
                                 dtype=torch.bfloat16, chunks=16,
                                 notes="chunked_bf16 forward + the zig-zag chunked backward"),
    "chunked_bwd_single_bf16": Workload("chunked_bwd_single_bf16", B=1, Tq=131072, H=8, D=128,
                                        num_blocks=4, dtype=torch.bfloat16, chunks=16,
                                        single_launch=True,
                                        notes="chunked_bwd_bf16 with one forward and one "
                                              "backward launch per emulated rank"),
    "varlen_zigzag_bf16": Workload("varlen_zigzag_bf16", B=1, Tq=32768, H=32, D=128,
                                   num_blocks=4, dtype=torch.bfloat16, chunks=16,
                                   doc_lengths=doc_lengths_multiple(32768, 256, 8192, 16, 0),
                                   notes="varlen_bf16's documents rounded to multiples of 16, "
                                         "each cut into 16 zig-zag chunks (emulated cp=8)"),
    "varlen_zigzag_single_bf16": Workload("varlen_zigzag_single_bf16", B=1, Tq=32768, H=32,
                                          D=128, num_blocks=4, dtype=torch.bfloat16, chunks=16,
                                          doc_lengths=doc_lengths_multiple(32768, 256, 8192, 16,
                                                                           0),
                                          single_launch=True,
                                          notes="varlen_zigzag_bf16 with one forward and one "
                                                "backward launch per emulated rank over every "
                                                "document's chunks"),
    "frozen_target_bf16": Workload("frozen_target_bf16", B=1, Tq=8192, H=32, D=128,
                                   num_blocks=1, dtype=torch.bfloat16, Tk=65536,
                                   q_pos_offset=57344, backward=False,
                                   notes="query shard at global offset 57344 vs 65536 keys"),
}


def make_tensors(B: int, Tq: int, H: int, D: int, num_blocks: int, dtype: torch.dtype,
                 Tk: int | None = None, seed: int = 0, grad: bool = True,
                 device: str | torch.device = "cpu") -> dict[str, torch.Tensor]:
    """q [B,Tq,H,D], cache_k / cache_v [B,NB,Tk,H,D], grad_out [B,Tq,H,D]."""
    Tk = Tq if Tk is None else Tk
    g = torch.Generator().manual_seed(seed)
    out = {}
    out["q"] = torch.randn((B, Tq, H, D), generator=g, dtype=torch.float32).to(dtype)
    out["cache_k"] = torch.randn((B, num_blocks, Tk, H, D), generator=g,
                                 dtype=torch.float32).to(dtype)
    out["cache_v"] = torch.randn((B, num_blocks, Tk, H, D), generator=g,
                                 dtype=torch.float32).to(dtype)
    if grad:
        out["grad_out"] = torch.randn((B, Tq, H, D), generator=g, dtype=torch.float32).to(dtype)
    if str(device) != "cpu":
        out = {k: v.to(device) for k, v in out.items()}
    return out


def make_workload(w: Workload, device: str | torch.device = "cpu") -> dict:
    """Tensors plus the mask description of workload ``w``."""
    t = make_tensors(w.B, w.Tq, w.H, w.D, w.num_blocks, w.dtype, Tk=w.tk, seed=w.seed,
                     grad=w.backward, device=device)
    t["cu_seqlens"] = None if w.doc_lengths is None else cu_seqlens(w.doc_lengths)
    t["max_seqlen"] = None if w.doc_lengths is None else max(w.doc_lengths)
    t["scale"] = w.scale
    t["q_pos_offset"] = w.q_pos_offset
    t["k_pos_offset"] = w.k_pos_offset
    return t
