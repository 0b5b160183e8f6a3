"""Shapes, seeded weights and seeded prompts for the looped nGPT model.

Input recipe (the same for every consumer):

* Every weight matrix is stored ``[out, in]``. Its entries are standard
  normal draws that are then divided, row by row, by the row's L2 norm (rows
  of the ``[out, in]`` matrix, each of length ``in``).  For bf16 shapes the
  float32 result is rounded to nearest-even bf16.
* Tensors are numbered in a fixed order: the embedding, then for each physical
  layer its attention matrices (q, k, v, o) or its MLP matrices (gate, up,
  down), then the LM head.  Rows are drawn in blocks of ``ROW_BLOCK``; block
  ``b`` of tensor ``i`` uses ``PCG64(SeedSequence([seed, i, b]))``.  Blocks are
  independent streams, so generation can run on several host threads and the
  result does not depend on the thread count.
* Prompts are uniform integers in ``[0, vocab)`` from
  ``PCG64(SeedSequence([seed, PROMPT_STREAM, length]))``.

Nothing here computes any part of the model.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, replace

import numpy as np

ROW_BLOCK = 2048
PROMPT_STREAM = 0x70726F6D  # separates prompt streams from weight streams


@dataclass(frozen=True)
class Shape:
    """Integer shape of a looped nGPT model.

    ``n_in``, ``n_rec`` and ``n_out`` count *physical* layers (an attention
    sublayer and an MLP sublayer are one physical layer each).  Physical layers
    alternate attention and MLP with attention first; attention layer ``j``
    (counted over the whole stack) uses full causal attention when
    ``j % full_every == full_phase`` and sliding-window attention otherwise.
    """

    name: str
    d_model: int
    vocab: int
    n_heads: int
    head_dim: int
    n_kv_heads: int
    d_ff: int
    n_in: int
    n_rec: int
    n_out: int
    swa_window: int
    full_every: int = 4
    full_phase: int = 3
    dtype: str = "f32"  # "f32" or "bf16": storage type of weights and KV

    @property
    def n_layers(self) -> int:
        return self.n_in + self.n_rec + self.n_out

    @property
    def q_dim(self) -> int:
        return self.n_heads * self.head_dim

    @property
    def kv_dim(self) -> int:
        return self.n_kv_heads * self.head_dim

    def with_(self, **kw) -> "Shape":
        return replace(self, **kw)


# Tiny fp32 model: d=256, vocab 1024, 8 heads of 32, 2 KV heads, SwiGLU 1024,
# 2 + 4 + 2 physical layers, window 16, attention 3 SWA : 1 full.
TINY = Shape("tiny", 256, 1024, 8, 32, 2, 1024, 2, 4, 2, 16, dtype="f32")
# The same shape stored in bf16 (exercises the bf16 kernels with ring wrap).
TINY_BF16 = TINY.with_(name="tiny_bf16", dtype="bf16")
# 4B-shaped model: d=2560, vocab 131072, 20 heads x 128, 4 KV heads,
# SwiGLU 10240, 16 + 40 + 16 physical layers, window 4096.
DORY_4B = Shape("dory4b", 2560, 131072, 20, 128, 4, 10240, 16, 40, 16, 4096, dtype="bf16")

# Small bf16 shape with 128-wide heads (the 4B head shape) and a short window,
# so long chunks and ring wrap-around reach the bf16 attention kernels cheaply.
SMALL128 = Shape("small128", 512, 2048, 4, 128, 1, 1024, 2, 4, 2, 32, dtype="bf16")

SHAPES = {s.name: s for s in (TINY, TINY_BF16, DORY_4B, SMALL128)}


def layer_kinds(shape: Shape) -> list[str]:
    """'attn' or 'mlp' for each physical layer (which weight tensors exist)."""
    return ["attn" if l % 2 == 0 else "mlp" for l in range(shape.n_layers)]


def weight_specs(shape: Shape) -> list[tuple[str, tuple[int, int]]]:
    """(name, [out, in]) of every weight tensor, in generation order."""
    d = shape.d_model
    specs: list[tuple[str, tuple[int, int]]] = [("embed", (shape.vocab, d))]
    for l, kind in enumerate(layer_kinds(shape)):
        if kind == "attn":
            specs += [
                (f"L{l}.wq", (shape.q_dim, d)),
                (f"L{l}.wk", (shape.kv_dim, d)),
                (f"L{l}.wv", (shape.kv_dim, d)),
                (f"L{l}.wo", (d, shape.q_dim)),
            ]
        else:
            specs += [
                (f"L{l}.wg", (shape.d_ff, d)),
                (f"L{l}.wu", (shape.d_ff, d)),
                (f"L{l}.wdown", (d, shape.d_ff)),
            ]
    specs.append(("lm_head", (shape.vocab, d)))
    return specs


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 to nearest-even bfloat16; returns the uint16 bit patterns."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    rounding = ((u >> 16) & 1) + np.uint32(0x7FFF)
    return ((u + rounding) >> 16).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float32."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _block(seed: int, tidx: int, bidx: int, rows: int, cols: int, bf16: bool) -> np.ndarray:
    g = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, tidx, bidx])))
    a = g.standard_normal((rows, cols), dtype=np.float32)
    norm = np.sqrt(np.einsum("ij,ij->i", a, a, dtype=np.float64))
    a = (a / norm[:, None]).astype(np.float32)
    return f32_to_bf16_bits(a) if bf16 else a


def make_weights(shape: Shape, seed: int, threads: int | None = None) -> dict[str, np.ndarray]:
    """All weight tensors of ``shape``: float32 arrays for f32 shapes, uint16
    bf16 bit patterns for bf16 shapes, each ``[out, in]`` and C-contiguous."""
    bf16 = shape.dtype == "bf16"
    out: dict[str, np.ndarray] = {}
    jobs = []
    for tidx, (name, (rows, cols)) in enumerate(weight_specs(shape)):
        arr = np.empty((rows, cols), dtype=np.uint16 if bf16 else np.float32)
        out[name] = arr
        for bidx, r0 in enumerate(range(0, rows, ROW_BLOCK)):
            jobs.append((arr, tidx, bidx, r0, min(ROW_BLOCK, rows - r0), cols))

    def run(job):
        arr, tidx, bidx, r0, nr, cols = job
        arr[r0:r0 + nr] = _block(seed, tidx, bidx, nr, cols, bf16)

    n = threads or min(32, os.cpu_count() or 1)
    if n <= 1 or len(jobs) < 4:
        for j in jobs:
            run(j)
    else:
        with ThreadPoolExecutor(n) as ex:
            list(ex.map(run, jobs))
    return out


def make_prompt(seed: int, length: int, vocab: int) -> np.ndarray:
    """Uniform random token ids in [0, vocab), int32."""
    g = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, PROMPT_STREAM, length])))
    return g.integers(0, vocab, size=length, dtype=np.int64).astype(np.int32)
