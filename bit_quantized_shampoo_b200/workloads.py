"""Seeded synthetic workloads for the 4-bit Shampoo preconditioner step.

This module only *draws inputs*: parameter shapes and gradient matrices.  It
holds none of the method's arithmetic (no partitioning, no statistics, no
quantization), so both the CUDA path and the CPU oracle can take their inputs
from here without sharing any computation.

The five workloads are synthetic stand-ins for the layer families that the
"4-bit Shampoo for Memory-Efficient Network Training" abstract evaluates on
(image classifiers and language models); no dataset or trained weight is used.

Seeding: every gradient matrix is drawn from its own numpy
``Generator(PCG64(seed))`` with ``seed = 1000*config + 17*matrix + step``.
"""
from __future__ import annotations

import dataclasses
import numpy as np

__all__ = ["Workload", "WORKLOADS", "resnet50_conv_shapes", "gradient",
           "gradients", "u_like"]


def resnet50_conv_shapes() -> list[tuple[int, int]]:
    """The 53 convolution weights of a ResNet-50, reshaped out x (in*kh*kw).

    Built from the architecture's published stage layout: a 7x7 stem with 64
    filters, then four stages of bottleneck blocks (3, 4, 6, 3 blocks; widths
    64, 128, 256, 512; expansion 4), each stage's first block carrying a 1x1
    projection shortcut.  The fully connected head is not a convolution and
    is not included.
    """
    shapes = [(64, 3 * 7 * 7)]
    in_ch = 64
    for width, blocks in zip((64, 128, 256, 512), (3, 4, 6, 3)):
        for b in range(blocks):
            shapes.append((width, in_ch))            # 1x1 reduce
            shapes.append((width, width * 9))        # 3x3
            shapes.append((4 * width, width))        # 1x1 expand
            if b == 0:
                shapes.append((4 * width, in_ch))    # projection shortcut
            in_ch = 4 * width
    return shapes


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic workload: the parameter shapes and how G is drawn."""
    index: int                     # 1..5
    name: str
    shapes: tuple                  # ((rows, cols), ...)
    dist: str                      # "normal" | "normal_lowrank" | "student_t"
    scale: float                   # std (normal) or scale parameter (t)
    steps: int
    refresh_every: int             # T
    beta: float = 0.95
    eps: float = 1e-6
    bjorck_iters: int = 5
    max_block: int = 1024
    quant_block: int = 64

    @property
    def nparams(self) -> int:
        return len(self.shapes)


_TRANSFORMER_LAYER = ((768, 2304), (768, 768), (768, 3072), (3072, 768))

WORKLOADS = {
    1: Workload(1, "single 128x128 fp32 weight", ((128, 128),), "normal", 1.0,
                steps=10, refresh_every=1),
    2: Workload(2, "single 1024x1024 layer, N(0,0.02^2) + rank-16 term",
                ((1024, 1024),), "normal_lowrank", 0.02, steps=100,
                refresh_every=10),
    3: Workload(3, "ResNet-50 conv batch (53 matrices), Student-t nu=4 x 0.01",
                tuple(resnet50_conv_shapes()), "student_t", 0.01, steps=20,
                refresh_every=10),
    4: Workload(4, "transformer stack, 12 blocks of d=768",
                _TRANSFORMER_LAYER * 12, "normal", 0.01, steps=20,
                refresh_every=10),
    5: Workload(5, "Llama-style layers: 8 x 4096x11008 + 8 x 4096x4096",
                ((4096, 11008),) * 8 + ((4096, 4096),) * 8, "normal", 0.01,
                steps=3, refresh_every=1000),
}


def _seed(config: int, matrix: int, step: int) -> int:
    return 1000 * config + 17 * matrix + step


def _lowrank_factors(rows: int, cols: int, config: int, matrix: int):
    # Fixed across steps: drawn from step index -1 so it never collides with
    # a per-step stream.
    rng = np.random.Generator(np.random.PCG64(_seed(config, matrix, 0) + 999_983))
    a = rng.standard_normal((rows, 16))
    b = rng.standard_normal((cols, 16))
    return a, b


def gradient(w: Workload, matrix: int, step: int) -> np.ndarray:
    """G for parameter ``matrix`` at optimizer step ``step`` (1-based), fp32.

    normal         : N(0, scale^2)
    normal_lowrank : N(0, scale^2) fresh each step + 0.1 * A B^T / 4 with
                     A (rows x 16), B (cols x 16) ~ N(0, 1) fixed over steps
                     (per-entry std of that term is 0.1)
    student_t      : Student-t with 4 degrees of freedom times ``scale``
    """
    rows, cols = w.shapes[matrix]
    rng = np.random.Generator(np.random.PCG64(_seed(w.index, matrix, step)))
    if w.dist == "normal":
        g = rng.standard_normal((rows, cols), dtype=np.float32) * np.float32(w.scale)
    elif w.dist == "normal_lowrank":
        e = rng.standard_normal((rows, cols)) * w.scale
        a, b = _lowrank_factors(rows, cols, w.index, matrix)
        g = (e + 0.1 * (a @ b.T) / 4.0).astype(np.float32)
    elif w.dist == "student_t":
        g = (rng.standard_t(4.0, size=(rows, cols)) * w.scale).astype(np.float32)
    else:
        raise ValueError(w.dist)
    return np.ascontiguousarray(g, dtype=np.float32)


def gradients(w: Workload, step: int) -> list[np.ndarray]:
    return [gradient(w, i, step) for i in range(w.nparams)]


def u_like(d: int, seed: int, count: int = 1) -> np.ndarray:
    """U-shaped codec input: ``count`` d x d matrices with N(0, 1/d) entries,
    the entry distribution of a random orthogonal matrix's columns."""
    rng = np.random.Generator(np.random.PCG64(seed))
    return (rng.standard_normal((count, d, d), dtype=np.float32)
            * np.float32(1.0 / np.sqrt(d)))
