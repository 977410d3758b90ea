"""Seeded synthetic workloads: shapes of the five denoising workloads and their inputs.

This module draws random numbers and rounds them to bf16; it holds none of the
attention-state arithmetic.  It imports nothing from the rest of the package
(so it never loads the CUDA library) and nothing from the oracle.  Tests, the
benchmark and the smoke check feed the SAME bytes it produces to both the CUDA
path and the CPU oracle.

Input recipe (one reading of the workload descriptions; the pages print no
data):
  * numpy ``Generator(PCG64(seed))``, seed 0 unless a case says otherwise;
  * step 1: Q, K, V drawn in that order, each ``[H][S][D]`` in C order, as
    float32 masters ``N(0,1)/sqrt(D)``;
  * step t >= 2: for Q, K, V in that order, ``master += sigma * N(0,1)``
    (an absolute perturbation, drawn independently per tensor);
  * the device input of a step is ``bf16(master)`` with round-to-nearest-even,
    delivered as raw uint16 bit patterns so both sides read identical bytes.

The latent grids (4x16x16 frames, 32x32 and 128x128 patch grids, 21x30x52
video latents) only fix S; tokens are flattened frame-major, row-major.
"""

from __future__ import annotations

import dataclasses
import math
from typing import Iterator, List, Optional, Tuple

import numpy as np

TILE = 128


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic workload: geometry, schedule and the plan family."""

    name: str
    H: int
    S: int
    D: int
    P: int                    # context partitions (1 in window mode)
    steps: int
    sigma: float              # per-step perturbation
    reuse: Tuple[int, ...]    # r values: KV partitions reused per query partition
    window: int = 0           # W > 0 selects the window + residual plan mode
    seed: int = 0

    @property
    def mode(self) -> str:
        return "window" if self.window > 0 else "proximity"


# The five workloads (1 sample each).  r is "reuse ratio x P".
WORKLOADS: List[Workload] = [
    Workload("tiny_4x16x16_h2_d64_p4", H=2, S=1024, D=64, P=4, steps=2,
             sigma=0.05, reuse=(2,)),
    Workload("dit_xl2_512_32x32_h16_d72_p8", H=16, S=1024, D=72, P=8, steps=4,
             sigma=0.05, reuse=(0, 2, 4, 6)),
    Workload("pixart_2048_128x128_h16_d72_p16", H=16, S=16384, D=72, P=16,
             steps=4, sigma=0.03, reuse=(8,)),
    Workload("video_21x30x52_h40_d128_p16", H=40, S=32760, D=128, P=16,
             steps=6, sigma=0.03, reuse=(0, 4, 8, 12)),
    Workload("window_128x128_h16_d72_w1024", H=16, S=16384, D=72, P=1,
             steps=4, sigma=0.03, reuse=(0,), window=1024),
]

BY_NAME = {w.name: w for w in WORKLOADS}


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 (nearest, ties to even); return uint16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns exactly to float32."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32)
            << np.uint32(16)).view(np.float32)


class InputStream:
    """Per-step Q, K, V for one workload (or any custom shape).

    ``next_step()`` returns ``(q, k, v)`` as uint16 bf16 bit arrays of shape
    ``[H][S][D]`` for steps 1, 2, ... in order.
    """

    def __init__(self, H: int, S: int, D: int, sigma: float, seed: int = 0,
                 scale: Optional[float] = None):
        self.H, self.S, self.D, self.sigma = H, S, D, sigma
        self.rng = np.random.Generator(np.random.PCG64(seed))
        self.scale = (1.0 / math.sqrt(D)) if scale is None else scale
        self.step = 0
        self.master: Optional[List[np.ndarray]] = None

    def next_step(self) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
        shape = (self.H, self.S, self.D)
        if self.master is None:
            self.master = []
            for _ in range(3):
                m = self.rng.standard_normal(shape, dtype=np.float32)
                m *= np.float32(self.scale)
                self.master.append(m)
        else:
            for m in self.master:
                noise = self.rng.standard_normal(shape, dtype=np.float32)
                noise *= np.float32(self.sigma)
                m += noise
        self.step += 1
        return tuple(f32_to_bf16_bits(m) for m in self.master)  # type: ignore


def stream_for(w: Workload) -> InputStream:
    return InputStream(w.H, w.S, w.D, w.sigma, seed=w.seed)


def steps(w: Workload, n: Optional[int] = None) -> Iterator[Tuple[np.ndarray, np.ndarray, np.ndarray]]:
    s = stream_for(w)
    for _ in range(w.steps if n is None else n):
        yield s.next_step()


def stress_inputs(H: int, S: int, D: int, kind: str, seed: int = 1):
    """Parity-only stress sets (never timed).

    ``"unit"``: Q, K ~ N(0,1) so logits have std ~ sqrt(D)/sqrt(D) = 1 after the
    1/sqrt(D) softmax scale.  ``"spiky"``: as ``unit`` plus a few keys aligned
    with some queries so that a handful of logits exceed 20, exercising the
    running-max subtraction.  Returns bf16 bit arrays.
    """
    rng = np.random.Generator(np.random.PCG64(seed))
    q = rng.standard_normal((H, S, D), dtype=np.float32)
    k = rng.standard_normal((H, S, D), dtype=np.float32)
    v = rng.standard_normal((H, S, D), dtype=np.float32)
    if kind == "spiky":
        n = max(1, S // 97)
        rows = rng.choice(S, size=n, replace=False)
        cols = rng.choice(S, size=n, replace=False)
        for h in range(H):
            for r, c in zip(rows, cols):
                # logit = q.k / sqrt(D); put |q||k|cos ~ 25 sqrt(D)
                k[h, c] = q[h, r] * np.float32(25.0 * math.sqrt(D) / float(np.dot(q[h, r], q[h, r])))
    elif kind != "unit":
        raise ValueError(kind)
    return f32_to_bf16_bits(q), f32_to_bf16_bits(k), f32_to_bf16_bits(v)
