"""Seeded synthetic inputs shared by the CPU oracle and the CUDA path.

This module draws random numbers and describes shapes.  It holds none of the
looped model's arithmetic (no quantiser, no norm, no attention): the oracle and
the CUDA library each implement that on their own from these draws.

Sources of the workload shapes:
  * "Dynamic-L Inference", "Measured Performance Spectrum" (32-token prompt,
    32 decode tokens, L in {2,4,8,16,32}) and "L-Aware Batching" (per-lane L).
  * "Benchmark Comparison" (measured benchmarks) section 1 (seq_len 128, L=8,
    no logits) and section 2 (shared 1024-token prefix).
  * The model definitions of the five workloads: RMSNorm eps 1e-5, SwiGLU FFN,
    RoPE base 1e4, weights N(0, 0.02) drawn from seed 0, symmetric INT4 with an
    FP16 scale per group of 32 or 128, or BF16 weights.

Weight draw order (one PCG64 stream, float64, scaled by 0.02):
  embed [V, d];
  then for every pre block, then for every loop-body layer:
      wqkv [3d, d]  (rows q | k | v),  wo [d, d],  wg [F, d],  wu [F, d],  wd [d, F];
  then head [V, d].
RMSNorm gains are not drawn: they are ones, unless a test asks for random gains
from their own seed.
"""
from __future__ import annotations

from dataclasses import dataclass, replace
from typing import Iterator, Tuple

import numpy as np

INT4 = "int4"
BF16 = "bf16"


@dataclass(frozen=True)
class ModelShape:
    vocab: int
    d: int
    n_heads: int
    ffn: int
    n_pre: int
    n_loop_layers: int
    fmt_pre: str
    fmt_loop: str
    fmt_embed_head: str
    group: int
    rms_eps: float = 1e-5
    rope_base: float = 1e4

    @property
    def head_dim(self) -> int:
        return self.d // self.n_heads

    def fmt_of(self, name: str) -> str:
        if name in ("embed", "head"):
            return self.fmt_embed_head
        if name.startswith("pre"):
            return self.fmt_pre
        return self.fmt_loop


# Tiny looped LM: vocab 512, d 128, 4 heads x 32, FFN 512, 1 pre + 1 loop, INT4 g32.
TINY = ModelShape(512, 128, 4, 512, 1, 1, INT4, INT4, INT4, 32)
# 407M-class: vocab 50257, d 1024, 16 x 64, FFN 4096, 2 pre + 1 loop, INT4 g128.
M407 = ModelShape(50257, 1024, 16, 4096, 2, 1, INT4, INT4, INT4, 128)
# Same model with an unquantised (BF16) loop block.
M407_BF16LOOP = replace(M407, fmt_loop=BF16)
# 1.4B-class shared-prefix model: vocab 49152, d 2048, 16 x 128, FFN 5632,
# no pre blocks, 24-layer loop body, BF16 everywhere.
M1B4 = ModelShape(49152, 2048, 16, 5632, 0, 24, BF16, BF16, BF16, 0)

# The same layout at test size (every structural feature of M1B4: BF16
# everywhere, 128-wide heads, no pre blocks, a multi-layer loop body, a vocab
# and FFN that are not multiples of the 128-row tile).
M1B4_MINI = ModelShape(4000, 256, 2, 704, 0, 3, BF16, BF16, BF16, 0)

SHAPES = {"tiny": TINY, "m407": M407, "m407_bf16loop": M407_BF16LOOP, "m1b4": M1B4, "m1b4_mini": M1B4_MINI}


def matrix_shapes(shape: ModelShape) -> list[Tuple[str, Tuple[int, int]]]:
    """Names and [rows, cols] of every weight matrix, in draw order."""
    d, F, V = shape.d, shape.ffn, shape.vocab
    out = [("embed", (V, d))]
    blocks = [f"pre{b}" for b in range(shape.n_pre)] + [f"loop{m}" for m in range(shape.n_loop_layers)]
    for blk in blocks:
        out += [(f"{blk}.wqkv", (3 * d, d)), (f"{blk}.wo", (d, d)), (f"{blk}.wg", (F, d)),
                (f"{blk}.wu", (F, d)), (f"{blk}.wd", (d, F))]
    out.append(("head", (V, d)))
    return out


def gain_names(shape: ModelShape) -> list[str]:
    blocks = [f"pre{b}" for b in range(shape.n_pre)] + [f"loop{m}" for m in range(shape.n_loop_layers)]
    names = []
    for blk in blocks:
        names += [f"{blk}.g1", f"{blk}.g2"]
    names.append("final.g")
    return names


def master_weights(shape: ModelShape, seed: int = 0) -> Iterator[Tuple[str, np.ndarray]]:
    """Yield (name, float64 matrix) in draw order: N(0, 0.02) from PCG64(seed)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    for name, (r, c) in matrix_shapes(shape):
        yield name, rng.standard_normal((r, c)) * 0.02


def gains(shape: ModelShape, random_seed: int | None = None) -> dict[str, np.ndarray]:
    """RMSNorm gains: ones, or 1 + 0.1 N(0,1) from PCG64(random_seed)."""
    if random_seed is None:
        return {n: np.ones(shape.d) for n in gain_names(shape)}
    rng = np.random.Generator(np.random.PCG64(random_seed))
    return {n: 1.0 + 0.1 * rng.standard_normal(shape.d) for n in gain_names(shape)}


def prompts(n_lanes: int, T: int, vocab: int, seed: int = 1) -> np.ndarray:
    """Uniform-random token ids, int32 [n_lanes, T]."""
    rng = np.random.Generator(np.random.PCG64(seed))
    return rng.integers(0, vocab, (n_lanes, T)).astype(np.int32)


def poisson_L(n_lanes: int, mean: float = 8.0, lo: int = 2, hi: int = 32, seed: int = 2) -> np.ndarray:
    """Per-lane loop counts: Poisson(mean) clamped to [lo, hi], int32 [n_lanes]."""
    rng = np.random.Generator(np.random.PCG64(seed))
    return np.clip(rng.poisson(mean, n_lanes), lo, hi).astype(np.int32)


def uniform_L(n_lanes: int, lo: int = 1, hi: int = 4, seed: int = 2) -> np.ndarray:
    """Per-lane loop counts uniform in {lo..hi}, int32 [n_lanes]."""
    rng = np.random.Generator(np.random.PCG64(seed))
    return rng.integers(lo, hi + 1, n_lanes).astype(np.int32)


def random_vectors(shape: Tuple[int, ...], seed: int, scale: float = 1.0) -> np.ndarray:
    """Plain N(0, scale^2) float64 draws for kernel-level tests."""
    rng = np.random.Generator(np.random.PCG64(seed))
    return rng.standard_normal(shape) * scale


@dataclass(frozen=True)
class Workload:
    """A decode or scoring workload on one model shape."""
    name: str
    shape: ModelShape
    n_lanes: int
    prompt_len: int
    n_new: int
    per_lane_L: Tuple[int, ...]
    ee_tau: float = 0.0
    ee_min_L: int = 2
    ee_patience: int = 0
    ee_peek_every: int = 1
    shared_prefix: int = 0


def workload(name: str) -> Workload:
    """The named workloads, with their seeded per-lane L draws."""
    if name == "tiny":
        return Workload("tiny", TINY, 2, 16, 8, (2, 4))
    if name == "m407_score":
        return Workload("m407_score", M407, 1, 128, 0, (8,))
    if name.startswith("m407_decode_L"):
        L = int(name.rsplit("L", 1)[1])
        return Workload(name, M407, 1, 32, 32, (L,))
    if name.startswith("m407_bf16loop_decode_L"):
        L = int(name.rsplit("L", 1)[1])
        return Workload(name, M407_BF16LOOP, 1, 32, 32, (L,))
    if name == "m407_cdb64":
        return Workload("m407_cdb64", M407, 64, 512, 128, tuple(int(x) for x in poisson_L(64)),
                        ee_tau=0.1, ee_min_L=2, ee_patience=2, ee_peek_every=1)
    if name == "m1b4_prefix256":
        return Workload("m1b4_prefix256", M1B4, 256, 64, 64, tuple(int(x) for x in uniform_L(256)),
                        shared_prefix=1024)
    if name == "m1b4_mini_prefix":
        return Workload("m1b4_mini_prefix", M1B4_MINI, 4, 8, 4, tuple(int(x) for x in uniform_L(4)),
                        shared_prefix=96)
    raise KeyError(name)


def prefix_prompts(wl: Workload) -> Tuple[np.ndarray, np.ndarray]:
    """Shared-prefix workloads: the common prefix (int32 [shared_prefix], from
    PCG64(1)) and each lane's suffix (int32 [n_lanes, prompt_len], from
    PCG64(3)); lane i's prompt is prefix + suffix[i]."""
    pre = prompts(1, wl.shared_prefix, wl.shape.vocab, seed=1)[0]
    suf = prompts(wl.n_lanes, wl.prompt_len, wl.shape.vocab, seed=3)
    return pre, suf
