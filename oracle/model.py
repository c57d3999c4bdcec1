"""Oracle: the weight-shared looped transformer in float64.

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).

Pipeline ("Benchmark Comparison" (vs generic runtimes), "Where Generic Runtimes
Lose On Looped Checkpoints"):  embed -> pre blocks -> shared loop block x L -> head.
L is a runtime argument over the same weights ("Dynamic-L Inference", "The Core
Idea").  Every pre block and every loop iteration keeps its own K/V, i.e. each
iteration is its own "layer" of cache ("Benchmark Comparison" (measured
benchmarks), section 9: storage for "2 pre + 8 loop" blocks; "CLI Reference",
TINYLOOP_KV_H_MODE: one buffer per layer).

Block math (workload model definitions; the pages do not spell it out):
  a = RMSNorm(x; g1, eps) ; [q|k|v] = a Wqkv^T ; RoPE(q, k, position)
  o = causal softmax(q k^T / sqrt(hd)) v over this cache slot, per head
  x = x + o Wo^T
  b = RMSNorm(x; g2, eps) ; x = x + (silu(b Wg^T) * (b Wu^T)) Wd^T
  logits = RMSNorm(h; g_final, eps) Whead^T
Readings (where the pages are silent): pre-norm blocks, no biases, every head
has its own K/V, NeoX "rotate-half" RoPE pairing (i, i + hd/2) with angle
p * base^(-2i/hd) at the absolute position p (the same p at every iteration),
no re-injection of the embedding between iterations, untied head.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

from synthetic import ModelShape, INT4, BF16
from . import quant


# ---------------------------------------------------------------- weights ----

@dataclass
class BlockWeights:
    g1: np.ndarray
    wqkv: np.ndarray
    wo: np.ndarray
    g2: np.ndarray
    wg: np.ndarray
    wu: np.ndarray
    wd: np.ndarray


@dataclass
class Weights:
    shape: ModelShape
    embed: np.ndarray
    pre: list
    loop: list
    g_final: np.ndarray
    head: np.ndarray
    int4: dict = field(default_factory=dict)   # name -> (packed, scales) for INT4 matrices


def effective_matrix(name: str, w: np.ndarray, shape: ModelShape, keep: dict | None = None) -> np.ndarray:
    """The matrix the model computes with: INT4 dequant of the master, or its BF16 rounding."""
    fmt = shape.fmt_of(name)
    if fmt == INT4:
        packed, scale = quant.quantize_int4(w, shape.group)
        if keep is not None:
            keep[name] = (packed, scale)
        return quant.dequantize_int4(packed, scale, shape.group)
    if fmt == BF16:
        return quant.round_bf16(w)
    raise ValueError(fmt)


def build_weights(shape: ModelShape, masters, gains: dict, keep_int4: bool = False) -> Weights:
    """masters: iterable of (name, float64 master) in draw order; gains: name -> [d]."""
    eff = {}
    keep = {} if keep_int4 else None
    for name, w in masters:
        eff[name] = effective_matrix(name, w, shape, keep)

    def blk(p):
        return BlockWeights(gains[f"{p}.g1"], eff[f"{p}.wqkv"], eff[f"{p}.wo"], gains[f"{p}.g2"],
                            eff[f"{p}.wg"], eff[f"{p}.wu"], eff[f"{p}.wd"])

    return Weights(shape, eff["embed"], [blk(f"pre{b}") for b in range(shape.n_pre)],
                   [blk(f"loop{m}") for m in range(shape.n_loop_layers)], gains["final.g"],
                   eff["head"], keep or {})


# ------------------------------------------------------------- primitives ----

def rmsnorm(x: np.ndarray, g: np.ndarray, eps: float) -> np.ndarray:
    """x / sqrt(mean(x^2) + eps) * g over the last axis."""
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps) * g


def silu(x: np.ndarray) -> np.ndarray:
    return x / (1.0 + np.exp(-x))


def rope_cos_sin(pos: np.ndarray, hd: int, base: float):
    """cos/sin [T, hd/2] of angle p * base^(-2i/hd)."""
    i = np.arange(hd // 2, dtype=np.float64)
    theta = base ** (-2.0 * i / hd)
    ang = np.asarray(pos, dtype=np.float64)[:, None] * theta[None, :]
    return np.cos(ang), np.sin(ang)


def apply_rope(x: np.ndarray, pos: np.ndarray, base: float) -> np.ndarray:
    """x [T, H, hd]: rotate pairs (i, i + hd/2) by the angle of position pos[t]."""
    hd = x.shape[-1]
    half = hd // 2
    c, s = rope_cos_sin(pos, hd, base)
    c, s = c[:, None, :], s[:, None, :]
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def attend(q: np.ndarray, K: np.ndarray, V: np.ndarray, q_pos: np.ndarray, k_pos: np.ndarray) -> np.ndarray:
    """Causal multi-head attention. q [T,H,hd], K/V [S,H,hd]; key s is visible to
    query t iff k_pos[s] <= q_pos[t].  Max-subtracted softmax, scale 1/sqrt(hd)."""
    hd = q.shape[-1]
    # per head: scores = Q K^T [T, S], then softmax(scores) V [T, hd] (batched matrix products over heads)
    scores = np.matmul(q.transpose(1, 0, 2), K.transpose(1, 2, 0)) / np.sqrt(hd)
    visible = k_pos[None, :] <= q_pos[:, None]
    scores = np.where(visible[None], scores, -np.inf)
    scores = scores - scores.max(axis=-1, keepdims=True)
    p = np.exp(scores)
    p = p / p.sum(axis=-1, keepdims=True)
    return np.matmul(p, V.transpose(1, 0, 2)).transpose(1, 0, 2)


# ---------------------------------------------------------------- KV cache ----

class KVCache:
    """Per-lane cache: one (K, V) slab per slot; a slot is a pre block ("pre", b)
    or a loop iteration and body layer ("loop", l, m), l counted from 1.

    deep_fallback (the reading for a lane whose L rises, e.g. after an L-warmup
    phase; the pages do not say what a deeper iteration attends to at positions
    computed shallower): a position with no entry in ("loop", l, m) is read from
    the deepest iteration l' < l that holds it at the same body layer m."""

    def __init__(self, shape: ModelShape, max_seq: int, deep_fallback: bool = False):
        self.shape = shape
        self.max_seq = max_seq
        self.slots: dict = {}
        self.deep_fallback = deep_fallback

    def slab(self, slot):
        if slot not in self.slots:
            H, hd = self.shape.n_heads, self.shape.head_dim
            self.slots[slot] = (np.zeros((self.max_seq, H, hd)), np.zeros((self.max_seq, H, hd)),
                                np.zeros(self.max_seq, dtype=bool))
        return self.slots[slot]

    def write(self, slot, pos, k, v):
        K, V, filled = self.slab(slot)
        K[pos] = k
        V[pos] = v
        filled[pos] = True

    def read_upto(self, slot, p_max: int):
        """K, V, positions of all filled entries at positions <= p_max (with
        deep_fallback, loop-slot gaps filled from shallower iterations)."""
        K, V, filled = self.slab(slot)
        if not (self.deep_fallback and slot[0] == "loop"):
            idx = np.nonzero(filled[: p_max + 1])[0]
            return K[idx], V[idx], idx
        _, l, m = slot
        Kf, Vf, have = K[: p_max + 1].copy(), V[: p_max + 1].copy(), filled[: p_max + 1].copy()
        for lower in range(l - 1, 0, -1):  # deepest first
            if ("loop", lower, m) not in self.slots:
                continue
            Kl, Vl, fl = self.slots[("loop", lower, m)]
            take = ~have & fl[: p_max + 1]
            Kf[take], Vf[take] = Kl[: p_max + 1][take], Vl[: p_max + 1][take]
            have |= take
        idx = np.nonzero(have)[0]
        return Kf[idx], Vf[idx], idx


# ------------------------------------------------------------------ blocks ----

def block(bw: BlockWeights, shape: ModelShape, x: np.ndarray, pos: np.ndarray, cache: KVCache, slot) -> np.ndarray:
    """One transformer block on rows x [T, d] at positions pos [T] (ascending).
    Appends this block's K/V for the rows, then attends over the slot."""
    d, H, hd, eps = shape.d, shape.n_heads, shape.head_dim, shape.rms_eps
    a = rmsnorm(x, bw.g1, eps)
    qkv = a @ bw.wqkv.T
    q = qkv[:, :d].reshape(-1, H, hd)
    k = qkv[:, d:2 * d].reshape(-1, H, hd)
    v = qkv[:, 2 * d:].reshape(-1, H, hd)
    q = apply_rope(q, pos, shape.rope_base)
    k = apply_rope(k, pos, shape.rope_base)
    cache.write(slot, pos, k, v)
    K, V, kpos = cache.read_upto(slot, int(pos.max()))
    o = attend(q, K, V, pos, kpos).reshape(-1, d)
    x = x + o @ bw.wo.T
    b = rmsnorm(x, bw.g2, eps)
    u = silu(b @ bw.wg.T) * (b @ bw.wu.T)
    return x + u @ bw.wd.T


def embed(W: Weights, tokens) -> np.ndarray:
    return W.embed[np.asarray(tokens, dtype=np.int64)].copy()


def pre_blocks(W: Weights, x, pos, cache: KVCache):
    for b, bw in enumerate(W.pre):
        x = block(bw, W.shape, x, pos, cache, ("pre", b))
    return x


def loop_iteration(W: Weights, x, pos, cache: KVCache, l: int):
    """Iteration l (1-based) of the shared loop body: every body layer once."""
    for m, bw in enumerate(W.loop):
        x = block(bw, W.shape, x, pos, cache, ("loop", l, m))
    return x


def head_logits(W: Weights, h: np.ndarray) -> np.ndarray:
    return rmsnorm(h, W.g_final, W.shape.rms_eps) @ W.head.T


def argmax_lowest(logits: np.ndarray) -> np.ndarray:
    """Greedy token: the largest logit, the lowest id among equal maxima."""
    return np.argmax(logits, axis=-1)   # numpy returns the first maximal index


def top2_margin(logits: np.ndarray) -> np.ndarray:
    s = np.sort(logits, axis=-1)
    return s[..., -1] - s[..., -2]


def forward(W: Weights, tokens, L: int, cache: KVCache | None = None, pos0: int = 0):
    """Score a token sequence at loop count L: returns the final hidden rows [T, d]
    (no head), with the whole sequence run as one causal batch."""
    tokens = np.asarray(tokens)
    T = len(tokens)
    if cache is None:
        cache = KVCache(W.shape, pos0 + T)
    pos = np.arange(pos0, pos0 + T)
    x = pre_blocks(W, embed(W, tokens), pos, cache)
    for l in range(1, L + 1):
        x = loop_iteration(W, x, pos, cache, l)
    return x, cache
