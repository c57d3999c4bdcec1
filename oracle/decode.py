"""Oracle: greedy decode with per-lane L, hidden-state early exit, monotonic clamp,
and continuous depth batching at loop-iteration granularity.

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).

Passages followed:
  * "Dynamic-L Inference", "L-Aware Batching": one batch call, a loop count per lane.
  * "CLI Reference", generate options --early-exit-patience / -min-L / -tau /
    -peek-every: stop the loop once the relative L2 change of the hidden state
    stayed below tau for N consecutive iterations past min_L, probing only every
    peek_every iterations past min_L; L never rises again within a generation
    once reduced (monotonic clamp keeps the cache consistent).  Early exit is a
    cached-decode feature, so the prompt always runs the full requested L.
  * "CLI Reference", generate option --early-exit-logit-margin: when positive,
    the probe's stability metric becomes the top-1 minus top-2 margin of the
    head's logits at that iteration instead of the hidden-state change (a head
    projection per probe); the lane stops when the model is confident.
  * "CLI Reference", "Current Behavior": max_seq = prompt tokens + max tokens.
  * "Depth-adaptive Inference of Looped Language Models via Continuous Depth
    Batching", CDB design: scheduling at loop-iteration granularity, boundary
    stages (embedding, LM head) queued apart from loop steps, exit decided one
    step ahead.

Readings (pages silent or loose):
  * delta_l = ||h_l - h_{l-1}|| / ||h_{l-1}|| over the residual stream after the
    whole loop body, h_0 = the loop input; delta = inf when ||h_{l-1}|| = 0.
  * A probe happens at iteration l when l > min_L and (l - min_L - 1) is a
    multiple of peek_every.  The streak goes up by one when delta < tau and
    returns to zero otherwise; iterations without a probe leave it unchanged; it
    starts at zero for every token.  The lane exits at l once streak >= patience.
  * Early exit is off when tau <= 0 or patience == 0 (hidden-state mode), or
    logit_margin <= 0 or patience == 0 (margin mode).
  * Margin mode: a probe succeeds when margin >= logit_margin (the pages say
    the loop stops when the prediction is confident; the threshold itself is
    read as confident enough); success extends the streak, failure resets it,
    as in hidden-state mode.  Only the per-lane definition (generate_lane)
    implements it.
  * After a token ran D iterations the lane's cap becomes D; the next token runs
    min(L_requested, cap) iterations.
  * N emitted tokens: the first comes from the last prompt position; the N-th
    emitted token is not fed back.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

from . import model as M


@dataclass(frozen=True)
class EarlyExit:
    tau: float = 0.0
    min_L: int = 2
    patience: int = 0
    peek_every: int = 1
    logit_margin: float = 0.0   # > 0: margin mode (tau is then unused)

    @property
    def margin_mode(self) -> bool:
        return self.logit_margin > 0

    @property
    def enabled(self) -> bool:
        if self.margin_mode:
            return self.patience > 0
        return self.tau > 0 and self.patience > 0

    def is_probe(self, l: int) -> bool:
        return self.enabled and l > self.min_L and (l - self.min_L - 1) % self.peek_every == 0


def probe_succeeds(ee: EarlyExit, metric: float) -> bool:
    """Hidden-state mode: the relative change is below tau; margin mode: the
    top-1 / top-2 logit margin reaches logit_margin."""
    return metric >= ee.logit_margin if ee.margin_mode else metric < ee.tau


def streak_update(ee: EarlyExit, l: int, delta: float, streak: int) -> tuple[int, bool]:
    """The rule after iteration l (delta: the probe's metric): returns (new
    streak, exit now)."""
    if not ee.is_probe(l):
        return streak, False
    streak = streak + 1 if probe_succeeds(ee, delta) else 0
    return streak, streak >= ee.patience


def exit_iteration(deltas, L_run: int, ee: EarlyExit) -> int:
    """deltas[l-1] is delta after iteration l; returns the number of iterations a
    token runs under early exit with run length L_run."""
    streak = 0
    for l in range(1, L_run + 1):
        streak, exit_now = streak_update(ee, l, deltas[l - 1], streak)
        if exit_now:
            return l
    return L_run


def rel_l2(h: np.ndarray, h_prev: np.ndarray) -> float:
    den = float(np.sqrt(np.sum(h_prev * h_prev)))
    num = float(np.sqrt(np.sum((h - h_prev) ** 2)))
    return np.inf if den == 0.0 else num / den


@dataclass
class Probe:
    token: int          # index of the emitted token this iteration belongs to
    l: int              # iteration (1-based)
    delta: float        # the probe's metric: relative change (or top-2 logit margin in margin mode)
    below: bool         # the probe succeeded (delta < tau, or margin >= logit_margin)

    def margin(self, tau: float) -> float:
        """|delta / tau - 1|: how far the decision sits from the threshold."""
        return abs(self.delta / tau - 1.0)


@dataclass
class LaneResult:
    tokens: np.ndarray               # int [n_new]
    depths: np.ndarray               # int [n_new] executed iterations behind each token
    logits: np.ndarray | None        # float64 [n_new, V]
    probes: list = field(default_factory=list)
    prompt_hidden: np.ndarray | None = None


def _probe_step(ee: EarlyExit, t: int, l: int, h, h_prev, streak: int, probes: list, W=None):
    """Record the probe after iteration l (if any) and apply the rule.  In
    margin mode the metric is the head's top-2 margin at h (needs W)."""
    if not ee.is_probe(l):
        return streak, False
    metric = float(M.top2_margin(M.head_logits(W, h))) if ee.margin_mode else rel_l2(h, h_prev)
    probes.append(Probe(t, l, metric, probe_succeeds(ee, metric)))
    return streak_update(ee, l, metric, streak)


def generate_lane(W: M.Weights, prompt, L_req: int, n_new: int, ee: EarlyExit = EarlyExit(),
                  forced_depths=None, keep_logits: bool = True, keep_prompt_hidden: bool = False,
                  warmup_tokens: int = 0, warmup_L: int = 2) -> LaneResult:
    """The definition: one lane, token by token, iteration by iteration.

    forced_depths[t] (t >= 1), when given, replaces the early-exit decision of
    token t by that depth (used to follow another implementation's decision at a
    probe that sits on the threshold); probes are still recorded.

    warmup_tokens > 0 ("Dynamic-L Inference", L scheduling; "CLI Reference",
    --l-warmup-tokens / --l-warmup-L): decode tokens 1..warmup_tokens run
    min(warmup_L, L_req) iterations and leave the cap alone; later tokens run
    the full schedule, their deeper iterations reading the warmup positions
    through KVCache.deep_fallback.  The prompt runs the full L_req."""
    if L_req < 1:
        raise ValueError("L must be >= 1")
    prompt = np.asarray(prompt)
    T = len(prompt)
    cache = M.KVCache(W.shape, T + max(n_new - 1, 0), deep_fallback=warmup_tokens > 0)
    x, _ = M.forward(W, prompt, L_req, cache)
    tokens = np.zeros(n_new, dtype=np.int64)
    depths = np.zeros(n_new, dtype=np.int64)
    logits_all = np.zeros((n_new, W.shape.vocab)) if keep_logits else None
    probes: list = []
    h = x[-1:]
    L_cap = L_req
    for t in range(n_new):
        if t == 0:
            depth = L_req
        else:
            p = T + t - 1
            pos = np.array([p])
            h = M.pre_blocks(W, M.embed(W, [tokens[t - 1]]), pos, cache)
            warm = t <= warmup_tokens
            L_run = min(warmup_L, L_req) if warm else min(L_req, L_cap)
            target = None if forced_depths is None else int(forced_depths[t])
            if target is not None and not (1 <= target <= L_run):
                raise ValueError("forced depth out of range")
            streak = 0
            depth = L_run
            for l in range(1, L_run + 1):
                h_prev = h
                h = M.loop_iteration(W, h, pos, cache, l)
                streak, exit_now = _probe_step(ee, t, l, h[0], h_prev[0], streak, probes, W)
                if target is not None:
                    exit_now = l == target
                if exit_now:
                    depth = l
                    break
            if not warm:
                L_cap = depth
        lg = M.head_logits(W, h[0])
        tokens[t] = M.argmax_lowest(lg)
        depths[t] = depth
        if keep_logits:
            logits_all[t] = lg
    return LaneResult(tokens, depths, logits_all, probes, x if keep_prompt_hidden else None)


def speculative_lane(W: M.Weights, prompt, L_draft: int, L_verify: int, n_new: int, draft_ahead: int):
    """Self-speculative greedy decode of one lane ("CLI Reference", speculate:
    --draft-loops, --verify-loops, --draft-ahead, temperature 0): the same
    weights and one cache for both passes.  Each round drafts up to draft_ahead
    tokens at L_draft, one position at a time; then runs the drafted positions
    at L_verify as one causal batch, keeps the drafted tokens up to the first
    one the verify pass's greedy choice disagrees with, and takes the verify
    pass's own token there.  The verify pass recomputes iterations 1..L_draft
    of the drafted positions (their values equal the draft's, since the hidden
    state at iteration j does not depend on L >= j); every position is
    rewritten before anything later reads it.  Returns (tokens int [n_new],
    rounds).  With greedy choices the tokens are those of a plain greedy run at
    L_verify; the draft only decides how many positions one verify pass covers."""
    if not (1 <= L_draft and 1 <= L_verify and draft_ahead >= 1):
        raise ValueError("bad speculation parameters")
    prompt = np.asarray(prompt)
    T = len(prompt)
    cache = M.KVCache(W.shape, T + n_new + draft_ahead)
    x, _ = M.forward(W, prompt, L_verify, cache)
    tokens = [int(M.argmax_lowest(M.head_logits(W, x[-1])))]
    rounds = 0
    while len(tokens) < n_new:
        rounds += 1
        p0 = T + len(tokens) - 1          # position of the last token taken (not computed yet)
        k = min(draft_ahead, n_new - len(tokens))
        draft, prev = [], tokens[-1]
        for j in range(k):                # draft: one position at a time, shallow
            pos = np.array([p0 + j])
            h = M.pre_blocks(W, M.embed(W, [prev]), pos, cache)
            for l in range(1, L_draft + 1):
                h = M.loop_iteration(W, h, pos, cache, l)
            prev = int(M.argmax_lowest(M.head_logits(W, h[0])))
            draft.append(prev)
        pos = np.arange(p0, p0 + k)       # verify: the same positions together, deep
        h = M.pre_blocks(W, M.embed(W, [tokens[-1]] + draft[:-1]), pos, cache)
        for l in range(1, L_verify + 1):
            h = M.loop_iteration(W, h, pos, cache, l)
        for j in range(k):
            choice = int(M.argmax_lowest(M.head_logits(W, h[j])))
            tokens.append(choice)
            if choice != draft[j]:
                break
    return np.array(tokens[:n_new], dtype=np.int64), rounds


# ------------------------------------------------ continuous depth batching ----

LOOP, BOUNDARY, DONE = 0, 1, 2


@dataclass
class _Lane:
    L_req: int
    L_cap: int
    cache: M.KVCache
    T: int
    n_new: int
    phase: int = BOUNDARY
    l: int = 0               # iterations done for the current token
    L_run: int = 0
    streak: int = 0
    h: np.ndarray | None = None
    h_in: np.ndarray | None = None
    n_emitted: int = 0
    depth: int = 0
    tokens: list = field(default_factory=list)
    depths: list = field(default_factory=list)
    logits: list = field(default_factory=list)
    probes: list = field(default_factory=list)


def generate_cdb(W: M.Weights, prompts, per_lane_L, n_new: int, ee: EarlyExit = EarlyExit(),
                 keep_logits: bool = True):
    """All lanes together, one loop iteration per step for every lane in its loop
    phase (each at its own iteration index), boundary stages queued apart.

    Each step: (1) gather the rows of lanes in the loop phase and run one loop
    iteration on them as a batch, every row against its own lane's cache slot;
    (2) decide per row whether its loop is finished (early exit or L_run
    reached), which moves the lane to the boundary queue before the next step is
    formed; (3) run the boundary queue: head + greedy token, then embed + pre
    blocks for lanes that still have tokens to emit.  Returns (per-lane
    LaneResult list, number of loop steps)."""
    if ee.margin_mode:
        raise NotImplementedError("margin-mode early exit is defined per lane (generate_lane) only")
    shape = W.shape
    d, H, hd = shape.d, shape.n_heads, shape.head_dim
    lanes = []
    for i, prompt in enumerate(prompts):
        prompt = np.asarray(prompt)
        T = len(prompt)
        L = int(per_lane_L[i])
        cache = M.KVCache(shape, T + max(n_new - 1, 0))
        x, _ = M.forward(W, prompt, L, cache)
        lane = _Lane(L, L, cache, T, n_new)
        lane.h = x[-1:].copy()
        lane.depth = L
        lanes.append(lane)

    steps = 0
    while True:
        # boundary stage queue
        for lane in lanes:
            if lane.phase != BOUNDARY:
                continue
            lg = M.head_logits(W, lane.h[0])
            tok = int(M.argmax_lowest(lg))
            lane.tokens.append(tok)
            lane.depths.append(lane.depth)
            if keep_logits:
                lane.logits.append(lg)
            lane.n_emitted += 1
            lane.L_cap = lane.depth
            if lane.n_emitted == lane.n_new:
                lane.phase = DONE
                continue
            p = lane.T + lane.n_emitted - 1
            lane.h = M.pre_blocks(W, M.embed(W, [tok]), np.array([p]), lane.cache)
            lane.L_run = min(lane.L_req, lane.L_cap)
            lane.l = 0
            lane.streak = 0
            lane.phase = LOOP
        rows = [lane for lane in lanes if lane.phase == LOOP]
        if not rows:
            break
        steps += 1
        # one loop iteration for all rows, batched through the projections
        X = np.concatenate([lane.h for lane in rows], axis=0)
        X_in = X.copy()
        for m, bw in enumerate(W.loop):
            a = M.rmsnorm(X, bw.g1, shape.rms_eps)
            qkv = a @ bw.wqkv.T
            O = np.zeros((len(rows), d))
            for r, lane in enumerate(rows):
                l = lane.l + 1
                p = lane.T + lane.n_emitted - 1
                pos = np.array([p])
                q = M.apply_rope(qkv[r:r + 1, :d].reshape(1, H, hd), pos, shape.rope_base)
                k = M.apply_rope(qkv[r:r + 1, d:2 * d].reshape(1, H, hd), pos, shape.rope_base)
                v = qkv[r:r + 1, 2 * d:].reshape(1, H, hd)
                slot = ("loop", l, m)
                lane.cache.write(slot, pos, k, v)
                K, V, kpos = lane.cache.read_upto(slot, p)
                O[r] = M.attend(q, K, V, pos, kpos).reshape(d)
            X = X + O @ bw.wo.T
            b = M.rmsnorm(X, bw.g2, shape.rms_eps)
            X = X + (M.silu(b @ bw.wg.T) * (b @ bw.wu.T)) @ bw.wd.T
        # exit decisions, taken before the next step's batch is formed
        for r, lane in enumerate(rows):
            lane.l += 1
            lane.h = X[r:r + 1]
            lane.streak, exit_now = _probe_step(ee, lane.n_emitted, lane.l, X[r], X_in[r],
                                                lane.streak, lane.probes)
            if exit_now or lane.l == lane.L_run:
                lane.depth = lane.l
                lane.phase = BOUNDARY
    results = [LaneResult(np.array(l.tokens), np.array(l.depths),
                          np.array(l.logits) if keep_logits else None, l.probes) for l in lanes]
    return results, steps
