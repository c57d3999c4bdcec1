"""Pins for the oracle's decode: early-exit rule, clamp, per-lane L batching."""
import os

import numpy as np
import pytest

import synthetic as S
import oracle as O
from oracle import decode as D

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


@pytest.fixture(scope="module")
def tiny():
    sh = S.TINY
    return O.build_weights(sh, S.master_weights(sh), S.gains(sh))


def _schedule_rows():
    rows = []
    with open(os.path.join(GOLDEN, "ee_schedule.txt")) as f:
        for line in f:
            if not line.strip() or line.startswith("#"):
                continue
            head, deltas, probes, depth = [p.strip() for p in line.split("|")]
            tau, min_L, pat, peek, L = head.split()
            ee = D.EarlyExit(float(tau), int(min_L), int(pat), int(peek))
            rows.append((ee, int(L), [float(x) for x in deltas.split()],
                         [] if probes == "-" else [int(x) for x in probes.split()], int(depth)))
    return rows


def test_golden_exit_schedule():
    for ee, L, deltas, probes, depth in _schedule_rows():
        assert [l for l in range(1, L + 1) if ee.is_probe(l)] == probes
        assert D.exit_iteration(deltas, L, ee) == depth, (ee, deltas)


def test_golden_exit_schedule_incremental():
    # the incremental form both decode paths use, fed one delta at a time
    for ee, L, deltas, probes, depth in _schedule_rows():
        streak, got, seen = 0, L, []
        for l in range(1, L + 1):
            if ee.is_probe(l):
                seen.append(l)
            streak, exit_now = D.streak_update(ee, l, deltas[l - 1], streak)
            if exit_now:
                got = l
                break
        assert got == depth
        assert seen == [p for p in probes if p <= got]


def test_rel_l2():
    h0 = np.array([3.0, 4.0])
    assert D.rel_l2(h0 + np.array([0.3, 0.4]), h0) == pytest.approx(0.1, abs=1e-15)
    assert D.rel_l2(np.ones(2), np.zeros(2)) == np.inf


def test_cdb_batch_equals_lanes_alone(tiny):
    P = S.prompts(3, 12, tiny.shape.vocab, seed=41)
    Ls = [2, 5, 3]
    ee = D.EarlyExit(tau=0.9, min_L=1, patience=2)
    res, steps = D.generate_cdb(tiny, P, Ls, 6, ee)
    total = 0
    for i in range(3):
        alone = D.generate_lane(tiny, P[i], Ls[i], 6, ee)
        assert np.array_equal(res[i].depths, alone.depths)
        assert np.array_equal(res[i].tokens, alone.tokens)
        assert np.allclose(res[i].logits, alone.logits, rtol=0, atol=1e-12)
        total = max(total, int(alone.depths[1:].sum()))
    # at iteration granularity the step count is the deepest lane's work
    assert steps == total
    assert any(r.depths[-1] < Ls[i] for i, r in enumerate(res))  # some lane exited early


def test_clamp_binds_in_both_paths(tiny):
    # token 1 exits at l=5; without the clamp token 2 would first drop below tau at l=6
    P = S.prompts(1, 10, tiny.shape.vocab, seed=52)[0]
    ee = D.EarlyExit(tau=0.33, min_L=1, patience=1)
    free = D.generate_lane(tiny, P, 8, 6, D.EarlyExit(tau=1e9, min_L=0, patience=100))
    d2 = [p.delta for p in free.probes if p.token == 2]
    assert next(l for l in range(1, 9) if d2[l - 1] < 0.33) == 6
    alone = D.generate_lane(tiny, P, 8, 6, ee)
    assert alone.depths.tolist() == [8, 5, 5, 5, 5, 5]
    res, _ = D.generate_cdb(tiny, P[None], [8], 6, ee)
    assert np.array_equal(res[0].depths, alone.depths)
    assert np.allclose(res[0].logits, alone.logits, rtol=0, atol=1e-12)


def test_disabled_early_exit_equals_fixed_L(tiny):
    P = S.prompts(1, 8, tiny.shape.vocab, seed=42)[0]
    fixed = D.generate_lane(tiny, P, 5, 5)
    for ee in (D.EarlyExit(tau=0.0, patience=2), D.EarlyExit(tau=-1.0, patience=2),
               D.EarlyExit(tau=1e9, patience=0)):
        r = D.generate_lane(tiny, P, 5, 5, ee)
        assert np.array_equal(r.depths, [5] * 5)
        assert np.array_equal(r.logits, fixed.logits)


def test_huge_tau_exits_at_earliest_then_clamps(tiny):
    P = S.prompts(1, 8, tiny.shape.vocab, seed=43)[0]
    ee = D.EarlyExit(tau=1e9, min_L=2, patience=2)
    r = D.generate_lane(tiny, P, 7, 5, ee)
    assert r.depths.tolist() == [7, 4, 4, 4, 4]
    # equals a fixed run at L=4 for every decode token: prompt at 7, then L capped to 4
    forced = D.generate_lane(tiny, P, 7, 5, forced_depths=[0, 4, 4, 4, 4])
    assert np.array_equal(forced.logits, r.logits)


def test_patience_beyond_range_never_exits(tiny):
    P = S.prompts(1, 8, tiny.shape.vocab, seed=44)[0]
    r = D.generate_lane(tiny, P, 5, 4, D.EarlyExit(tau=1e9, min_L=2, patience=4))
    assert r.depths.tolist() == [5] * 4


def test_depths_follow_rule_on_recorded_deltas_and_never_rise(tiny):
    P = S.prompts(2, 10, tiny.shape.vocab, seed=45)
    ee = D.EarlyExit(tau=0.4, min_L=2, patience=1, peek_every=2)
    for i, L in enumerate((9, 6)):
        r = D.generate_lane(tiny, P[i], L, 8, ee)
        assert all(a >= b for a, b in zip(r.depths, r.depths[1:]))
        cap = L
        for t in range(1, 8):
            pr = {p.l: p.delta for p in r.probes if p.token == t}
            deltas = [pr.get(l, np.inf) for l in range(1, cap + 1)]
            assert r.depths[t] == D.exit_iteration(deltas, cap, ee)
            cap = r.depths[t]


def test_forcing_natural_depths_reproduces_run(tiny):
    P = S.prompts(1, 8, tiny.shape.vocab, seed=46)[0]
    ee = D.EarlyExit(tau=0.45, min_L=2, patience=1)
    r = D.generate_lane(tiny, P, 8, 6, ee)
    f = D.generate_lane(tiny, P, 8, 6, ee, forced_depths=r.depths)
    assert np.array_equal(f.logits, r.logits) and np.array_equal(f.depths, r.depths)


def test_edge_cases(tiny):
    P = S.prompts(1, 4, tiny.shape.vocab, seed=47)[0]
    r = D.generate_lane(tiny, P, 1, 1)
    assert r.depths.tolist() == [1] and r.logits.shape == (1, tiny.shape.vocab)
    with pytest.raises(ValueError):
        D.generate_lane(tiny, P, 0, 2)
    with pytest.raises(ValueError):
        D.generate_lane(tiny, P, 3, 3, forced_depths=[0, 4, 1])


# ------------------------------------------------ logit-margin early exit ----

def test_margin_mode_huge_threshold_never_exits(tiny):
    P = S.prompts(1, 8, tiny.shape.vocab, seed=61)[0]
    ee = D.EarlyExit(min_L=1, patience=1, logit_margin=1e9)
    r = D.generate_lane(tiny, P, 6, 4, ee)
    assert r.depths.tolist() == [6] * 4
    assert r.probes and not any(p.below for p in r.probes)
    fixed = D.generate_lane(tiny, P, 6, 4)
    assert np.array_equal(fixed.logits, r.logits)


def test_margin_mode_tiny_threshold_exits_at_earliest_then_clamps(tiny):
    # every probe with a non-zero margin succeeds: exit at min_L + 1 + (patience - 1) * peek_every
    P = S.prompts(1, 8, tiny.shape.vocab, seed=62)[0]
    ee = D.EarlyExit(min_L=2, patience=2, peek_every=2, logit_margin=1e-12)
    r = D.generate_lane(tiny, P, 8, 4, ee)
    assert r.depths.tolist() == [8, 5, 5, 5]
    forced = D.generate_lane(tiny, P, 8, 4, forced_depths=[0, 5, 5, 5])
    assert np.array_equal(forced.logits, r.logits)


def test_margin_probe_metric_is_the_heads_top2_margin(tiny):
    # the metric recorded at iteration l of token 1 equals the top-2 margin of the
    # logits a run stopped at l emits for token 1 (same hidden state, same head)
    P = S.prompts(1, 8, tiny.shape.vocab, seed=63)[0]
    ee = D.EarlyExit(min_L=1, patience=9, logit_margin=1e9)  # probes at l = 2, 3, 4 and no exit
    r = D.generate_lane(tiny, P, 4, 2, ee)
    got = {p.l: p.delta for p in r.probes if p.token == 1}
    assert sorted(got) == [2, 3, 4]
    for l in (2, 3, 4):
        stopped = D.generate_lane(tiny, P, 4, 2, forced_depths=[0, l])
        s = np.sort(stopped.logits[1])
        assert got[l] == s[-1] - s[-2]


def test_margin_mode_rule_on_recorded_margins(tiny):
    P = S.prompts(1, 8, tiny.shape.vocab, seed=64)[0]
    probe_all = D.EarlyExit(min_L=0, patience=99, logit_margin=1e9)
    margins = [p.delta for p in D.generate_lane(tiny, P, 6, 2, probe_all).probes if p.token == 1]
    thr = float(np.median(margins))
    ee = D.EarlyExit(min_L=0, patience=1, logit_margin=thr)
    r = D.generate_lane(tiny, P, 6, 2, ee)
    first = next(l for l, m in enumerate(margins, start=1) if m >= thr)
    assert r.depths[1] == first


def test_margin_mode_is_per_lane_only(tiny):
    with pytest.raises(NotImplementedError):
        D.generate_cdb(tiny, S.prompts(1, 4, tiny.shape.vocab), [2], 2, D.EarlyExit(patience=1, logit_margin=1.0))


# ------------------------------------------------------------- L warmup ----

def test_kv_deep_fallback_reads_the_deepest_shallower_iteration():
    from oracle import model as M
    sh = S.TINY
    c = M.KVCache(sh, 8, deep_fallback=True)
    H, hd = sh.n_heads, sh.head_dim
    for l, upto in ((1, 5), (2, 3), (3, 2)):  # iteration l holds positions 0..upto-1
        for p in range(upto):
            c.write(("loop", l, 0), np.array([p]), np.full((1, H, hd), 10.0 * l + p), np.full((1, H, hd), -10.0 * l - p))
    K, V, idx = c.read_upto(("loop", 3, 0), 4)
    assert idx.tolist() == [0, 1, 2, 3, 4]
    assert [float(K[i, 0, 0]) for i in range(5)] == [30.0, 31.0, 22.0, 13.0, 14.0]
    assert [float(V[i, 0, 0]) for i in range(5)] == [-30.0, -31.0, -22.0, -13.0, -14.0]
    plain = M.KVCache(sh, 8)
    plain.slots = c.slots
    assert plain.read_upto(("loop", 3, 0), 4)[2].tolist() == [0, 1]  # without the reading: only its own entries


def test_warmup_schedule_and_its_degenerate_cases(tiny):
    P = S.prompts(1, 8, tiny.shape.vocab, seed=71)[0]
    r = D.generate_lane(tiny, P, 6, 6, warmup_tokens=3, warmup_L=2)
    assert r.depths.tolist() == [6, 2, 2, 2, 6, 6]     # the prompt at full L, 3 shallow tokens, then full L again
    plain = D.generate_lane(tiny, P, 6, 6)
    # warmup at the full depth, or no warmup tokens, is the plain run
    assert np.array_equal(D.generate_lane(tiny, P, 6, 6, warmup_tokens=3, warmup_L=6).logits, plain.logits)
    assert np.array_equal(D.generate_lane(tiny, P, 6, 6, warmup_tokens=0, warmup_L=2).logits, plain.logits)
    # the shallow tokens are those of a plain run forced to depth 2 (their keys are all present)
    forced = D.generate_lane(tiny, P, 6, 4, forced_depths=[0, 2, 2, 2])
    assert np.array_equal(forced.logits, r.logits[:4])


def test_warmup_deep_tokens_read_the_warmup_positions(tiny, monkeypatch):
    # after the warmup, iterations 3..6 of token 4 read the 3 warmup positions through their
    # iteration-2 entries: a cache without that reading (which sees only the prompt and the
    # token itself there) gives different logits, while every token before it is unchanged
    P = S.prompts(1, 8, tiny.shape.vocab, seed=72)[0]
    r = D.generate_lane(tiny, P, 6, 5, warmup_tokens=3, warmup_L=2)
    from oracle import model as M

    class NoReading(M.KVCache):
        def __init__(self, shape, max_seq, deep_fallback=False):
            super().__init__(shape, max_seq, deep_fallback=False)
    monkeypatch.setattr(D.M, "KVCache", NoReading)
    other = D.generate_lane(tiny, P, 6, 5, warmup_tokens=3, warmup_L=2)
    assert np.array_equal(other.logits[:4], r.logits[:4])
    assert not np.allclose(other.logits[4], r.logits[4])


# ------------------------------------------------ self-speculative decode ----

@pytest.mark.parametrize("L_draft,draft_ahead", [(1, 1), (2, 4), (3, 3), (6, 2)])
def test_speculative_tokens_equal_greedy_at_the_verify_depth(tiny, L_draft, draft_ahead):
    P = S.prompts(1, 10, tiny.shape.vocab, seed=81)[0]
    ref = D.generate_lane(tiny, P, 6, 9)
    from oracle import model as M
    assert min(M.top2_margin(lg) for lg in ref.logits) > 1e-9  # no near-tie for the batched verify to flip
    tok, rounds = D.speculative_lane(tiny, P, L_draft, 6, 9, draft_ahead)
    assert tok.tolist() == ref.tokens.tolist()
    assert -(-8 // draft_ahead) <= rounds <= 8
    if L_draft == 6:  # the draft is the verify model: every drafted token is accepted
        assert rounds == -(-8 // draft_ahead)


def test_golden_margin_exit_schedule():
    with open(os.path.join(GOLDEN, "ee_margin_schedule.txt")) as f:
        rows = [l for l in f if l.strip() and not l.startswith("#")]
    assert rows
    for line in rows:
        head, metrics, probes, depth = [p.strip() for p in line.split("|")]
        thr, min_L, pat, peek, L = head.split()
        ee = D.EarlyExit(min_L=int(min_L), patience=int(pat), peek_every=int(peek), logit_margin=float(thr))
        L = int(L)
        want = [] if probes == "-" else [int(x) for x in probes.split()]
        assert [l for l in range(1, L + 1) if ee.is_probe(l)] == want
        assert D.exit_iteration([float(x) for x in metrics.split()], L, ee) == int(depth), line
