"""End-to-end parity of the CUDA path against the fp64 oracle, through the C ABI.

Bars (floating point): logits max-abs <= 1e-2 and relative L2 <= 2e-3 per
position, prompt hidden states relative L2 <= 2e-3.  Exact: per-lane depth
schedules, exit masks, and greedy tokens wherever the oracle's top-1/top-2
margin exceeds 1e-3."""
import numpy as np
import pytest

import synthetic as S
from oracle import decode as D
from oracle import model as M

from gpu_helpers import (assert_logits_close, gpu_model, oracle_weights, rel_l2, status_clean, teacher_forced,
                         MARGIN)

pytestmark = pytest.mark.gpu


def _check_tokens(ref_tokens, ref_logits, got_tokens):
    """Greedy tokens must agree wherever the oracle's margin exceeds 1e-3; after
    the first near-tie the sequences may legitimately part."""
    for t in range(len(ref_tokens)):
        if M.top2_margin(ref_logits[t]) <= MARGIN:
            return t
        assert int(got_tokens[t]) == int(ref_tokens[t]), f"token {t}"
    return len(ref_tokens)


# --------------------------------------------------------------- tiny model ----

@pytest.mark.parametrize("gain_seed", [None, 7])
def test_tiny_generate_end_to_end(gain_seed):
    wl = S.workload("tiny")
    W = oracle_weights("tiny", gain_seed)
    P = S.prompts(wl.n_lanes, wl.prompt_len, wl.shape.vocab)
    m = gpu_model("tiny", gain_seed, max_lanes=2, max_seq=32, L_max=8)
    tok, dep = m.generate(P, wl.per_lane_L, wl.n_new)
    status_clean(m)
    for i, L in enumerate(wl.per_lane_L):
        r = D.generate_lane(W, P[i], L, wl.n_new)
        assert dep[i].tolist() == [L] * wl.n_new
        _check_tokens(r.tokens, r.logits, tok[i])


def test_tiny_teacher_forced_logits():
    wl = S.workload("tiny")
    W = oracle_weights("tiny", 7)
    P = S.prompts(wl.n_lanes, wl.prompt_len, wl.shape.vocab)
    m = gpu_model("tiny", 7, max_lanes=2, max_seq=32, L_max=8)
    ref, lg, am, dep = teacher_forced(m, W, P, list(wl.per_lane_L), wl.n_new)
    status_clean(m)
    for i in range(wl.n_lanes):
        for t in range(wl.n_new):
            assert_logits_close(lg[i, t], ref[i].logits[t], f"lane {i} token {t}")
            if M.top2_margin(ref[i].logits[t]) > MARGIN:
                assert am[i, t] == ref[i].tokens[t]
        assert dep[i].tolist() == ref[i].depths.tolist()


def test_tiny_single_lane_equals_batch():
    # a lane's result does not depend on the other lanes in the step
    wl = S.workload("tiny")
    P = S.prompts(3, 12, wl.shape.vocab, seed=41)
    Ls = [2, 5, 3]
    m = gpu_model("tiny", None, max_lanes=3, max_seq=32, L_max=8)
    tok_b, dep_b = m.generate(P, Ls, 6)
    for i in range(3):
        m1 = gpu_model("tiny", None, max_lanes=1, max_seq=32, L_max=8)
        t1, d1 = m1.generate(P[i:i + 1], Ls[i:i + 1], 6)
        assert np.array_equal(t1[0], tok_b[i]) and np.array_equal(d1[0], dep_b[i])


def _probe_margins(ref, tau):
    return [p.margin(tau) for r in ref for p in r.probes]


@pytest.mark.parametrize("ee", [D.EarlyExit(0.9, 1, 2, 1), D.EarlyExit(0.33, 1, 1, 1), D.EarlyExit(0.5, 2, 1, 2),
                                D.EarlyExit(1e9, 2, 2, 1)])
def test_tiny_early_exit_schedules(ee):
    W = oracle_weights("tiny")
    P = S.prompts(3, 12, 512, seed=52)
    Ls = [8, 5, 3]
    ref = [D.generate_lane(W, P[i], Ls[i], 6, ee) for i in range(3)]
    m = gpu_model("tiny", None, max_lanes=3, max_seq=32, L_max=8)
    m.set_early_exit(ee.tau, ee.min_L, ee.patience, ee.peek_every)
    tok, dep = m.generate(P, Ls, 6)
    status_clean(m)
    near = [x for x in _probe_margins(ref, ee.tau) if x <= 1e-2]
    assert not near, f"probes within 1% of tau: {near}"
    for i in range(3):
        assert dep[i].tolist() == ref[i].depths.tolist(), i
        _check_tokens(ref[i].tokens, ref[i].logits, tok[i])


def test_tiny_exit_masks_per_step():
    import torch
    W = oracle_weights("tiny")
    P = S.prompts(2, 10, 512, seed=52)
    ee = D.EarlyExit(0.33, 1, 1, 1)
    Ls = [8, 6]
    ref, lg, am, dep = teacher_forced(gpu_model("tiny", None, max_lanes=2, max_seq=32, L_max=8), W, P, Ls, 5, ee)
    for i in range(2):
        assert dep[i].tolist() == ref[i].depths.tolist()
        for t in range(5):
            assert_logits_close(lg[i, t], ref[i].logits[t], f"lane {i} token {t}")


def test_tiny_raising_L_is_refused():
    from dynamic_depth_b200 import TlError
    m = gpu_model("tiny", None, max_lanes=2, max_seq=32, L_max=8)
    P = S.prompts(2, 8, 512, seed=3)
    m.prefill(0, P[0], 3)
    m.prefill(1, P[1], 3)
    with pytest.raises(TlError) as e:
        m.decode([3, 4], 2)
    assert e.value.status == -4  # TL_EKV
    with pytest.raises(TlError):
        m.prefill(0, P[0], 0)
    with pytest.raises(TlError):
        m.prefill(0, np.array([600], dtype=np.int32), 2)  # token outside the vocabulary


# ---------------------------------------------------------- 407M-class model ----

def test_m407_prefill_hidden_T128_L8():
    import torch
    W = oracle_weights("m407")
    wl = S.workload("m407_score")
    P = S.prompts(1, wl.prompt_len, S.M407.vocab)
    want, _ = M.forward(W, P[0], 8)
    m = gpu_model("m407", None, max_lanes=1, max_seq=128, L_max=8)
    hid = torch.zeros((128, S.M407.d), dtype=torch.float32, device="cuda")
    m.prefill(0, P[0], 8, hidden_out=hid)
    status_clean(m)
    got = hid.cpu().numpy()
    assert rel_l2(got, want) <= 2e-3
    for t in (0, 1, 63, 127):
        assert rel_l2(got[t], want[t]) <= 2e-3, t


@pytest.mark.parametrize("L", [2, 32])
def test_m407_decode_logits_teacher_forced(L):
    W = oracle_weights("m407")
    P = S.prompts(1, 32, S.M407.vocab)
    m = gpu_model("m407", None, max_lanes=1, max_seq=40, L_max=32)
    ref, lg, am, dep = teacher_forced(m, W, P, [L], 4)
    status_clean(m)
    for t in range(4):
        assert_logits_close(lg[0, t], ref[0].logits[t], f"L={L} token {t}")
        if M.top2_margin(ref[0].logits[t]) > MARGIN:
            assert am[0, t] == ref[0].tokens[t]


# ------------------------------------------- wide batches (tensor-core path) ----

def test_tiny_wide_batch_tensor_core_decode():
    # 12 lanes: more rows than the CUDA-core GEMV takes, so loop steps run on tcgen05
    W = oracle_weights("tiny", 7)
    P = S.prompts(12, 16, 512, seed=71)
    Ls = [2, 3, 4, 5] * 3
    m = gpu_model("tiny", 7, max_lanes=12, max_seq=32, L_max=8)
    ref, lg, am, dep = teacher_forced(m, W, P, Ls, 4)
    status_clean(m)
    for i in range(12):
        assert dep[i].tolist() == ref[i].depths.tolist()
        for t in range(4):
            assert_logits_close(lg[i, t], ref[i].logits[t], f"lane {i} token {t}")


def test_tiny_wide_batch_generate_matches_oracle():
    W = oracle_weights("tiny")
    P = S.prompts(16, 20, 512, seed=72)
    Ls = [1, 2, 3, 4, 5, 6, 7, 8] * 2
    m = gpu_model("tiny", None, max_lanes=16, max_seq=40, L_max=8)
    tok, dep = m.generate(P, Ls, 8)
    status_clean(m)
    for i in range(16):
        r = D.generate_lane(W, P[i], Ls[i], 8)
        assert dep[i].tolist() == r.depths.tolist()
        _check_tokens(r.tokens, r.logits, tok[i])


def test_m407_wide_decode_logits():
    W = oracle_weights("m407")
    P = S.prompts(16, 24, S.M407.vocab, seed=73)
    Ls = [3] * 16
    m = gpu_model("m407", None, max_lanes=16, max_seq=32, L_max=4)
    ref, lg, am, dep = teacher_forced(m, W, P, Ls, 3)
    status_clean(m)
    for i in range(16):
        for t in range(3):
            assert_logits_close(lg[i, t], ref[i].logits[t], f"lane {i} token {t}")


@pytest.mark.parametrize("mode", [1, 2, 3])
def test_tiny_tick_layouts_match_oracle(mode):
    # every layout of a decode tick (entering lanes' first iteration in the boundary stage, at the next
    # tick beside the other lanes' loop step, or boundary stages on their own stream) gives each lane its
    # own schedule and tokens
    W = oracle_weights("tiny", 7)
    P = S.prompts(16, 12, 512, seed=75)
    Ls = [1, 2, 3, 4, 5, 6, 7, 8] * 2
    m = gpu_model("tiny", 7, max_lanes=16, max_seq=32, L_max=8)
    m.set_tick_overlap(mode)
    tok, dep = m.generate(P, Ls, 7)
    st = status_clean(m)
    assert st["entry_in_boundary"] == (1 if mode == 1 else 0)
    assert st["tick_layout"] == mode
    assert st["tokens_emitted"] >= 16 * 7
    for i in range(16):
        r = D.generate_lane(W, P[i], Ls[i], 7)
        assert dep[i].tolist() == r.depths.tolist()
        _check_tokens(r.tokens, r.logits, tok[i])


def _tau_clear_of_probes(W, P, Ls, n_new, candidates, min_L=1, patience=1, peek=1):
    """The first threshold whose oracle run has no probe within 1% of it and exits somewhere early:
    (early-exit rule, oracle results)."""
    for tau in candidates:
        ee = D.EarlyExit(tau, min_L, patience, peek)
        ref = [D.generate_lane(W, P[i], Ls[i], n_new, ee) for i in range(len(Ls))]
        clear = not [x for x in _probe_margins(ref, tau) if x <= 1e-2]
        fired = any(int(d) < L for r, L in zip(ref, Ls) for d in r.depths[1:])
        if clear and fired:
            return ee, ref
    raise AssertionError("no candidate threshold clear of the probes")


@pytest.mark.parametrize("exit_rule", [False, True])
def test_tiny_async_stages_early_exit_and_repeat(exit_rule):
    # boundary stages apart from the loop steps: exact schedules with the exit rule, twice on one model
    # (the second run replays the captured graphs)
    W = oracle_weights("tiny")
    P = S.prompts(24, 10, 512, seed=76)
    Ls = [8, 1, 5, 3, 7, 2, 6, 4] * 3
    m = gpu_model("tiny", None, max_lanes=24, max_seq=40, L_max=8)
    m.set_tick_overlap(3)
    if exit_rule:
        # probes every second iteration from l = 3, two successes in a row: the oracle's probe values leave
        # a wide gap around 0.45
        ee, ref = _tau_clear_of_probes(W, P, Ls, 9, [0.446, 0.43, 0.46, 0.257], min_L=2, patience=2, peek=2)
        m.set_early_exit(ee.tau, ee.min_L, ee.patience, ee.peek_every)
    else:
        ref = [D.generate_lane(W, P[i], Ls[i], 9) for i in range(24)]
    for _ in range(2):
        b0 = m.stats()["boundary_stages"]
        tok, dep = m.generate(P, Ls, 9)
        st = status_clean(m)
        assert st["tick_layout"] == 3
        assert st["boundary_stages"] > b0
        for i in range(24):
            assert dep[i].tolist() == ref[i].depths.tolist(), i
            _check_tokens(ref[i].tokens, ref[i].logits, tok[i])
