"""L warmup on the GPU path against the fp64 oracle ("Dynamic-L Inference",
L scheduling; "CLI Reference", --l-warmup-tokens / --l-warmup-L): decode
tokens 1..N run min(Lw, L) iterations without lowering the cap, later tokens
run the full schedule and, at iterations deeper than a warmup position was
computed, attend to that position's deepest computed iteration (the reading
the oracle's KVCache(deep_fallback=True) defines).

Exact: depth schedules (with early exit too); float: logits per position
within max-abs 1e-2 / relative L2 2e-3, teacher-forced so every position is
compared; greedy tokens equal wherever the oracle's top-2 margin > 1e-3."""
import numpy as np
import pytest

import synthetic as S
from oracle import decode as D
from oracle import model as M

from gpu_helpers import MARGIN, assert_logits_close, gpu_model, oracle_weights, status_clean, teacher_forced

pytestmark = pytest.mark.gpu


def _tokens_agree(ref, got):
    for t in range(len(ref.tokens)):
        if M.top2_margin(ref.logits[t]) <= MARGIN:
            return
        assert int(got[t]) == int(ref.tokens[t]), t


@pytest.mark.parametrize("N,Lw", [(3, 2), (2, 1), (4, 9)])
def test_tiny_warmup_teacher_forced(N, Lw):
    W = oracle_weights("tiny", 7)
    P = S.prompts(3, 12, 512, seed=101)
    Ls = [8, 5, 3]
    m = gpu_model("tiny", 7, max_lanes=3, max_seq=32, L_max=8)
    ref, lg, am, dep = teacher_forced(m, W, P, Ls, 7, warmup=(N, Lw))
    status_clean(m)
    for i in range(3):
        want = [Ls[i]] + [min(Lw, Ls[i])] * N + [Ls[i]] * (6 - N)
        assert ref[i].depths.tolist() == want
        assert dep[i].tolist() == want, i
        for t in range(7):
            assert_logits_close(lg[i, t], ref[i].logits[t], f"lane {i} token {t}")


def test_tiny_warmup_generate_with_early_exit():
    W = oracle_weights("tiny")
    P = S.prompts(3, 12, 512, seed=102)
    Ls = [8, 6, 4]
    ee = D.EarlyExit(0.9, 1, 2, 1)
    ref = [D.generate_lane(W, P[i], Ls[i], 8, ee, warmup_tokens=3, warmup_L=3) for i in range(3)]
    near = [p.margin(ee.tau) for r in ref for p in r.probes if p.margin(ee.tau) <= 1e-2]
    assert not near, near
    m = gpu_model("tiny", None, max_lanes=3, max_seq=32, L_max=8)
    m.set_early_exit(ee.tau, ee.min_L, ee.patience, ee.peek_every)
    m.set_l_warmup(3, 3)
    tok, dep = m.generate(P, Ls, 8)
    status_clean(m)
    for i in range(3):
        assert dep[i].tolist() == ref[i].depths.tolist(), i
        _tokens_agree(ref[i], tok[i])


def test_m407_warmup_teacher_forced():
    W = oracle_weights("m407")
    P = S.prompts(2, 20, S.M407.vocab, seed=103)
    Ls = [8, 5]
    m = gpu_model("m407", None, max_lanes=2, max_seq=32, L_max=8)
    ref, lg, am, dep = teacher_forced(m, W, P, Ls, 5, warmup=(2, 2))
    status_clean(m)
    for i in range(2):
        assert dep[i].tolist() == [Ls[i], 2, 2, Ls[i], Ls[i]]
        for t in range(5):
            assert_logits_close(lg[i, t], ref[i].logits[t], f"lane {i} token {t}")


def test_warmup_off_is_the_plain_schedule():
    W = oracle_weights("tiny")
    P = S.prompts(2, 10, 512, seed=104)
    m = gpu_model("tiny", None, max_lanes=2, max_seq=32, L_max=8)
    m.set_l_warmup(3, 2)
    m.set_l_warmup(0, 2)
    tok, dep = m.generate(P, [6, 3], 5)
    status_clean(m)
    for i, L in enumerate([6, 3]):
        r = D.generate_lane(W, P[i], L, 5)
        assert dep[i].tolist() == [L] * 5
        _tokens_agree(r, tok[i])
