"""Logit-margin early exit on the GPU path against the fp64 oracle ("CLI
Reference", --early-exit-logit-margin: the probe's metric is the top-1 minus
top-2 margin of the head's logits at that iteration; "Current Behavior": the
mode that fires).  Exact: depth schedules and exit masks; greedy tokens equal
wherever the oracle's top-2 margin > 1e-3; logits within the usual bars.

A threshold is only used where exits fire and no oracle probe sits within a
guard band of it (the GPU's fp32 logits may differ from the oracle's by far
less than the band, so every decision is the oracle's)."""
import numpy as np
import pytest

import synthetic as S
from oracle import decode as D
from oracle import model as M

from gpu_helpers import MARGIN, assert_logits_close, gpu_model, oracle_weights, status_clean

pytestmark = pytest.mark.gpu

BAND = 2e-3
CANDS = [round(0.04 + 0.0113 * k, 4) for k in range(24)]  # 0.04 .. 0.30


def _pick(W, P, Ls, n_new, cands, min_L, patience, peek):
    """The first candidate threshold whose oracle run exits early somewhere
    with no probe margin within BAND of it."""
    for thr in cands:
        ee = D.EarlyExit(min_L=min_L, patience=patience, peek_every=peek, logit_margin=thr)
        ref = [D.generate_lane(W, P[i], Ls[i], n_new, ee) for i in range(len(Ls))]
        near = [p.delta for r in ref for p in r.probes if abs(p.delta - thr) <= BAND]
        fired = any(int(r.depths[t]) < min(Ls[i], int(r.depths[t - 1]))
                    for i, r in enumerate(ref) for t in range(1, n_new))
        if fired and not near:
            return ee, ref
    pytest.fail("no candidate threshold both fires and stays clear of every probe")


def _tokens_agree(ref, got):
    for t in range(len(ref.tokens)):
        if M.top2_margin(ref.logits[t]) <= MARGIN:
            return
        assert int(got[t]) == int(ref.tokens[t]), t


@pytest.mark.parametrize("min_L,patience,peek", [(1, 1, 1), (2, 2, 1), (1, 1, 2)])
def test_tiny_margin_exit_generate(min_L, patience, peek):
    W = oracle_weights("tiny")
    P = S.prompts(4, 12, 512, seed=111)
    Ls = [8, 6, 5, 3]
    ee, ref = _pick(W, P, Ls, 8, CANDS, min_L, patience, peek)
    m = gpu_model("tiny", None, max_lanes=4, max_seq=32, L_max=8)
    m.set_early_exit_logit_margin(ee.logit_margin, ee.min_L, ee.patience, ee.peek_every)
    tok, dep = m.generate(P, Ls, 8)
    status_clean(m)
    for i in range(4):
        assert dep[i].tolist() == ref[i].depths.tolist(), (i, ee)
        _tokens_agree(ref[i], tok[i])


def test_tiny_margin_exit_teacher_forced_masks_and_logits():
    import torch
    W = oracle_weights("tiny", 7)
    P = S.prompts(3, 10, 512, seed=112)
    Ls = [8, 7, 4]
    n_new = 6
    ee, ref = _pick(W, P, Ls, n_new, CANDS, 1, 1, 1)
    m = gpu_model("tiny", 7, max_lanes=3, max_seq=32, L_max=8)
    m.set_early_exit_logit_margin(ee.logit_margin, ee.min_L, ee.patience, ee.peek_every)
    for i in range(3):
        m.prefill(i, P[i], Ls[i])
    dev = m.device
    logits = torch.zeros((3, 512), dtype=torch.float32, device=dev)
    argmax = torch.zeros(3, dtype=torch.int32, device=dev)
    mask = torch.ones(3, dtype=torch.uint8, device=dev)
    exit_mask = torch.zeros(3, dtype=torch.uint8, device=dev)
    for t in range(n_new):
        if t > 0:
            tok = torch.tensor([int(r.tokens[t - 1]) for r in ref], dtype=torch.int32, device=dev)
            m.embed_next(mask, tok)
            done = np.zeros(3, dtype=bool)
            it = 0
            while not done.all():
                m.loop_step(None, mask, exit_mask)
                it += 1
                em = exit_mask.cpu().numpy().astype(bool)
                # the exit mask of every step is the oracle's: a lane finishes exactly at its depth
                for i in range(3):
                    if not done[i]:
                        assert em[i] == (it == int(ref[i].depths[t])), (i, t, it)
                done |= em
        m.head_logits(mask, logits, argmax)
        lg = logits.cpu().numpy()
        for i in range(3):
            assert_logits_close(lg[i], ref[i].logits[t], f"lane {i} token {t}")
    status_clean(m)


def test_m407_margin_exit_generate():
    W = oracle_weights("m407")
    P = S.prompts(3, 16, S.M407.vocab, seed=113)
    Ls = [8, 6, 4]
    ee, ref = _pick(W, P, Ls, 6, [round(0.1 + 0.0413 * k, 4) for k in range(12)], 2, 1, 1)
    m = gpu_model("m407", None, max_lanes=3, max_seq=32, L_max=8)
    m.set_early_exit_logit_margin(ee.logit_margin, ee.min_L, ee.patience, ee.peek_every)
    tok, dep = m.generate(P, Ls, 6)
    status_clean(m)
    for i in range(3):
        assert dep[i].tolist() == ref[i].depths.tolist(), (i, ee)
        _tokens_agree(ref[i], tok[i])


def test_tiny_margin_exit_wide_batch_tensor_core_probes():
    # 12 lanes: probes of more than 8 rows take the tensor-core head
    W = oracle_weights("tiny")
    P = S.prompts(12, 12, 512, seed=114)
    Ls = [8, 7, 6, 5] * 3
    ee, ref = _pick(W, P, Ls, 6, CANDS, 1, 1, 1)
    m = gpu_model("tiny", None, max_lanes=12, max_seq=32, L_max=8)
    m.set_early_exit_logit_margin(ee.logit_margin, ee.min_L, ee.patience, ee.peek_every)
    tok, dep = m.generate(P, Ls, 6)
    status_clean(m)
    for i in range(12):
        assert dep[i].tolist() == ref[i].depths.tolist(), (i, ee)
        _tokens_agree(ref[i], tok[i])
