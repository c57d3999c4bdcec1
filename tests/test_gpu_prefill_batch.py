"""Batched prompts (tl_prefill_batch): several lanes with different prompt
lengths and loop counts in one pass over the weights, against the fp64 oracle.
Bars as in the other parity tests (logits max-abs <= 1e-2, relative L2 <=
2e-3 per position, exact depth schedules)."""
import numpy as np
import pytest

import synthetic as S
from oracle import model as M

from gpu_helpers import assert_logits_close, gpu_model, oracle_weights, status_clean, teacher_forced, MARGIN

pytestmark = pytest.mark.gpu


def _ragged_prompts(n, lengths, vocab, seed):
    P = S.prompts(n, max(lengths), vocab, seed=seed)
    return [P[i, :lengths[i]].copy() for i in range(n)]


def _batch_once(m, lanes, prompts, Ls, **kw):
    done = []

    def prefill(i, ln):  # the first lane's turn prefills all of them together
        if not done:
            m.prefill_batch(lanes, prompts, Ls, **kw)
            done.append(1)
    return prefill


@pytest.mark.parametrize("gains", [None, 7])
def test_tiny_prompt_batch_teacher_forced(gains):
    # 5 lanes, lengths 1..70 (tiles of 64 rows with ragged ends), L from 1 to 8
    W = oracle_weights("tiny", gains)
    lens = [70, 1, 33, 64, 9]
    Ls = [3, 8, 1, 5, 8]
    P = _ragged_prompts(5, lens, 512, seed=91)
    m = gpu_model("tiny", gains, max_lanes=5, max_seq=80, L_max=8, max_prefill_tokens=200)
    ref, lg, am, dep = teacher_forced(m, W, P, Ls, 3, prefill=_batch_once(m, list(range(5)), P, Ls))
    status_clean(m)
    for i in range(5):
        assert dep[i].tolist() == ref[i].depths.tolist()
        for t in range(3):
            assert_logits_close(lg[i, t], ref[i].logits[t], f"lane {i} token {t}")
            if M.top2_margin(ref[i].logits[t]) > MARGIN:
                assert am[i, t] == ref[i].tokens[t]


def test_m407_prompt_batch_logits():
    # the 407M-class model: 6 lanes in one pass run on the tensor-core path
    W = oracle_weights("m407")
    lens = [40, 17, 64, 5, 33, 40]
    Ls = [3, 8, 1, 5, 8, 2]
    P = _ragged_prompts(6, lens, S.M407.vocab, seed=92)
    m = gpu_model("m407", None, max_lanes=6, max_seq=72, L_max=8, max_prefill_tokens=256)
    ref, lg, am, dep = teacher_forced(m, W, P, Ls, 2, prefill=_batch_once(m, list(range(6)), P, Ls))
    status_clean(m)
    for i in range(6):
        for t in range(2):
            assert_logits_close(lg[i, t], ref[i].logits[t], f"lane {i} token {t}")


def test_mini_prompt_batch_with_shared_prefix():
    wl = S.workload("m1b4_mini_prefix")
    pre, suf = S.prefix_prompts(wl)
    prompts = [np.concatenate([pre, suf[i]]).astype(np.int32) for i in range(wl.n_lanes)]
    W = oracle_weights("m1b4_mini", 5)
    m = gpu_model("m1b4_mini", 5, max_lanes=5, max_seq=112, L_max=4, kv_page_tokens=32, max_prefill_tokens=128)
    m.prefill(4, pre, 4)
    Ls = list(wl.per_lane_L)
    pf = _batch_once(m, [0, 1, 2, 3], prompts, Ls, share_from=4, shared_tokens=wl.shared_prefix)
    ref, lg, am, dep = teacher_forced(m, W, prompts, Ls, 2, lanes=[0, 1, 2, 3], prefill=pf)
    status_clean(m)
    for i in range(wl.n_lanes):
        assert dep[i].tolist() == ref[i].depths.tolist()
        for t in range(2):
            assert_logits_close(lg[i, t], ref[i].logits[t], f"lane {i} token {t}")


def test_prompt_batch_rejects_bad_arguments():
    from dynamic_depth_b200 import TlError
    m = gpu_model("tiny", None, max_lanes=4, max_seq=32, L_max=4, max_prefill_tokens=40)
    P = _ragged_prompts(3, [20, 20, 20], 512, seed=93)
    with pytest.raises(TlError):  # 60 rows > 40
        m.prefill_batch([0, 1, 2], P, [2, 2, 2])
    with pytest.raises(TlError):  # a lane twice
        m.prefill_batch([0, 0], P[:2], [2, 2])
    with pytest.raises(TlError):  # L above L_max
        m.prefill_batch([0, 1], P[:2], [2, 5])
    m.prefill_batch([0, 1], P[:2], [2, 3])
    status_clean(m)


# ------------------------------------------- >= 512 prompt rows: persistent GEMM

@pytest.mark.parametrize("name,gains,n,T,Ls,max_seq", [
    ("tiny", 7, 8, 70, [3, 8, 1, 5, 8, 2, 6, 4], 80),
    ("tiny", None, 8, 70, [2] * 8, 80),  # every stage wide: the last block's residual is added after it
    ("m407", None, 4, 160, [2, 4, 3, 1], 168),
    ("m1b4_mini", 5, 6, 100, [1, 2, 3, 4, 4, 2], 108),
])
def test_wide_prompt_batch_persistent_gemm(name, gains, n, T, Ls, max_seq):
    # 512+ prompt rows in one pass: every projection of the prompt runs on the
    # persistent tensor-core kernel (INT4 and BF16, single matrix and gate/up pair),
    # and the residual projections leave their sums to the next norm kernel,
    # including across a stage that drops below 512 rows
    sh = S.SHAPES[name]
    W = oracle_weights(name, gains)
    P = list(S.prompts(n, T, sh.vocab, seed=94))
    m = gpu_model(name, gains, max_lanes=n, max_seq=max_seq, L_max=8, max_prefill_tokens=n * T)
    ref, lg, am, dep = teacher_forced(m, W, P, Ls, 2, prefill=_batch_once(m, list(range(n)), P, Ls))
    status_clean(m)
    for i in range(n):
        assert dep[i].tolist() == ref[i].depths.tolist()
        for t in range(2):
            assert_logits_close(lg[i, t], ref[i].logits[t], f"{name} lane {i} token {t}")
