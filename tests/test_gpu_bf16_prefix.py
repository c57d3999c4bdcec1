"""Parity of the BF16 weight paths, 128-wide heads, a multi-layer loop body
with no pre blocks, and shared-prefix KV pages (the layout of the 1.4B-class
shared-prefix workload at test size), plus the 407M-class model with a BF16
loop block.  Same bars as the other parity tests: logits max-abs <= 1e-2 and
relative L2 <= 2e-3 per position, exact depth schedules, and greedy tokens
wherever the oracle's top-1/top-2 margin exceeds 1e-3."""
import numpy as np
import pytest

import synthetic as S
from oracle import decode as D
from oracle import model as M

from gpu_helpers import assert_logits_close, gpu_model, oracle_weights, status_clean, teacher_forced, MARGIN

pytestmark = pytest.mark.gpu

GAINS = 5  # random RMSNorm gains, so a wrong gain index shows


def _prefix_case():
    wl = S.workload("m1b4_mini_prefix")
    pre, suf = S.prefix_prompts(wl)
    prompts = [np.concatenate([pre, suf[i]]).astype(np.int32) for i in range(wl.n_lanes)]
    return wl, pre, prompts


def _model(max_lanes, max_seq=112, L_max=4):
    return gpu_model("m1b4_mini", GAINS, max_lanes=max_lanes, max_seq=max_seq, L_max=L_max, kv_page_tokens=32,
                     max_prefill_tokens=min(104, max_seq))


def test_mini_bf16_shared_prefix_teacher_forced():
    # lane 4 holds the prefix at the deepest L; lanes 0..3 map its 3 pages of
    # every slot and compute only their own suffix positions
    wl, pre, prompts = _prefix_case()
    W = oracle_weights("m1b4_mini", GAINS)
    m = _model(5)
    m.prefill(4, pre, 4)
    Ls = list(wl.per_lane_L)

    def shared(i, ln):
        m.prefill(ln, prompts[i], Ls[i], share_from=4, shared_tokens=wl.shared_prefix)

    ref, lg, am, dep = teacher_forced(m, W, prompts, Ls, wl.n_new, lanes=[0, 1, 2, 3], prefill=shared)
    status_clean(m)
    for i in range(wl.n_lanes):
        assert dep[i].tolist() == ref[i].depths.tolist()
        for t in range(wl.n_new):
            assert_logits_close(lg[i, t], ref[i].logits[t], f"lane {i} token {t}")
            if M.top2_margin(ref[i].logits[t]) > MARGIN:
                assert am[i, t] == ref[i].tokens[t]


def test_mini_bf16_shared_prefix_decode_matches_oracle():
    wl, pre, prompts = _prefix_case()
    W = oracle_weights("m1b4_mini", GAINS)
    m = _model(5)
    m.prefill(4, pre, 4)
    for i in range(wl.n_lanes):
        m.prefill(i, prompts[i], wl.per_lane_L[i], share_from=4, shared_tokens=wl.shared_prefix)
    import torch
    tok = torch.zeros((wl.n_lanes, wl.n_new), dtype=torch.int32, device="cuda")
    dep = torch.zeros_like(tok)
    m.decode(list(wl.per_lane_L), wl.n_new, tok, dep)
    status_clean(m)
    tok, dep = tok.cpu().numpy(), dep.cpu().numpy()
    for i in range(wl.n_lanes):
        r = D.generate_lane(W, prompts[i], wl.per_lane_L[i], wl.n_new)
        assert dep[i].tolist() == r.depths.tolist()
        for t in range(wl.n_new):
            if M.top2_margin(r.logits[t]) <= MARGIN:
                break
            assert int(tok[i, t]) == int(r.tokens[t]), (i, t)


def test_mini_shared_prefix_needs_deep_enough_donor():
    from dynamic_depth_b200 import TlError
    wl, pre, prompts = _prefix_case()
    m = _model(5)
    m.prefill(4, pre, 2)
    with pytest.raises(TlError) as e:
        m.prefill(0, prompts[0], 3, share_from=4, shared_tokens=wl.shared_prefix)
    assert e.value.status == -1  # TL_EINVAL: the donor has no iteration-3 pages
    m.prefill(0, prompts[0], 2, share_from=4, shared_tokens=wl.shared_prefix)
    status_clean(m)


def test_mini_bf16_wide_batch_tensor_cores():
    # 12 lanes: the loop body runs on the tensor-core path with BF16 weights,
    # 128-wide heads and FFN / vocab tiles with ragged ends
    W = oracle_weights("m1b4_mini", GAINS)
    P = S.prompts(12, 20, S.M1B4_MINI.vocab, seed=81)
    Ls = [1, 2, 3, 4] * 3
    m = _model(12, max_seq=32, L_max=4)
    ref, lg, am, dep = teacher_forced(m, W, P, Ls, 3)
    status_clean(m)
    for i in range(12):
        assert dep[i].tolist() == ref[i].depths.tolist()
        for t in range(3):
            assert_logits_close(lg[i, t], ref[i].logits[t], f"lane {i} token {t}")


@pytest.mark.parametrize("L", [2, 8])
def test_m407_bf16_loop_block_decode_logits(L):
    W = oracle_weights("m407_bf16loop")
    P = S.prompts(1, 32, S.M407.vocab)
    m = gpu_model("m407_bf16loop", None, max_lanes=1, max_seq=40, L_max=8)
    ref, lg, am, dep = teacher_forced(m, W, P, [L], 3)
    status_clean(m)
    for t in range(3):
        assert_logits_close(lg[0, t], ref[0].logits[t], f"L={L} token {t}")
        if M.top2_margin(ref[0].logits[t]) > MARGIN:
            assert am[0, t] == ref[0].tokens[t]
