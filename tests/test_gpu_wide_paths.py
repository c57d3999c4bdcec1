"""The 407M-class model on the kernel paths the 64-lane continuous-depth
workload takes at full size, against the fp64 oracle through the C ABI.

* 64 lanes with 520-token prompts and the workload's per-lane L draw
  (Poisson(8) clamped to [2, 32], seed 2): loop steps start at 64 rows on the
  tensor cores (fp16 operands, fp16-rounded dequantised weights) and shrink
  through the CUDA-core GEMV as lanes finish; decode attention runs one
  context split per (row, head), so every CTA chains 17+ key blocks through
  the online-softmax rescale.  Teacher-forced for 3 tokens (the oracle's
  tokens for the compared lanes, the GPU's own greedy tokens for the rest);
  8 lanes spanning the drawn L values are compared with the oracle.
* 16 lanes at L = 32 on the tensor-core path (the deepest iteration count the
  logits tolerance is stated for).

Bars: logits max-abs <= 1e-2 and relative L2 <= 2e-3 per position; depths
exact; greedy tokens equal wherever the oracle's top-1/top-2 margin > 1e-3
("Dynamic-L Inference", "L-Aware Batching": a batch with a loop count per lane
gives each lane what it gives alone)."""
import numpy as np
import pytest

import synthetic as S
from oracle import decode as D
from oracle import model as M

from gpu_helpers import MARGIN, assert_logits_close, gpu_model, oracle_weights, status_clean

pytestmark = pytest.mark.gpu


def _spanning_lanes(Ls, k):
    """k lanes whose L values span the draw: the lowest, the highest and evenly spaced ranks between."""
    order = np.argsort(np.asarray(Ls), kind="stable")
    picks = [int(order[round(j * (len(order) - 1) / (k - 1))]) for j in range(k)]
    return sorted(set(picks))


def _teacher_forced_subset(m, ref, check, n_lanes, n_new, V):
    """Drive all n_lanes lanes (already prefilled) for n_new tokens: lanes in
    `check` take the oracle's tokens, the others their own greedy tokens.
    Returns GPU logits [len(check), n_new, V], argmax and depths for `check`."""
    import torch
    dev = m.device
    logits = torch.zeros((n_lanes, V), dtype=torch.float32, device=dev)
    argmax = torch.zeros(n_lanes, dtype=torch.int32, device=dev)
    mask = torch.ones(n_lanes, dtype=torch.uint8, device=dev)
    exit_mask = torch.zeros(n_lanes, dtype=torch.uint8, device=dev)
    out_lg = np.zeros((len(check), n_new, V))
    out_am = np.zeros((len(check), n_new), dtype=np.int64)
    depths = np.zeros((n_lanes, n_new), dtype=np.int64)
    widths = []
    for t in range(n_new):
        if t > 0:
            tok = argmax.clone()
            for j, ln in enumerate(check):
                tok[ln] = int(ref[j].tokens[t - 1])
            m.embed_next(mask, tok)
            done = np.zeros(n_lanes, dtype=bool)
            it = 0
            while not done.all():
                widths.append(int((~done).sum()))
                m.loop_step(None, mask, exit_mask)
                it += 1
                em = exit_mask.cpu().numpy().astype(bool)
                depths[em & ~done, t] = it
                done |= em
                assert it <= 40
        m.head_logits(mask, logits, argmax)
        lg = logits.cpu().numpy()
        am = argmax.cpu().numpy()
        for j, ln in enumerate(check):
            out_lg[j, t] = lg[ln]
            out_am[j, t] = am[ln]
    return out_lg, out_am, depths, widths


def _compare(ref, lg, am, depths, check, Ls, n_new):
    worst = (0.0, 0.0)
    for j, ln in enumerate(check):
        assert depths[ln, 1:].tolist() == [Ls[ln]] * (n_new - 1), f"lane {ln}"
        for t in range(n_new):
            mx, rl = assert_logits_close(lg[j, t], ref[j].logits[t], f"lane {ln} (L={Ls[ln]}) token {t}")
            worst = (max(worst[0], mx), max(worst[1], rl))
            if M.top2_margin(ref[j].logits[t]) > MARGIN:
                assert am[j, t] == ref[j].tokens[t], f"lane {ln} token {t}"
    return worst


def test_m407_64_lanes_520_token_prompts_workload_L():
    n, T, n_new = 64, 520, 3
    wl = S.workload("m407_cdb64")
    Ls = [int(x) for x in wl.per_lane_L]
    assert len(Ls) == n and max(Ls) >= 12
    V = S.M407.vocab
    W = oracle_weights("m407")
    P = S.prompts(n, T, V, seed=91)
    check = _spanning_lanes(Ls, 8)
    assert len(check) == 8 and min(Ls[c] for c in check) == min(Ls) and max(Ls[c] for c in check) == max(Ls)
    ref = [D.generate_lane(W, P[ln], Ls[ln], n_new) for ln in check]
    m = gpu_model("m407", None, max_lanes=n, max_seq=T + n_new, L_max=max(Ls), max_prefill_tokens=n * T)
    m.prefill_batch(list(range(n)), list(P), Ls)
    lg, am, depths, widths = _teacher_forced_subset(m, ref, check, n, n_new, V)
    status_clean(m)
    assert max(widths) == n and min(widths) <= 8  # tensor-core widths down to the GEMV's
    _compare(ref, lg, am, depths, check, Ls, n_new)


def test_m407_16_lanes_L32_tensor_core_path():
    n, T, n_new, L = 16, 24, 2, 32
    V = S.M407.vocab
    W = oracle_weights("m407")
    P = S.prompts(n, T, V, seed=92)
    Ls = [L] * n
    ref = [D.generate_lane(W, P[i], L, n_new) for i in range(n)]
    m = gpu_model("m407", None, max_lanes=n, max_seq=T + n_new, L_max=L, max_prefill_tokens=n * T)
    m.prefill_batch(list(range(n)), list(P), Ls)
    lg, am, depths, widths = _teacher_forced_subset(m, ref, list(range(n)), n, n_new, V)
    status_clean(m)
    assert min(widths) == n  # every step of the decoded token ran all 16 rows on the tensor cores
    _compare(ref, lg, am, depths, list(range(n)), Ls, n_new)
