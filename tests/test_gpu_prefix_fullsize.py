"""Shared-prefix serving at full size, checked on a lane subset the oracle computes.

The 1.4B-class BF16 model (d 2048, 16 x 128 heads, 24-layer loop body) with 256
lanes that share one 1024-token prefix and add 64-token suffixes, per-lane L
uniform in {1..4}, in the benchmark's launch configuration: the prefix prefilled
once on a donor lane at the deepest L, every lane's suffix in one batched pass
with the donor's pages mapped ("Benchmark Comparison" (measured benchmarks),
section 2), the cascade attention on.  Eight lanes, two per L value, are
compared with the fp64 oracle (prefix once, then each lane's suffix and tokens):
the first token's logits after the batched suffix pass, the second token's
logits teacher-forced with the oracle's first token (loop steps over all 256
lanes at their own L), and the greedy tokens of a two-token decode of all lanes
wherever the oracle's top-1/top-2 margin exceeds 1e-3.  Bars: logits max-abs
<= 1e-2 and relative L2 <= 2e-3 per position."""

import numpy as np
import pytest

import synthetic as S
import oracle as O
from oracle import model as M

from gpu_helpers import assert_logits_close, status_clean, MARGIN

pytestmark = pytest.mark.gpu

def _subset(Ls, per_L=2):
    picked = []
    for L in (1, 2, 3, 4):
        picked += [i for i, x in enumerate(Ls) if x == L][:per_L]
    return picked

def _oracle_lane_logits(W, pre_cache, Tp, suffix, L, n_tokens_forced):
    """Logits of the first token (end of the suffix) and of the next, fed the
    oracle's own first token; the lane reads the prefix cache's slots of its
    iterations (a position's hidden state at iteration l does not depend on the
    L it was computed at)."""
    cache = M.KVCache(W.shape, pre_cache.max_seq)
    for slot, (K, V, filled) in pre_cache.slots.items():
        if slot[0] == "loop" and slot[1] <= L:
            cache.slots[slot] = (K.copy(), V.copy(), filled.copy())
    h, cache = M.forward(W, suffix, L, cache, pos0=Tp)
    out = [M.head_logits(W, h[-1:])[0]]
    pos = Tp + len(suffix)
    for _ in range(n_tokens_forced):
        tok = int(M.argmax_lowest(out[-1]))
        h, cache = M.forward(W, [tok], L, cache, pos0=pos)
        out.append(M.head_logits(W, h[-1:])[0])
        pos += 1
    return out

def test_m1b4_prefix256_lane_subset_against_oracle():
    import torch
    import dynamic_depth_b200 as T
    from dynamic_depth_b200 import weights as Wt

    wl = S.workload("m1b4_prefix256")
    sh = wl.shape
    pre, suf = S.prefix_prompts(wl)
    Ls = [int(x) for x in wl.per_lane_L]
    n, Tp, Ts, Lmax, page = wl.n_lanes, wl.shared_prefix, wl.prompt_len, 4, 64
    n_new = 2
    max_seq = Tp + Ts + n_new
    pps = -(-max_seq // page)
    slots = sh.n_pre + Lmax * sh.n_loop_layers
    own = pps - Tp // page
    pool = slots * pps + sum((sh.n_pre + L * sh.n_loop_layers) * own for L in Ls)
    donor = n
    cfg = T.config_from_shape(sh, max_lanes=n + 1, max_seq=max_seq, L_max=Lmax, kv_page_tokens=page,
                              kv_pool_pages=pool, max_prefill_tokens=max(Tp + Ts, n * Ts))
    dev = "cuda:0"
    masters = list(S.master_weights(sh))  # drawn once for both sides
    m = T.LoopedLM(cfg, dev)
    m.load_weights(Wt.build_blob(cfg, masters, S.gains(sh), dev))
    prompts = [np.concatenate([pre, suf[i]]) for i in range(n)]
    m.prefill(donor, pre, Lmax)
    m.prefill_batch(list(range(n)), prompts, np.array(Ls, dtype=np.int32), share_from=donor, shared_tokens=Tp)

    V = sh.vocab
    lg = torch.zeros((n + 1, V), dtype=torch.float32, device=dev)
    am = torch.zeros(n + 1, dtype=torch.int32, device=dev)
    mask = torch.zeros(n + 1, dtype=torch.uint8, device=dev)
    mask[:n] = 1
    m.head_logits(mask, lg, am)
    first = lg[:n].double().cpu().numpy()

    # the oracle: the prefix once at the deepest L, then the subset lanes
    W = O.build_weights(sh, masters, S.gains(sh))
    del masters
    _, pre_cache = M.forward(W, pre, Lmax, M.KVCache(sh, max_seq))
    sub = _subset(Ls)
    assert len(sub) == 8
    ref = {i: _oracle_lane_logits(W, pre_cache, Tp, suf[i], Ls[i], 1) for i in sub}
    del pre_cache

    for i in sub:
        assert_logits_close(first[i], ref[i][0], f"lane {i} (L={Ls[i]}) first token")

    # the second token, teacher-forced: every lane takes a token (the oracle's on the subset), then loop
    # steps at each lane's L until every loop finished
    tok = am.clone()
    for i in sub:
        tok[i] = int(M.argmax_lowest(ref[i][0]))
    m.embed_next(mask, tok)
    exit_mask = torch.zeros(n + 1, dtype=torch.uint8, device=dev)
    done = np.zeros(n, dtype=bool)
    for _ in range(Lmax):
        m.loop_step(None, mask, exit_mask)
        done |= exit_mask[:n].cpu().numpy().astype(bool)
        if done.all():
            break
    assert done.all()
    m.head_logits(mask, lg, am)
    second = lg[:n].double().cpu().numpy()
    for i in sub:
        assert_logits_close(second[i], ref[i][1], f"lane {i} (L={Ls[i]}) second token")
    status_clean(m)

    # the decode path (CUDA graphs, cascade): greedy tokens of all lanes, two per lane
    m.prefill_batch(list(range(n)), prompts, np.array(Ls, dtype=np.int32), share_from=donor, shared_tokens=Tp)
    tok_out = torch.zeros((n, n_new), dtype=torch.int32, device=dev)
    dep_out = torch.zeros_like(tok_out)
    m.decode(np.array(Ls, dtype=np.int32), n_new, tok_out, dep_out)
    st = status_clean(m)
    assert st["tokens_emitted"] > 0
    tk = tok_out.cpu().numpy()
    dp = dep_out.cpu().numpy()
    for i in sub:
        assert dp[i].tolist() == [Ls[i]] * n_new
        for t in range(n_new):
            if M.top2_margin(ref[i][t]) <= MARGIN:
                break
            assert int(tk[i, t]) == int(M.argmax_lowest(ref[i][t])), f"lane {i} token {t}"
