"""Helpers for the GPU parity tests: build the oracle and the CUDA model from
the same seeded inputs, drive the CUDA path through the C ABI, and compare."""
from __future__ import annotations

import functools

import numpy as np

import synthetic as S
import oracle as O


@functools.lru_cache(maxsize=4)
def oracle_weights(name: str, gain_seed=None):
    sh = S.SHAPES[name]
    return O.build_weights(sh, S.master_weights(sh), S.gains(sh, gain_seed))


def gpu_model(name: str, gain_seed=None, device="cuda:0", **capacity):
    import dynamic_depth_b200 as T
    from dynamic_depth_b200 import weights as Wt
    sh = S.SHAPES[name]
    cfg = T.config_from_shape(sh, **capacity)
    m = T.LoopedLM(cfg, device)
    blob = Wt.build_blob(cfg, S.master_weights(sh), S.gains(sh, gain_seed), device)
    m.load_weights(blob)
    return m


def rel_l2(a, b) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


LOGIT_MAX_ABS = 1e-2
LOGIT_REL_L2 = 2e-3
MARGIN = 1e-3


def assert_logits_close(got, want, where=""):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    mx = float(np.max(np.abs(got - want)))
    rl = rel_l2(got, want)
    assert mx <= LOGIT_MAX_ABS and rl <= LOGIT_REL_L2, f"{where}: max-abs {mx:.3g}, rel-L2 {rl:.3g}"
    return mx, rl


def status_clean(m):
    st = m.stats()
    assert st["device_status"] == 0, f"device status word {st['device_status']:#x}"
    return st


def teacher_forced(m, W, prompts, Ls, n_new, ee=None, lanes=None, torch=None, prefill=None, warmup=(0, 2)):
    """Drive the CUDA path with the oracle's tokens (prefill, head, then
    embed_next + loop steps until every lane's loop finished, head again).
    prefill(i, lane) replaces the plain m.prefill of prompt i when given.
    Returns (oracle results, GPU logits [n_lanes, n_new, V], GPU argmax, GPU
    depths [n_lanes, n_new])."""
    import torch as _t
    torch = torch or _t
    from oracle import decode as D
    ee = ee or D.EarlyExit()
    n = len(prompts)
    lanes = list(range(n)) if lanes is None else lanes
    ref = [D.generate_lane(W, prompts[i], Ls[i], n_new, ee, warmup_tokens=warmup[0], warmup_L=warmup[1])
           for i in range(n)]
    V = W.shape.vocab
    max_lanes = m.cfg.max_lanes
    dev = m.device
    logits = torch.zeros((max_lanes, V), dtype=torch.float32, device=dev)
    argmax = torch.zeros(max_lanes, dtype=torch.int32, device=dev)
    mask = torch.zeros(max_lanes, dtype=torch.uint8, device=dev)
    mask[lanes] = 1
    exit_mask = torch.zeros(max_lanes, dtype=torch.uint8, device=dev)
    tok = torch.zeros(max_lanes, dtype=torch.int32, device=dev)
    m.set_early_exit(ee.tau, ee.min_L, ee.patience, ee.peek_every)
    m.set_l_warmup(warmup[0], warmup[1])
    for i, ln in enumerate(lanes):
        if prefill is None:
            m.prefill(ln, prompts[i], Ls[i])
        else:
            prefill(i, ln)
    out_logits = np.zeros((n, n_new, V))
    out_arg = np.zeros((n, n_new), dtype=np.int64)
    depths = np.zeros((n, n_new), dtype=np.int64)
    depths[:, 0] = [Ls[i] for i in range(n)]
    for t in range(n_new):
        if t > 0:
            tok[lanes] = torch.tensor([int(r.tokens[t - 1]) for r in ref], dtype=torch.int32, device=dev)
            m.embed_next(mask, tok)
            done = np.zeros(n, dtype=bool)
            it = 0
            while not done.all():
                m.loop_step(None, mask, exit_mask)
                it += 1
                em = exit_mask.cpu().numpy()
                for i, ln in enumerate(lanes):
                    if not done[i] and em[ln]:
                        done[i] = True
                        depths[i, t] = it
                assert it <= 64
        m.head_logits(mask, logits, argmax)
        lg = logits.cpu().numpy()
        am = argmax.cpu().numpy()
        for i, ln in enumerate(lanes):
            out_logits[i, t] = lg[ln]
            out_arg[i, t] = am[ln]
    return ref, out_logits, out_arg, depths
