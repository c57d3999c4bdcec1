"""Shared-prefix ("cascade") attention on the GPU path ("Benchmark
Comparison" (measured benchmarks), section 2, SHARED prefix reuse): lanes map
one donor's prefix pages; every decode attention step attends all rows at one
loop iteration to the prefix together on the tensor cores, then each row's own
positions, merged by log-sum-exp.  Checked against the fp64 oracle (each lane
alone, recomputing its whole prompt) on a subset of lanes, with more lanes
than one 128-row cascade tile, for head widths 128 and 64, and against the
same GPU run with the cascade off."""
import numpy as np
import pytest

import synthetic as S
from oracle import decode as D

from gpu_helpers import gpu_model, oracle_weights, status_clean
from test_gpu_wide_paths import _compare, _teacher_forced_subset

pytestmark = pytest.mark.gpu


def _run(name, n, Tp, Ts, n_new, page, check, gain_seed=None, cascade=True, seed=131, act_split=0):
    sh = S.SHAPES[name]
    rng = np.random.Generator(np.random.PCG64(seed))
    pre = rng.integers(0, sh.vocab, Tp).astype(np.int32)
    suf = rng.integers(0, sh.vocab, (n, Ts)).astype(np.int32)
    Ls = [int(x) for x in rng.integers(1, 5, n)]
    prompts = [np.concatenate([pre, suf[i]]) for i in range(n)]
    donor = n
    m = gpu_model(name, gain_seed, max_lanes=n + 1, max_seq=Tp + Ts + n_new, L_max=4, kv_page_tokens=page,
                  max_prefill_tokens=max(Tp + Ts, n * Ts), act_split=act_split)
    m.set_cascade(cascade)
    m.prefill(donor, pre, 4)
    m.prefill_batch(list(range(n)), prompts, Ls, share_from=donor, shared_tokens=Tp)
    W = oracle_weights(name, gain_seed)
    ref = [D.generate_lane(W, prompts[i], Ls[i], n_new) for i in check]
    lg, am, dep, widths = _teacher_forced_subset(m, ref, check, n + 1, n_new, sh.vocab)
    status_clean(m)
    return ref, lg, am, dep, Ls + [4]


def test_cascade_140_lanes_hd128():
    check = [0, 1, 63, 64, 127, 128, 129, 139]
    ref, lg, am, dep, Ls = _run("m1b4_mini", 140, 96, 8, 3, 32, check, gain_seed=5)
    _compare(ref, lg, am, dep, check, Ls, 3)


def test_cascade_70_lanes_hd64():
    check = [0, 17, 34, 69]
    ref, lg, am, dep, Ls = _run("m407", 70, 128, 6, 3, 64, check)
    _compare(ref, lg, am, dep, check, Ls, 3)


def test_cascade_on_off_agree():
    check = [0, 5, 9]
    r1, lg1, _, d1, _ = _run("m1b4_mini", 10, 96, 8, 3, 32, check, gain_seed=5, cascade=True)
    r0, lg0, _, d0, _ = _run("m1b4_mini", 10, 96, 8, 3, 32, check, gain_seed=5, cascade=False)
    assert np.array_equal(d1, d0)
    assert np.max(np.abs(lg1 - lg0)) < 2e-3
