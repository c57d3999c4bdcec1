"""Split activations for the tensor-core projections (tl_config.act_split = 1):
every fp16 activation copy (norm output, attention output, SwiGLU output) is
stored as hi = fp16(x) and lo = fp16(x - hi), and every tensor-core projection
multiplies both halves by the same weights.  Checked against the fp64 oracle
through the C ABI on the paths that produce or consume those copies: decode
projections on the tensor cores (INT4 and BF16), the persistent prompt GEMM
over 512+ rows (INT4 with in-kernel dequant, BF16 through the fp16 staging),
tensor-core prompt attention (hd 64, 128) and the CUDA-core one (hd 32), and
the shared-prefix cascade merge.  With the split, the logits' error against
the oracle is below that of single fp16 activations on the same inputs.  Bars
as elsewhere: logits max-abs <= 1e-2 and relative L2 <= 2e-3 per position,
depths exact."""
import numpy as np
import pytest

import synthetic as S
from oracle import decode as D

from gpu_helpers import assert_logits_close, gpu_model, oracle_weights, rel_l2, status_clean, teacher_forced
from test_gpu_cascade import _run as cascade_run
from test_gpu_wide_paths import _compare, _teacher_forced_subset

pytestmark = pytest.mark.gpu


def _m407_l32_errors(act_split):
    n, T, n_new, L = 16, 24, 2, 32
    V = S.M407.vocab
    W = oracle_weights("m407")
    P = S.prompts(n, T, V, seed=92)
    Ls = [L] * n
    ref = [D.generate_lane(W, P[i], L, n_new) for i in range(n)]
    m = gpu_model("m407", None, max_lanes=n, max_seq=T + n_new, L_max=L, max_prefill_tokens=n * T,
                  act_split=act_split)
    m.prefill_batch(list(range(n)), list(P), Ls)
    lg, am, depths, widths = _teacher_forced_subset(m, ref, list(range(n)), n, n_new, V)
    status_clean(m)
    assert min(widths) == n  # every loop step on the tensor cores
    _compare(ref, lg, am, depths, list(range(n)), Ls, n_new)
    return [rel_l2(lg[i, t], ref[i].logits[t]) for i in range(n) for t in range(n_new)]


def test_m407_l32_tensor_cores_split_activations_closer_to_the_oracle():
    split = _m407_l32_errors(1)
    single = _m407_l32_errors(2)
    assert np.mean(split) < np.mean(single), (np.mean(split), np.mean(single))


@pytest.mark.parametrize("name,gains,n,T,Ls,max_seq", [
    ("tiny", 7, 8, 70, [3, 8, 1, 5, 8, 2, 6, 4], 80),
    ("m407", None, 4, 160, [2, 4, 3, 1], 168),
    ("m1b4_mini", 5, 6, 100, [1, 2, 3, 4, 4, 2], 108),
])
def test_split_activations_wide_prompt_batch(name, gains, n, T, Ls, max_seq):
    sh = S.SHAPES[name]
    W = oracle_weights(name, gains)
    P = list(S.prompts(n, T, sh.vocab, seed=94))
    m = gpu_model(name, gains, max_lanes=n, max_seq=max_seq, L_max=8, max_prefill_tokens=n * T, act_split=1)

    def prefill(i, ln):
        if i == 0:
            m.prefill_batch(list(range(n)), P, Ls)

    ref, lg, am, dep = teacher_forced(m, W, P, Ls, 2, prefill=prefill)
    status_clean(m)
    for i in range(n):
        assert dep[i].tolist() == ref[i].depths.tolist()
        for t in range(2):
            assert_logits_close(lg[i, t], ref[i].logits[t], f"{name} lane {i} token {t}")


def test_split_activations_tiny_wide_decode():
    # 12 lanes: loop steps above 8 rows run on the tensor cores; hd 32 prompt attention on CUDA cores
    W = oracle_weights("tiny", 7)
    P = S.prompts(12, 16, 512, seed=71)
    Ls = [2, 3, 4, 5] * 3
    m = gpu_model("tiny", 7, max_lanes=12, max_seq=32, L_max=8, act_split=1)
    ref, lg, am, dep = teacher_forced(m, W, P, Ls, 4)
    status_clean(m)
    for i in range(12):
        assert dep[i].tolist() == ref[i].depths.tolist()
        for t in range(4):
            assert_logits_close(lg[i, t], ref[i].logits[t], f"lane {i} token {t}")


def test_split_activations_cascade_hd128():
    check = [0, 63, 128, 139]
    ref, lg, am, dep, Ls = cascade_run("m1b4_mini", 140, 96, 8, 3, 32, check, gain_seed=5, act_split=1)
    _compare(ref, lg, am, dep, check, Ls, 3)
