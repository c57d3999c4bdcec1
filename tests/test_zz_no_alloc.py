"""The allocation-free greedy head (tl_head_argmax_static) against the
workspace-based head (tl_head_logits) on the same model and lanes.

tl_head_argmax_static is for callers that cannot allocate device memory when
they run the head (memory reserved once at start-up, an allocator owned by a
host framework, or code running during stream capture): it keeps its scratch
in a fixed array inside the library instead of a tl_create workspace.  This
file is collected last so that a run stopping at the first failure has run
every other test before it."""
import ctypes as C

import numpy as np
import pytest

import synthetic as S

from gpu_helpers import assert_logits_close, gpu_model, status_clean

pytestmark = pytest.mark.gpu

LANE_STATE_BYTES = 13 * 4  # int32 fields of one lane's scheduling state


def _head_inputs(name, n_lanes, prompt_len, L):
    import torch
    import dynamic_depth_b200 as T
    from dynamic_depth_b200 import weights as Wt
    sh = S.SHAPES[name]
    cfg = T.config_from_shape(sh, max_lanes=n_lanes, max_seq=prompt_len + 4, L_max=L)
    blob = Wt.build_blob(cfg, S.master_weights(sh), S.gains(sh, 7), "cuda:0")
    m = T.LoopedLM(cfg, "cuda:0")
    m.load_weights(blob)
    P = S.prompts(n_lanes, prompt_len, sh.vocab, seed=81)
    for i in range(n_lanes):
        m.prefill(i, P[i], L)
    # the workspace-based head on every lane
    mask = torch.ones(n_lanes, dtype=torch.uint8, device="cuda")
    ref_logits = torch.zeros((n_lanes, sh.vocab), dtype=torch.float32, device="cuda")
    ref_arg = torch.zeros(n_lanes, dtype=torch.int32, device="cuda")
    m.head_logits(mask, ref_logits, ref_arg)
    snap = m.lane_state_save()
    torch.cuda.synchronize()
    status_clean(m)
    h = snap[LANE_STATE_BYTES * n_lanes:].view(torch.float32).reshape(n_lanes, sh.d).clone()
    # head weights and final gain in the blob's layout
    V, d, g = sh.vocab, sh.d, cfg.group
    head_bytes = V * d // 2 + V * (d // g) * 2
    gains_bytes = (2 * (sh.n_pre + sh.n_loop_layers) + 1) * d * 4
    head = blob[len(blob) - gains_bytes - head_bytes: len(blob) - gains_bytes]
    packed = torch.from_numpy(head[:V * d // 2].copy()).cuda()
    scales = torch.from_numpy(head[V * d // 2:].copy().view(np.int16)).cuda()
    g_final = torch.from_numpy(blob[len(blob) - d * 4:].copy().view(np.float32)).cuda()
    return cfg, sh, h, g_final, packed, scales, ref_logits.cpu().numpy(), ref_arg.cpu().numpy()


def _call_static(cfg, sh, h_rows, g_final, packed, scales):
    import torch
    from dynamic_depth_b200 import check, lib
    rows = h_rows.shape[0]
    logits = torch.full((rows, sh.vocab), float("nan"), dtype=torch.float32, device="cuda")
    arg = torch.full((rows,), -1, dtype=torch.int32, device="cuda")
    check(lib().tl_head_argmax_static(h_rows.data_ptr(), rows, g_final.data_ptr(), C.c_float(cfg.rms_eps),
                                      packed.data_ptr(), scales.data_ptr(), sh.vocab, sh.d, cfg.group,
                                      logits.data_ptr(), arg.data_ptr(), torch.cuda.current_stream().cuda_stream),
          "tl_head_argmax_static")
    torch.cuda.synchronize()
    return logits.cpu().numpy(), arg.cpu().numpy()


def _check(got_logits, got_arg, ref_logits, ref_arg, lanes):
    for k, i in enumerate(lanes):
        assert_logits_close(got_logits[k], ref_logits[i], f"lane {i}")
        s = np.sort(ref_logits[i])
        if s[-1] - s[-2] > 1e-3:
            assert int(got_arg[k]) == int(ref_arg[i]), f"lane {i}"


@pytest.mark.parametrize("name,n_lanes,prompt_len,L", [("tiny", 6, 16, 3), ("m407", 3, 24, 2)])
def test_static_head_matches_workspace_head_on_consecutive_calls(name, n_lanes, prompt_len, L):
    cfg, sh, h, g_final, packed, scales, ref_logits, ref_arg = _head_inputs(name, n_lanes, prompt_len, L)
    # first call: all lanes
    lg, arg = _call_static(cfg, sh, h, g_final, packed, scales)
    _check(lg, arg, ref_logits, ref_arg, list(range(n_lanes)))
    # second call right after, on fewer rows in another order: nothing left over from the first call shows
    sel = list(range(n_lanes - 1, 0, -1))
    lg2, arg2 = _call_static(cfg, sh, h[sel].contiguous(), g_final, packed, scales)
    _check(lg2, arg2, ref_logits, ref_arg, sel)


def test_static_head_64_rows_and_the_oracle():
    """The array's full row count (rows 32..63 take the second half of every
    per-lane slot), checked against the workspace head and, on the same hidden
    rows, against the fp64 oracle's head."""
    import oracle as O
    from oracle import model as M
    n = 6
    cfg, sh, h, g_final, packed, scales, ref_logits, ref_arg = _head_inputs("tiny", n, 16, 3)
    sel = [(7 * i + 3) % n for i in range(64)]
    h64 = h[sel].contiguous()
    lg, arg = _call_static(cfg, sh, h64, g_final, packed, scales)
    _check(lg, arg, ref_logits, ref_arg, sel)
    W = O.build_weights(sh, S.master_weights(sh), S.gains(sh, 7))
    want = M.head_logits(W, h64.cpu().numpy().astype(np.float64))
    for r in range(64):
        assert_logits_close(lg[r], want[r], f"row {r} vs oracle")
        s_ = np.sort(want[r])
        if s_[-1] - s_[-2] > 1e-3:
            assert int(arg[r]) == int(np.argmax(want[r])), r


def test_static_head_rejects_misaligned_head_pointer():
    import torch
    from dynamic_depth_b200 import lib
    x = torch.zeros((2, 128), dtype=torch.float32, device="cuda")
    g = torch.ones(128, dtype=torch.float32, device="cuda")
    q = torch.zeros(512 * 64 + 16, dtype=torch.uint8, device="cuda")
    s = torch.zeros((512, 4), dtype=torch.int16, device="cuda")
    a = torch.zeros(2, dtype=torch.int32, device="cuda")
    st = lib().tl_head_argmax_static(x.data_ptr(), 2, g.data_ptr(), C.c_float(1e-5), q.data_ptr() + 8, s.data_ptr(),
                                     512, 128, 32, None, a.data_ptr(), None)
    assert st == -1  # TL_EINVAL, nothing enqueued


def test_static_head_rejects_sizes_beyond_its_array():
    import torch
    from dynamic_depth_b200 import lib
    x = torch.zeros((65, 128), dtype=torch.float32, device="cuda")
    g = torch.ones(128, dtype=torch.float32, device="cuda")
    q = torch.zeros((512, 64), dtype=torch.uint8, device="cuda")
    s = torch.zeros((512, 4), dtype=torch.int16, device="cuda")
    a = torch.zeros(65, dtype=torch.int32, device="cuda")
    st = lib().tl_head_argmax_static(x.data_ptr(), 65, g.data_ptr(), C.c_float(1e-5), q.data_ptr(), s.data_ptr(),
                                     512, 128, 32, None, a.data_ptr(), None)
    assert st == -2  # TL_ENOMEM: more rows than the static array holds

    # a width beyond 4096 and a vocabulary beyond 262144 rows
    d = 4128
    x = torch.zeros((2, d), dtype=torch.float32, device="cuda")
    g = torch.ones(d, dtype=torch.float32, device="cuda")
    q = torch.zeros((512, d // 2), dtype=torch.uint8, device="cuda")
    s = torch.zeros((512, d // 32), dtype=torch.int16, device="cuda")
    st = lib().tl_head_argmax_static(x.data_ptr(), 2, g.data_ptr(), C.c_float(1e-5), q.data_ptr(), s.data_ptr(),
                                     512, d, 32, None, a.data_ptr(), None)
    assert st == -2
    st = lib().tl_head_argmax_static(x.data_ptr(), 2, g.data_ptr(), C.c_float(1e-5), q.data_ptr(), s.data_ptr(),
                                     262145, 128, 32, None, a.data_ptr(), None)
    assert st == -2
