"""bench.py's algorithmic accounting on CPU: byte counts against the block and
head sizes of the 407M-class configuration, and the per-tick schedule counts
against an independent tick-by-tick simulation of continuous depth batching
(each tick: lanes whose loop finished emit a token and, if they have more to
produce, enter at the next position; then every lane in its loop runs one
iteration)."""
import numpy as np

import bench
import synthetic as S


def test_weight_bytes_of_the_407m_class_model():
    # INT4 packed + fp16 scales at group 128: QKV 1,572,864 + 49,152; O 524,288 + 16,384;
    # gate/up 4,194,304 + 131,072; down 2,097,152 + 65,536 bytes
    assert bench.loop_block_weight_bytes(S.M407) == 8_650_752
    assert bench.head_weight_bytes(S.M407) == 50257 * 1024 // 2 + 50257 * 8 * 2 == 26_535_696


def _simulate(depths, T, n_pre, d):
    n, n_new = depths.shape
    nxt = [1] * n            # next token to compute
    left = [0] * n           # loop iterations left for it (0: at a boundary)
    done = [False] * n
    boundary, entered, loop_rows, attn = [], [], [], 0
    while not all(done):
        b = e = 0
        for i in range(n):
            if done[i] or left[i] > 0:
                continue
            b += 1                                # emits token nxt[i] - 1
            if nxt[i] >= n_new:
                done[i] = True
                continue
            e += 1                                # enters at position T + nxt[i] - 1
            left[i] = int(depths[i, nxt[i]])
            attn += (n_pre + left[i]) * (T + nxt[i]) * 4 * d
            nxt[i] += 1
        rows = sum(1 for i in range(n) if not done[i] and left[i] > 0)
        for i in range(n):
            if not done[i] and left[i] > 0:
                left[i] -= 1
        boundary.append(b)
        entered.append(e)
        loop_rows.append(rows)
    return boundary, entered, loop_rows, attn


def _simulate_next_tick(depths, T, n_pre, d):
    """Entering lanes run their loop from the next tick on: each tick, the lanes
    in their loop at its start run one iteration while the waiting lanes take a
    token (concurrently, on disjoint lanes)."""
    n, n_new = depths.shape
    nxt, left, done = [1] * n, [0] * n, [False] * n
    boundary, entered, loop_rows, attn = [], [], [], 0
    while not all(done):
        looping = [i for i in range(n) if not done[i] and left[i] > 0]
        waiting = [i for i in range(n) if not done[i] and left[i] == 0]
        for i in looping:
            left[i] -= 1
        b = e = 0
        for i in waiting:
            b += 1
            if nxt[i] >= n_new:
                done[i] = True
                continue
            e += 1
            left[i] = int(depths[i, nxt[i]])
            attn += (n_pre + left[i]) * (T + nxt[i]) * 4 * d
            nxt[i] += 1
        boundary.append(b)
        entered.append(e)
        loop_rows.append(len(looping))
    return boundary, entered, loop_rows, attn


def test_schedule_counts_match_a_tick_by_tick_simulation_next_tick_entry():
    rng = np.random.Generator(np.random.PCG64(6))
    n, n_new, T = 7, 6, 20
    depths = rng.integers(1, 6, (n, n_new)).astype(np.int32)

    class Wl:
        prompt_len, n_new = T, 6
    u = bench.schedule_units(S.M407, Wl, depths, same_tick=False)
    b, e, rows, attn = _simulate_next_tick(depths, T, S.M407.n_pre, S.M407.d)
    assert u["ticks"] == len(b)
    assert list(u["boundary"]) == b
    assert list(u["entered"]) == e
    assert list(u["loop_rows"]) == rows
    assert u["attn_bytes"] == attn


def test_schedule_counts_match_a_tick_by_tick_simulation():
    rng = np.random.Generator(np.random.PCG64(5))
    n, n_new, T = 7, 6, 20
    depths = rng.integers(1, 6, (n, n_new)).astype(np.int32)

    class Wl:
        prompt_len, n_new = T, 6
    u = bench.schedule_units(S.M407, Wl, depths)
    b, e, rows, attn = _simulate(depths, T, S.M407.n_pre, S.M407.d)
    assert u["ticks"] == len(b)
    assert list(u["boundary"]) == b
    assert list(u["entered"]) == e
    assert list(u["loop_rows"]) == rows
    assert u["attn_bytes"] == attn


def test_whole_job_rate_counts_every_replica():
    assert bench.whole_job_rate(8192, 1000.0, 1) == 8192.0
    assert bench.whole_job_rate(8192, 1000.0, 8) == 8 * 8192.0
