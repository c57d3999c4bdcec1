"""Pins for the oracle's block math: closed forms, invariants, brute force."""
import math

import numpy as np
import pytest

import synthetic as S
import oracle as O
from oracle import model as M


@pytest.fixture(scope="module")
def tiny():
    sh = S.TINY
    return O.build_weights(sh, S.master_weights(sh), S.gains(sh, random_seed=7))


# ---------------------------------------------------------------- RMSNorm ----

def test_rmsnorm_constant_vector_closed_form():
    for c in (0.3, -2.0, 1e-3):
        x = np.full((1, 16), c)
        y = M.rmsnorm(x, np.ones(16), 1e-5)
        assert np.allclose(y, math.copysign(1.0, c) / math.sqrt(1 + 1e-5 / c ** 2), rtol=0, atol=1e-15)


def test_rmsnorm_gain_and_rms():
    x = S.random_vectors((5, 64), seed=1)
    g = S.random_vectors((64,), seed=2)
    y = M.rmsnorm(x, np.ones(64), 0.0)
    assert np.allclose(np.sqrt(np.mean(y * y, axis=1)), 1.0, atol=1e-14)
    assert np.allclose(M.rmsnorm(x, g, 0.0), y * g, atol=1e-14)
    # eps pulls small vectors towards zero
    assert np.all(np.abs(M.rmsnorm(1e-4 * x, np.ones(64), 1e-5)) < np.abs(y))


# ------------------------------------------------------------------- RoPE ----

def test_rope_identity_at_zero_and_norm_preserved():
    x = S.random_vectors((3, 4, 32), seed=3)
    assert np.allclose(M.apply_rope(x, np.zeros(3), 1e4), x, atol=0)
    y = M.apply_rope(x, np.array([1, 17, 900]), 1e4)
    assert np.allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x, axis=-1), atol=1e-13)


def test_rope_two_dim_rotation_direction():
    # hd = 2: theta_0 = 1, so position p rotates (1, 0) to (cos p, sin p).
    x = np.array([[[1.0, 0.0]]])
    y = M.apply_rope(x, np.array([0.5]), 1e4)
    assert np.allclose(y[0, 0], [math.cos(0.5), math.sin(0.5)], atol=1e-15)


def test_rope_pairs_i_with_i_plus_half():
    x = np.zeros((1, 1, 8))
    x[0, 0, 1] = 1.0
    y = M.apply_rope(x, np.array([3.0]), 1e4)[0, 0]
    nz = set(np.nonzero(np.abs(y) > 1e-15)[0].tolist())
    assert nz == {1, 5}
    # frequency of pair 1 is base^(-2/8)
    ang = 3.0 * 1e4 ** (-2.0 / 8)
    assert np.allclose([y[1], y[5]], [math.cos(ang), math.sin(ang)], atol=1e-15)


def test_rope_relative_position_property():
    q = S.random_vectors((1, 2, 16), seed=4)
    k = S.random_vectors((1, 2, 16), seed=5)

    def dot(p, pp):
        return np.sum(M.apply_rope(q, np.array([p]), 1e4) * M.apply_rope(k, np.array([pp]), 1e4), axis=-1)

    assert np.allclose(dot(7, 3), dot(104, 100), atol=1e-12)
    assert np.allclose(dot(0, 0), np.sum(q * k, axis=-1), atol=1e-12)


# -------------------------------------------------------------- attention ----

def test_attention_single_key_returns_value():
    q = S.random_vectors((1, 2, 8), seed=6)
    K = S.random_vectors((1, 2, 8), seed=7)
    V = S.random_vectors((1, 2, 8), seed=8)
    assert np.allclose(M.attend(q, K, V, np.array([0]), np.array([0])), V, atol=1e-15)


def test_attention_equal_keys_average_values():
    q = S.random_vectors((1, 2, 8), seed=9)
    K = np.repeat(S.random_vectors((1, 2, 8), seed=10), 5, axis=0)
    V = S.random_vectors((5, 2, 8), seed=11)
    out = M.attend(q, K, V, np.array([4]), np.arange(5))
    assert np.allclose(out[0], V.mean(axis=0), atol=1e-15)


def test_attention_is_causal():
    q = S.random_vectors((3, 2, 8), seed=12)
    K = S.random_vectors((3, 2, 8), seed=13)
    V = S.random_vectors((3, 2, 8), seed=14)
    a = M.attend(q, K, V, np.arange(3), np.arange(3))
    K2, V2 = K.copy(), V.copy()
    K2[2] += 5.0
    V2[2] -= 3.0
    b = M.attend(q, K2, V2, np.arange(3), np.arange(3))
    assert np.allclose(a[:2], b[:2], atol=0) and not np.allclose(a[2], b[2])


def _brute_block(bw, sh, x, pos):
    """One block on a fresh cache, with explicit loops (tiny shapes only)."""
    d, H, hd, F, eps = sh.d, sh.n_heads, sh.head_dim, sh.ffn, sh.rms_eps
    T = len(pos)

    def norm(v, g):
        ms = sum(e * e for e in v) / len(v)
        return [v[i] / math.sqrt(ms + eps) * g[i] for i in range(len(v))]

    def matvec(W, v):  # W[out][in]
        return [sum(W[o][i] * v[i] for i in range(len(v))) for o in range(len(W))]

    def rot(v, p):
        out = list(v)
        half = hd // 2
        for i in range(half):
            ang = p * sh.rope_base ** (-2.0 * i / hd)
            c, s = math.cos(ang), math.sin(ang)
            out[i] = v[i] * c - v[i + half] * s
            out[i + half] = v[i + half] * c + v[i] * s
        return out

    Q, Kc, Vc = [], [], []
    for t in range(T):
        a = norm(list(x[t]), bw.g1)
        qkv = matvec(bw.wqkv, a)
        Q.append([rot(qkv[h * hd:(h + 1) * hd], pos[t]) for h in range(H)])
        Kc.append([rot(qkv[d + h * hd:d + (h + 1) * hd], pos[t]) for h in range(H)])
        Vc.append([qkv[2 * d + h * hd:2 * d + (h + 1) * hd] for h in range(H)])
    out = []
    for t in range(T):
        o = []
        for h in range(H):
            sc = [sum(Q[t][h][i] * Kc[s][h][i] for i in range(hd)) / math.sqrt(hd) for s in range(t + 1)]
            mx = max(sc)
            e = [math.exp(v - mx) for v in sc]
            z = sum(e)
            o += [sum(e[s] / z * Vc[s][h][i] for s in range(t + 1)) for i in range(hd)]
        xr = [x[t][i] + v for i, v in enumerate(matvec(bw.wo, o))]
        b = norm(xr, bw.g2)
        gt, up = matvec(bw.wg, b), matvec(bw.wu, b)
        u = [gt[i] / (1 + math.exp(-gt[i])) * up[i] for i in range(F)]
        out.append([xr[i] + v for i, v in enumerate(matvec(bw.wd, u))])
    return np.array(out)


def test_block_matches_brute_force():
    sh = S.ModelShape(64, 16, 2, 24, 0, 1, S.INT4, S.INT4, S.INT4, 8)
    W = O.build_weights(sh, S.master_weights(sh, seed=21), S.gains(sh, random_seed=22))
    x = S.random_vectors((4, 16), seed=23, scale=0.5)
    pos = np.array([0, 1, 2, 3])
    got = M.block(W.loop[0], sh, x, pos, M.KVCache(sh, 4), ("loop", 1, 0))
    assert np.allclose(got, _brute_block(W.loop[0], sh, x, pos), rtol=0, atol=1e-12)


def test_causal_prefill_equals_incremental(tiny):
    toks = S.prompts(1, 10, tiny.shape.vocab, seed=31)[0]
    full, _ = M.forward(tiny, toks, 3)
    cache = M.KVCache(tiny.shape, 10)
    rows = []
    for p in range(10):
        x, _ = M.forward(tiny, toks[p:p + 1], 3, cache, pos0=p)
        rows.append(x[0])
    assert np.allclose(np.array(rows), full, atol=1e-12)


def test_L_equals_k_applications_of_one_block(tiny):
    toks = S.prompts(1, 6, tiny.shape.vocab, seed=32)[0]
    pos = np.arange(6)
    x = M.pre_blocks(tiny, M.embed(tiny, toks), pos, M.KVCache(tiny.shape, 6))
    for k in range(1, 5):
        # a fresh cache per application: iteration l only ever sees its own K/V
        x = M.block(tiny.loop[0], tiny.shape, x, pos, M.KVCache(tiny.shape, 6), "any")
        got, _ = M.forward(tiny, toks, k)
        assert np.allclose(got, x, atol=1e-13), k


def test_hidden_at_j_independent_of_L(tiny):
    toks = S.prompts(1, 5, tiny.shape.vocab, seed=33)[0]
    a, ca = M.forward(tiny, toks, 2)
    b, cb = M.forward(tiny, toks, 6)
    for slot in [("pre", 0), ("loop", 1, 0), ("loop", 2, 0)]:
        assert np.array_equal(ca.slots[slot][0], cb.slots[slot][0])
    assert not np.allclose(a, b)


def test_argmax_lowest_index_on_ties():
    lg = np.array([[0.0, 3.0, 1.0, 3.0], [5.0, 5.0, 5.0, 5.0]])
    assert M.argmax_lowest(lg).tolist() == [1, 0]


def test_silu_special_values():
    assert M.silu(np.array([0.0]))[0] == 0.0
    assert abs(M.silu(np.array([40.0]))[0] - 40.0) < 1e-12
    assert abs(M.silu(np.array([-40.0]))[0]) < 1e-15


def test_weight_draw_order_and_effective_values():
    sh = S.TINY
    ws = dict(S.master_weights(sh))
    rng = np.random.Generator(np.random.PCG64(0))
    assert np.array_equal(ws["embed"], rng.standard_normal((sh.vocab, sh.d)) * 0.02)
    assert np.array_equal(ws["pre0.wqkv"][:sh.d], rng.standard_normal((sh.d, sh.d)) * 0.02)
    assert [n for n, _ in S.matrix_shapes(sh)][-1] == "head"
    W = O.build_weights(sh, S.master_weights(sh), S.gains(sh))
    assert np.max(np.abs(W.head - ws["head"])) < 0.02 * 5 / 7 / 2 * 1.01 + 1e-3


# ------------------------------------------------------- embed and head ----

def _scalar_int4_row(packed_row, scales_row, group):
    """One row of an INT4 matrix, element by element: byte k // 2 holds element
    k in its low nibble when k is even and in its high nibble when k is odd;
    the value is (nibble - 8) * the fp16 scale of group k // group."""
    out = []
    for k in range(2 * len(packed_row)):
        byte = int(packed_row[k // 2])
        u = (byte & 0xF) if k % 2 == 0 else (byte >> 4)
        out.append((u - 8) * float(scales_row[k // group]))
    return out


@pytest.fixture(scope="module")
def tiny_kept():
    sh = S.TINY
    gains = S.gains(sh, random_seed=5)
    W = O.build_weights(sh, S.master_weights(sh), gains, keep_int4=True)
    return sh, gains, W


def test_embed_is_the_dequantised_embedding_row(tiny_kept):
    sh, _, W = tiny_kept
    packed, scales = W.int4["embed"]
    toks = [0, 7, sh.vocab - 1, 7]
    got = M.embed(W, toks)
    for r, t in enumerate(toks):
        assert got[r].tolist() == _scalar_int4_row(packed[t], scales[t], sh.group), t
    # the embedding table is the first matrix drawn from the seed-0 stream
    master = np.random.Generator(np.random.PCG64(0)).standard_normal((sh.vocab, sh.d)) * 0.02
    s = scales.astype(np.float64)
    assert np.all(np.abs(got - master[toks]) <= np.repeat(s[toks], sh.group, axis=1) / 2 + 1e-18)


def test_head_logits_match_scalar_loops(tiny_kept):
    """logits[v] = sum_i RMSNorm(h; g_final)[i] * Whead[v, i] with the final
    gain (not a block's), the norm applied, and the head's own matrix (untied:
    the last matrix drawn, not the embedding)."""
    sh, gains, W = tiny_kept
    d, eps = sh.d, sh.rms_eps
    h = S.random_vectors((2, d), seed=61, scale=3.0)   # RMS ~3: a dropped norm cannot pass
    got = M.head_logits(W, h)
    packed, scales = W.int4["head"]
    g = gains["final.g"]
    rows = [_scalar_int4_row(packed[v], scales[v], sh.group) for v in range(sh.vocab)]
    for r in range(2):
        ms = sum(float(x) * float(x) for x in h[r]) / d
        y = [float(h[r][i]) / math.sqrt(ms + eps) * float(g[i]) for i in range(d)]
        want = [sum(y[i] * row[i] for i in range(d)) for row in rows]
        assert np.allclose(got[r], want, rtol=0, atol=1e-12)
    # the head matrix is the last draw of the seed-0 stream
    rng = np.random.Generator(np.random.PCG64(0))
    last = None
    for _, (nr, nc) in S.matrix_shapes(sh):
        last = rng.standard_normal((nr, nc)) * 0.02
    dq = np.array(rows)
    assert np.all(np.abs(dq - last) <= np.repeat(scales.astype(np.float64), sh.group, axis=1) / 2 + 1e-18)
    # and it is not the embedding table, nor does a block gain stand in for g_final
    assert not np.array_equal(W.int4["head"][0], W.int4["embed"][0])
    assert not np.allclose(got, M.rmsnorm(h, gains["pre0.g1"], eps) @ W.head.T, atol=1e-6)
