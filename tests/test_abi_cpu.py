"""C-ABI checks that need no GPU: the library loads, exports every symbol
include/tl.h declares, validates configurations, and sizes its weight blob and
workspace by formulas checked here independently."""
import ctypes as C
import os
import re

import pytest

import synthetic as S
import dynamic_depth_b200 as T
from dynamic_depth_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_functions():
    src = open(os.path.join(ROOT, "include", "tl.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(tl_[a-z0-9_]+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    lib = _lib.lib()
    names = header_functions()
    assert len(names) >= 17
    for n in names:
        assert hasattr(lib, n), n
        assert n in _lib.SIGNATURES, n


def test_strerror_names_every_status():
    lib = _lib.lib()
    seen = set()
    for s in range(0, -8, -1):
        msg = lib.tl_strerror(s).decode()
        assert msg and msg != "unknown status"
        seen.add(msg)
    assert len(seen) == 8
    assert lib.tl_strerror(-99).decode() == "unknown status"


def _blob_formula(shape, group):
    """Bytes of the weight blob, counted from the shapes."""
    d, F, V = shape.d, shape.ffn, shape.vocab

    def mat(fmt, n, k):
        return n * k // 2 + n * (k // group) * 2 if fmt == "int4" else n * k * 2

    total = 8 + 48
    total += 2 * mat(shape.fmt_embed_head, V, d)
    for b in range(shape.n_pre + shape.n_loop_layers):
        f = shape.fmt_pre if b < shape.n_pre else shape.fmt_loop
        total += mat(f, 3 * d, d) + mat(f, d, d) + 2 * mat(f, F, d) + mat(f, d, F)
    total += (2 * (shape.n_pre + shape.n_loop_layers) + 1) * d * 4
    return total


@pytest.mark.parametrize("name", ["tiny", "m407", "m407_bf16loop", "m1b4"])
def test_weight_blob_size_formula(name):
    sh = S.SHAPES[name]
    cfg = T.config_from_shape(sh, max_lanes=4, max_seq=128, L_max=8)
    assert T.weights_bytes(cfg) == _blob_formula(sh, cfg.group)


def test_407m_int4_loop_block_bytes():
    # one loop iteration of the 407M-class model reads 8,650,752 bytes of INT4 weights + scales
    sh = S.M407
    d, F, g = sh.d, sh.ffn, sh.group
    per = sum(n * k // 2 + n * (k // g) * 2 for n, k in [(3 * d, d), (d, d), (F, d), (F, d), (d, F)])
    assert per == 8_650_752


def test_workspace_grows_with_capacity_and_kv_formula():
    sh = S.M407
    a = T.workspace_bytes(T.config_from_shape(sh, max_lanes=1, max_seq=128, L_max=8))
    b = T.workspace_bytes(T.config_from_shape(sh, max_lanes=2, max_seq=128, L_max=8))
    # one more lane adds at least its KV: (n_pre + L_max) slots x 2 pages x page bytes
    page = 2 * sh.n_heads * 64 * sh.head_dim * 2
    assert b - a >= (sh.n_pre + 8) * 2 * page
    c = T.workspace_bytes(T.config_from_shape(sh, max_lanes=1, max_seq=128, L_max=8, kv_pool_pages=10))
    assert a - c >= ((sh.n_pre + 8) * 2 - 10) * page


@pytest.mark.parametrize("field,value", [("d", 100), ("n_heads", 3), ("group", 48), ("kv_page_tokens", 48),
                                         ("ffn", 544),  # a multiple of 32 but not of 64
                                         ("ffn", 2048),  # 64 scale groups of 32 across ffn
                                         ("kv_page_tokens", 16), ("max_lanes", 0), ("max_lanes", 2048),
                                         ("L_max", 0), ("fmt_loop", 7), ("max_prefill_tokens", -1),
                                         ("act_split", 3), ("act_split", -1)])
def test_invalid_configs_rejected(field, value):
    cfg = T.config_from_shape(S.TINY, max_lanes=2, max_seq=64, L_max=4)
    setattr(cfg, field, value)
    n = C.c_size_t()
    assert _lib.lib().tl_workspace_bytes(C.byref(cfg), C.byref(n)) == _lib.TL_EINVAL
    assert _lib.lib().tl_weights_bytes(C.byref(cfg), C.byref(n)) == _lib.TL_EINVAL


def test_null_arguments_rejected_without_cuda():
    lib = _lib.lib()
    cfg = T.config_from_shape(S.TINY, max_lanes=2, max_seq=64, L_max=4)
    h = C.c_void_p()
    assert lib.tl_create(C.byref(cfg), None, 1 << 20, None, C.byref(h)) == _lib.TL_EINVAL
    assert lib.tl_create(C.byref(cfg), 0x1001, 1 << 20, None, C.byref(h)) == _lib.TL_EINVAL  # unaligned
    assert lib.tl_load_weights(None, None, 0) == _lib.TL_EINVAL
    assert lib.tl_decode(None, None, 1, 1, None, None) == _lib.TL_EINVAL
    assert lib.tl_quantize_int4(None, 4, 64, 32, None, None, None) == _lib.TL_EINVAL
    assert lib.tl_quantize_int4(0x1000, 4, 48, 32, 0x1000, 0x1000, None) == _lib.TL_EINVAL
    assert lib.tl_set_early_exit(None, 0.1, 2, 2, 1) == _lib.TL_EINVAL


def test_blob_header_layout():
    from dynamic_depth_b200 import weights as Wt
    cfg = T.config_from_shape(S.TINY, max_lanes=2, max_seq=64, L_max=4)
    h = Wt.header(cfg)
    assert len(h) == 56 and h[:8] == b"TLWBLOB1"
    assert Wt.gain_order(cfg) == S.gain_names(S.TINY)
    assert len(Wt.matrix_formats(cfg)) == len(S.matrix_shapes(S.TINY))


def test_prompt_rows_may_exceed_one_sequence():
    # a batched prefill computes the prompts of several lanes at once
    cfg = T.config_from_shape(S.TINY, max_lanes=8, max_seq=64, L_max=4, max_prefill_tokens=512)
    small = T.config_from_shape(S.TINY, max_lanes=8, max_seq=64, L_max=4)
    assert T.workspace_bytes(cfg) > T.workspace_bytes(small)


def _ws(sh, **kw):
    return T.workspace_bytes(T.config_from_shape(sh, **kw))


def test_split_activations_double_the_fp16_activation_copies():
    # act_split = 1 stores every fp16 activation copy as [hi | lo] rows: three copies (norm output,
    # attention output: d wide; SwiGLU output: ffn wide) for the prompt rows and again for the boundary
    # stage's scratch (max_lanes rows), each twice as wide
    sh = S.M407
    cap = dict(max_lanes=4, max_seq=128, L_max=8, max_prefill_tokens=512)
    single = _ws(sh, act_split=2, **cap)
    split = _ws(sh, act_split=1, **cap)
    rows, lanes = 512, 4
    extra = (rows + lanes) * (2 * sh.d + sh.ffn) * 2
    assert extra <= split - single <= extra + 6 * 256  # up to one alignment pad per region


def test_split_activations_automatic_past_48_blocks():
    # automatic: split when n_pre + L_max * n_loop_layers > 48 (the 407M-class model at L_max = 32 crosses
    # 34 blocks, the 1.4B-class layout at L_max = 4 crosses 96)
    m407 = dict(max_lanes=2, max_seq=64, max_prefill_tokens=64)
    assert _ws(S.M407, L_max=32, act_split=0, **m407) == _ws(S.M407, L_max=32, act_split=2, **m407)
    assert _ws(S.M407, L_max=47, act_split=0, **m407) == _ws(S.M407, L_max=47, act_split=1, **m407)
    mini = dict(max_lanes=2, max_seq=64, max_prefill_tokens=64)
    assert _ws(S.M1B4_MINI, L_max=16, act_split=0, **mini) == _ws(S.M1B4_MINI, L_max=16, act_split=2, **mini)
    assert _ws(S.M1B4_MINI, L_max=17, act_split=0, **mini) == _ws(S.M1B4_MINI, L_max=17, act_split=1, **mini)


def test_workspace_holds_a_resident_fp16_copy_of_every_block():
    # every block's five matrices in fp16: (3d*d + d*d + 2*ffn*d + d*ffn) halves per block
    sh = S.M407
    cfg = T.config_from_shape(sh, max_lanes=1, max_seq=64, L_max=2)
    ws = T.workspace_bytes(cfg)
    weights = T.weights_bytes(cfg)
    copies = (sh.n_pre + sh.n_loop_layers) * (4 * sh.d * sh.d + 3 * sh.d * sh.ffn) * 2
    assert ws > weights + copies
