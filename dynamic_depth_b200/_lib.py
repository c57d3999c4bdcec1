"""ctypes declarations of libtl.so (include/tl.h).  Marshalling only.

Loading fails loudly when the library has not been built: there is no
fallback path of any kind.
"""
from __future__ import annotations

import ctypes as C
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libtl.so")

TL_OK, TL_EINVAL, TL_ENOMEM, TL_ESTATE, TL_EKV, TL_ECUDA, TL_ETIMEOUT, TL_EDEVICE = 0, -1, -2, -3, -4, -5, -6, -7
TL_FMT_INT4, TL_FMT_BF16 = 0, 1
TL_PROF_NONE, TL_PROF_ATTN, TL_PROF_PROJ, TL_PROF_HEAD = 0, 1, 2, 3


class TlConfig(C.Structure):
    _fields_ = [
        ("vocab", C.c_int32), ("d", C.c_int32), ("n_heads", C.c_int32), ("ffn", C.c_int32),
        ("n_pre", C.c_int32), ("n_loop_layers", C.c_int32), ("fmt_pre", C.c_int32),
        ("fmt_loop", C.c_int32), ("fmt_embed_head", C.c_int32), ("group", C.c_int32),
        ("rms_eps", C.c_float), ("rope_base", C.c_float),
        ("max_lanes", C.c_int32), ("max_seq", C.c_int32), ("L_max", C.c_int32),
        ("kv_page_tokens", C.c_int32), ("kv_pool_pages", C.c_int32), ("max_prefill_tokens", C.c_int32),
        ("act_split", C.c_int32),
    ]


class TlStats(C.Structure):
    _fields_ = [
        ("loop_steps", C.c_int64), ("lane_iterations", C.c_int64), ("tokens_emitted", C.c_int64),
        ("prefill_tokens", C.c_int64), ("kernel_launches", C.c_int64), ("device_status", C.c_int32),
        ("kv_pages_used", C.c_int32), ("entry_in_boundary", C.c_int32), ("tick_layout", C.c_int32),
        ("boundary_stages", C.c_int64),
    ]


# name -> (restype, argtypes), in header order
SIGNATURES = {
    "tl_workspace_bytes": (C.c_int, [C.POINTER(TlConfig), C.POINTER(C.c_size_t)]),
    "tl_weights_bytes": (C.c_int, [C.POINTER(TlConfig), C.POINTER(C.c_size_t)]),
    "tl_create": (C.c_int, [C.POINTER(TlConfig), C.c_void_p, C.c_size_t, C.c_void_p, C.POINTER(C.c_void_p)]),
    "tl_destroy": (C.c_int, [C.c_void_p]),
    "tl_load_weights": (C.c_int, [C.c_void_p, C.c_void_p, C.c_size_t]),
    "tl_quantize_int4": (C.c_int, [C.c_void_p, C.c_int64, C.c_int64, C.c_int32, C.c_void_p, C.c_void_p, C.c_void_p]),
    "tl_dequant_int4": (C.c_int, [C.c_void_p, C.c_void_p, C.c_int64, C.c_int64, C.c_int32, C.c_void_p, C.c_void_p]),
    "tl_round_bf16": (C.c_int, [C.c_void_p, C.c_int64, C.c_void_p, C.c_void_p]),
    "tl_prefill": (C.c_int, [C.c_void_p, C.c_int32, C.c_void_p, C.c_int32, C.c_int32, C.c_int32, C.c_int32,
                             C.c_void_p]),
    "tl_prefill_batch": (C.c_int, [C.c_void_p, C.c_int32, C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p,
                                   C.c_int32, C.c_int32]),
    "tl_set_early_exit": (C.c_int, [C.c_void_p, C.c_double, C.c_int32, C.c_int32, C.c_int32]),
    "tl_set_early_exit_logit_margin": (C.c_int, [C.c_void_p, C.c_double, C.c_int32, C.c_int32, C.c_int32]),
    "tl_set_l_warmup": (C.c_int, [C.c_void_p, C.c_int32, C.c_int32]),
    "tl_loop_step": (C.c_int, [C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p]),
    "tl_head_logits": (C.c_int, [C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p]),
    "tl_embed_next": (C.c_int, [C.c_void_p, C.c_void_p, C.c_void_p]),
    "tl_decode": (C.c_int, [C.c_void_p, C.c_void_p, C.c_int32, C.c_int32, C.c_void_p, C.c_void_p]),
    "tl_generate": (C.c_int, [C.c_void_p, C.c_void_p, C.c_int32, C.c_int32, C.c_void_p, C.c_int32, C.c_void_p,
                              C.c_void_p]),
    "tl_speculate": (C.c_int, [C.c_void_p, C.c_int32, C.c_int32, C.c_int32, C.c_int32, C.c_int32, C.c_void_p,
                               C.c_void_p]),
    "tl_set_tick_overlap": (C.c_int, [C.c_void_p, C.c_int32]),
    "tl_set_cascade": (C.c_int, [C.c_void_p, C.c_int32]),
    "tl_set_graphs": (C.c_int, [C.c_void_p, C.c_int32]),
    "tl_lane_state_bytes": (C.c_int, [C.c_void_p, C.POINTER(C.c_size_t)]),
    "tl_lane_state_save": (C.c_int, [C.c_void_p, C.c_void_p]),
    "tl_lane_state_load": (C.c_int, [C.c_void_p, C.c_void_p]),
    "tl_profile_begin": (C.c_int, [C.c_void_p, C.c_int32]),
    "tl_profile_end": (C.c_int, [C.c_void_p, C.POINTER(C.c_int64), C.POINTER(C.c_double)]),
    "tl_head_argmax_static": (C.c_int, [C.c_void_p, C.c_int32, C.c_void_p, C.c_float, C.c_void_p, C.c_void_p,
                                         C.c_int32, C.c_int32, C.c_int32, C.c_void_p, C.c_void_p, C.c_void_p]),
    "tl_read_probe": (C.c_int, [C.c_void_p, C.c_size_t, C.c_int32, C.c_void_p, C.c_int32, C.c_void_p]),
    "tl_stats_get": (C.c_int, [C.c_void_p, C.POINTER(TlStats)]),
    "tl_strerror": (C.c_char_p, [C.c_int]),
    "tl_last_cuda_error": (C.c_char_p, []),
}

_lib = None


def lib() -> C.CDLL:
    """The loaded libtl.so (raises if it is missing)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libtl.so not built at {LIB_PATH}: run `python -m dynamic_depth_b200.build`")
        L = C.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


class TlError(RuntimeError):
    def __init__(self, status: int, what: str):
        msg = lib().tl_strerror(status).decode()
        if status == TL_ECUDA:
            msg += ": " + lib().tl_last_cuda_error().decode()
        super().__init__(f"{what}: {msg} ({status})")
        self.status = status


def check(status: int, what: str) -> None:
    if status != TL_OK:
        raise TlError(status, what)
