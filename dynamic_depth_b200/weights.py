"""Weight blob assembly (layout in include/tl.h) from float64 master matrices.

INT4 matrices are quantised on the device by tl_quantize_int4 and BF16 ones
rounded by tl_round_bf16; this module only orders the bytes.
"""
from __future__ import annotations

import struct

import numpy as np

from . import _lib
from ._lib import TL_FMT_INT4, TlConfig, check, lib

MAGIC = b"TLWBLOB1"


def header(cfg: TlConfig) -> bytes:
    ints = [cfg.vocab, cfg.d, cfg.n_heads, cfg.ffn, cfg.n_pre, cfg.n_loop_layers, cfg.fmt_pre, cfg.fmt_loop,
            cfg.fmt_embed_head, cfg.group]
    return MAGIC + struct.pack("<10i2f", *ints, cfg.rms_eps, cfg.rope_base)


def matrix_formats(cfg: TlConfig) -> list[int]:
    """Storage format of every matrix, in blob order."""
    out = [cfg.fmt_embed_head]
    for b in range(cfg.n_pre + cfg.n_loop_layers):
        out += [cfg.fmt_pre if b < cfg.n_pre else cfg.fmt_loop] * 5
    out.append(cfg.fmt_embed_head)
    return out


def gain_order(cfg: TlConfig) -> list[str]:
    names = []
    for b in range(cfg.n_pre):
        names += [f"pre{b}.g1", f"pre{b}.g2"]
    for m in range(cfg.n_loop_layers):
        names += [f"loop{m}.g1", f"loop{m}.g2"]
    return names + ["final.g"]


def quantize_int4_device(w: np.ndarray, group: int, device="cuda:0", stream=None):
    """float64 [N, K] -> (packed uint8 [N, K/2], fp16 scale bits uint16 [N, K/group]) via tl_quantize_int4."""
    import torch
    N, K = w.shape
    dw = torch.from_numpy(np.ascontiguousarray(w, dtype=np.float64)).to(device)
    packed = torch.empty((N, K // 2), dtype=torch.uint8, device=device)
    scales = torch.empty((N, K // group), dtype=torch.int16, device=device)
    s = stream or torch.cuda.current_stream(device)
    check(lib().tl_quantize_int4(dw.data_ptr(), N, K, group, packed.data_ptr(), scales.data_ptr(), s.cuda_stream),
          "tl_quantize_int4")
    return packed.cpu().numpy(), scales.cpu().numpy().view(np.uint16)


def round_bf16_device(w: np.ndarray, device="cuda:0", stream=None) -> np.ndarray:
    import torch
    dw = torch.from_numpy(np.ascontiguousarray(w, dtype=np.float64)).to(device)
    out = torch.empty(dw.shape, dtype=torch.int16, device=device)
    s = stream or torch.cuda.current_stream(device)
    check(lib().tl_round_bf16(dw.data_ptr(), dw.numel(), out.data_ptr(), s.cuda_stream), "tl_round_bf16")
    return out.cpu().numpy().view(np.uint16)


def build_blob(cfg: TlConfig, matrices, gains: dict, device="cuda:0") -> np.ndarray:
    """matrices: iterable of (name, float64 [N, K]) in blob order; gains: name -> [d]."""
    parts = [np.frombuffer(header(cfg), dtype=np.uint8)]
    fmts = matrix_formats(cfg)
    n = 0
    for i, (_, w) in enumerate(matrices):
        if fmts[i] == TL_FMT_INT4:
            packed, scales = quantize_int4_device(w, cfg.group, device)
            parts += [packed.reshape(-1), scales.reshape(-1).view(np.uint8)]
        else:
            parts.append(round_bf16_device(w, device).reshape(-1).view(np.uint8))
        n += 1
    if n != len(fmts):
        raise ValueError(f"expected {len(fmts)} matrices, got {n}")
    for name in gain_order(cfg):
        parts.append(np.ascontiguousarray(gains[name], dtype=np.float32).view(np.uint8))
    blob = np.concatenate(parts)
    want = _weights_bytes(cfg)
    if blob.nbytes != want:
        raise ValueError(f"blob is {blob.nbytes} bytes, expected {want}")
    return blob


def _weights_bytes(cfg: TlConfig) -> int:
    import ctypes as C
    n = C.c_size_t()
    check(lib().tl_weights_bytes(C.byref(cfg), C.byref(n)), "tl_weights_bytes")
    return n.value


__all__ = ["build_blob", "quantize_int4_device", "round_bf16_device", "header", "matrix_formats", "gain_order",
           "_lib"]
