"""Per-lane-depth decode of a weight-shared looped transformer on B200.

A thin Python face over libtl.so (include/tl.h): every step of the model runs
in the library's CUDA kernels; this module only marshals arguments.  PyTorch
provides device memory (the workspace, caller-owned buffers) and streams.
"""
from __future__ import annotations

import ctypes as C

import numpy as np

from . import _lib
from ._lib import TlConfig, TlError, TL_FMT_INT4, TL_FMT_BF16, check, lib  # noqa: F401

__all__ = ["TlConfig", "TlError", "LoopedLM", "make_config", "TL_FMT_INT4", "TL_FMT_BF16"]

_FMT = {"int4": TL_FMT_INT4, "bf16": TL_FMT_BF16}


def make_config(vocab, d, n_heads, ffn, n_pre, n_loop_layers, fmt_pre="int4", fmt_loop="int4",
                fmt_embed_head="int4", group=128, rms_eps=1e-5, rope_base=1e4, *, max_lanes=1,
                max_seq=256, L_max=32, kv_page_tokens=64, kv_pool_pages=0, max_prefill_tokens=0,
                act_split=0) -> TlConfig:
    f = lambda x: _FMT[x] if isinstance(x, str) else int(x)  # noqa: E731
    return TlConfig(vocab, d, n_heads, ffn, n_pre, n_loop_layers, f(fmt_pre), f(fmt_loop), f(fmt_embed_head),
                    group, rms_eps, rope_base, max_lanes, max_seq, L_max, kv_page_tokens, kv_pool_pages,
                    max_prefill_tokens, act_split)


def config_from_shape(shape, **capacity) -> TlConfig:
    """Build a TlConfig from any object with the model-shape attributes."""
    return make_config(shape.vocab, shape.d, shape.n_heads, shape.ffn, shape.n_pre, shape.n_loop_layers,
                       shape.fmt_pre, shape.fmt_loop, shape.fmt_embed_head, shape.group or 32,
                       shape.rms_eps, shape.rope_base, **capacity)


def workspace_bytes(cfg: TlConfig) -> int:
    n = C.c_size_t()
    check(lib().tl_workspace_bytes(C.byref(cfg), C.byref(n)), "tl_workspace_bytes")
    return n.value


def weights_bytes(cfg: TlConfig) -> int:
    n = C.c_size_t()
    check(lib().tl_weights_bytes(C.byref(cfg), C.byref(n)), "tl_weights_bytes")
    return n.value


def _ptr(t) -> int | None:
    """Device (or host) address of a torch tensor / numpy array, None for None."""
    if t is None:
        return None
    if isinstance(t, np.ndarray):
        return t.ctypes.data
    return t.data_ptr()


class LoopedLM:
    """One libtl context: a workspace on `device`, bound to `stream`."""

    def __init__(self, cfg: TlConfig, device="cuda:0", stream=None):
        import torch
        self.torch = torch
        self.cfg = cfg
        self.device = torch.device(device)
        self.stream = stream if stream is not None else torch.cuda.current_stream(self.device)
        self.workspace = torch.empty(workspace_bytes(cfg), dtype=torch.uint8, device=self.device)
        h = C.c_void_p()
        check(lib().tl_create(C.byref(cfg), self.workspace.data_ptr(), self.workspace.numel(),
                              self.stream.cuda_stream, C.byref(h)), "tl_create")
        self.h = h

    def close(self):
        if self.h:
            lib().tl_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # ---------------------------------------------------------------- weights
    def load_weights(self, blob: np.ndarray):
        blob = np.ascontiguousarray(blob, dtype=np.uint8)
        check(lib().tl_load_weights(self.h, blob.ctypes.data, blob.nbytes), "tl_load_weights")

    # ------------------------------------------------------------------ lanes
    def prefill(self, lane: int, tokens, L: int, share_from: int = -1, shared_tokens: int = 0, hidden_out=None):
        tok = np.ascontiguousarray(tokens, dtype=np.int32)
        check(lib().tl_prefill(self.h, lane, tok.ctypes.data, len(tok), L, share_from, shared_tokens,
                               _ptr(hidden_out)), "tl_prefill")

    def prefill_batch(self, lanes, prompts, per_lane_L, share_from: int = -1, shared_tokens: int = 0):
        """Prompts of several lanes in one pass (tl_prefill_batch); prompts: a list of int sequences."""
        ln = np.ascontiguousarray(lanes, dtype=np.int32)
        toks = [np.ascontiguousarray(p, dtype=np.int32) for p in prompts]
        T = np.array([len(t) for t in toks], dtype=np.int32)
        L = np.ascontiguousarray(per_lane_L, dtype=np.int32)
        if not (len(ln) == len(toks) == len(L)):
            raise ValueError("lanes, prompts and per_lane_L differ in length")
        flat = np.concatenate(toks) if toks else np.zeros(0, np.int32)
        check(lib().tl_prefill_batch(self.h, len(ln), ln.ctypes.data, flat.ctypes.data, T.ctypes.data, L.ctypes.data,
                                     share_from, shared_tokens), "tl_prefill_batch")

    def set_early_exit(self, tau: float, min_L: int = 2, patience: int = 0, peek_every: int = 1):
        check(lib().tl_set_early_exit(self.h, float(tau), min_L, patience, peek_every), "tl_set_early_exit")

    def set_early_exit_logit_margin(self, margin: float, min_L: int = 2, patience: int = 1, peek_every: int = 1):
        check(lib().tl_set_early_exit_logit_margin(self.h, float(margin), min_L, patience, peek_every),
              "tl_set_early_exit_logit_margin")

    def set_l_warmup(self, warmup_tokens: int, warmup_L: int = 2):
        check(lib().tl_set_l_warmup(self.h, warmup_tokens, warmup_L), "tl_set_l_warmup")

    def loop_step(self, per_lane_L=None, active_mask=None, exit_mask_out=None):
        check(lib().tl_loop_step(self.h, _ptr(per_lane_L), _ptr(active_mask), _ptr(exit_mask_out)),
              "tl_loop_step")

    def head_logits(self, lane_mask=None, logits=None, argmax=None):
        check(lib().tl_head_logits(self.h, _ptr(lane_mask), _ptr(logits), _ptr(argmax)), "tl_head_logits")

    def embed_next(self, lane_mask, tokens):
        check(lib().tl_embed_next(self.h, _ptr(lane_mask), _ptr(tokens)), "tl_embed_next")

    def decode(self, per_lane_L, n_new: int, tokens_out=None, depths_out=None):
        L = np.ascontiguousarray(per_lane_L, dtype=np.int32)
        check(lib().tl_decode(self.h, L.ctypes.data, len(L), n_new, _ptr(tokens_out), _ptr(depths_out)),
              "tl_decode")

    def generate(self, prompts, per_lane_L, n_new: int, tokens_out=None, depths_out=None):
        """Host in, host out.  prompts int32 [n_lanes, T]; returns (tokens, depths) int32 [n_lanes, n_new]."""
        P = np.ascontiguousarray(prompts, dtype=np.int32)
        L = np.ascontiguousarray(per_lane_L, dtype=np.int32)
        n = P.shape[0]
        tok = tokens_out if tokens_out is not None else np.zeros((n, n_new), np.int32)
        dep = depths_out if depths_out is not None else np.zeros((n, n_new), np.int32)
        check(lib().tl_generate(self.h, _ptr(P), n, P.shape[1], L.ctypes.data, n_new, _ptr(tok), _ptr(dep)),
              "tl_generate")
        return tok, dep

    def speculate(self, lane: int, n_new: int, L_draft: int, L_verify: int, draft_ahead: int):
        """Self-speculative greedy decode of a freshly prefilled lane: (tokens int32 [n_new], verify rounds)."""
        tok = np.zeros(n_new, np.int32)
        rounds = C.c_int32(0)
        check(lib().tl_speculate(self.h, lane, n_new, L_draft, L_verify, draft_ahead, tok.ctypes.data,
                                 C.byref(rounds)), "tl_speculate")
        return tok, rounds.value

    def set_tick_overlap(self, mode: int):
        """0 automatic, 1 entering lanes iterate in the boundary stage, 2 they join at the next tick,
        3 boundary stages and loop steps on two streams with no join per tick."""
        check(lib().tl_set_tick_overlap(self.h, mode), "tl_set_tick_overlap")

    def set_cascade(self, enabled: bool):
        check(lib().tl_set_cascade(self.h, 1 if enabled else 0), "tl_set_cascade")

    def set_graphs(self, enabled: bool):
        check(lib().tl_set_graphs(self.h, 1 if enabled else 0), "tl_set_graphs")

    def lane_state_save(self):
        """Snapshot of every lane's scheduling state and hidden row (a device tensor)."""
        n = C.c_size_t()
        check(lib().tl_lane_state_bytes(self.h, C.byref(n)), "tl_lane_state_bytes")
        buf = self.torch.empty(n.value, dtype=self.torch.uint8, device=self.device)
        check(lib().tl_lane_state_save(self.h, buf.data_ptr()), "tl_lane_state_save")
        return buf

    def lane_state_load(self, buf):
        check(lib().tl_lane_state_load(self.h, buf.data_ptr()), "tl_lane_state_load")

    def profile_begin(self, kind_mask: int):
        """Time launch groups of the kinds in kind_mask (bit 1 attention, 2 projections, 3 head)."""
        check(lib().tl_profile_begin(self.h, kind_mask), "tl_profile_begin")

    def profile_end(self):
        """(groups[4], ms[4]) indexed by kind."""
        g, ms = (C.c_int64 * 4)(), (C.c_double * 4)()
        check(lib().tl_profile_end(self.h, g, ms), "tl_profile_end")
        return list(g), list(ms)

    def stats(self) -> dict:
        s = _lib.TlStats()
        check(lib().tl_stats_get(self.h, C.byref(s)), "tl_stats_get")
        return {k: getattr(s, k) for k, _ in s._fields_}


def read_bandwidth_gbs(n_bytes: int, reps: int, device="cuda:0", trials: int = 5) -> float:
    """Read bandwidth (GB/s) of tl_read_probe over an n_bytes device buffer read
    reps times per launch: best of `trials` event-timed launches after one
    untimed launch (which also brings an L2-sized buffer into L2)."""
    import torch
    dev = torch.device(device)
    buf = torch.ones(n_bytes // 4, dtype=torch.int32, device=dev)
    n_sink = 4 * torch.cuda.get_device_properties(dev).multi_processor_count
    sink = torch.zeros(n_sink, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def launch():
        check(lib().tl_read_probe(buf.data_ptr(), buf.numel() * 4, reps, sink.data_ptr(), n_sink, stream.cuda_stream),
              "tl_read_probe")
    launch()
    best = float("inf")
    for _ in range(trials):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        launch()
        e1.record(stream)
        e1.synchronize()
        best = min(best, e0.elapsed_time(e1))
    return buf.numel() * 4 * reps / 1e9 / (best / 1e3)
