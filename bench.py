#!/usr/bin/env python
"""Decode throughput of L-aware continuous depth batching on B200.

Workload (one "step" = one whole decode pass of the batch): the 407M-class
looped model (vocab 50257, d 1024, 16 heads x 64, SwiGLU FFN 4096, 2 pre
blocks + 1 shared loop block, INT4 group 128, random N(0, 0.02) weights from
seed 0); 64 lanes with uniform-random 512-token prompts; 128 greedy tokens per
lane; per-lane L drawn Poisson(8) clamped to [2, 32]; early exit on the
relative-L2 hidden delta < 0.1 after min_L 2 with patience 2; exited lanes are
compacted out of every loop step on the device.  The prompts are prefilled once
before timing; every step restores the post-prompt lane state and decodes all
64 x 128 tokens.  Inputs larger than L2: the KV cache the decode reads is
~1.7 GB (plus 79 MB of weights) against a 126 MB L2, so no flush is needed.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun (N > 1) every rank runs its own replica of the whole batch
(weak scaling, no collective on the data path); rank 0 prints one JSON line.
`--impl reference` times the fp64 CPU oracle (the only reference this work
has) on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synthetic as S  # noqa: E402

METRIC = "decode tokens/s (L-aware continuous depth batching, per-lane L)"
UNIT = "tokens/s"
WORKLOAD = "m407_cdb64"


def workload_config(wl):
    return {"workload": f"407M-class looped LM, {wl.n_lanes} lanes x ({wl.prompt_len}-token prompt + {wl.n_new} "
                        "greedy tokens), per-lane L ~ clamp(Poisson(8), 2, 32), rel-L2 early exit tau 0.1 / min_L 2 / "
                        "patience 2" + ("" if (wl.n_lanes, wl.prompt_len, wl.n_new) == (64, 512, 128)
                                        else " [reduced case]"),
            "model": "vocab 50257, d 1024, 16x64 heads, SwiGLU 4096, 2 pre + 1 loop block, INT4 g128",
            "lanes": wl.n_lanes, "prompt_len": wl.prompt_len, "new_tokens": wl.n_new,
            "per_lane_L": list(wl.per_lane_L), "weights": "random N(0,0.02) seed 0",
            "l2": "inputs larger than L2 (KV cache ~1.7 GB read per decode pass), no flush"}


# ------------------------------------------------------------------ clocks --

class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.p = None

    def __enter__(self):
        try:
            self.p = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                                       "--format=csv,noheader,nounits", "-lms", "200"],
                                      stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.p = None
        return self

    def __exit__(self, *a):
        self.rows = []
        if self.p is None:
            return
        time.sleep(0.25)
        self.p.terminate()
        try:
            out, _ = self.p.communicate(timeout=5)
        except Exception:
            self.p.kill()
            out = ""
        for line in out.strip().splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) == 7:
                self.rows.append(parts)

    def summary(self):
        if not getattr(self, "rows", None):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm = [float(r[0]) for r in self.rows if r[0].replace(".", "").isdigit()]
        mx = [float(r[1]) for r in self.rows if r[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in self.rows for i in range(4) if r[3 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(self.rows)}


def gpu_id(dev) -> str:
    """nvidia-smi -i selector for a torch device (UUID when torch exposes it)."""
    import torch
    try:
        u = str(torch.cuda.get_device_properties(dev).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        return str(torch.device(dev).index or 0)


# -------------------------------------------------------------- algorithmic --

def loop_block_weight_bytes(sh) -> int:
    d, F, g = sh.d, sh.ffn, sh.group
    return sum(n * k // 2 + n * (k // g) * 2 for n, k in [(3 * d, d), (d, d), (F, d), (F, d), (d, F)])


def schedule_units(sh, wl, depths):
    """Counts behind the algorithmic bytes, from the executed depth schedule.

    Lane i runs one loop iteration in every tick k < S_i = sum of its decode
    depths (the boundary stage of a tick feeds the same tick's loop), and takes
    a new token (pre blocks) at tick 0 and whenever a token's loop finished."""
    T, n_new = wl.prompt_len, wl.n_new
    S_i = depths[:, 1:].sum(axis=1)
    ticks = int(S_i.max()) + 1
    loop_rows = np.array([(S_i > k).sum() for k in range(ticks)])
    entered = np.zeros(ticks, dtype=np.int64)
    boundary = np.zeros(ticks, dtype=np.int64)
    kv_bytes_per_pos = 2 * sh.d * 2  # K and V, fp16
    attn_bytes = 0
    attn_rows = 0
    for i in range(depths.shape[0]):
        tick = 0
        boundary[0] += 1
        for t in range(1, n_new):
            ctx = T + t  # the row at position T + t - 1 attends to positions 0 .. T + t - 1
            entered[tick] += 1
            attn_bytes += (sh.n_pre + int(depths[i, t])) * ctx * kv_bytes_per_pos
            attn_rows += sh.n_pre + int(depths[i, t])
            tick += int(depths[i, t])
            boundary[tick] += 1
    return {"ticks": ticks, "loop_rows": loop_rows, "entered": entered, "boundary": boundary,
            "attn_bytes": attn_bytes, "attn_rows": attn_rows}


def head_weight_bytes(sh) -> int:
    return sh.vocab * sh.d // 2 + sh.vocab * (sh.d // sh.group) * 2


def workload_from_args(args):
    """The benchmark workload, or a reduced case of it (profiling captures) when
    --lanes / --prompt-len / --new-tokens are given."""
    import dataclasses
    wl = S.workload(WORKLOAD)
    kw = {}
    if args.lanes:
        kw["n_lanes"] = args.lanes
        kw["per_lane_L"] = tuple(wl.per_lane_L[i % len(wl.per_lane_L)] for i in range(args.lanes))
    if args.prompt_len:
        kw["prompt_len"] = args.prompt_len
    if args.new_tokens:
        kw["n_new"] = args.new_tokens
    return dataclasses.replace(wl, **kw) if kw else wl


# -------------------------------------------------------------------- ours --

def run_ours(args, rank, world, local_rank):
    import torch
    import dynamic_depth_b200 as T
    from dynamic_depth_b200 import weights as Wt

    dev = f"cuda:{local_rank}"
    torch.cuda.set_device(dev)
    wl = workload_from_args(args)
    sh = wl.shape
    cfg = T.config_from_shape(sh, max_lanes=wl.n_lanes, max_seq=wl.prompt_len + wl.n_new, L_max=32,
                              max_prefill_tokens=wl.prompt_len)
    m = T.LoopedLM(cfg, dev)
    m.load_weights(Wt.build_blob(cfg, S.master_weights(sh), S.gains(sh), dev))
    m.set_early_exit(wl.ee_tau, wl.ee_min_L, wl.ee_patience, wl.ee_peek_every)
    if args.eager:
        m.set_graphs(False)
    P = S.prompts(wl.n_lanes, wl.prompt_len, sh.vocab)
    Ls = np.array(wl.per_lane_L, dtype=np.int32)

    # prompts (timed separately)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    for i in range(wl.n_lanes):
        m.prefill(i, P[i], int(Ls[i]))
    torch.cuda.synchronize()
    prefill_s = time.perf_counter() - t0
    snap = m.lane_state_save()
    tok = torch.zeros((wl.n_lanes, wl.n_new), dtype=torch.int32, device=dev)
    dep = torch.zeros((wl.n_lanes, wl.n_new), dtype=torch.int32, device=dev)

    def step():
        m.lane_state_load(snap)
        m.decode(Ls, wl.n_new, tok, dep)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    st0 = m.stats()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(gpu_id(dev)) as clk:
        torch.cuda.nvtx.range_push("timed")
        ev0.record(stream)
        for _ in range(args.steps):
            step()
        ev1.record(stream)
        torch.cuda.synchronize()
        torch.cuda.nvtx.range_pop()
    if world > 1:
        torch.distributed.barrier()
    st1 = m.stats()
    assert st1["device_status"] == 0, f"device status {st1['device_status']:#x}"
    ms = ev0.elapsed_time(ev1)
    if world > 1:
        t = torch.tensor([ms], device=dev, dtype=torch.float64)
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        ms = float(t.item())
    tokens_per_step = wl.n_lanes * wl.n_new
    value = world * tokens_per_step * args.steps / (ms / 1e3)
    # the same steps again with per-kind event timing (kept out of the headline timing)
    m.profile_begin(args.profile_mask)
    ev0.record(stream)
    for _ in range(args.steps):
        step()
    ev1.record(stream)
    torch.cuda.synchronize()
    prof = m.profile_end()
    ms_profiled = ev0.elapsed_time(ev1)
    depths = dep.cpu().numpy()

    # roofline of the dominant kernel kind, from the live event timings
    units = schedule_units(sh, wl, depths)
    groups, kind_ms = prof
    kinds = {}
    for k, name in ((1, "attention"), (2, "projections"), (3, "head")):
        if groups[k] > 0:
            kinds[name] = {"groups_per_step": groups[k] / args.steps, "ms_per_step": kind_ms[k] / args.steps}
    pk_path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    peaks = json.load(open(pk_path)) if os.path.exists(pk_path) else {}
    hbm = float(peaks.get("hbm_gbs", 6650.0))
    hbm_src = "of measured (MEASURED_PEAKS.json hbm_gbs)" if "hbm_gbs" in peaks else "of fallback 6650 GB/s"
    # algorithmic bytes per step of each kind: what the schedule must read at least once
    alg = {
        "attention": (units["attn_bytes"], "attn_decode: paged per-iteration KV read (fp16 K+V of every attended "
                                            "position, pre blocks and loop iterations)"),
        "projections": ((int((units["loop_rows"] > 0).sum()) + sh.n_pre * int((units["entered"] > 0).sum()))
                        * loop_block_weight_bytes(sh),
                        "W4A16 block projections: INT4 weights + fp16 scales, once per step that has rows"),
        "head": (int((units["boundary"] > 0).sum()) * head_weight_bytes(sh),
                 "head GEMV + argmax: INT4 head weights once per tick with boundary rows"),
    }
    roof = None
    if kinds:
        dom = max(kinds, key=lambda k: kinds[k]["ms_per_step"])
        bytes_step, what = alg[dom]
        a = bytes_step / 1e9 / (kinds[dom]["ms_per_step"] / 1e3)
        roof = {"kernel": what, "bound": "hbm", "achieved": round(a, 1), "peak": hbm, "unit": "GB/s",
                "frac": round(a / hbm, 4), "traffic": None, "algorithmic_bytes_per_step": int(bytes_step),
                "peak_source": hbm_src}
        for k in kinds:
            b, _ = alg[k]
            kinds[k]["algorithmic_GB_per_s"] = round(b / 1e9 / (kinds[k]["ms_per_step"] / 1e3), 1)

    # end to end through tl_generate: pinned host prompts in, host tokens out
    e2e = None
    if not args.no_e2e:
        hp = torch.from_numpy(P.astype(np.int32)).pin_memory()
        ht = torch.zeros((wl.n_lanes, wl.n_new), dtype=torch.int32).pin_memory()
        hd = torch.zeros((wl.n_lanes, wl.n_new), dtype=torch.int32).pin_memory()
        m.generate(hp.numpy(), Ls, wl.n_new, ht, hd)  # warm
        torch.cuda.synchronize()
        reps = max(1, min(args.steps, 3))
        t0 = time.perf_counter()
        for _ in range(reps):
            m.generate(hp.numpy(), Ls, wl.n_new, ht, hd)
        e2e_s = (time.perf_counter() - t0) / reps
        if world > 1:
            t = torch.tensor([e2e_s], device=dev, dtype=torch.float64)
            torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
            e2e_s = float(t.item())
        e2e = {"value": round(world * tokens_per_step / e2e_s, 1), "unit": UNIT,
               "h2d_bytes_per_step": int(P.nbytes + Ls.nbytes),
               "d2h_bytes_per_step": int(2 * wl.n_lanes * wl.n_new * 4),
               "includes": "prompt upload, 64 x 512-token prefill, decode, token download (tl_generate)"}
        assert np.array_equal(ht.numpy(), tok.cpu().numpy()), "tl_generate tokens differ from tl_decode"

    out = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms / args.steps, 3), "higher_is_better": True,
        "ms_per_step_profiled_pass": round(ms_profiled / args.steps, 3),
        "launch_mode": "eager" if args.eager else "cuda graph per tick (conditional nodes)",
        "scaling": "weak", "vs_baseline": None, "dtype": "fp32 accumulate; INT4 weights; fp16 KV",
        "data": "synthetic (seeded random weights and token ids)",
        "config": dict(workload_config(wl), parallelism=f"replicas x{world} (lanes independent, no collective)"),
        "prefill_s": round(prefill_s, 3),
        "gpu_launches": int(st1["kernel_launches"] - st0["kernel_launches"]),
        "lane_iterations_per_step": int(st1["lane_iterations"] - st0["lane_iterations"]) // args.steps,
        "lane_iterations_no_exit": int(sum(int(L) * (wl.n_new - 1) for L in Ls)),
        "depth_histogram": {int(k): int(v) for k, v in zip(*np.unique(depths[:, 1:], return_counts=True))},
        "ticks_per_step": units["ticks"],
        "kernel_time": kinds,
        "roofline": roof,
        "clocks": clk.summary(),
        "e2e": e2e,
    }
    return out, m, P, Ls


# ---------------------------------------------------------- cpu / oracle ----

def oracle_sample(n_tokens: int = 8):
    """The fp64 oracle on a bounded sample of the workload: lane 0's 512-token
    prompt at its L, then n_tokens greedy tokens.  Returns (decode tokens/s,
    seconds of decode, seconds of prompt, cores)."""
    import oracle as O
    from oracle import decode as D
    wl = S.workload(WORKLOAD)
    sh = wl.shape
    W = O.build_weights(sh, S.master_weights(sh), S.gains(sh))
    P = S.prompts(wl.n_lanes, wl.prompt_len, sh.vocab)
    L = int(wl.per_lane_L[0])
    ee = D.EarlyExit(wl.ee_tau, wl.ee_min_L, wl.ee_patience, wl.ee_peek_every)
    t0 = time.perf_counter()
    D.generate_lane(W, P[0], L, 1, ee, keep_logits=False)
    t1 = time.perf_counter()
    D.generate_lane(W, P[0], L, n_tokens + 1, ee, keep_logits=False)
    t2 = time.perf_counter()
    prompt_s = t1 - t0
    decode_s = max((t2 - t1) - prompt_s, 1e-9)
    return n_tokens / decode_s, decode_s, prompt_s, len(os.sched_getaffinity(0)), L


def run_reference(args, rank, world):
    if rank != 0:
        return None
    vals = []
    for k in range(args.warmup + args.steps):
        v, dec_s, pr_s, cores, L = oracle_sample(4)
        if k >= args.warmup:
            vals.append(v)
    value = statistics.median(vals)
    wl = S.workload(WORKLOAD)
    sample = (f"lane 0 (L={L}) of the workload: 512-token prompt then 4 greedy tokens per step; "
              f"tokens/s = 4 / decode seconds (prompt excluded)")
    return {"impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(4 / value * 1e3, 1),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded random weights and token ids)",
            "config": workload_config(wl),
            "cpu_baseline": {"value": round(value, 4), "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(value, 4), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


# -------------------------------------------------------------------- main --

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--profile-mask", type=int, default=0b1110)
    ap.add_argument("--eager", action="store_true", help="launch every kernel of a tick individually "
                    "(for profilers that cannot look inside graphs with conditional nodes)")
    ap.add_argument("--lanes", type=int, default=0, help="reduced case: lanes (profiling captures only)")
    ap.add_argument("--prompt-len", type=int, default=0, help="reduced case: prompt tokens")
    ap.add_argument("--new-tokens", type=int, default=0, help="reduced case: generated tokens")
    args = ap.parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        out = run_reference(args, rank, world)
        if out is not None:
            print(json.dumps(out))
        return 0
    if args.warmup < 3:
        args.warmup = 3
    if world > 1:
        import datetime
        import torch
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=600))
    out, m, P, Ls = run_ours(args, rank, world, local_rank)
    if rank == 0 and not args.no_cpu_baseline:
        v, dec_s, pr_s, cores, L = oracle_sample(8)
        out["cpu_baseline"] = {"value": round(v, 4), "unit": UNIT, "cores": cores, "kind": "oracle",
                               "sample": f"lane 0 (L={L}): 512-token prompt ({pr_s:.1f} s, excluded) then 8 greedy "
                                         f"tokens in {dec_s:.1f} s; fp64 NumPy"}
    if world > 1:
        import torch
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(out))
    return 0


if __name__ == "__main__":
    sys.exit(main())
