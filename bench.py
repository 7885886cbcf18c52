#!/usr/bin/env python
"""Benchmark of the LoopVQ decode hot path on B200.

A step is one decode step of the looped model over the whole batch: decode
attention for every (loop step, layer), loop-step-major as the looped forward
runs them (T x L calls of loopvq_decode_attn), against a cache that was
encoded on the GPU (loopvq_encode) from seeded synthetic keys and values.

Default workload (ctx32k): 24 layers, 16 KV / 16 query heads of dimension 128,
4 loop steps coded as one block, c = 4 (G = 16, K = 256: 0.5 bit per element),
batch 8, 32768-token cache, per-sequence lengths uniform in [16384, 32768].

The JSON line reports algorithmic cache bytes per second (whole job), the time
per step and per call, the roofline of the dominant call, the clocks seen while
timing, an end-to-end figure through the public API with host buffers, and the
CPU checker timed on a bounded sample as a reported baseline.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl loopvq|reference]
"""
from __future__ import annotations

import argparse
import datetime
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from synth import (WORKLOADS, lengths, random_indices, queries, bf16_bits_to_f32, codebook, codebooks,  # noqa: E402
                   tasq_weights, tasq_perm, kv_loops)

METRIC = "LoopVQ decode-attn µs/step & GB/s at 32K ctx, 0.5 bit; % of roofline"
SMEM_BYTES_PER_CLK_SM = 128
FP32_FLOPS_PER_CLK_SM = 256          # 128 fp32 lanes x one fused multiply-add
N_SM = 148


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="ctx32k", choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="loopvq", choices=["loopvq", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--layers", type=int, default=0, help="override the layer count (profiling runs)")
    ap.add_argument("--batch", type=int, default=0, help="override the batch size (profiling runs)")
    ap.add_argument("--no-compare", action="store_true",
                    help="skip the bf16-cache comparison and the bf16-window layout measurement")
    return ap.parse_args()


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def max_over_ranks(x, dist=None, device="cpu"):
    """Maximum of a per-rank float over all ranks (the slowest rank sets every timed figure)."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(x)
    import torch
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world, bytes_per_step_per_rank, ms_per_step_max):
    """Whole-job algorithmic bytes per second (GB/s) under weak scaling: every rank serves its own batch."""
    return world * bytes_per_step_per_rank / (ms_per_step_max * 1e-3) / 1e9


def decode_kernel_name(w):
    """The split kernel a decode call of workload w runs: decode_mha_kernel for one query head per KV
    head at D = 128 with groups of 4 channels (plain or TaSQ keys) or of 16 (plain keys),
    decode_gqa_kernel for 4 query heads per KV head at D = 128 with groups of 8 (plain keys), all with a
    shared codebook; decode_split_kernel otherwise."""
    if w.D == 128 and w.ncb == 1:
        if w.Hq == w.Hkv and (w.c == 4 or (w.c == 16 and not w.tasq)):
            return "decode_mha"                   # plain or TaSQ keys
        if w.c == 8 and w.Hq == 4 * w.Hkv and not w.tasq:
            return "decode_gqa"
    return "decode_split"


def _code_only(src: bytes) -> bytes:
    """C++ source without its comments and with whitespace runs collapsed, so that editing a comment
    does not mark a profile as stale."""
    import re
    src = re.sub(rb"/\*.*?\*/", b" ", src, flags=re.S)
    src = re.sub(rb"//[^\n]*", b" ", src)
    return re.sub(rb"\s+", b" ", src).strip()


def kernel_sources_hash(kern):
    """Hash of what decides a decode split kernel's code and launch: its headers, and for the MHA and GQA
    kernels the line of decode_attn.cu that fixes their launch shape (the whole file otherwise), each
    without comments."""
    import hashlib
    csrc = os.path.join(ROOT, "looped_lm_decode_b200", "csrc")
    h = hashlib.sha256()
    heads = {"decode_mha": ("decode_mha.cuh", "decode_kernel.cuh"),
             "decode_gqa": ("decode_gqa.cuh", "decode_kernel.cuh")}.get(kern, ("decode_split.cuh", "decode_kernel.cuh"))
    for src in heads:
        with open(os.path.join(csrc, src), "rb") as f:
            h.update(_code_only(f.read()))
    with open(os.path.join(csrc, "decode_attn.cu"), "rb") as f:
        attn = f.read()
    tag = {"decode_mha": b"static constexpr int kMhaWarps", "decode_gqa": b"static constexpr int kGqaWarps"}.get(kern)
    h.update(_code_only(attn if tag is None else next(ln for ln in attn.splitlines() if ln.startswith(tag))))
    return h.hexdigest()[:16]


def profiled_traffic(w):
    """DRAM bytes per launch of the decode split kernel from the committed ncu summary, if that summary
    was taken from the kernel sources as they are now (else None)."""
    kern = decode_kernel_name(w)
    path = os.path.join(ROOT, "profiles", f"{kern}_{w.name}.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        prof = json.load(f)
    if kernel_sources_hash(kern) != prof.get("kernel_sources_sha256_16"):
        return None
    return prof["dram_bytes_read_per_launch"] + prof["dram_bytes_write_per_launch"]


def graph_of(fn):
    """A CUDA graph of fn(stream): one eager run first (so every kernel's attributes are set), then a
    capture on a side stream.  Replaying it re-issues the same launches with no host work per call, as a
    serving loop replays its decode step."""
    import torch
    cur = torch.cuda.current_stream()
    fn(cur)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream()
    cap.wait_stream(cur)
    with torch.cuda.graph(g, stream=cap):
        fn(cap)
    cur.wait_stream(cap)
    torch.cuda.synchronize()
    return g


def replay_ms(g, reps, stream):
    """Mean device time of one replay of g over reps back-to-back replays (CUDA events on `stream`)."""
    import torch
    g.replay()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(reps):
        g.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / reps


def bf16_and_window(w, cache, lens, lens_np, max_len, qs, ws, stream, reps=3):
    """Same decode calls on a cache held entirely in bf16 (the pages' comparison, LoopVQ paper Sec. 5.3),
    and on the pages' serving layout: 8 sink + 64 recent tokens in a bf16 window, the rest coded, combined
    through the log-sum-exps (Sec. 4.3 "Cache layout", "Attention").  Timed as CUDA graph replays with CUDA
    events, like the coded calls."""
    import torch
    import looped_lm_decode_b200 as LQ
    from synth import gpu as SG
    dev = qs.device
    nl = min(2, w.L)                                # two bf16 layers: every call streams > L2
    tmp = torch.empty((1, w.B, w.Nmax, w.Hkv, w.D), dtype=torch.bfloat16, device=dev)
    caches = []
    for layer in range(nl):
        kv = []
        for k in range(2):
            SG.fill_kv(w, layer, k, 1, 1, tmp)
            kv.append(tmp[0].permute(0, 2, 1, 3).contiguous())
        caches.append(LQ.Bf16Cache(kv[0], kv[1], w.Hq))
    del tmp
    ws_b = torch.empty(max(LQ.bf16_decode_workspace_bytes(caches[0], max_len), 16), dtype=torch.uint8, device=dev)
    out_b = torch.empty((w.B, w.Hq, w.D), dtype=torch.float32, device=dev)
    lse_b = torch.empty((w.B, w.Hq), dtype=torch.float32, device=dev)

    def timed(fn, calls):
        def seq(st):
            for i in range(calls):
                fn(i, st)
        return replay_ms(graph_of(seq), reps, stream) / calls

    calls = w.T * nl
    bf_ms = timed(lambda i, st: LQ.bf16_decode_attn(caches[i % nl], qs[i], lens, max_len, out=out_b, lse=lse_b,
                                                    workspace=ws_b, stream=st), calls)
    bf_bytes = int(lens_np.astype(np.int64).sum()) * w.Hkv * 2 * w.D * 2 + w.B * w.Hq * (w.D * 2 + w.D * 4 + 4)
    del caches

    # ---- the serving layout through the window API: a full decode step is one advance (a page roll for
    # full windows every 8 steps), then per (loop step, layer) an append and a windowed attention call
    peak, kind = peaks()
    bf16_line = {"us_per_call": bf_ms * 1e3, "gbs": bf_bytes / (bf_ms * 1e-3) / 1e9,
                 "frac": bf_bytes / (bf_ms * 1e-3) / 1e9 / peak, "peak": peak, "peak_kind": kind,
                 "bytes_per_call": bf_bytes,
                 "kernel": "loopvq_bf16_decode_attn over a bf16 cache of the same shape (keys stored rotated)"}
    if w.ncb > 1 or w.tasq:                           # the window's page encoder codes plain, shared-codebook keys
        return {"bf16_cache": bf16_line, "windowed": None}
    n_sink, n_recent = 8, 64
    win = LQ.Window(cache, n_sink=n_sink, n_recent=n_recent, device=dev)
    tmp = torch.empty((1, w.B, win.W, w.Hkv, w.D), dtype=torch.bfloat16, device=dev)
    for dst, k in ((win.k_rot, 0), (win.k_pre, 0), (win.v, 1)):
        SG.fill_kv(w.replace(Nmax=win.W), 0, k, 0, 0, tmp)
        dst.copy_(tmp[0].permute(0, 2, 1, 3).reshape(1, 1, w.B, w.Hkv, win.W, w.D).expand_as(dst))
    del tmp
    coded = np.maximum(n_sink + ((lens_np - n_sink - n_recent) // 8) * 8, n_sink).astype(np.int32)
    win.coded_end.copy_(torch.from_numpy(coded))
    win.fill.copy_(torch.from_numpy((n_sink + lens_np - coded).astype(np.int32)))
    tok = [win.k_rot[0, 0, :, :, 0].contiguous(), win.k_pre[0, 0, :, :, 0].contiguous(), win.v[0, 0, :, :, 0].contiguous()]
    ws_w = torch.empty(max(LQ.window_workspace_bytes(win, cache, w.Nmax), 16), dtype=torch.uint8, device=dev)
    out_c = torch.empty_like(out_b)
    lse_c = torch.empty_like(lse_b)
    def wstep(st):                                    # the token appended by the windowed call itself
        LQ.window_advance(win, cache, stream=st)
        for t in range(w.T):
            for layer in range(w.L):
                LQ.window_append_decode_attn(win, cache, layer, t, tok[0], tok[1], tok[2], qs[t * w.L + layer],
                                             w.Nmax, out=out_c, lse=lse_c, workspace=ws_w, stream=st)

    def wstep_separate(st):                           # the same step with a separate append launch
        LQ.window_advance(win, cache, stream=st)
        for t in range(w.T):
            for layer in range(w.L):
                LQ.window_append(win, layer, t, tok[0], tok[1], tok[2], stream=st)
                LQ.window_decode_attn(win, cache, layer, t, qs[t * w.L + layer], w.Nmax, out=out_c, lse=lse_c,
                                      workspace=ws_w, stream=st)

    def wcalls(st):                                   # the attention calls of a step alone
        for t in range(w.T):
            for layer in range(w.L):
                LQ.window_decode_attn(win, cache, layer, t, qs[t * w.L + layer], w.Nmax, out=out_c, lse=lse_c,
                                      workspace=ws_w, stream=st)

    nsteps = 16                                       # two page rolls for every sequence
    win_step_ms = replay_ms(graph_of(wstep), nsteps, stream)      # the window state lives on the device
    win_step_sep_ms = replay_ms(graph_of(wstep_separate), nsteps, stream)
    win_call_ms = replay_ms(graph_of(wcalls), 2, stream) / (w.T * w.L)
    del win

    return {
        "bf16_cache": bf16_line,
        "windowed": {"us_per_call": win_call_ms * 1e3, "us_per_step": win_step_ms * 1e3,
                     "us_per_step_separate_append": win_step_sep_ms * 1e3, "steps": nsteps,
                     "sink": n_sink, "recent": n_recent,
                     "calls": "per step: loopvq_window_advance (page roll every 8 steps), then per (loop step, "
                              "layer) loopvq_window_append_decode_attn (coded split kernel + merge kernel, which "
                              "writes the new token into the window and attends to the window slots); "
                              "us_per_step_separate_append: the same step with loopvq_window_append + "
                              "loopvq_window_decode_attn"},
    }


def workload_desc(w, world=1):
    return {
        "parallelism": "replicas" if world > 1 else "single GPU",
        "workload": f"{w.name}: looped decoder, {w.L} layers x {w.T} loop steps (blocks of {w.Tc}), "
                    f"{w.Hkv} KV / {w.Hq} q heads, D={w.D}, c={w.c} (G={w.G}, K={w.K}, {8 / w.G:g} bit), "
                    f"batch {w.B}, cache {w.Nmax} tokens",
        "batch": w.B, "context": w.Nmax,
        "lengths": (f"uniform in [{w.len_lo}, {w.Nmax}] (seeded)" if w.len_lo >= 0 else "all full"),
        "layers": w.L, "loop_steps": w.T, "kv_heads": w.Hkv, "q_heads": w.Hq, "head_dim": w.D,
        "codebooks": "shared by the channel groups" if w.ncb == 1 else f"one per channel group ({w.ncb})",
        "keys": "TaSQ transform before coupling (seeded weights and pair orders)" if w.tasq else "plain",
        "bits_per_element": 8 / w.G,
        "l2": "inputs larger than L2: every call streams its layer's index words (> 126 MB), "
              "successive calls touch different layers",
    }


def call_bytes(w, lens):
    """Algorithmic bytes of one decode call: index words, codebook slices, query, output, lse; with TaSQ
    keys also the fp16 token scales (one per token, shared by the heads) and each head's channel weights
    (fp32) and pair order (int16)."""
    idx = int(np.sum(lens)) * w.Hkv * 2 * (w.D // w.c)
    slices = 2 * w.Hkv * w.K * w.c * 2
    q = w.B * w.Hq * w.D * 2
    out = w.B * w.Hq * w.D * 4 + w.B * w.Hq * 4
    tasq = int(np.sum(lens)) * 2 + w.Hkv * (w.D * 4 + (w.D // 2) * 2) if w.tasq else 0
    return idx + slices + q + out + tasq


def gather_bytes(w, lens):
    """Shared-memory gather bytes of one call: D bf16 key and D bf16 value per token and KV head."""
    return int(np.sum(lens)) * w.Hkv * 2 * w.D * 2


def call_flops(w, lens):
    """Algorithmic fp32 work of one call: per token and KV head, the RoPE rotation of the rebuilt key
    (3D) once, then per query head its score (2D) and its value sum (2D): 7D with one query head,
    3D + 4D per query head with several."""
    return int(np.sum(lens)) * w.Hkv * (3 * w.D + 4 * w.D * (w.Hq // w.Hkv))


def floors(w, lens, sm_mhz, hbm_gbs):
    """The three per-call floors (µs) and the peaks behind them: HBM (algorithmic bytes at the measured
    copy bandwidth), shared-memory gathers (128 B/clk/SM x 148 SMs x the sampled SM clock) and fp32
    (128 lanes x 2 flops/clk/SM x 148 SMs x the clock).  The largest binds."""
    smem_gbs = SMEM_BYTES_PER_CLK_SM * N_SM * sm_mhz * 1e6 / 1e9
    fp32_tflops = FP32_FLOPS_PER_CLK_SM * N_SM * sm_mhz * 1e6 / 1e12
    cb, gb, fl = call_bytes(w, lens), gather_bytes(w, lens), call_flops(w, lens)
    return {
        "hbm": {"us": cb / (hbm_gbs * 1e9) * 1e6, "per_call": cb, "peak": hbm_gbs, "unit": "GB/s"},
        "smem": {"us": gb / (smem_gbs * 1e9) * 1e6, "per_call": gb, "peak": smem_gbs, "unit": "GB/s"},
        "fp32": {"us": fl / (fp32_tflops * 1e12) * 1e6, "per_call": fl, "peak": fp32_tflops, "unit": "TFLOP/s"},
    }


class Clocks:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.idx = gpu_index
        self.f = tempfile.NamedTemporaryFile(mode="w+", suffix=".csv", delete=False)
        self.p = None

    def start(self):
        try:
            self.p = subprocess.Popen(["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.FIELDS}",
                                       "--format=csv,noheader,nounits", "-lms", "100"], stdout=self.f,
                                      stderr=subprocess.DEVNULL)
        except FileNotFoundError:
            self.p = None

    def stop(self):
        if self.p is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.p.terminate()
        self.p.wait()
        self.f.flush()
        self.f.seek(0)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.f.read().splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        os.unlink(self.f.name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "samples": len(sm), "reasons": sorted(reasons)}


_CPU_INPUTS = {}


def _cpu_inputs(w, layer, t, b, hq):
    key = (w.name, layer, t, b, hq)
    if key not in _CPU_INPUTS:
        blk = t // w.Tc
        h = hq // (w.Hq // w.Hkv)
        n = int(lengths(w)[b])
        _CPU_INPUTS[key] = (
            bf16_bits_to_f32(queries(w, layer, t, b=[b], hq=[hq])[0, 0]).astype(np.float64),
            random_indices(w, layer, blk, 0, b, h, range(n)), random_indices(w, layer, blk, 1, b, h, range(n)),
            bf16_bits_to_f32(_codebook(w, layer, blk, 0, h)), bf16_bits_to_f32(_codebook(w, layer, blk, 1, h)))
    return _CPU_INPUTS[key]


_TASQ = {}


def _tasq_params(w):
    """Seeded TaSQ weights and pair orders of a workload (host copies)."""
    if w.name not in _TASQ:
        _TASQ[w.name] = (tasq_weights(w), tasq_perm(w))
    return _TASQ[w.name]


def _codebook(w, layer, blk, kv, h):
    """[K][G] bits of a shared codebook, [NCB][K][G] with one per channel group."""
    return codebook(w, layer, blk, kv, h) if w.ncb == 1 else codebooks(w, layer, blk, kv, h)


def cpu_sample(w, seconds, layer=0, t=1):
    """Time the CPU checker's decode on (sequence, query head) units of one call until `seconds` pass.
    Codes for the sampled units are regenerated uniform codes of the same shape (the checker's
    work does not depend on code values); regeneration is not timed."""
    from oracle import oracle as O
    lens = lengths(w)
    m = t % w.Tc
    total_s, nbytes, units = 0.0, 0, 0
    order = [(b, hq) for b in range(w.B) for hq in range(w.Hq)]
    for b, hq in order:
        n = int(lens[b])
        q, ik, iv, Ek, Ev = _cpu_inputs(w, layer, t, b, hq)
        t0 = time.perf_counter()
        if w.tasq:
            h = hq // (w.Hq // w.Hkv)
            O.tasq_decode(q, ik, iv, Ek, Ev, _tasq_params(w)[1][layer, t // w.Tc, h], _tasq_params(w)[0][layer, t, h],
                          np.ones(n), w.c, w.Tc, m, w.theta, 1 / math.sqrt(w.D))
        else:
            (O.decode_pg if w.ncb > 1 else O.decode)(q, ik, iv, Ek, Ev, w.c, w.Tc, m, w.theta, 1 / math.sqrt(w.D))
        total_s += time.perf_counter() - t0
        nbytes += n * 2 * (w.D // w.c)
        units += 1
        if total_s >= seconds:
            break
    return total_s, nbytes, units


def cpu_model():
    """CPU model name of the host (first /proc/cpuinfo entry)."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def host_threads():
    """Cores this process may run on."""
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def cpu_sample_all_cores(w, seconds_1core_per_unit, threads, budget_s, layer=0, t=1):
    """The checker's decode on `threads` host cores at once: (sequence, query head) units of one call, one
    per thread at a time.  The checker's ctypes calls release the GIL, so the threads run on separate
    cores.  The number of units is bounded so the run takes about budget_s; inputs are regenerated before
    the clock starts."""
    from concurrent.futures import ThreadPoolExecutor
    from oracle import oracle as O
    lens = lengths(w)
    m = t % w.Tc
    order = [(b, hq) for b in range(w.B) for hq in range(w.Hq)]
    nunits = max(threads, int(threads * budget_s / max(seconds_1core_per_unit, 1e-3)))
    nunits = min(nunits, len(order))
    units = [_cpu_inputs(w, layer, t, b, hq) + (b, hq) for b, hq in order[:nunits]]

    def one(u):
        q, ik, iv, Ek, Ev, b, hq = u
        if w.tasq:
            h = hq // (w.Hq // w.Hkv)
            n = len(ik)
            O.tasq_decode(q, ik, iv, Ek, Ev, _tasq_params(w)[1][layer, t // w.Tc, h], _tasq_params(w)[0][layer, t, h],
                          np.ones(n), w.c, w.Tc, m, w.theta, 1 / math.sqrt(w.D))
        else:
            (O.decode_pg if w.ncb > 1 else O.decode)(q, ik, iv, Ek, Ev, w.c, w.Tc, m, w.theta, 1 / math.sqrt(w.D))
        return len(ik) * 2 * (w.D // w.c)

    with ThreadPoolExecutor(max_workers=threads) as ex:
        t0 = time.perf_counter()
        nbytes = sum(ex.map(one, units))
        wall = time.perf_counter() - t0
    return wall, nbytes, nunits


def _unpack_codes(words, Nmax, NP):
    """Index words of one (layer, block, sequence, KV head) -> [Nmax][2NP] K and V codes (the word
    layout of include/loopvq.h: tiles of 4 tokens, [Nmax/4][NP][4]; bytes K p, K p+NP, V p, V p+NP)."""
    wd = words.reshape(Nmax // 4, NP, 4).transpose(0, 2, 1).reshape(Nmax, NP).astype(np.uint32)
    k = np.concatenate([wd & 0xFF, (wd >> 8) & 0xFF], axis=1).astype(np.uint8)
    v = np.concatenate([(wd >> 16) & 0xFF, (wd >> 24) & 0xFF], axis=1).astype(np.uint8)
    return k, v


def tie_sample(w, threads):
    """The tokens the encode baseline and the tie count use: one (sequence, KV head) per thread, a run of
    `chunk` tokens each."""
    chunk = min(4096, w.Nmax)
    return chunk, [((j * 7) % w.B, (j * 5) % w.Hkv, (j * 997) % max(1, w.Nmax - chunk)) for j in range(threads)]


def gpu_sample_codes(w, cache, threads, layer=0, blk=0):
    """The GPU's key and value codes of the tie sample's tokens, copied to the host.  Taken right after the
    cache is encoded: the windowed comparison later rolls window pages into the same cache, which replaces
    the codes of the tokens it rolls."""
    NP = w.D // (2 * w.c)
    chunk, sample = tie_sample(w, threads)
    per_bh = w.Nmax * NP
    codes = {}
    for b, h, tok0 in sample:
        base = ((layer * w.NB + blk) * w.B + b) * w.Hkv + h
        words = cache.idx[base * per_bh:(base + 1) * per_bh].cpu().numpy().view(np.uint32)
        ck, cv = _unpack_codes(words, w.Nmax, NP)
        codes[(b, h, tok0)] = (ck[tok0:tok0 + chunk].copy(), cv[tok0:tok0 + chunk].copy())
    return codes


def cpu_encode_and_ties(w, gpu_codes, threads, budget_s, layer=0, blk=0):
    """The checker's encode of sampled tokens of one (layer, block) on `threads` cores, timed and
    extrapolated to the whole (layer, block) unit (labelled as such), and the GPU's codes for the same
    tokens (`gpu_sample_codes`) compared with it: a code that differs counts as a near-tie when the two
    fp64 distances differ by at most 1e-5 relative, anything else as a mismatch.  Runs after the timed
    region."""
    from concurrent.futures import ThreadPoolExecutor
    from oracle import oracle as O
    if w.tasq:
        return None, {"checked": 0, "note": "TaSQ codes are checked by the GPU tests, not here"}
    chunk, sample = tie_sample(w, threads)
    jobs = []
    for b, h, tok0 in sample:
        toks = range(tok0, tok0 + chunk)
        for kv in range(2):
            x = kv_loops(w, layer, kv, blk * w.Tc, blk * w.Tc + w.Tc - 1, [b], toks, [h])[:, 0, :, 0, :]
            E = bf16_bits_to_f32(_codebook(w, layer, blk, kv, h))
            jobs.append((b, h, kv, tok0, np.ascontiguousarray(bf16_bits_to_f32(x)), np.ascontiguousarray(E)))
    enc = O.encode_pg if w.ncb > 1 else O.encode

    def one(job):
        return enc(job[4], job[5], w.c)

    with ThreadPoolExecutor(max_workers=threads) as ex:
        t0 = time.perf_counter()
        refs = list(ex.map(one, jobs))
        wall = time.perf_counter() - t0
    vec_sample = len(jobs) * chunk * (w.D // w.c)
    vec_unit = 2 * w.B * w.Nmax * w.Hkv * (w.D // w.c)
    enc_line = {"ms_per_layer_block": wall * vec_unit / vec_sample * 1e3, "cores": threads, "extrapolated": True,
                "sample": f"{len(jobs)} runs of {chunk} tokens (one sequence and KV head each, K and V) of "
                          f"layer {layer}, block {blk}: {vec_sample} coupled vectors timed in {wall:.2f} s on "
                          f"{threads} threads, scaled to the {vec_unit} vectors of the (layer, block)"}
    # the GPU codes of the same tokens
    checked = ties = other = 0
    for (b, h, kv, tok0, x, E), ref in zip(jobs, refs):
        gpu = gpu_codes[(b, h, tok0)][kv]
        checked += gpu.size
        for i, g in zip(*np.nonzero(gpu != ref)):
            if w.ncb > 1:
                dg = O.dist64_pg(x, E, w.c, int(i), int(g), int(gpu[i, g]))
                do = O.dist64_pg(x, E, w.c, int(i), int(g), int(ref[i, g]))
            else:
                dg = O.dist64(x, E, w.c, int(i), int(g), int(gpu[i, g]))
                do = O.dist64(x, E, w.c, int(i), int(g), int(ref[i, g]))
            if abs(dg - do) <= 1e-5 * max(dg, do):
                ties += 1
            else:
                other += 1
    return enc_line, {"checked": checked, "near_ties": ties, "mismatches": other,
                      "rule": "a differing code is a near-tie when its fp64 distance is within 1e-5 relative "
                              "of the checker's; any other difference is a mismatch"}


def run_reference(args):
    """The CPU checker as the reference arm: each step decodes a bounded sample of the workload."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    w = WORKLOADS[args.workload]
    nthr = host_threads()
    per_step = max(0.1, min(2.0, 60.0 / max(1, args.steps + args.warmup)))
    s1, _, u1 = cpu_sample(w, min(per_step, 2.0))            # one unit's single-thread time sizes the steps
    per_unit = s1 / max(u1, 1)
    for _ in range(args.warmup):
        cpu_sample_all_cores(w, per_unit, nthr, per_step)
    tot_s, tot_b, tot_u = 0.0, 0, 0
    for _ in range(args.steps):
        s, b, u = cpu_sample_all_cores(w, per_unit, nthr, per_step)
        tot_s, tot_b, tot_u = tot_s + s, tot_b + b, tot_u + u
    gbs = tot_b / tot_s / 1e9
    sample = (f"{tot_u} (sequence, query head) units of the layer-0, loop-step-2 call over {args.steps} steps, "
              f"one unit per thread at a time on {nthr} threads; fp64 dequant, RoPE and softmax per unit")
    line = {"impl": "reference", "metric": METRIC, "value": gbs, "unit": "GB/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot_s / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_desc(w, int(os.environ.get("WORLD_SIZE", "1"))),
            "cpu_baseline": {"value": gbs, "unit": "GB/s", "cores": nthr, "kind": "oracle", "sample": sample,
                             "cpu_model": cpu_model()},
            "e2e": {"value": gbs, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
        return

    import torch
    import looped_lm_decode_b200 as LQ
    from synth import gpu as SG

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    w = WORKLOADS[args.workload]
    if args.layers > 0:
        w = w.replace(L=args.layers)
    if args.batch > 0:
        w = w.replace(B=args.batch)

    # ---------------- set-up: codebooks, slices, RoPE table, GPU encode of every (layer, block)
    cache = LQ.Cache(w.L, w.T, w.Tc, w.Hkv, w.Hq, w.D, w.c, w.K, w.B, w.Nmax, w.theta, device=dev, ncb=w.ncb)
    SG.fill_codebook(w, cache.codebook)
    LQ.prepare(cache)
    tq = None
    if w.tasq:
        tw, tp = _tasq_params(w)
        tq = LQ.Tasq(cache, w=torch.from_numpy(tw).to(dev), perm=torch.from_numpy(tp).to(dev), device=dev)
    xk = torch.empty((w.Tc, w.B, w.Nmax, w.Hkv, w.D), dtype=torch.bfloat16, device=dev)
    xv = torch.empty_like(xk)
    enc_ms = []
    for layer in range(w.L):
        for blk in range(w.NB):
            SG.fill_kv(w, layer, 0, blk * w.Tc, blk * w.Tc + w.Tc - 1, xk)
            SG.fill_kv(w, layer, 1, blk * w.Tc, blk * w.Tc + w.Tc - 1, xv)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            if tq is not None:
                LQ.tasq_encode(cache, tq, layer, blk, xk, xv)
            else:
                LQ.encode(cache, layer, blk, xk, xv)
            e1.record()
            torch.cuda.synchronize()
            enc_ms.append(e0.elapsed_time(e1))
    del xk, xv
    torch.cuda.empty_cache()

    lens_np = lengths(w)
    lens = torch.from_numpy(lens_np).to(dev)
    max_len = int(lens_np.max())
    ncall = w.L * w.T
    qs = torch.empty((ncall, w.B, w.Hq, w.D), dtype=torch.bfloat16, device=dev)
    for t in range(w.T):
        for layer in range(w.L):
            SG.fill_q(w, layer, t, qs[t * w.L + layer])
    out = torch.empty((ncall, w.B, w.Hq, w.D), dtype=torch.float32, device=dev)
    lse = torch.empty((ncall, w.B, w.Hq), dtype=torch.float32, device=dev)
    ws = torch.empty(LQ.decode_workspace_bytes(cache, max_len), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step(st=None):
        st = stream if st is None else st
        for t in range(w.T):
            for layer in range(w.L):
                i = t * w.L + layer
                if tq is not None:
                    LQ.tasq_decode_attn(cache, tq, layer, t, qs[i], lens, max_len, 0.0, out=out[i], lse=lse[i],
                                        workspace=ws, stream=st)
                else:
                    LQ.decode_attn(cache, layer, t, qs[i], lens, max_len, 0.0, out=out[i], lse=lse[i], workspace=ws,
                                   stream=st)

    def barrier():
        torch.cuda.synchronize()
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()

    for _ in range(max(args.warmup, 3)):
        step()
    graph = graph_of(step)                # the step's L x T calls as one CUDA graph
    for _ in range(max(args.warmup, 3)):
        graph.replay()
    clocks = Clocks(local)
    barrier()
    clocks.start()
    time.sleep(0.3)                       # let the sampler start before the timed region
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for k in range(args.steps):
        graph.replay()
    t1.record(stream)
    barrier()
    clk = clocks.stop()
    ms_total = t0.elapsed_time(t1)
    ms_step_local = ms_total / args.steps
    call_ms_local = ms_step_local / ncall  # one call = split kernel + merge kernel

    # ---------------- end to end through the public API with host buffers
    q_host = torch.empty(qs.shape, dtype=qs.dtype, pin_memory=True)
    q_host.copy_(qs)
    lens_host = torch.from_numpy(lens_np.copy()).pin_memory()
    out_host = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
    lse_host = torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True)
    e2e_steps = max(3, min(args.steps, 20))

    def e2e_step():
        qs.copy_(q_host, non_blocking=True)
        lens.copy_(lens_host, non_blocking=True)
        step()
        out_host.copy_(out, non_blocking=True)
        lse_host.copy_(lse, non_blocking=True)

    e2e_step()
    barrier()
    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    a1.record(stream)
    barrier()
    e2e_ms_local = a0.elapsed_time(a1) / e2e_steps
    h2d = q_host.numel() * q_host.element_size() + lens_host.numel() * 4
    d2h = out_host.numel() * 4 + lse_host.numel() * 4

    tie_codes = None
    if world == 1 and not args.no_cpu_baseline and not w.tasq:
        tie_codes = gpu_sample_codes(w, cache, host_threads())
    compare = None
    if not args.no_compare and rank == 0:
        compare = bf16_and_window(w, cache, lens, lens_np, max_len, qs, ws, stream)

    ms_step = max_over_ranks(ms_step_local, dist, dev)
    e2e_ms = max_over_ranks(e2e_ms_local, dist, dev)
    avg_call_ms = max_over_ranks(call_ms_local, dist, dev)

    if rank == 0:
        cb = call_bytes(w, lens_np)
        gb = gather_bytes(w, lens_np)
        step_bytes = cb * ncall
        value = job_throughput(world, step_bytes, ms_step)
        hbm_peak, peak_kind = peaks()
        sm_mhz = clk.get("sm_mhz") or 1965.0
        fl = floors(w, lens_np, sm_mhz, hbm_peak)
        bound = max(fl, key=lambda k: fl[k]["us"])
        call_us = avg_call_ms * 1e3
        scale_unit = {"GB/s": 1e9, "TFLOP/s": 1e12}
        achieved = fl[bound]["per_call"] / (call_us * 1e-6) / scale_unit[fl[bound]["unit"]]
        floor_line = {k: {"floor_us": v["us"], "frac": v["us"] / call_us, "peak": v["peak"], "unit": v["unit"],
                          "per_call": v["per_call"]} for k, v in fl.items()}
        floor_line["hbm"]["peak_kind"] = f"{peak_kind} copy bandwidth"
        floor_line["smem"]["peak_kind"] = f"derived: {SMEM_BYTES_PER_CLK_SM} B/clk/SM x {N_SM} SMs x median SM clock"
        floor_line["fp32"]["peak_kind"] = (f"derived: {FP32_FLOPS_PER_CLK_SM} flop/clk/SM x {N_SM} SMs x median SM "
                                           "clock; algorithmic flops 3D + 4D per query head per token and KV head")
        line = {
            "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": max(args.warmup, 3), "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": workload_desc(w, world),
            "us_per_step": ms_step * 1e3, "us_per_call": avg_call_ms * 1e3, "calls_per_step": ncall,
            "roofline": {"bound": bound, "achieved": achieved, "peak": fl[bound]["peak"], "unit": fl[bound]["unit"],
                         "frac": achieved / fl[bound]["peak"], "traffic": profiled_traffic(w),
                         "peak_kind": floor_line[bound]["peak_kind"],
                         "kernel": f"one loopvq_decode_attn call ({decode_kernel_name(w)}_kernel + merge_kernel)",
                         "per_launch": fl[bound]["per_call"], "bytes_per_launch": cb,
                         "floors": floor_line},
            "clocks": clk,
            "e2e": {"value": job_throughput(world, step_bytes, e2e_ms), "unit": "GB/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
            "gpu_launches": args.steps * ncall * 2,
            "encode": {"ms_per_layer_block": statistics.median(enc_ms),
                       "tokens_per_s": w.B * w.Nmax / (statistics.median(enc_ms) * 1e-3),
                       "input_gbs": 2 * w.Tc * w.B * w.Nmax * w.Hkv * w.D * 2 / (statistics.median(enc_ms) * 1e-3) / 1e9,
                       "kernel": ("tasq_sigma_kernel + encode_tc_kernel with TaSQ keys (u split into three "
                                  "bf16 parts along the contraction)" if w.tasq else
                                  "encode_tc_kernel (tcgen05 bf16 distance contraction + TMEM arg-max)" if w.ncb == 1
                                  else "encode_tc_kernel, one codebook per channel group (tiles of 128 tokens of "
                                       "one group, that group's codebook as the B operand)")},
        }
        if compare is not None:
            line["bf16_cache"] = compare["bf16_cache"]
            line["bf16_cache"]["loopvq_speedup"] = compare["bf16_cache"]["us_per_call"] / (avg_call_ms * 1e3)
            if compare["windowed"] is not None:
                line["windowed"] = compare["windowed"]
        if world == 1 and not args.no_cpu_baseline:
            s1, nb1, u1 = cpu_sample(w, args.cpu_seconds)
            nthr = host_threads()
            sa, nba, ua = cpu_sample_all_cores(w, s1 / max(u1, 1), nthr, args.cpu_seconds)
            enc_cpu, ties = cpu_encode_and_ties(w, tie_codes, nthr, args.cpu_seconds)
            line["cpu_baseline"] = {
                "value": nb1 / s1 / 1e9, "unit": "GB/s", "cores": 1, "kind": "oracle", "cpu_model": cpu_model(),
                "sample": f"{u1} (sequence, query head) units of the layer-0, loop-step-2 call, {s1:.1f} s "
                          f"single-threaded",
                "all_cores": {"value": nba / sa / 1e9, "unit": "GB/s", "cores": nthr,
                              "sample": f"{ua} units of the same call on {nthr} threads (one unit per thread at a "
                                        f"time), {sa:.1f} s wall"},
                "encode": enc_cpu}
            line["near_ties"] = ties
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
