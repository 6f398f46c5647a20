#!/usr/bin/env python
"""Benchmark of the dMel front end on B200: dMel tokens/s (waveform to 6144-d bf16 vector) and
the fraction of the HBM roofline.

Headline workload: ragged1024, 1024 clips of 1-30 s of 16 kHz fp32 audio (pink noise, harmonic
tones, both, silence), concatenated with an offsets array and no padding: 318,044 frames, bf16
table 1280 x 6144 ~ N(0, 0.02), RMSNorm on (eps 1e-6), bf16 out. A step is one dmel_forward over
the whole batch with inputs resident in HBM (1.0 GB in, 3.9 GB out: larger than L2), each step
timed with its own CUDA events on the launching stream. `e2e` is the same batch through
dmel_forward_host: page-locked host waveforms in, the 6144-d vectors back in page-locked host
memory, every copy inside the timed region.

Context lines (each with its own roofline fractions and CPU baseline): one_clip_2s (latency of a
40-frame call, fp32 table and output, no RMSNorm), batch64_10s (12,800 frames), long_20min
(24,000 frames), streams4096 (1000 successive calls of 4096 streams x 800 new samples plus the
carried tail), and the ShortConv and hMLP kernels.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

N > 1 runs under torchrun: every rank runs its own copy of the batch on its own GPU (replicas,
no collective on the data path); the step time is the max over ranks. --impl reference times
the CPU oracle on the host cores instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "dMel tokens/sec (waveform to 6144-d bf16 embed); % of HBM roofline"
DIM = 6144
DESCR = {
    "one_clip_2s": "one_clip_2s: 1 clip, 2.0 s of 16 kHz mono fp32 (3 sines + N(0, 0.01^2) noise), 40 frames, "
                   "fp32 table 1280x6144 N(0,0.02), no RMSNorm, fp32 out",
    "batch64_10s": "batch64_10s: 64 clips x 10 s of 16 kHz mono fp32 (pink noise + linear chirp, 10% silent, "
                   "5% clipped), 12,800 frames, bf16 table 1280x6144 N(0,0.02), RMSNorm on (eps 1e-6, "
                   "w~N(1,0.1)), bf16 out",
    "long_20min": "long_20min: 1 clip of 20 min of 16 kHz mono fp32 (AR(12) noise bursts of 50-400 ms, 20% "
                  "silence), 24,000 frames, bf16 table, RMSNorm on, bf16 out",
    "ragged1024": "ragged1024: 1024 clips of 1-30 s of 16 kHz mono fp32 (pink noise, harmonic tones, both, "
                  "silence), concatenated with offsets and no padding, 318,044 frames, bf16 table 1280x6144 "
                  "N(0,0.02), RMSNorm on (eps 1e-6, w~N(1,0.1)), bf16 out",
    "streams4096": "streams4096: 4096 streams x (800 new + 800 carried samples) per call, 1000 successive calls, "
                   "white noise + tone, bf16 table, RMSNorm on, bf16 out",
}
HEADLINE = "ragged1024"
# algorithmic HBM bytes per frame: the path (800 new fp32 samples in, the vector out), and each
# stage: codes (samples in, 80 code bytes out), embedding (codes in, vector out)
IN_BYTES = 800 * 4
CODES_BYTES = 80


def out_bytes(out_es: int) -> int:
    return DIM * out_es


# DRAM bytes (read + write) of each stage's kernels per call, from the ncu capture of the headline
# workload itself (318,044 frames, profiles/dram_traffic_ragged1024.md, the kernels as they are
# now): codes_kernel_entry; and the embedding call's six kernels, gram_kernel, gram_combine_kernel,
# gram_diag_kernel (G), norm_partials_kernel, norm_finalize_kernel (the scales) and
# embed_sp_kernel<kScaled>. Other frame counts have no capture of the current kernels: null.
TRAFFIC_MEASURED = {318044: {"codes": 1024211456 + 27772160,
                             "embed": (15749120 + 7212544 + 15735040) + (29174528 + 21165056) + (69979648 + 68096)
                             + (42732288 + 3851324416)}}
# the tensor cores' work per frame in the one-hot product: 2 * 1280 * 6144 logical flops, run as a
# 2:4-sparse product whose peak is twice the dense bf16 peak (nominal 4.5 vs 2.25 PFLOP/s)
ONEHOT_FLOP_PER_FRAME = 2 * 1280 * DIM
SPARSE_PEAK_RATIO = 2.0


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        try:
            d = json.load(open(p))
            return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                    "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                    "source": "measured"}
        except (KeyError, TypeError, ValueError) as e:  # a file of another shape: the fallback, said so
            return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                    "source": f"fallback (MEASURED_PEAKS.json unreadable: {type(e).__name__})"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


class ClockSampler:
    """nvidia-smi samples (every 200 ms) of one GPU while the timed region runs."""

    FIELDS = ["clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.active",
              "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
              "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]

    def __init__(self, uuid: str | None):
        self.uuid = uuid
        self.proc = None
        self.lines: list[str] = []
        self.thread = None

    def start(self):
        cmd = ["nvidia-smi", f"--query-gpu={','.join(self.FIELDS)}", "--format=csv,noheader,nounits", "-lms", "200"]
        if self.uuid:
            cmd += ["-i", self.uuid]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < len(self.FIELDS):
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------------------------ workloads

def load_workload(name: str) -> dict:
    """Host inputs of a workload: waveforms, sample offsets, table (fp32), RMSNorm weight or None,
    output element size."""
    from encoder_free_audio_b200 import synth
    if name == "one_clip_2s":
        wav, off = synth.one_clip_2s()
        return {"wav": wav, "off": off, "table": synth.table(), "g": None, "bf16": False}
    fn = {"batch64_10s": synth.batch64_10s, "long_20min": synth.long_20min, "ragged1024": synth.ragged1024}[name]
    wav, off = fn()
    return {"wav": wav, "off": off, "table": synth.table(), "g": synth.rms_weight(), "bf16": True}


def oracle_sample(wav, off, table64, g64, budget_s: float, seed: int, tails=None) -> dict:
    """The oracle as it stands (codes + embedding [+ RMSNorm], fp64) on a bounded random sample of
    the workload's frames, on this host's cores; tokens/s."""
    from oracle import oracle
    oracle.build()
    fo = oracle.frame_offsets(off)
    F = int(fo[-1])
    rng = np.random.default_rng(seed)

    def run(n):
        ids = np.sort(rng.choice(F, n, replace=False)).astype(np.int64)
        t0 = time.perf_counter()
        c = oracle.codes(wav, off, tails=tails, frame_ids=ids, want_lhat=False)
        oracle.embed(c, table64, g64, 1e-6)
        return time.perf_counter() - t0

    n0 = min(F, 32)
    t0 = run(n0)
    n = int(min(F, max(n0, n0 * budget_s / max(t0, 1e-6))))
    t = run(n)
    return {"value": n / t, "unit": "tokens/s", "cores": oracle.threads(), "kind": "oracle",
            "sample": f"{n} random frames of the {F}-frame workload (codes + embedding"
                      f"{' + RMSNorm' if g64 is not None else ''}, fp64)"}


def host_tables(torch, wl):
    """The table and RMSNorm weight as the oracle sees them: the bf16 values (exactly) in fp64."""
    dt = torch.bfloat16 if wl["bf16"] else torch.float32
    tb = torch.from_numpy(wl["table"]).to(dt).double().numpy()
    gb = None if wl["g"] is None else torch.from_numpy(wl["g"]).to(dt).double().numpy()
    return tb, gb


class Timer:
    """CUDA-event timing of calls on one stream (after warm-up; optional L2 flush before each)."""

    def __init__(self, torch, stream, flush=None):
        self.torch, self.stream, self.flush = torch, stream, flush

    def run(self, fn, steps: int, warmup: int, launches: list | None = None):
        torch = self.torch
        for _ in range(warmup):
            if self.flush is not None:
                self.flush.zero_()
            fn()
        torch.cuda.synchronize()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        for i in range(steps):
            if self.flush is not None:
                self.flush.zero_()
            evs[i][0].record(self.stream)
            fn()
            evs[i][1].record(self.stream)
            if launches is not None:
                from encoder_free_audio_b200 import dmel
                launches.append(dmel.dmel_last_launch_count())
        torch.cuda.synchronize()
        return [a.elapsed_time(b) for a, b in evs]


def stage_lines(F, codes_ms, embed_ms, out_es, pk) -> dict:
    """Roofline of each stage (algorithmic bytes of one launch / its mean event-timed duration)."""
    def line(name, ms, bytes_per_frame, kernel):
        s = statistics.mean(ms) / 1e3
        achieved = bytes_per_frame * F / s / 1e9
        traffic = TRAFFIC_MEASURED[F][name] if F in TRAFFIC_MEASURED else None
        return {"bound": "hbm", "achieved": achieved, "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / pk["hbm_gbs"], "traffic": traffic,
                "ms": statistics.mean(ms), "kernel": kernel, "peak_source": pk["source"]}
    norm = ("RMSNorm scales from G = T T^T, then the 2:4-sparse one-hot product" if F >= 16384 else
            "2:4-sparse one-hot product, RMSNorm by row-sum exchange")
    return {"codes": line("codes", codes_ms, IN_BYTES + CODES_BYTES, "codes_kernel_entry (fp64 DFT, fp32 mel/log/levels)"),
            "embed": line("embed", embed_ms, CODES_BYTES + out_bytes(out_es), f"dmel_embed call ({norm})")}


def run_batch(torch, dev, dmel, FrontEnd, name, wl, steps, warmup, pk, flush, with_cpu, cpu_budget,
              with_e2e=True, e2e_steps=None):
    """One batch workload: device-resident steps, the two stages alone, e2e from host memory."""
    stream = torch.cuda.current_stream()
    dt = torch.bfloat16 if wl["bf16"] else torch.float32
    T = torch.from_numpy(wl["table"]).to(dt).to(dev)
    G = None if wl["g"] is None else torch.from_numpy(wl["g"]).to(dt).to(dev)
    fe = FrontEnd(T, G, 1e-6, dt)
    plan = fe.plan(wl["off"])
    F = plan.n_frames
    out_es = 2 if wl["bf16"] else 4
    wav_d = torch.from_numpy(wl["wav"]).to(dev)
    timer = Timer(torch, stream, flush)
    launches: list = []
    step_ms = timer.run(lambda: fe.forward(wav_d, plan), steps, warmup, launches)
    prepared_ms = None
    if G is not None and wl["bf16"]:
        # the same step with the table prepared once (RMSNorm scales from a G computed up front)
        fe_p = FrontEnd(T, G, 1e-6, dt, prepare=True)
        prepared_ms = timer.run(lambda: fe_p.forward(wav_d, plan), steps, warmup) if fe_p.prepared is not None else None
        del fe_p
    # the two stages alone (same kernels), each bracketed by events on the launching stream
    codes_ms = timer.run(lambda: dmel.dmel_codes(wav_d, plan.sample_offsets, plan.frame_offsets, F, plan.codes),
                         steps, warmup)
    embed_ms = timer.run(lambda: dmel.dmel_embed(plan.codes, T, plan.out, rms_weight=G, eps=1e-6,
                                                 workspace=plan.workspace), steps, warmup)
    res = {"frames": F, "step_ms": step_ms, "prepared_ms": prepared_ms, "launches": launches,
           "stages": stage_lines(F, codes_ms, embed_ms, out_es, pk),
           "path_bytes_per_frame": IN_BYTES + out_bytes(out_es)}
    del wav_d
    if with_e2e:
        # end to end: page-locked host waveforms in, vectors back in page-locked host memory
        wav_h = torch.from_numpy(wl["wav"]).pin_memory()
        out_h = torch.empty((F, DIM), dtype=dt, pin_memory=True)
        ws = torch.empty(max(1, dmel.dmel_forward_host_workspace_size(wl["off"], DIM, dmel._dtype_code(T),
                                                                       dmel._dtype_code(out_h), G is not None)),
                         dtype=torch.uint8, device=dev)
        fwd = lambda: dmel.dmel_forward_host(wav_h, wl["off"], T, out_h, rms_weight=G, eps=1e-6, workspace=ws)
        e2e_ms = Timer(torch, stream, None).run(fwd, e2e_steps or steps, min(warmup, 3))
        res["e2e"] = {"ms": e2e_ms, "h2d_bytes_per_step": int(wl["wav"].nbytes),
                      "d2h_bytes_per_step": int(F * DIM * out_es)}
        del wav_h, out_h, ws
    if with_cpu:
        tb, gb = host_tables(torch, wl)
        res["cpu_baseline"] = oracle_sample(wl["wav"], wl["off"], tb, gb, cpu_budget, 77)
    del plan, fe
    torch.cuda.empty_cache()
    return res


def context_line(name, r, pk, world) -> dict:
    F = r["frames"]
    ms = statistics.mean(r["step_ms"])
    st = r["stages"]
    dom = max(st, key=lambda k: st[k]["ms"])
    line = {"workload": DESCR[name], "frames": F, "tokens_per_s": F / (ms / 1e3), "ms_per_call": ms,
            "hbm_roofline_frac": r["path_bytes_per_frame"] * F / (ms / 1e3) / 1e9 / pk["hbm_gbs"],
            "roofline": st[dom], "stages": {k: {"ms": v["ms"], "frac": v["frac"]} for k, v in st.items()},
            "launches_per_call": r["launches"][-1] if r["launches"] else None}
    if r.get("prepared_ms"):
        line["prepared_table_ms_per_call"] = statistics.mean(r["prepared_ms"])
    if "e2e" in r:
        e = r["e2e"]
        line["e2e"] = {"value": F / (statistics.mean(e["ms"]) / 1e3), "unit": "tokens/s",
                       "ms_per_call": statistics.mean(e["ms"]), "h2d_bytes_per_step": e["h2d_bytes_per_step"],
                       "d2h_bytes_per_step": e["d2h_bytes_per_step"]}
    if "cpu_baseline" in r:
        line["cpu_baseline"] = r["cpu_baseline"]
    return line


def latency_line(torch, dev, dmel, FrontEnd, pk, calls: int, with_cpu: bool) -> dict:
    """one_clip_2s: a single 40-frame call (fp32 table and output, no RMSNorm): p50 / p99 device
    latency per call, and the same from host memory (dmel_forward_host)."""
    wl = load_workload("one_clip_2s")
    stream = torch.cuda.current_stream()
    T = torch.from_numpy(wl["table"]).to(dev)
    fe = FrontEnd(T, None, 1e-6, torch.float32)
    plan = fe.plan(wl["off"])
    F = plan.n_frames
    wav_d = torch.from_numpy(wl["wav"]).to(dev)
    timer = Timer(torch, stream, None)
    ms = sorted(timer.run(lambda: fe.forward(wav_d, plan), calls, 10))
    wav_h = torch.from_numpy(wl["wav"]).pin_memory()
    out_h = torch.empty((F, DIM), dtype=torch.float32, pin_memory=True)
    ws = torch.empty(max(1, dmel.dmel_forward_host_workspace_size(wl["off"], DIM, dmel.DMEL_F32, dmel.DMEL_F32, False)),
                     dtype=torch.uint8, device=dev)
    e2e = sorted(timer.run(lambda: dmel.dmel_forward_host(wav_h, wl["off"], T, out_h, workspace=ws), calls, 10))
    p50, p99 = ms[len(ms) // 2], ms[min(len(ms) - 1, int(0.99 * len(ms)))]
    path = (IN_BYTES + out_bytes(4)) * F
    line = {"workload": DESCR["one_clip_2s"], "frames": F, "calls": calls, "p50_us": 1e3 * p50, "p99_us": 1e3 * p99,
            "tokens_per_s": F / (statistics.mean(ms) / 1e3),
            "hbm_roofline_frac": path / (p50 / 1e3) / 1e9 / pk["hbm_gbs"],
            "e2e": {"p50_us": 1e3 * e2e[len(e2e) // 2], "value": F / (statistics.mean(e2e) / 1e3), "unit": "tokens/s",
                    "h2d_bytes_per_step": int(wl["wav"].nbytes), "d2h_bytes_per_step": int(F * DIM * 4)},
            "note": "latency-bound: one 40-frame call; the HBM fraction is the call's bytes over its p50 latency"}
    if with_cpu:
        tb, _ = host_tables(torch, wl)
        line["cpu_baseline"] = oracle_sample(wl["wav"], wl["off"], tb, None, 2.0, 71)
    return line


def streaming_line(torch, dev, dmel, FrontEnd, pk, calls: int, warmup: int, with_cpu: bool) -> dict:
    """streams4096: 4096 streams, each call brings 800 new samples per stream plus the carried
    800-sample tail (one frame per stream); `calls` successive calls, per-call device time with
    CUDA events. The calls' inputs are generated up front and kept on the device."""
    from encoder_free_audio_b200 import synth
    S = synth.Streams4096()
    wl = {"table": synth.table(), "g": synth.rms_weight(), "bf16": True}
    T = torch.from_numpy(wl["table"]).to(torch.bfloat16).to(dev)
    G = torch.from_numpy(wl["g"]).to(torch.bfloat16).to(dev)
    fe = FrontEnd(T, G, 1e-6, torch.bfloat16)
    plan = fe.plan(synth.offsets_from_lengths([800] * S.n))
    n_in = min(calls, 64)  # distinct inputs, cycled (13 MB each)
    xs = [torch.from_numpy(S.call(k)).to(dev).reshape(-1) for k in range(n_in)]
    # two tail buffers, alternating: call k reads tails[k % 2] and writes tails[(k + 1) % 2] (the
    # codes kernel writes them; updating one buffer in place takes a copy kernel after it)
    tails = [torch.zeros((S.n, 800), device=dev), torch.zeros((S.n, 800), device=dev)]
    stream = torch.cuda.current_stream()
    for k in range(warmup):
        fe.forward(xs[k % n_in], plan, tails=tails[k % 2], tails_out=tails[(k + 1) % 2])
    tails[0].zero_()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(calls)]
    for k in range(calls):
        evs[k][0].record(stream)
        fe.forward(xs[k % n_in], plan, tails=tails[k % 2], tails_out=tails[(k + 1) % 2])
        evs[k][1].record(stream)
    torch.cuda.synchronize()
    ms = [a.elapsed_time(b) for a, b in evs]
    srt = sorted(ms)
    per_frame = IN_BYTES + 2 * 800 * 4 + out_bytes(2)  # new samples, tail in and out, vector out
    line = {"workload": DESCR["streams4096"], "frames_per_call": S.n, "calls": calls,
            "p50_us": 1e3 * srt[len(srt) // 2], "p99_us": 1e3 * srt[min(len(srt) - 1, int(0.99 * len(srt)))],
            "tokens_per_s": S.n * calls / (sum(ms) / 1e3),
            "hbm_roofline_frac": per_frame * S.n * calls / (sum(ms) / 1e3) / 1e9 / pk["hbm_gbs"],
            "launches_per_call": dmel.dmel_last_launch_count()}
    if with_cpu:
        tb, gb = host_tables(torch, wl)
        wav = S.call(0).reshape(-1)
        line["cpu_baseline"] = oracle_sample(wav, synth.offsets_from_lengths([800] * S.n), tb, gb, 2.0, 72,
                                             tails=np.zeros((S.n, 800), np.float32))
        line["cpu_baseline"]["sample"] += " (call 0, zero tails)"
    return line


def shortconv_context(torch, dev, dmel, pk: dict, warmup: int, steps: int = 20, with_oracle: bool = False) -> dict:
    """ShortConv (the decoder's width-4 per-channel causal conv) over 12,800 frame vectors as 64
    sequences of 200 tokens, bf16, with carried state in and out: HBM-bound, so reported against
    the measured copy bandwidth. Inputs larger than L2 are rotated between calls."""
    T, C, n_seq = 12800, DIM, 64
    g = torch.Generator(device=dev).manual_seed(9)
    xs = [torch.randn((T, C), device=dev, generator=g).to(torch.bfloat16) for _ in range(2)]
    y = torch.empty_like(xs[0])
    w = (0.5 * torch.randn((C, 4), device=dev, generator=g)).contiguous()
    off = torch.arange(0, T + 1, T // n_seq, dtype=torch.int64, device=dev)
    st = torch.zeros((n_seq, 3, C), dtype=torch.bfloat16, device=dev)
    st_out = torch.empty_like(st)
    for k in range(warmup):
        dmel.dmel_shortconv(xs[k % 2], off, w, y, state=st, state_out=st_out)
    s = torch.cuda.current_stream()
    # back-to-back calls (a decoder layer's stream of them) between one pair of events on the
    # launching stream; the inputs alternate between two 157 MB buffers, so no call finds its
    # input in L2
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    ev0.record(s)
    for k in range(steps):
        dmel.dmel_shortconv(xs[k % 2], off, w, y, state=st, state_out=st_out)
    ev1.record(s)
    torch.cuda.synchronize()
    ms = ev0.elapsed_time(ev1) / steps
    launches = dmel.dmel_last_launch_count()
    # this GPU's own device-to-device copy of the same bytes (x's size, read + write), timed the
    # same way: the attainable rate for a read-one-write-one stream on this machine
    for k in range(3):
        y.copy_(xs[k % 2])
    torch.cuda.synchronize()
    ev0.record(s)
    for k in range(steps):
        y.copy_(xs[k % 2])
    ev1.record(s)
    torch.cuda.synchronize()
    copy_gbs = 2 * T * C * 2 / (ev0.elapsed_time(ev1) / steps / 1e3) / 1e9
    algo = 2 * T * C * 2 + C * 16 + 2 * n_seq * 3 * C * 2  # x in, y out, weights, state in + out
    line = {"workload": "12,800 tokens x 6144 channels bf16, 64 sequences, state in/out", "us_per_call": ms * 1e3,
            "achieved_gbs": algo / (ms / 1e3) / 1e9, "peak_gbs": pk["hbm_gbs"],
            "frac": algo / (ms / 1e3) / 1e9 / pk["hbm_gbs"], "bytes_per_call": algo,
            "copy_gbs_this_gpu": copy_gbs, "frac_of_copy_this_gpu": algo / (ms / 1e3) / 1e9 / copy_gbs,
            "tokens_per_s": T / (ms / 1e3), "launches_per_call": launches}
    if with_oracle:
        # the oracle beside it: 8 of the 64 sequences on the host (fp64, one thread), as tokens/s
        from oracle import oracle
        xh = xs[0][: 8 * (T // n_seq)].float().cpu().numpy()
        t0 = time.perf_counter()
        oracle.shortconv(xh, np.arange(0, xh.shape[0] + 1, T // n_seq), w.cpu().numpy(),
                         st[:8].float().cpu().numpy())
        dt = time.perf_counter() - t0
        line["cpu_baseline"] = {"value": xh.shape[0] / dt, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                                "sample": f"8 of 64 sequences ({xh.shape[0]} tokens x {C} channels)"}
    return line


def hmlp_context(torch, dev, dmel, pk: dict, warmup: int, steps: int = 10, with_oracle: bool = False) -> dict:
    """The hMLP patchifier of the vision path on 4 images of 800 x 800 (1,600 patches of 40 x 40),
    widths 1536 / 1536 / 1536 / 6144, bf16, synthetic weights: dense GEMMs, so reported against the
    sustained bf16 tensor peak."""
    n, H, W = 4, 800, 800
    d1 = d2 = d3 = DIM // 4
    g = torch.Generator(device=dev).manual_seed(11)

    def rn(*shape, scale=1.0):
        return (scale * torch.randn(shape, device=dev, generator=g)).contiguous()
    params = {"W1": rn(75, d1, scale=75 ** -0.5).to(torch.bfloat16), "W2": rn(4 * d1, d2, scale=(4 * d1) ** -0.5).to(
        torch.bfloat16), "W3": rn(4 * d2, d3, scale=(4 * d2) ** -0.5).to(torch.bfloat16),
        "W4": rn(4 * d3, DIM, scale=(4 * d3) ** -0.5).to(torch.bfloat16)}
    for k, d in (("b1", d1), ("b2", d2), ("b3", d3), ("b4", DIM)):
        params[k] = rn(d, scale=0.1)
    for s_, d in ((1, d1), (2, d2), (3, d3)):
        params[f"g{s_}"] = (1 + rn(d, scale=0.1)).contiguous()
        params[f"be{s_}"] = rn(d, scale=0.1)
    img = rn(n, H, W, 3).clamp(-1, 1).to(torch.bfloat16).contiguous()
    P = n * (H // 40) * (W // 40)
    out = torch.empty((P, DIM), dtype=torch.bfloat16, device=dev)
    ws = torch.empty(dmel.dmel_hmlp_workspace_size(P, params), dtype=torch.uint8, device=dev)
    for _ in range(warmup):
        dmel.dmel_hmlp(img, params, out, ws)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    s = torch.cuda.current_stream()
    torch.cuda.synchronize()
    for k in range(steps):
        evs[k][0].record(s)
        dmel.dmel_hmlp(img, params, out, ws)
        evs[k][1].record(s)
    torch.cuda.synchronize()
    ms = sum(a.elapsed_time(b) for a, b in evs) / steps
    flop = 2 * P * (64 * 75 * d1 + 16 * 4 * d1 * d2 + 4 * 4 * d2 * d3 + 4 * d3 * DIM)
    line = {"workload": "4 images 800x800 bf16 = 1,600 patches, widths 1536/1536/1536/6144", "us_per_call": ms * 1e3,
            "patches_per_s": P / (ms / 1e3), "achieved_tflops": flop / (ms / 1e3) / 1e12,
            "peak_tflops": pk["bf16_tflops_sustained"],
            "frac": flop / (ms / 1e3) / 1e12 / pk["bf16_tflops_sustained"], "flop_per_call": flop,
            "launches_per_call": dmel.dmel_last_launch_count(),
            "gemms": "stage 1 in one tcgen05 kernel; stages 2-4 on the tcgen05 CTA-pair GEMM, each followed by its row kernel"}
    if with_oracle:
        from oracle import oracle
        host = {k: v.double().cpu().numpy() for k, v in params.items()}
        t0 = time.perf_counter()
        oracle.hmlp(img[:1, :40, :40].double().cpu().numpy(), host)
        dt = time.perf_counter() - t0
        line["cpu_baseline"] = {"value": 1.0 / dt, "unit": "patches/s", "cores": 1, "kind": "oracle",
                                "sample": "1 patch of 40 x 40"}
    return line


# ------------------------------------------------------------------------------------ arms

def run_profile(args):
    """Profiling mode (no timing, no JSON line): dmel_codes and dmel_embed (RMSNorm, bf16 out) on
    one workload, args.steps times, so a profiler can capture the path's kernels on a call of that
    size. The form of RMSNorm follows the library's rule for the call size (DMEL_EMBED_NORM
    overrides it)."""
    import torch
    from encoder_free_audio_b200 import build, dmel
    build.build()
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    if args.profile in ("shortconv", "hmlp"):
        fn = shortconv_context if args.profile == "shortconv" else hmlp_context
        line = fn(torch, dev, dmel, peaks(), 3, steps=args.steps)
        print(f"profile {args.profile}: {args.steps} calls after 3 warm-ups, device error bits "
              f"{dmel.dmel_get_device_error(clear=True)}", flush=True)
        return 0
    wl = load_workload(args.profile)
    fo = dmel.dmel_frame_offsets(wl["off"])
    F = int(fo[-1])
    dt = torch.bfloat16 if wl["bf16"] else torch.float32
    T = torch.from_numpy(wl["table"]).to(dt).to(dev)
    G = None if wl["g"] is None else torch.from_numpy(wl["g"]).to(dt).to(dev)
    w = torch.from_numpy(wl["wav"]).to(dev)
    so, fod = torch.from_numpy(wl["off"]).to(dev), torch.from_numpy(fo).to(dev)
    codes = torch.empty((F, 80), dtype=torch.uint8, device=dev)
    out = torch.empty((F, DIM), dtype=dt, device=dev)
    n = dmel.dmel_workspace_size(F, DIM, dmel._dtype_code(T), G is not None, True)
    ws = torch.empty(max(1, n), dtype=torch.uint8, device=dev)
    for _ in range(args.steps):
        dmel.dmel_codes(w, so, fod, F, codes)
        dmel.dmel_embed(codes, T, out, rms_weight=G, eps=1e-6, workspace=ws)
    torch.cuda.synchronize()
    print(f"profile {args.profile}: {F} frames x {args.steps} calls, device error bits "
          f"{dmel.dmel_get_device_error(clear=True)}", flush=True)
    return 0


def run_reference(args):
    """The oracle on the host cores, on the headline workload: each step a bounded random sample
    of its frames (codes + embedding + RMSNorm, fp64)."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from oracle import oracle
    import torch
    wl = load_workload(HEADLINE)
    tb, gb = host_tables(torch, wl)
    oracle.build()
    F = int(oracle.frame_offsets(wl["off"])[-1])
    rng = np.random.default_rng(78)
    per_step = 96
    times = []
    for i in range(args.warmup + args.steps):
        ids = np.sort(rng.choice(F, per_step, replace=False)).astype(np.int64)
        t0 = time.perf_counter()
        c = oracle.codes(wl["wav"], wl["off"], frame_ids=ids, want_lhat=False)
        oracle.embed(c, tb, gb, 1e-6)
        dt = time.perf_counter() - t0
        if i >= args.warmup:
            times.append(dt)
    total = sum(times)
    value = per_step * len(times) / total
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / len(times),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": DESCR[HEADLINE], "step": f"{per_step} random frames of the workload per step"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": oracle.threads(), "kind": "oracle",
                         "sample": f"{per_step} random frames per step, {args.steps} timed steps"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def run_ours(args):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=dev)

    from encoder_free_audio_b200 import build, dmel, replicas
    from encoder_free_audio_b200.frontend import FrontEnd
    build.build()
    pk = peaks()
    solo = rank == 0 and world == 1
    with_cpu = solo and not args.no_cpu_baseline

    def barrier():
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    # ---------------------------------------------------------- headline: ragged1024
    wl = load_workload(HEADLINE)
    barrier()
    uuid = None
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        uuid = None
    sampler = ClockSampler(uuid)
    sampler.start()
    head = run_batch(torch, dev, dmel, FrontEnd, HEADLINE, wl, args.steps, args.warmup, pk, None, False, 0.0,
                     with_e2e=True, e2e_steps=max(3, args.steps // 2))
    clocks = sampler.stop()
    barrier()
    F = head["frames"]
    total_ms = replicas.max_over_ranks(sum(head["step_ms"]), world, dev)
    e2e_ms = replicas.max_over_ranks(sum(head["e2e"]["ms"]), world, dev)
    e2e_steps = len(head["e2e"]["ms"])

    # ---------------------------------------------------------- context lines
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    nvtx = torch.cuda.nvtx
    ctx = {}
    for name in ("batch64_10s", "long_20min"):
        nvtx.range_push(name)
        r = run_batch(torch, dev, dmel, FrontEnd, name, load_workload(name), args.steps, args.warmup, pk, flush,
                      with_cpu, 3.0)
        ctx[name] = context_line(name, r, pk, world)
        nvtx.range_pop()
    nvtx.range_push("one_clip_2s")
    ctx["one_clip_2s"] = latency_line(torch, dev, dmel, FrontEnd, pk, max(100, 10 * args.steps), with_cpu)
    nvtx.range_pop()
    nvtx.range_push("streaming")
    ctx["streams4096"] = streaming_line(torch, dev, dmel, FrontEnd, pk, args.stream_calls, args.warmup, with_cpu)
    nvtx.range_pop()
    nvtx.range_push("shortconv")
    ctx["shortconv"] = shortconv_context(torch, dev, dmel, pk, args.warmup, with_oracle=with_cpu)
    nvtx.range_pop()
    nvtx.range_push("hmlp")
    ctx["hmlp"] = hmlp_context(torch, dev, dmel, pk, args.warmup, with_oracle=with_cpu)
    nvtx.range_pop()
    err_bits = dmel.dmel_get_device_error(clear=True)

    if rank != 0:
        if world > 1:
            dist.barrier()
            dist.destroy_process_group()
        return 0

    value = replicas.job_throughput([F * args.steps] * world, total_ms / 1e3)
    st = head["stages"]
    dom = max(st, key=lambda k: st[k]["ms"])
    emb_s = st["embed"]["ms"] / 1e3
    line = {
        "metric": METRIC,
        "value": value,
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": total_ms / args.steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": DESCR[HEADLINE], "frames_per_gpu": F, "parallelism": f"replicas x{world}",
                   "l2": "inputs larger than L2 (1.02 GB of samples in, 3.9 GB of vectors out per step)",
                   "compute": "fp64 transform, 2:4-sparse bf16 x bf16 -> fp32 tensor-core sum, bf16 out"},
        "hbm_roofline_frac": head["path_bytes_per_frame"] * value / world / (pk["hbm_gbs"] * 1e9),
        "clocks": {"sm_mhz": clocks["sm_mhz"], "sm_max_mhz": clocks["sm_max_mhz"], "reasons": clocks["reasons"]},
        "e2e": {"value": world * F * e2e_steps / (e2e_ms / 1e3), "unit": "tokens/s",
                "h2d_bytes_per_step": head["e2e"]["h2d_bytes_per_step"],
                "d2h_bytes_per_step": head["e2e"]["d2h_bytes_per_step"],
                "api": "dmel_forward_host (page-locked host samples in, page-locked host vectors out)"},
        "gpu_launches": int(sum(head["launches"])),
        "roofline": {k: v for k, v in st[dom].items() if k != "ms"},
        "roofline_stages": st,
        "roofline_tensor": {"achieved": ONEHOT_FLOP_PER_FRAME * F / emb_s / 1e12,
                            "peak": SPARSE_PEAK_RATIO * pk["bf16_tflops_sustained"], "unit": "TFLOP/s",
                            "frac": ONEHOT_FLOP_PER_FRAME * F / emb_s / 1e12
                            / (SPARSE_PEAK_RATIO * pk["bf16_tflops_sustained"]),
                            "note": "embedding's one-hot product, 2*1280*6144 logical flops per frame, against the "
                                    "2:4-sparse bf16 peak = measured sustained dense bf16 x 2 (nominal ratio)"},
        "context": ctx,
        "device_error_bits": err_bits,
    }
    if with_cpu:
        tb, gb = host_tables(torch, wl)
        line["cpu_baseline"] = oracle_sample(wl["wav"], wl["off"], tb, gb, 12.0, 77)
    print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--stream-calls", type=int, default=1000)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile", choices=["batch64_10s", "long_20min", "one_clip_2s", "ragged1024", "shortconv", "hmlp"],
                    default=None, help="run the path's kernels on one workload --steps times, untimed (for "
                    "profilers); shortconv / hmlp: the context line's calls, --steps of them after 3 warm-ups")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)  # at least 3 untimed warm-up steps
    if args.profile:
        return run_profile(args)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
