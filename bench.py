"""Benchmark of the GDN token mixer on B200.

A step is one gdn_prefill call of the long-prefill workload (1 sequence x
32768 tokens, 32 heads, dk = dv = 128, bf16 inputs and output, fp32 state,
S0 ~ N(0, 0.02)): ShortConv, SiLU, L2Norm, gates, the chunked gated delta rule
and the gated RMSNorm output.  The decode workload (256 sequences x 32 heads,
fp32 state updated in place, 1000 consecutive steps) is timed in the same run
and reported under "decode".

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With N > 1 (one process per GPU under torchrun) every rank runs its own
independent long-prefill problem (weak scaling, no collective on the data
path); the step time is the max over ranks.  `--impl reference` times the fp64
CPU oracle (the only reference this method has) on a bounded sample.
"""
import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time
from dataclasses import replace

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from linear_attention_token_shortconv_b200 import dist as rankio  # noqa: E402
from linear_attention_token_shortconv_b200 import gdn  # noqa: E402
from linear_attention_token_shortconv_b200.workloads import (DECODE, LONG, PRETRAIN, QSA, VARLEN,  # noqa: E402
                                                             make_decode_inputs, make_layer_inputs,
                                                             make_prefill_inputs, make_qsa_inputs, to_oracle_bits)

METRIC = "GDN prefill tokens/s at T=32K H=32 (% TC peak); decode state GB/s (% HBM)"
# Algorithmic work per token-head of the fused chunked prefill (chunk C = 64, d = 128):
# MMA flops C(6dk+4dv) + 6 dk dv, and one pass over bf16 q,k,v,z, the two gate
# logits and a bf16 output.
PREFILL_FLOP_PER_TOKEN_HEAD = 64 * (6 * 128 + 4 * 128) + 6 * 128 * 128   # 180,224
PREFILL_BYTES_PER_TOKEN_HEAD = 4 * 128 * 2 + 2 * 2 + 128 * 2           # 1,284
# Backward (fp32, d = 128), per token-head.  Bytes that must move: q, k, v, z and
# d_out read, dq, dk, dv and d_z written (fp32 rows of 128), two gate logits read
# and their two gradients written: 4,624 B.  SIMT arithmetic of the token-level
# recurrence: the forward step re-run (S^T k, S^T q, the update: 6 d^2 flop) and
# the backward step (D += q dy^T, D^T k, P dy, P de, D e, <D, P>, the decay of D:
# 14 d^2 flop) = 20 d^2 = 327,680 flop.
BACKWARD_BYTES_PER_TOKEN_HEAD = 9 * 128 * 4 + 4 * 4
BACKWARD_FLOP_PER_TOKEN_HEAD = 20 * 128 * 128
# fp32 SIMT peak: 148 SMs x 128 fp32 lanes x 2 flop (FMA) x 1.965 GHz (max SM clock)
FP32_SIMT_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12
# Per-kernel roofline units (a few (sequence, head) chains run as one fused
# persistent kernel; many chains as chunk_prep / chunk_chain launches per
# segment).  chunk_prep reads q, k, v and the two logits: 772 of
# the 1,284 B above; the rest (z in, the output out) belongs to chunk_chain, whose
# algorithmic work is, though, the state-dependent MMAs of the chunk form:
# 2 C dk dv (U) + 2 C dk dv (Q S) + 2 C^2 dv (Aqk U) + 2 C dk dv (S update) per
# chunk = 114,688 flop per token-head (chunk_prep's state-independent MMAs are the
# other 65,536 of the 180,224 above).  Each kernel is reported against its bound.
KERNEL_ROOFLINE = {"chunk_prep": ("hbm", 3 * 128 * 2 + 2 * 2),                      # 772 B
                   "chunk_chain": ("tensor", 3 * 2 * 128 * 128 + 2 * 64 * 128),        # 114,688 flop
                   # both in one persistent launch: the whole pass's 1,284 B
                   "prefill_fused": ("hbm", PREFILL_BYTES_PER_TOKEN_HEAD)}
# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) per unit from one
# ncu capture of each kernel (profiles/), valid only while the kernel's sources
# are the ones captured (sha1 over them); otherwise the JSON reports traffic null.
#   prefill_fused: `bench.py --profile-case prefill 8192` (T = 8192, H = 32): 347.4 MB read +
#     332.6 MB written for 262,144 token-heads; per token-head, scaled to the launch.
NCU_TRAFFIC = {
    "prefill_fused": {"sources": ["prefill_tc.cu", "prep_body.cuh", "chain_body.cuh"],
                      "sha1": "736a70aa4f6290e66b2141af8ad45a411a4f9a00",
                      "bytes_per_unit": (347.356160e6 + 332.615680e6) / (8192 * 32)},
}


def kernel_traffic(name, units):
    """ncu DRAM bytes for one launch of `name` processing `units` (token-heads),
    or None when no capture of the kernel's current sources exists."""
    rec = NCU_TRAFFIC.get(name)
    if rec is None:
        return None
    import hashlib
    h = hashlib.sha1()
    try:
        for f in rec["sources"]:
            with open(os.path.join(ROOT, "linear_attention_token_shortconv_b200", "csrc", f), "rb") as fh:
                h.update(fh.read())
    except OSError:
        return None
    return rec["bytes_per_unit"] * units if h.hexdigest() == rec["sha1"] else None


# Peaks used only when MEASURED_PEAKS.json is absent: an earlier measurement on
# the same B200 pool (STREAM-style copy; cuBLAS bf16 burst and sustained).
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return FALLBACK_PEAKS, "fallback"


def wait_event(ev):
    """Wait for a recorded event by polling it with short sleeps: the clock
    sampler's thread runs meanwhile (a device synchronisation can keep it out)."""
    while not ev.query():
        time.sleep(0.0002)


class ClockSampler:
    """SM clock, power and clock-event (throttle) reasons sampled during a
    region: NVML polled every millisecond from a thread (the counters
    nvidia-smi prints; a 16 ms timed region still gets several samples), else
    nvidia-smi every 200 ms.  Read-only: no setting is changed."""
    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown"}
    SMI_FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                  "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                  "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.rows = []          # (sm_mhz, max_mhz, watts, set of reason names)
        self.source = None
        self._stop = None
        self._thread = None
        self._proc = None
        self._path = None

    def _nvml_handle(self):
        import pynvml
        pynvml.nvmlInit()
        try:
            p = torch.cuda.get_device_properties(self.index)
            bus = f"{p.pci_domain_id:08x}:{p.pci_bus_id:02x}:{p.pci_device_id:02x}.0"
            return pynvml, pynvml.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.index)

    def _poll(self, nv, h):
        get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        mx = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
        while not self._stop.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                w = nv.nvmlDeviceGetPowerUsage(h) / 1000.0
                r = get_reasons(h)
                self.rows.append((float(sm), float(mx), w,
                                  {n for bit, n in self.REASONS.items() if r & bit}))
            except Exception:
                break
            self._polling.set()
            self._stop.wait(0.001)
        self._polling.set()

    def __enter__(self):
        import threading
        try:
            nv, h = self._nvml_handle()
            self._stop = threading.Event()
            self._polling = threading.Event()
            self._thread = threading.Thread(target=self._poll, args=(nv, h), daemon=True)
            self._thread.start()
            self._polling.wait(timeout=2.0)   # the poll loop is running before the region starts
            self.rows.clear()                 # samples from before the region
            self.source = "nvml 1 ms"
            return self
        except Exception:
            pass
        try:
            fd, self._path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self._fh = open(self._path, "w")
            self._proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.SMI_FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"], stdout=self._fh,
                stderr=subprocess.DEVNULL)
            time.sleep(0.3)
            self.source = "nvidia-smi 200 ms"
        except (OSError, ValueError):
            self._proc = None
        return self

    def __exit__(self, *exc):
        if self._thread is not None:
            self._stop.set()
            self._thread.join(timeout=5)
        if self._proc is not None:
            self._proc.terminate()
            try:
                self._proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self._proc.kill()
            self._fh.close()
            names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
            for line in open(self._path):
                parts = [p.strip() for p in line.split(",")]
                try:
                    self.rows.append((float(parts[0]), float(parts[1]), float(parts[2]),
                                      {names[i] for i, v in enumerate(parts[4:8]) if v == "Active"}))
                except (ValueError, IndexError):
                    continue
            os.unlink(self._path)

    def summary(self):
        if not self.rows:
            return {"sm_mhz": None, "sm_max_mhz": None,
                    "reasons": ["no samples" if self.source else "no clock source"]}
        reasons = sorted(set().union(*(r[3] for r in self.rows)))
        return {"sm_mhz": statistics.median(r[0] for r in self.rows),
                "sm_max_mhz": max(r[1] for r in self.rows),
                "sm_mhz_min": min(r[0] for r in self.rows),
                "power_w_max": max(r[2] for r in self.rows), "samples": len(self.rows),
                "source": self.source, "reasons": reasons}


def barrier(world):
    rankio.barrier(world)


def max_over_ranks(x, world):
    return rankio.max_over_ranks(x, world, "cuda")


def prefill_call(inp, out, S_final):
    gdn.prefill(inp["q"], inp["k"], inp["v"], inp["conv_w"], inp["a_logit"], inp["b_logit"],
                inp["A"], inp["b_alpha"], inp["z"], inp["norm_w"], S0=inp["S0"],
                cu_seqlens=inp["cu_seqlens"], num_seqs=S_final.shape[0], out=out, S_final=S_final)


def bench_prefill(cfg, steps, warmup, world, rank, dev):
    """Times `steps` gdn_prefill calls.  Besides the whole-call events (on the
    caller's stream, which the library forks from and joins), every kernel
    launch is bracketed by its own pair of events on the stream it runs on."""
    inp = make_prefill_inputs(cfg, dev, seed=rankio.shard_seed(cfg.seed, rank))
    n_tok, H = cfg.total_tokens, cfg.H
    out = torch.empty((n_tok, H, cfg.dv), dtype=torch.bfloat16, device=dev)
    S_final = torch.empty((cfg.num_seqs, H, cfg.dk, cfg.dv), dtype=torch.float32, device=dev)
    for _ in range(warmup):
        prefill_call(inp, out, S_final)
    n_slot = gdn.last_call_slots()
    torch.cuda.synchronize()
    mk = lambda n: [torch.cuda.Event(enable_timing=True) for _ in range(n)]
    evb, eve = mk(steps), mk(steps)
    kb, ke = [mk(n_slot) for _ in range(steps)], [mk(n_slot) for _ in range(steps)]
    for e in evb + eve + sum(kb, []) + sum(ke, []):   # materialise the CUDA handles
        e.record()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    launches = 0
    with ClockSampler(dev.index) as clk:
        start.record()
        for i in range(steps):
            gdn.set_timing_events(evb[i], eve[i])
            gdn.set_kernel_events(kb[i], ke[i])
            prefill_call(inp, out, S_final)
            launches += gdn.last_call_launches()
        end.record()
        gdn.set_timing_events(None, None)
        gdn.set_kernel_events()
        wait_event(end)
        torch.cuda.synchronize()
    barrier(world)
    ms = max_over_ranks(start.elapsed_time(end) / steps, world)
    kern_ms = max_over_ranks(sum(b.elapsed_time(e) for b, e in zip(evb, eve)) / steps, world)
    # launch slots: the fused persistent kernel (with its task-list builder for
    # unequal lengths), or chunk_prep / chunk_chain per segment
    names = ("prefill_fused",) if n_slot == 1 else ("chunk_prep", "chunk_chain")
    per = {n: [] for n in names}
    for i in range(steps):
        for j in range(n_slot):
            per[names[j % len(names)]].append(kb[i][j].elapsed_time(ke[i][j]))
    kernels = {}
    for name, xs in per.items():
        kernels[name] = {"launches_per_step": len(xs) // steps,
                         "avg_launch_ms": max_over_ranks(statistics.fmean(xs), world),
                         "ms_per_step": max_over_ranks(sum(xs) / steps, world)}
    return ms, kern_ms, clk.summary(), kernels, launches, inp


def prefill_summary(cfg, steps, ms, kern_ms, kernels, pk):
    """Whole-call throughput and roofline fractions of one timed prefill workload,
    with each kernel's share of the call (from its per-launch events)."""
    th = cfg.total_tokens * cfg.H
    gbs = PREFILL_BYTES_PER_TOKEN_HEAD * th / (kern_ms * 1e-3) / 1e9
    tf = PREFILL_FLOP_PER_TOKEN_HEAD * th / (kern_ms * 1e-3) / 1e12
    total = sum(k["ms_per_step"] for k in kernels.values()) or 1.0
    return {"workload": cfg.name, "steps": steps, "ms_per_step": ms, "call_ms": kern_ms,
            "tokens_per_s": cfg.total_tokens / (ms * 1e-3),
            "hbm": {"bytes_per_token_head": PREFILL_BYTES_PER_TOKEN_HEAD, "achieved_gbs": gbs,
                    "peak_gbs": pk["hbm_gbs"], "frac": gbs / pk["hbm_gbs"]},
            "tc": {"flop_per_token_head": PREFILL_FLOP_PER_TOKEN_HEAD, "achieved_tflops": tf,
                   "peak_tflops": pk["bf16_tflops"], "frac": tf / pk["bf16_tflops"]},
            "kernels": {n: {"launches_per_step": k["launches_per_step"], "ms_per_step": k["ms_per_step"],
                            "avg_launch_ms": k["avg_launch_ms"], "share": k["ms_per_step"] / total}
                        for n, k in kernels.items()}}


def bench_e2e(cfg, steps, warmup, world, rank, dev):
    """Same metric through the public API with the inputs in pinned host memory:
    every step copies the step's inputs host->device and reads out + S_final back.
    Steps are pipelined as a serving loop would run them: two sets of device
    buffers, the host->device copies on one stream, gdn_prefill on the caller's
    stream, the device->host reads on a third, ordered by events, so that step
    i + 1's inputs travel and step i - 1's results come back while step i
    computes.  The timed region starts before the first copy and ends after the
    last read-back."""
    src = make_prefill_inputs(cfg, dev, seed=rankio.shard_seed(cfg.seed, rank))
    host = {k: (None if v is None else v.cpu().pin_memory()) for k, v in src.items()}
    n_tok, H = cfg.total_tokens, cfg.H
    sets = []
    for _ in range(2):
        sets.append({"in": {k: (None if v is None else torch.empty_like(v)) for k, v in src.items()},
                     "out": torch.empty((n_tok, H, cfg.dv), dtype=torch.bfloat16, device=dev),
                     "S": torch.empty((cfg.num_seqs, H, cfg.dk, cfg.dv), dtype=torch.float32, device=dev),
                     "computed": torch.cuda.Event(), "drained": torch.cuda.Event(), "loaded": torch.cuda.Event()})
    del src
    out_h = torch.empty(sets[0]["out"].shape, dtype=torch.bfloat16, pin_memory=True)
    S_h = torch.empty(sets[0]["S"].shape, dtype=torch.float32, pin_memory=True)
    h2d = sum(v.numel() * v.element_size() for v in host.values() if v is not None)
    d2h = out_h.numel() * out_h.element_size() + S_h.numel() * S_h.element_size()
    compute = torch.cuda.current_stream(dev)
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def step(i):
        b = sets[i % 2]
        with torch.cuda.stream(s_in):
            s_in.wait_event(b["computed"])   # step i - 2 is done reading these inputs
            for k, v in host.items():
                if v is not None:
                    b["in"][k].copy_(v, non_blocking=True)
            b["loaded"].record(s_in)
        compute.wait_event(b["loaded"])
        compute.wait_event(b["drained"])     # step i - 2's results have left these buffers
        prefill_call(b["in"], b["out"], b["S"])
        b["computed"].record(compute)
        with torch.cuda.stream(s_out):
            s_out.wait_event(b["computed"])
            out_h.copy_(b["out"], non_blocking=True)
            S_h.copy_(b["S"], non_blocking=True)
            b["drained"].record(s_out)

    def run(n):
        first = torch.cuda.Event(enable_timing=True)
        first.record(compute)
        s_in.wait_event(first)
        s_out.wait_event(first)
        for i in range(n):
            step(i)
        last = torch.cuda.Event()
        last.record(s_out)
        compute.wait_event(last)
        done = torch.cuda.Event(enable_timing=True)
        done.record(compute)
        return first, done

    run(max(warmup, 2))
    torch.cuda.synchronize()
    barrier(world)
    start, end = run(steps)
    torch.cuda.synchronize()
    barrier(world)
    ms = max_over_ranks(start.elapsed_time(end) / steps, world)
    return ms, h2d, d2h


def bench_decode(cfg, steps, dev):
    d = make_decode_inputs(cfg, dev)
    S, hist = d["S"], d["ring"]
    out = torch.empty((cfg.B, cfg.H, cfg.dv), dtype=torch.bfloat16, device=dev)
    P = cfg.pool

    def step(t):
        p = t % P
        gdn.decode_step(d["q"][p], d["k"][p], d["v"][p], d["conv_w"], hist, d["a_logit"][p],
                        d["b_logit"][p], d["A"], d["b_alpha"], d["z"][p], d["norm_w"], S, out=out)

    for t in range(5):
        step(t)
    torch.cuda.synchronize()
    evb = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    eve = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    for e in evb + eve:
        e.record()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    launches = 0
    with ClockSampler(dev.index) as clk:
        start.record()
        for t in range(steps):
            gdn.set_timing_events(evb[t], eve[t])
            step(t)
            launches += gdn.last_call_launches()
        end.record()
        gdn.set_timing_events(None, None)
        wait_event(end)
        torch.cuda.synchronize()
    ms = start.elapsed_time(end) / steps
    kern_ms = sum(b.elapsed_time(e) for b, e in zip(evb, eve)) / steps
    state_bytes = 2 * cfg.B * cfg.H * cfg.dk * cfg.dv * 4
    return ms, kern_ms, state_bytes, launches, clk.summary()


def bench_backward(steps, dev):
    """gdn_prefill_backward on the pretraining shape (4 sequences x 4096 tokens,
    H = 16, d = 128) in fp32, gradients of every input; inputs (0.54 GB of fp32
    token rows plus d_out) are larger than L2."""
    cfg = replace(PRETRAIN, in_dtype=torch.float32)
    inp = make_prefill_inputs(cfg, dev)
    g = torch.Generator(device=dev)
    g.manual_seed(cfg.seed + 100)
    d_out = torch.randn((cfg.total_tokens, cfg.H, cfg.dv), generator=g, device=dev)

    def call():
        return gdn.prefill_backward(inp["q"], inp["k"], inp["v"], inp["conv_w"], inp["a_logit"], inp["b_logit"],
                                    inp["A"], inp["b_alpha"], inp["z"], inp["norm_w"], d_out, S0=inp.get("S0"),
                                    num_seqs=cfg.num_seqs)

    for _ in range(3):
        call()
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    launches = 0
    s.record()
    for _ in range(steps):
        call()
        launches += gdn.last_call_launches()
    e.record()
    torch.cuda.synchronize()
    ms = s.elapsed_time(e) / steps
    del inp, d_out
    torch.cuda.empty_cache()
    return cfg, ms, launches


def bench_qsa(steps, dev):
    """gdn_qsa_indexer on one 32,768-token sequence (K = 2048, r = 4, 4 heads of
    128): the whole call, with the inputs resident; the score matrix (0.54 GB)
    is larger than L2."""
    cfg = QSA
    inp = make_qsa_inputs(cfg, dev)
    sel = torch.empty((cfg.B, cfg.n, cfg.budget // 4), dtype=torch.int32, device=dev)

    def call():
        gdn.qsa_indexer(inp["q"], inp["k"], inp["w_q"], inp["w_k"], budget=cfg.budget, sel=sel)

    for _ in range(3):
        call()
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    launches = 0
    s.record()
    for _ in range(steps):
        call()
        launches += gdn.last_call_launches()
    e.record()
    torch.cuda.synchronize()
    ms = s.elapsed_time(e) / steps
    n, nb = cfg.n, cfg.n // 4
    pairs = sum((i + 1) // 4 for i in range(n))           # (query, complete block) pairs
    flop = pairs * 4 * 128 * 2
    hbm = (n * 4 * 128 * 2 + n * 128 * 2                     # q, k read (bf16)
           + 2 * pairs * 4                                   # scores written, read back
           + n * (cfg.budget // 4) * 4)                      # selection written
    del inp, sel
    torch.cuda.empty_cache()
    return cfg, ms, launches, flop, hbm


def bench_layer(steps, dev, d_model=2048):
    """gdn_layer_forward on the pretraining shape (4 x 4096 tokens, H = 16, d = 128)
    with d_model = 2048: in-projection GEMMs, the mixer, W_o; bf16."""
    cfg = PRETRAIN
    inp = make_layer_inputs(cfg, d_model, dev)
    y = torch.empty((cfg.total_tokens, d_model), dtype=torch.bfloat16, device=dev)

    def call():
        gdn.layer_forward(inp["x"], inp["w_in"], inp["conv_w"], inp["A"], inp["b_alpha"], inp["norm_w"],
                          inp["w_o"], cfg.H, cfg.dk, cfg.dv, S0=inp["S0"], num_seqs=cfg.num_seqs, y=y)

    for _ in range(3):
        call()
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    launches = 0
    s.record()
    for _ in range(steps):
        call()
        launches += gdn.last_call_launches()
    e.record()
    torch.cuda.synchronize()
    ms = s.elapsed_time(e) / steps
    c_in = cfg.H * (2 * cfg.dk + 2 * cfg.dv) + 2 * cfg.H
    gemm_flop = 2 * cfg.total_tokens * d_model * (c_in + cfg.H * cfg.dv)
    mixer_flop = PREFILL_FLOP_PER_TOKEN_HEAD * cfg.total_tokens * cfg.H
    del inp, y
    torch.cuda.empty_cache()
    return cfg, d_model, ms, launches, gemm_flop, mixer_flop


def bench_decode_multi(cfg, T, steps, dev):
    """T consecutive tokens per sequence per step (gdn_decode_multi, all committed):
    the pool's entries [0, T) and [T, 2T) as two alternating multi-token inputs."""
    d = make_decode_inputs(cfg, dev)
    S, hist = d["S"], d["ring"]
    sets = [{key: d[key][o:o + T].transpose(0, 1).contiguous()
             for key in ("q", "k", "v", "z", "a_logit", "b_logit")} for o in (0, T)]
    out = torch.empty((cfg.B, T, cfg.H, cfg.dv), dtype=torch.bfloat16, device=dev)

    def step(t):
        m = sets[t % 2]
        gdn.decode_multi(m["q"], m["k"], m["v"], d["conv_w"], hist, m["a_logit"], m["b_logit"], d["A"],
                         d["b_alpha"], m["z"], d["norm_w"], S, out=out)

    for t in range(5):
        step(t)
    torch.cuda.synchronize()
    evb = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    eve = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    for e in evb + eve:
        e.record()
    torch.cuda.synchronize()
    launches = 0
    for t in range(steps):
        gdn.set_timing_events(evb[t], eve[t])
        step(t)
        launches += gdn.last_call_launches()
    gdn.set_timing_events(None, None)
    torch.cuda.synchronize()
    kern_ms = sum(b.elapsed_time(e) for b, e in zip(evb, eve)) / steps
    return kern_ms, launches


def oracle_sample_rate(inp, cfg, tokens, heads, n_threads):
    """Oracle (fp64, token by token) on `heads` chains of the first `tokens`
    tokens; returns (token-heads per second, seconds, threads used)."""
    import oracle
    idx = torch.arange(heads)
    dk, dv, H = cfg.dk, cfg.dv, cfg.H
    take = lambda k: to_oracle_bits(inp[k][:tokens].index_select(1, idx.to(inp[k].device)))
    rows = torch.cat([torch.arange(h * dk, (h + 1) * dk) for h in range(heads)] +
                     [H * dk + torch.arange(h * dk, (h + 1) * dk) for h in range(heads)] +
                     [2 * H * dk + torch.arange(h * dv, (h + 1) * dv) for h in range(heads)])
    cw = to_oracle_bits(inp["conv_w"].index_select(0, rows.to(inp["conv_w"].device)))
    S0 = None if inp["S0"] is None else to_oracle_bits(inp["S0"][:1].index_select(1, idx.to(inp["S0"].device)))
    args = (take("q"), take("k"), take("v"), cw, take("a_logit"), take("b_logit"),
            to_oracle_bits(inp["A"][:heads]), to_oracle_bits(inp["b_alpha"][:heads]), take("z"),
            to_oracle_bits(inp["norm_w"]))
    t0 = time.perf_counter()
    oracle.prefill(*args, S0=S0, n_threads=n_threads)
    dt = time.perf_counter() - t0
    return tokens * heads / dt, dt, oracle.threads(n_threads)


def run_reference(args, world, rank):
    """The fp64 CPU oracle on the host cores: each step a bounded sample (one
    head chain per core over 4096 tokens) of the long-prefill workload."""
    if rank != 0:
        return
    cfg = LONG
    inp = make_prefill_inputs(replace(cfg, lengths=(4096,)), "cpu")
    cores = os.cpu_count() or 1
    heads = min(cfg.H, cores)
    for _ in range(args.warmup):
        oracle_sample_rate(inp, cfg, 4096, heads, heads)
    total_th, total_s = 0.0, 0.0
    for _ in range(args.steps):
        rate, dt, thr = oracle_sample_rate(inp, cfg, 4096, heads, heads)
        total_th += 4096 * heads
        total_s += dt
    value = total_th / total_s / cfg.H
    sample = f"{heads} head chains x 4096 tokens per step of the T=32768 H=32 workload; tokens/s scaled to all 32 heads"
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total_s / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": cfg.name, "seq_len": 32768, "H": 32},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": thr, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}))


def profile_case(kind, size):
    """Small workloads for ncu captures (a few hundred MB on the device, inputs
    larger than L2), run through the public binding on cuda:0:
      prefill T   the long-prefill shape with T tokens (H = 32, d = 128, S0):
                  two warm-up calls, then one call
      pretrain T  the pretraining shape with 4 sequences of T tokens (H = 16):
                  two warm-up calls, then one call
      segmented T 4 sequences of T tokens with H = 40 (160 (sequence, head)
                  items, more than the SMs: the segmented prep + chain
                  pipeline): two warm-up calls, then one call
      decode B    decode steps for B sequences x 32 heads, d = 128: three steps
      decode4 B   multi-token decode steps (4 tokens per sequence, all committed)
                  for B sequences x 32 heads, d = 128: three steps
      backward T  prefill backward, 4 sequences x T tokens, H = 16, d = 128, fp32: three calls
      qsa n       QSA indexer on one sequence of n tokens, K = 2048: three calls
      layer T     layer forward, 4 sequences x T tokens, H = 16, d_model = 2048: three calls"""
    dev = torch.device("cuda", 0)
    if kind in ("prefill", "pretrain", "segmented"):
        cfg = (replace(LONG, lengths=(size,)) if kind == "prefill" else
               replace(PRETRAIN, lengths=(size,) * 4, H=40 if kind == "segmented" else PRETRAIN.H))
        inp = make_prefill_inputs(cfg, dev)
        out = torch.empty((cfg.total_tokens, cfg.H, cfg.dv), dtype=torch.bfloat16, device=dev)
        S = torch.empty((cfg.num_seqs, cfg.H, cfg.dk, cfg.dv), device=dev)
        for _ in range(3):
            prefill_call(inp, out, S)
        torch.cuda.synchronize()
        print("ok", float(out.float().abs().mean()))
    elif kind == "decode":
        cfg = replace(DECODE, B=size)
        d = make_decode_inputs(cfg, dev)
        out = torch.empty((cfg.B, cfg.H, cfg.dv), dtype=torch.bfloat16, device=dev)
        for t in range(3):
            gdn.decode_step(d["q"][t], d["k"][t], d["v"][t], d["conv_w"], d["ring"], d["a_logit"][t],
                            d["b_logit"][t], d["A"], d["b_alpha"], d["z"][t], d["norm_w"], d["S"], out=out)
        torch.cuda.synchronize()
        print("ok", float(out.float().abs().mean()))
    elif kind == "decode4":
        cfg = replace(DECODE, B=size)
        d = make_decode_inputs(cfg, dev)
        m = {key: d[key][:4].transpose(0, 1).contiguous() for key in ("q", "k", "v", "z", "a_logit", "b_logit")}
        out = torch.empty((cfg.B, 4, cfg.H, cfg.dv), dtype=torch.bfloat16, device=dev)
        for _ in range(3):
            gdn.decode_multi(m["q"], m["k"], m["v"], d["conv_w"], d["ring"], m["a_logit"], m["b_logit"], d["A"],
                             d["b_alpha"], m["z"], d["norm_w"], d["S"], out=out)
        torch.cuda.synchronize()
        print("ok", float(out.float().abs().mean()))
    elif kind == "backward":
        cfg = replace(PRETRAIN, lengths=(size,) * 4, in_dtype=torch.float32)
        inp = make_prefill_inputs(cfg, dev)
        g = torch.Generator(device=dev)
        g.manual_seed(cfg.seed + 100)
        d_out = torch.randn((cfg.total_tokens, cfg.H, cfg.dv), generator=g, device=dev)
        for _ in range(3):
            grads = gdn.prefill_backward(inp["q"], inp["k"], inp["v"], inp["conv_w"], inp["a_logit"],
                                         inp["b_logit"], inp["A"], inp["b_alpha"], inp["z"], inp["norm_w"],
                                         d_out, S0=inp.get("S0"), num_seqs=cfg.num_seqs)
        torch.cuda.synchronize()
        print("ok", float(grads["dq"].abs().mean()))
    elif kind == "layer":
        cfg = replace(PRETRAIN, lengths=(size,) * 4)
        inp = make_layer_inputs(cfg, 2048, dev)
        y = torch.empty((cfg.total_tokens, 2048), dtype=torch.bfloat16, device=dev)
        for _ in range(3):
            gdn.layer_forward(inp["x"], inp["w_in"], inp["conv_w"], inp["A"], inp["b_alpha"], inp["norm_w"],
                              inp["w_o"], cfg.H, cfg.dk, cfg.dv, S0=inp["S0"], num_seqs=cfg.num_seqs, y=y)
        torch.cuda.synchronize()
        print("ok", float(y.float().abs().mean()))
    elif kind == "qsa":
        cfg = replace(QSA, n=size)
        inp = make_qsa_inputs(cfg, dev)
        for _ in range(3):
            sel, _ = gdn.qsa_indexer(inp["q"], inp["k"], inp["w_q"], inp["w_k"], budget=cfg.budget)
        torch.cuda.synchronize()
        print("ok", int(sel[-1, -1, 0]))
    else:
        raise SystemExit(f"unknown profile case {kind!r}")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--decode-steps", type=int, default=1000)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--profile-case", nargs=2, metavar=("KIND", "SIZE"),
                    help="run one small workload for an ncu capture instead of the benchmark "
                         "(prefill T | pretrain T | segmented T | decode B | decode4 B | backward T | qsa n | layer T)")
    args = ap.parse_args()
    if args.profile_case:
        profile_case(args.profile_case[0], int(args.profile_case[1]))
        return
    if args.warmup < 3:
        ap.error("at least 3 warm-up steps")
    if args.gpus < 1:
        ap.error("--gpus must be at least 1")
    if "WORLD_SIZE" not in os.environ and args.gpus > 1:
        # not under a launcher: start one process per GPU (each re-enters here
        # with its rank in the environment) and pass on their exit status
        sys.exit(rankio.launch(args.gpus, os.path.abspath(__file__), sys.argv[1:]))
    if "WORLD_SIZE" in os.environ and rankio.env_ranks()[0] != args.gpus:
        print(f"bench.py: --gpus {args.gpus}, but the launcher started {rankio.env_ranks()[0]} ranks; "
              "timing the launcher's ranks", file=sys.stderr)

    world, rank, local = rankio.setup("nccl") if args.impl == "ours" else rankio.env_ranks()
    if args.impl == "reference":
        run_reference(args, world, rank)
        return
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    pk, pk_kind = peaks()

    cfg = LONG
    ms, kern_ms, clocks, kernels, launches, inp = bench_prefill(cfg, args.steps, args.warmup, world,
                                                                rank, dev)
    token_heads = cfg.total_tokens * cfg.H
    value = rankio.job_throughput(world, cfg.total_tokens, ms)
    path_gbs = PREFILL_BYTES_PER_TOKEN_HEAD * token_heads / (kern_ms * 1e-3) / 1e9
    tc_achieved = PREFILL_FLOP_PER_TOKEN_HEAD * token_heads / (kern_ms * 1e-3) / 1e12
    dom = max(kernels, key=lambda n: kernels[n]["ms_per_step"])
    kd = kernels[dom]
    units_per_launch = token_heads / kd["launches_per_step"]
    bound, per_unit = KERNEL_ROOFLINE[dom]
    rate = per_unit * units_per_launch / (kd["avg_launch_ms"] * 1e-3)
    if bound == "hbm":
        dom_ach, dom_peak, dom_unit = rate / 1e9, pk["hbm_gbs"], "GB/s"
    else:
        dom_ach, dom_peak, dom_unit = rate / 1e12, pk["bf16_tflops"], "TFLOP/s"
    traffic = kernel_traffic(dom, units_per_launch)
    for name, rec in kernels.items():   # every kernel against its own bound, for context
        b_, u_ = KERNEL_ROOFLINE[name]
        r_ = u_ * (token_heads / rec["launches_per_step"]) / (rec["avg_launch_ms"] * 1e-3)
        rec["bound"] = b_
        rec["frac"] = r_ / 1e9 / pk["hbm_gbs"] if b_ == "hbm" else r_ / 1e12 / pk["bf16_tflops"]

    result = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": "long prefill: 1 seq x T=32768, H=32, dk=dv=128, bf16 in/out, "
                               "fp32 state, S0~N(0,0.02), per GPU",
                   "global_batch": world, "seq_len": cfg.total_tokens, "parallelism": f"dp{world}",
                   "process_group_size": rankio.group_size(),
                   "l2": "inputs larger than L2 (1.07 GB of bf16 q,k,v,z read per step)"},
        "roofline": {"bound": bound, "achieved": dom_ach, "peak": dom_peak, "unit": dom_unit,
                     "frac": dom_ach / dom_peak, "traffic": traffic, "kernel": dom,
                     ("bytes_per_token_head" if bound == "hbm" else "flop_per_token_head"): per_unit,
                     "token_heads_per_launch": units_per_launch,
                     "avg_launch_ms": kd["avg_launch_ms"], "peak_kind": pk_kind,
                     "kernels": kernels,
                     "path": {"what": "whole gdn_prefill call (every kernel it launches)",
                              "call_ms": kern_ms, "bytes_per_token_head": PREFILL_BYTES_PER_TOKEN_HEAD,
                              "achieved_gbs": path_gbs, "frac": path_gbs / pk["hbm_gbs"]}},
        "tc": {"achieved_tflops": tc_achieved, "peak_tflops": pk["bf16_tflops"],
               "frac": tc_achieved / pk["bf16_tflops"], "peak_kind": pk_kind + " burst",
               "flop_per_token_head": PREFILL_FLOP_PER_TOKEN_HEAD, "over": "whole gdn_prefill call"},
        "gpu_launches": launches,
        "clocks": clocks,
    }
    del inp
    torch.cuda.empty_cache()

    if rank == 0:
        # the other prefill workloads (several sequences: the segmented pipeline of
        # chunk_prep / chunk_chain launches), timed on this rank alone
        for key, pcfg in (("pretrain", PRETRAIN), ("varlen", VARLEN)):
            p_ms, p_kern, _, p_kernels, p_launch, p_inp = bench_prefill(pcfg, 5, 3, 1, 0, dev)
            result[key] = prefill_summary(pcfg, 5, p_ms, p_kern, p_kernels, pk)
            result[key]["gpu_launches"] = p_launch
            del p_inp
            torch.cuda.empty_cache()

    if rank == 0 and args.decode_steps > 0:
        dms, dk_ms, sbytes, dlaunch, dclk = bench_decode(DECODE, args.decode_steps, dev)
        gbs = sbytes / (dk_ms * 1e-3) / 1e9
        result["decode"] = {"workload": DECODE.name, "steps": args.decode_steps,
                            "ms_per_step": dms, "kernel_ms": dk_ms,
                            "state_gbs": gbs, "peak_gbs": pk["hbm_gbs"],
                            "frac": gbs / pk["hbm_gbs"], "state_bytes_per_step": sbytes,
                            "kernel": "decode_stream", "gpu_launches": dlaunch, "clocks": dclk}
        torch.cuda.empty_cache()
        qcfg, q_ms, qlaunch, q_flop, q_hbm = bench_qsa(5, dev)
        result["qsa_indexer"] = {
            "workload": qcfg.name, "steps": 5, "ms_per_step": q_ms,
            "queries_per_s": qcfg.n / (q_ms * 1e-3),
            "bound": "hbm", "bytes_per_call": q_hbm, "achieved_gbs": q_hbm / (q_ms * 1e-3) / 1e9,
            "peak_gbs": pk["hbm_gbs"], "frac": q_hbm / (q_ms * 1e-3) / 1e9 / pk["hbm_gbs"],
            "tc": {"flop_per_call": q_flop, "achieved_tflops": q_flop / (q_ms * 1e-3) / 1e12,
                   "peak_tflops": pk["bf16_tflops"], "frac": q_flop / (q_ms * 1e-3) / 1e12 / pk["bf16_tflops"]},
            "kernels": "qsa_prep, qsa_score (tcgen05), qsa_topk", "gpu_launches": qlaunch}
        lcfg, l_dm, l_ms, llaunch, l_gemm, l_mix = bench_layer(5, dev)
        l_tf = (l_gemm + l_mix) / (l_ms * 1e-3) / 1e12
        result["layer"] = {
            "workload": f"layer forward, B=4 x T=4096, H=16, d=128, d_model={l_dm}, bf16 "
                        "(in-projection GEMMs and W_o on the library's tcgen05 GEMM, the mixer)",
            "steps": 5, "ms_per_step": l_ms, "tokens_per_s": lcfg.total_tokens / (l_ms * 1e-3),
            "bound": "tensor", "flop_per_call": l_gemm + l_mix, "achieved_tflops": l_tf,
            "peak_tflops": pk["bf16_tflops"], "frac": l_tf / pk["bf16_tflops"],
            "gemm_flop_share": l_gemm / (l_gemm + l_mix), "gpu_launches": llaunch}
        bcfg, b_ms, blaunch = bench_backward(5, dev)
        th = bcfg.total_tokens * bcfg.H
        b_tf = BACKWARD_FLOP_PER_TOKEN_HEAD * th / (b_ms * 1e-3) / 1e12
        b_gbs = BACKWARD_BYTES_PER_TOKEN_HEAD * th / (b_ms * 1e-3) / 1e9
        result["backward"] = {"workload": "prefill backward, pretraining shape B=4 x T=4096, H=16, d=128, fp32, "
                                          "gradients of every input",
                              "steps": 5, "ms_per_step": b_ms, "tokens_per_s": bcfg.total_tokens / (b_ms * 1e-3),
                              "bound": "alu", "achieved_tflops": b_tf, "peak_tflops": FP32_SIMT_TFLOPS,
                              "peak_kind": "derived: 148 SMs x 128 fp32 lanes x 2 x 1.965 GHz",
                              "frac": b_tf / FP32_SIMT_TFLOPS, "flop_per_token_head": BACKWARD_FLOP_PER_TOKEN_HEAD,
                              "hbm": {"bytes_per_token_head": BACKWARD_BYTES_PER_TOKEN_HEAD, "achieved_gbs": b_gbs,
                                      "frac": b_gbs / pk["hbm_gbs"]},
                              "kernel": "bwd_rec_kernel (dominant)", "gpu_launches": blaunch}
        T = 4
        mk_ms, mlaunch = bench_decode_multi(DECODE, T, max(50, args.decode_steps // 4), dev)
        mgbs = sbytes / (mk_ms * 1e-3) / 1e9
        result["decode_multi"] = {"workload": f"multi-token decode B={DECODE.B} H={DECODE.H} d=128, "
                                              f"T={T} tokens per sequence per step, all committed",
                                  "kernel_ms": mk_ms, "tokens_per_s": DECODE.B * T / (mk_ms * 1e-3),
                                  "single_token_steps_ms": T * dk_ms,
                                  "state_gbs": mgbs, "peak_gbs": pk["hbm_gbs"], "frac": mgbs / pk["hbm_gbs"],
                                  "kernel": "decode_stream (T <= 4)", "gpu_launches": mlaunch}
        torch.cuda.empty_cache()

    if not args.no_e2e:
        e_ms, h2d, d2h = bench_e2e(cfg, max(4, args.steps // 2), args.warmup, world, rank, dev)
        result["e2e"] = {"value": rankio.job_throughput(world, cfg.total_tokens, e_ms), "unit": "tokens/s",
                         "ms_per_step": e_ms, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                         "pipeline": "two device buffer sets; host->device copies, gdn_prefill and "
                                     "device->host reads on three streams, overlapping across steps"}
        torch.cuda.empty_cache()

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cores = os.cpu_count() or 1
        inp = make_prefill_inputs(cfg, "cpu")
        rate, dt, thr = oracle_sample_rate(inp, cfg, cfg.total_tokens, cfg.H, cores)
        result["cpu_baseline"] = {"value": rate / cfg.H, "unit": "tokens/s", "cores": thr,
                                  "kind": "oracle", "seconds": dt,
                                  "sample": "the whole T=32768 H=32 workload once (all 32 head "
                                            "chains, one OpenMP thread per chain)"}
    if rank == 0:
        print(json.dumps(result))
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
