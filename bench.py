"""Benchmark of the B200 attention library (one JSON line on stdout).

python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]

A step is one call of the hot path on one batch of seeded synthetic input
that is already resident in HBM:
  video      (default) O, LSE = attn_fwd(Q, K, V), B=1 H=40 S=32760 D=128 bf16,
             Q/K RMS-normalised per head -- the video-DiT self-attention;
  fp8        attn_fwd on e4m3 inputs with per-head descales, B=1 H=5 S=75600;
  llm_gqa    attn_fwd + attn_bwd_dsbuf (the backward that stores dS in an
             O(Sq x Sk) workspace), B=2 Hq=32 Hkv=8 S=2048 causal; the same
             step with the O(S)-memory attn_bwd and with attn_bwd_onepass
             are sub-results;
  streaming  attn_fwd_kvblocks over 21 blocks of 1560 keys + attn_fwd to 512
             text keys, B=1 H=40 Sq=1560;
  cross      attn_fwd, B=1 H=40 Sq=90000 Sk=512 (long-query cross-attention);
  window     attn_fwd, B=1 H=12 Sq=4680 Sk=51480 (window / sink KV).
The other workloads are measured too (``sub``) unless --no-sub, plus the e4m3
prologue (quantize_e4m3 of the fp8 config's Q, K, V; HBM-bound, in GB/s).

Timing: W untimed warm-up steps; then K steps, each preceded (outside its
CUDA events) by a 256 MB write that flushes L2, bracketed by a barrier and a
device synchronise on both sides; the step time is the sum of the per-step
event times on the launching stream, max over ranks.  Multi-GPU runs are
weak-scaled replicas: every rank runs the whole workload on its own GPU
(attention heads are independent; there is no collective on the data path).

``--impl reference`` times the CPU fp64 oracle (the only reference there is)
on a bounded sample of the same workload, on the host's cores.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import workloads  # noqa: E402
from workloads import make_bwd_inputs, make_fwd_inputs, make_kvblock_inputs, sample_rows  # noqa: E402

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 256 << 20
WORKLOAD_NAMES = {"tiny": "tiny self-attention fwd (B1 H2 S256 D128 bf16)",
                  "video": "video-DiT self-attention fwd (B1 H40 S32760 D128 bf16, Q/K RMS-norm)",
                  "fp8": "fp8 e4m3 attention fwd (B1 H5 S75600 D128, per-head descales)",
                  "llm_gqa": "LLM GQA causal fwd+bwd (B2 Hq32 Hkv8 S2048 D128 bf16; backward with stored dS, "
                             "attn_bwd_dsbuf, 537 MB workspace)",
                  "llm_gqa_attn_bwd": "LLM GQA causal fwd+bwd (B2 Hq32 Hkv8 S2048 D128 bf16; backward attn_bwd, "
                                      "O(S) workspace)",
                  "streaming": "streaming block-KV fwd (B1 H40 Sq1560, 21x1560 KV blocks + 512 text keys)",
                  "cross": "long-query cross-attention fwd (B1 H40 Sq90000 Sk512 D128 bf16)",
                  "window": "window/sink KV fwd (B1 H12 Sq4680 Sk51480 D128 bf16)",
                  "bf16_75600": "bf16 attention fwd at the fp8 shape (B1 H5 S75600 D128)",
                  "fp8_32760": "fp8 e4m3 attention fwd at the video shape (B1 H40 S32760 D128, Q/K RMS-norm)",
                  "fp8_prep": "e4m3 prologue of the fp8 config (Q, K RMS-normalised; V plain; per-head descales)",
                  "llm_gqa_onepass": "LLM GQA causal fwd + one-pass bwd (B2 Hq32 Hkv8 S2048 D128 bf16)",
                  "fp8_noscratch": "fp8 e4m3 attention fwd without scratch, V widened in shared memory "
                                   "(B1 H5 S75600 D128)",
                  "fp8_streaming": "streaming block-KV fwd over an FP8 e4m3 KV cache (B1 H40 Sq1560, 21x1560 blocks "
                                   "with per-block descales, + 512 e4m3 text keys)"}
FWD_WORKLOADS = ("video", "fp8", "tiny", "cross", "window", "bf16_75600", "fp8_32760")
SUB_ONLY = ("fp8_prep", "fp8_noscratch", "fp8_streaming", "llm_gqa_onepass", "llm_gqa_attn_bwd")   # sub-results only
KERNEL_SOURCES = ["head_attention_qk_b200/csrc/fwd_kernel.cuh", "head_attention_qk_b200/csrc/sm100.cuh"]


# ----------------------------------------------------------------------------- helpers

def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS if k in d}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_sha1():
    h = hashlib.sha1()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def recorded_traffic(workload):
    """DRAM bytes per launch of the dominant kernel from a committed ncu summary,
    or None if the kernel source changed since the counters were taken."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(workload)
    if not e or e.get("kernel_source_sha1") != kernel_source_sha1():
        return None
    return e.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples every 100 ms while running."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.Q,
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if not self.path or not os.path.exists(self.path):
            return None
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    rows.append((float(parts[1]), float(parts[2]), float(parts[3]), parts[5:9]))
                except ValueError:
                    continue
        os.unlink(self.path)
        if not rows:
            return None
        load = [r for r in rows if r[2] > 300.0] or rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in load for i, v in enumerate(r[3]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in load), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows), "samples_under_load": len(load),
                "power_w_max": max(r[2] for r in rows)}


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    return world, rank, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(x, world):
    """Maximum of a host scalar over all ranks (NCCL on GPUs, gloo on CPU)."""
    if world == 1:
        return x
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def whole_job_tflops(flops_per_step, steps, seconds_this_rank, world):
    """Weak scaling: every rank runs `steps` steps of its own units; the job's
    throughput is all ranks' FLOPs over the slowest rank's time."""
    slowest = max_over_ranks(seconds_this_rank, world)
    return world * flops_per_step * steps / slowest / 1e12, slowest


# ----------------------------------------------------------------------------- workloads

class Step:
    """One workload: device inputs, a step function and its FLOP count."""

    def __init__(self, name, h, heads=None, rank=0):
        self.name = name
        self.h = h
        base = {"fp8_prep": "fp8", "fp8_noscratch": "fp8", "fp8_streaming": "streaming",
                "llm_gqa_onepass": "llm_gqa", "llm_gqa_attn_bwd": "llm_gqa"}.get(name, name)
        self.w = workloads.get(base)
        if heads:
            self.w = workloads.get(base, Hq=heads, Hkv=max(1, heads * self.w.Hkv // self.w.Hq))
        if rank:
            # weak scaling: each rank attends over its own units (its own seeded draws)
            self.w = workloads.get(base, seed=self.w.seed + 7919 * rank, Hq=self.w.Hq, Hkv=self.w.Hkv)
        w = self.w
        self.launches = 1
        if name in FWD_WORKLOADS:
            x = make_fwd_inputs(w)
            self.host = x
            self.x = {k: v.cuda() for k, v in x.items()}
            self.out = torch.empty((w.B, w.Hq, w.Sq, w.D), dtype=torch.bfloat16, device="cuda")
            self.lse = torch.empty((w.B, w.Hq, w.Sq), dtype=torch.float32, device="cuda")
            self.flops = w.fwd_flops()
            self.dtype = w.dtype
            if w.dtype == "e4m3":
                self.launches = 2          # V widened to fp16, then the attention kernel
        elif name in ("llm_gqa", "llm_gqa_onepass", "llm_gqa_attn_bwd"):
            x = make_bwd_inputs(w)
            self.host = x
            self.x = {k: v.cuda() for k, v in x.items()}
            self.out = torch.empty_like(self.x["q"])
            self.lse = torch.empty((w.B, w.Hq, w.Sq), dtype=torch.float32, device="cuda")
            self.dq = torch.empty_like(self.x["q"])
            self.dk = torch.empty_like(self.x["k"])
            self.dv = torch.empty_like(self.x["v"])
            wsb = {"llm_gqa": h.bwd_dsbuf_workspace_size(w.B, w.Hq, w.Sq, w.Sk),
                   "llm_gqa_onepass": h.bwd_onepass_workspace_size(w.B, w.Hq, w.Sq),
                   "llm_gqa_attn_bwd": h.bwd_workspace_size(w.B, w.Hq, w.Sq)}[name]
            self.ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
            self.flops = w.fwd_flops() + w.bwd_flops()
            # fwd; then Delta + dK/dV + dQ product, Delta + dK/dV + dQ, or Delta + one pass
            self.launches = 3 if name == "llm_gqa_onepass" else 4
            self.dtype = "bf16"
        elif name == "fp8_prep":
            # the step before the fp8 forward: bf16 Q, K, V of the fp8 shape -> e4m3 + descales
            g = torch.Generator().manual_seed(w.seed)
            self.src = [torch.randn(w.B, H, S, w.D, generator=g).to(torch.bfloat16).cuda()
                        for H, S in ((w.Hq, w.Sq), (w.Hkv, w.Sk), (w.Hkv, w.Sk))]
            self.dst = [(torch.empty(t.shape, dtype=torch.float8_e4m3fn, device="cuda"),
                         torch.empty(t.shape[:2], dtype=torch.float32, device="cuda")) for t in self.src]
            self.flops = 0.0
            self.bytes = sum(5.0 * t.numel() for t in self.src)   # x read twice, codes written once
            self.launches = 6                                       # 3 x 2 kernels (and a memset each)
            self.dtype = "e4m3"
        elif name == "fp8_noscratch":
            x = make_fwd_inputs(w)
            self.host = x
            self.x = {k: v.cuda() for k, v in x.items()}
            self.out = torch.empty((w.B, w.Hq, w.Sq, w.D), dtype=torch.bfloat16, device="cuda")
            self.lse = torch.empty((w.B, w.Hq, w.Sq), dtype=torch.float32, device="cuda")
            self.flops = w.fwd_flops()
            self.dtype = "e4m3"
        elif name == "fp8_streaming":
            # an FP8 KV cache: every block (and the text keys) quantised with its
            # own per-head descales by the product prologue, outside the timed step
            x = make_kvblock_inputs(w)
            self.q, self.qd = h.quantize_e4m3(x["q"].cuda(), rmsnorm=True)
            n = len(x["blocks"])
            self.kds = torch.empty(n, w.B, w.Hkv, dtype=torch.float32, device="cuda")
            self.vds = torch.empty_like(self.kds)
            self.kb, self.vb = [], []
            for i, (kb, vb) in enumerate(x["blocks"]):
                self.kb.append(h.quantize_e4m3(kb.cuda(), rmsnorm=True, descale=self.kds[i])[0])
                self.vb.append(h.quantize_e4m3(vb.cuda(), descale=self.vds[i])[0])
            self.tk, self.tkd = h.quantize_e4m3(x["text"][0].cuda(), rmsnorm=True)
            self.tv, self.tvd = h.quantize_e4m3(x["text"][1].cuda())
            self.out = torch.empty((w.B, w.Hq, w.Sq, w.D), dtype=torch.bfloat16, device="cuda")
            self.lse = torch.empty((w.B, w.Hq, w.Sq), dtype=torch.float32, device="cuda")
            self.out_t = torch.empty_like(self.out)
            self.lse_t = torch.empty_like(self.lse)
            self.ws = torch.empty(h.fwd_workspace_size(w.B, w.Hkv, w.text_len, w.D, h.E4M3), dtype=torch.uint8,
                                  device="cuda")
            self.flops = 4.0 * w.B * w.Hq * w.Sq * w.D * (w.Sk + w.text_len)
            self.launches = 3                       # the block-KV kernel; text keys: V widening + attention
            self.dtype = "e4m3"
        elif name == "streaming":
            x = make_kvblock_inputs(w)
            self.host = x
            self.q = x["q"].cuda()
            self.kb = [k.cuda() for k, _ in x["blocks"]]
            self.vb = [v.cuda() for _, v in x["blocks"]]
            self.tk, self.tv = (t.cuda() for t in x["text"])
            self.out = torch.empty((w.B, w.Hq, w.Sq, w.D), dtype=torch.bfloat16, device="cuda")
            self.lse = torch.empty((w.B, w.Hq, w.Sq), dtype=torch.float32, device="cuda")
            self.out_t = torch.empty_like(self.out)
            self.lse_t = torch.empty_like(self.lse)
            self.ws = torch.empty(h.kvblocks_workspace_size(w.B, w.Hq, w.Sq, w.D, w.n_blocks), dtype=torch.uint8,
                                  device="cuda")
            self.flops = 4.0 * w.B * w.Hq * w.Sq * w.D * (w.Sk + w.text_len)
            self.launches = 3
            self.dtype = "bf16"
        else:
            raise ValueError(name)

    def __call__(self):
        h, w = self.h, self.w
        if self.name in FWD_WORKLOADS:
            x = self.x
            ds = {}
            if w.dtype == "e4m3":
                ds = dict(q_descale=x["q_descale"], k_descale=x["k_descale"], v_descale=x["v_descale"])
            h.attn_fwd(x["q"], x["k"], x["v"], out=self.out, lse=self.lse, **ds)
        elif self.name == "fp8_noscratch":
            x = self.x
            h.attn_fwd(x["q"], x["k"], x["v"], out=self.out, lse=self.lse, q_descale=x["q_descale"],
                       k_descale=x["k_descale"], v_descale=x["v_descale"], use_scratch=False)
        elif self.name == "fp8_streaming":
            h.attn_fwd_kvblocks(self.q, self.kb, self.vb, out=self.out, lse=self.lse, q_descale=self.qd,
                                k_descale=self.kds, v_descale=self.vds)
            h.attn_fwd(self.q, self.tk, self.tv, out=self.out_t, lse=self.lse_t, q_descale=self.qd,
                       k_descale=self.tkd, v_descale=self.tvd, workspace=self.ws)
        elif self.name == "fp8_prep":
            for i, (t, (c, d)) in enumerate(zip(self.src, self.dst)):
                h.quantize_e4m3(t, rmsnorm=i < 2, codes=c, descale=d)
        elif self.name in ("llm_gqa", "llm_gqa_onepass", "llm_gqa_attn_bwd"):
            x = self.x
            h.attn_fwd(x["q"], x["k"], x["v"], causal=True, out=self.out, lse=self.lse)
            bwd = {"llm_gqa": h.attn_bwd_dsbuf, "llm_gqa_onepass": h.attn_bwd_onepass,
                   "llm_gqa_attn_bwd": h.attn_bwd}[self.name]
            bwd(x["q"], x["k"], x["v"], self.out, self.lse, x["dout"], causal=True, workspace=self.ws,
                dq=self.dq, dk=self.dk, dv=self.dv)
        else:
            h.attn_fwd_kvblocks(self.q, self.kb, self.vb, workspace=self.ws, out=self.out, lse=self.lse)
            h.attn_fwd(self.q, self.tk, self.tv, out=self.out_t, lse=self.lse_t)


def time_steps(step, K, W, world, flush, sampler_index=None):
    for _ in range(W):
        step()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    sampler = ClockSampler(sampler_index) if sampler_index is not None else None
    if sampler:
        sampler.__enter__()
    barrier(world)
    torch.cuda.synchronize()
    for i in range(K):
        flush.zero_()
        evs[i][0].record(stream)
        step()
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    barrier(world)
    if sampler:
        sampler.__exit__()
    ms = [a.elapsed_time(b) for a, b in evs]
    return ms, (sampler.summary() if sampler else None)


def e2e_video_like(step, K, W):
    """Same metric through the public API with pinned HOST buffers: every step
    copies its inputs host -> device, calls attn_fwd and copies O and LSE back;
    all of it inside the timed region.  Steps are pipelined the way a server
    would run them: two buffer sets, the copy in of step k+1 and the copy out
    of step k-1 overlap the kernel of step k (separate streams, event-ordered)."""
    h = step.h
    names = ["q", "k", "v"] + (["q_descale", "k_descale", "v_descale"] if step.dtype == "e4m3" else [])
    host = {n: step.host[n].pin_memory() for n in names}
    sets = []
    for _ in range(2):
        sets.append({"in": {n: torch.empty_like(step.x[n]) for n in names},
                     "out": torch.empty_like(step.out), "lse": torch.empty_like(step.lse),
                     "out_h": torch.empty(step.out.shape, dtype=step.out.dtype).pin_memory(),
                     "lse_h": torch.empty(step.lse.shape, dtype=step.lse.dtype).pin_memory(),
                     "in_done": torch.cuda.Event(), "run_done": torch.cuda.Event(), "out_done": torch.cuda.Event()})
    s_in, s_run, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()

    def one(k):
        b = sets[k % 2]
        if k >= 2:
            s_in.wait_event(b["run_done"])          # step k-2 is done reading these inputs
        with torch.cuda.stream(s_in):
            for n in names:
                b["in"][n].copy_(host[n], non_blocking=True)
        b["in_done"].record(s_in)
        s_run.wait_event(b["in_done"])
        if k >= 2:
            s_run.wait_event(b["out_done"])         # step k-2's outputs have left the device
        ds = {}
        if step.dtype == "e4m3":
            ds = dict(q_descale=b["in"]["q_descale"], k_descale=b["in"]["k_descale"], v_descale=b["in"]["v_descale"])
        with torch.cuda.stream(s_run):
            h.attn_fwd(b["in"]["q"], b["in"]["k"], b["in"]["v"], out=b["out"], lse=b["lse"], stream=s_run, **ds)
        b["run_done"].record(s_run)
        s_out.wait_event(b["run_done"])
        with torch.cuda.stream(s_out):
            b["out_h"].copy_(b["out"], non_blocking=True)
            b["lse_h"].copy_(b["lse"], non_blocking=True)
        b["out_done"].record(s_out)

    for k in range(W):
        one(k)
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(s_in)
    for k in range(K):
        one(k)
    s_out.wait_event(sets[(K - 1) % 2]["out_done"])
    end.record(s_out)
    torch.cuda.synchronize()
    ms = start.elapsed_time(end) / K
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = sets[0]["out_h"].numel() * sets[0]["out_h"].element_size() + \
        sets[0]["lse_h"].numel() * sets[0]["lse_h"].element_size()
    return {"value": step.flops / (ms * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_step": ms,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "pipelining": "2 buffer sets; copy in of step k+1 and copy out of step k-1 overlap step k's kernel"}


# ----------------------------------------------------------------------------- oracle (CPU) timing

def oracle_sample_tflops(name, rows_per_head):
    """Time the CPU fp64 oracle on `rows_per_head` seeded query rows of every
    head of the workload; return (TFLOP/s of the sample, seconds, description)."""
    import oracle
    from workloads import bf16_bits, e4m3_bits

    w = workloads.get(name)
    if name == "streaming":
        x = make_kvblock_inputs(w)
        q = bf16_bits(x["q"])
        k = np.concatenate([bf16_bits(kb) for kb, _ in x["blocks"]], axis=2)
        v = np.concatenate([bf16_bits(vb) for _, vb in x["blocks"]], axis=2)
        ds = None
        Sk, causal = w.Sk, False
    else:
        x = make_fwd_inputs(w)
        conv = e4m3_bits if w.dtype == "e4m3" else bf16_bits
        q, k, v = (conv(x[n]) for n in ("q", "k", "v"))
        ds = None
        if w.dtype == "e4m3":
            ds = tuple(x[n].double().numpy().ravel() for n in ("q_descale", "k_descale", "v_descale"))
        Sk, causal = w.Sk, w.causal
    rows = sample_rows(w.Sq, rows_per_head, seed=w.seed)
    t0 = time.perf_counter()
    oracle.attn_fwd(q, k, v, w.scale, causal=causal, rows=rows, descales=ds)
    dt = time.perf_counter() - t0
    if causal:
        keys = sum(min(Sk, int(r) + Sk - w.Sq + 1) for r in rows)
    else:
        keys = len(rows) * Sk
    flops = 4.0 * w.B * w.Hq * keys * w.D
    desc = "%d seeded query rows per head x %d heads of the %s workload (fwd), fp64" % (len(rows), w.B * w.Hq, name)
    return flops / dt / 1e12, dt, desc, oracle.num_threads()


# ----------------------------------------------------------------------------- main

def run_reference(args, world, rank):
    if rank != 0:
        return 0
    name = args.workload
    w = workloads.get(name)
    rows = {"tiny": 256, "video": 16, "fp8": 32, "llm_gqa": 256, "streaming": 64, "cross": 256, "window": 48,
            "bf16_75600": 32, "fp8_32760": 16}[name]
    vals = []
    for _ in range(args.warmup):
        oracle_sample_tflops(name, rows)
    for _ in range(args.steps):
        v, dt, desc, cores = oracle_sample_tflops(name, rows)
        vals.append((v, dt))
    value = statistics.median(v for v, _ in vals)
    ms = statistics.median(dt for _, dt in vals) * 1e3
    line = {"metric": "attention fwd TFLOPS (bf16, FP8) and % of B200 dense tensor peak", "impl": "reference",
            "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOAD_NAMES[name], "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "Sq": w.Sq,
                       "Sk": w.Sk, "D": w.D, "causal": w.causal},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": desc},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))
    return 0


def sub_result(other, h, flush, steps, warmup, peaks, heads=None):
    """Time one workload on this GPU; its entry of the JSON line's ``sub``."""
    st = Step(other, h, heads=heads)
    oms, _ = time_steps(st, steps, warmup, 1, flush)
    if h.get_device_error() != 0:
        raise RuntimeError("a kernel reported a bounded-wait timeout")
    t = statistics.mean(oms)
    if other == "fp8_prep":
        gbs = st.bytes / (t * 1e-3) / 1e9
        r = {"workload": WORKLOAD_NAMES[other], "ms_per_step": t, "gbs": gbs,
             "frac_of_hbm": gbs / peaks["hbm_gbs"], "peak_gbs": peaks["hbm_gbs"],
             "bytes_per_step": st.bytes, "dtype": st.dtype, "launches_per_step": st.launches}
    else:
        pk = peaks["bf16_tflops"] * (2.0 if st.dtype == "e4m3" else 1.0)
        r = {"workload": WORKLOAD_NAMES[other], "ms_per_step": t, "tflops": st.flops / (t * 1e-3) / 1e12,
             "frac_of_peak": st.flops / (t * 1e-3) / 1e12 / pk, "peak_tflops": pk,
             "dtype": st.dtype, "launches_per_step": st.launches}
        traffic = recorded_traffic(other)
        if traffic is not None:
            # DRAM bytes per launch of the attention kernel (ncu, profiles/traffic.json)
            r["roofline"] = {"bound": "tensor", "traffic": traffic,
                             "algorithmic_flops_per_launch": st.flops}
    del st
    torch.cuda.empty_cache()
    return r


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=[n for n in WORKLOAD_NAMES if n not in SUB_ONLY], default="video")
    ap.add_argument("--no-sub", action="store_true", help="skip the other workloads")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--heads", type=int, default=0, help="smaller case: override the query head count")
    ap.add_argument("--only", choices=list(WORKLOAD_NAMES), default=None,
                    help="time just this workload (one GPU) and print its sub-result line; for profiling")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")

    world, rank, local = dist_setup() if args.impl == "ours" else (int(os.environ.get("WORLD_SIZE", "1")),
                                                                    int(os.environ.get("RANK", "0")), 0)
    if args.impl == "reference":
        return run_reference(args, world, rank)

    import head_attention_qk_b200 as h

    peaks, peak_src = load_peaks()
    torch.cuda.set_device(local)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device="cuda")
    if args.only:
        print(json.dumps({"only": args.only, **sub_result(args.only, h, flush, args.steps, args.warmup, peaks,
                                                           heads=args.heads or None)}))
        return 0
    name = args.workload
    step = Step(name, h, heads=args.heads or None, rank=rank)
    ms, clocks = time_steps(step, args.steps, args.warmup, world, flush,
                            sampler_index=local if rank == 0 else None)
    if h.get_device_error() != 0:
        raise RuntimeError("a kernel reported a bounded-wait timeout")
    value, total_s = whole_job_tflops(step.flops, args.steps, sum(ms) * 1e-3, world)
    ms_per_step = total_s * 1e3 / args.steps

    fp8 = step.dtype == "e4m3"
    peak_tensor = peaks["bf16_tflops"] * (2.0 if fp8 else 1.0)
    # the dominant kernel is the attention kernel; an e4m3 step also widens V
    # (an HBM-bound pass of about 0.5 % of the step), which this figure includes
    achieved = step.flops / (statistics.mean(ms) * 1e-3) / 1e12 if name in FWD_WORKLOADS else None
    w = step.w
    roofline = None
    if achieved is not None:
        traffic = recorded_traffic(name)
        roofline = {"bound": "tensor", "achieved": achieved, "peak": peak_tensor, "unit": "TFLOP/s",
                    "frac": achieved / peak_tensor, "traffic": traffic,
                    "kernel": "attn_fwd_kernel<%s>" % ("e4m3" if fp8 else "bf16"),
                    "peak_source": "%s (bf16 burst%s)" % (peak_src, " x2 nominal fp8:bf16 ratio" if fp8 else ""),
                    "algorithmic_flops_per_launch": step.flops}

    line = {"metric": "attention fwd TFLOPS (bf16, FP8) and % of B200 dense tensor peak",
            "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": step.dtype, "data": "synthetic (seeded N(0,1); no datasets or weights)",
            "config": {"workload": WORKLOAD_NAMES[name], "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "Sq": w.Sq,
                       "Sk": w.Sk, "D": w.D, "causal": w.causal, "qk_rmsnorm": w.qk_rmsnorm,
                       "parallelism": "replicas" if world > 1 else "single GPU",
                       "l2": "256 MB write before each timed step, outside its CUDA events"},
            "gpu_launches": step.launches * args.steps,
            "clocks": clocks, "roofline": roofline}
    if not args.no_e2e and name in FWD_WORKLOADS:
        e2e = e2e_video_like(step, max(2, args.steps // 2), 1)
        e2e["ms_per_step"] = max_over_ranks(e2e["ms_per_step"], world)
        e2e["value"] = world * step.flops / (e2e["ms_per_step"] * 1e-3) / 1e12
        line["e2e"] = e2e
    del step
    torch.cuda.empty_cache()

    if rank == 0 and world == 1 and not args.no_sub:
        sub = {}
        for other in WORKLOAD_NAMES:
            if other == name or other == "tiny":
                continue
            sub[other] = sub_result(other, h, flush, max(3, args.steps // 2), args.warmup, peaks)
        line["sub"] = sub

    if rank == 0 and world == 1 and not args.no_cpu:
        v, dt, desc, cores = oracle_sample_tflops(name, 256)
        line["cpu_baseline"] = {"value": v, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": desc,
                                "seconds": dt}

    if rank == 0:
        print(json.dumps(line))
    if world > 1:
        torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
