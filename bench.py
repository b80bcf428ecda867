#!/usr/bin/env python
"""Benchmark of the fused ShortConv K/V step (tokens/s and achieved HBM GB/s).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload long|single|varlen|decode|...] [--no-configs]

One step = one pass of the whole step (window assembly + causal conv, RMSNorm,
bf16 scatter into the paged cache, conv_state update) over one batch of
synthetic input, through the C ABI.  Default workload (the headline line):
the long-context chunked prefill -- one 1,048,576-token sequence, Hkv=8,
D=128, W=4, processed as 16 calls of 65,536 tokens with the conv_state
carried from call to call, paged cache (page 64, seeded page permutation).
A step of that workload is the whole sequence, i.e. 16 kernel launches.

Timing: W warm-up steps, then exactly K steps captured in one CUDA graph and
replayed once, bracketed by a barrier + synchronize on both sides and by CUDA
events on the replay stream; a sleep kernel queued in front of the start
event keeps the GPU busy while the host submits the graph, so the region
holds the launches only.  time / (K x launches per step) is the kernel's
average launch duration; max over ranks.  Inputs rotate over enough buffer
sets that each step's bytes exceed L2.

The `configs` key of the line times the other full-size workloads the same
way (8192-token single prefill, 32-sequence varlen batch, 1024-sequence
decode step, W=2 and W=8 65,536-token launches), each over enough launches
for a region of at least ~20 ms.

Under torchrun each rank runs its own independent batch (the step shards by
sequence with no exchange: weak scaling); rank 0 prints one JSON line.
`--impl reference` times the CPU oracle (test infrastructure) on the same
workload instead, on rank 0 only.
"""
import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from short_conv_kv_b200 import workloads as wl  # noqa: E402

L2_BYTES = 126 * 1024 * 1024
# A sleep kernel of about 2 ms at the B200's SM clock, queued ahead of each
# timed region (outside it) while the host submits the graph.
SLEEP_CYCLES = 4_000_000
PROFILE_DIR = os.path.join(ROOT, "profiles")
# Sources each kernel is built from (device code and its host-side launch
# geometry); a committed profile counts only while these are unchanged.
_CSRC = os.path.join(ROOT, "short_conv_kv_b200", "csrc")
KERNEL_SOURCES = {
    "prefill_tma_kernel": [os.path.join(_CSRC, f) for f in
                           ("common.cuh", "tma.cuh", "prefill_tma.cuh", "sconv_kv.cu")],
    "decode_tma_kernel": [os.path.join(_CSRC, f) for f in
                          ("common.cuh", "tma.cuh", "decode_tma.cuh", "sconv_kv.cu")],
}


# ------------------------------------------------------------------ helpers

def algorithmic_bytes(tokens, seqs, W, Hkv, D, slot_bytes=8, mx=False, ring=False):
    """Bytes the step must move: per token K+V rows in and K+V cache rows out
    (bf16, or with the MXFP8 store one E4M3 byte per channel plus one scale
    byte per 32 channels) plus the slot; per sequence the conv_state rows in
    and out (a ring-buffer state: W-1 rows in, one row out, plus the int64
    position -- counted for one-token decode steps); per launch the taps and
    gammas."""
    C = Hkv * D
    out = 2 * C + 2 * C // 32 if mx else 2 * C * 2
    per_token = 2 * C * 2 + out + slot_bytes
    row = 2 * C * 2
    per_seq = (W - 1) * row + (row + 8 if ring else (W - 1) * row)
    per_launch = 2 * W * C * 2 + 2 * D * 4
    return tokens * per_token + seqs * per_seq + per_launch


def strip_comments(src):
    """C/C++ source without its comments, whitespace runs collapsed (string
    and character literals kept as they are)."""
    out, i, n = [], 0, len(src)
    while i < n:
        c = src[i]
        if c in "\"'":
            j = i + 1
            while j < n and src[j] != c:
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        elif src.startswith("//", i):
            j = src.find("\n", i)
            i = n if j < 0 else j
        elif src.startswith("/*", i):
            j = src.find("*/", i + 2)
            out.append(" ")
            i = n if j < 0 else j + 2
        else:
            out.append(c)
            i += 1
    return " ".join("".join(out).split())


def source_hash(kernel):
    """Hash of the code of `kernel`'s sources (a key of KERNEL_SOURCES),
    comments and layout excluded: an edit to a comment keeps a profile."""
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[kernel]:
        with open(f, encoding="utf-8") as fh:
            h.update(strip_comments(fh.read()).encode())
    return h.hexdigest()[:16]


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return json.load(f), "measured"
    except Exception:
        return {"hbm_gbs": 6650.0}, "fallback"


def profile_traffic(kernel_tag):
    """DRAM bytes per launch from a committed ncu summary, only if the kernel
    sources are unchanged since the capture (else None)."""
    path = os.path.join(PROFILE_DIR, f"{kernel_tag}.md")
    if not os.path.exists(path):
        return None
    vals = {}
    for line in open(path):
        if line.startswith("- ") and ":" in line:
            k, v = line[2:].split(":", 1)
            vals[k.strip()] = v.strip().strip("`")
    kernel = "decode_tma_kernel" if kernel_tag.startswith("decode") else "prefill_tma_kernel"
    if vals.get("source_sha256") != source_hash(kernel):
        return None
    try:
        return float(vals["dram_bytes_per_launch_full"])
    except (KeyError, ValueError):
        return None


class ClockSampler:
    """Polls NVML (SM clock, throttle reasons) on a thread while running."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
        0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
        0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
        0x100: "display_clock_setting",
    }

    def __init__(self, index, period=0.002):
        self.samples, self.reasons, self.ok = [], 0, False
        self.period = period
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            # map the CUDA device to its NVML handle by UUID (CUDA and NVML
            # indices differ under CUDA_VISIBLE_DEVICES)
            uuid = str(torch.cuda.get_device_properties(index).uuid)
            uuid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
            self.h = pynvml.nvmlDeviceGetHandleByUUID(uuid)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.max_mhz = None
        self._stop = threading.Event()

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                self.reasons |= int(nv.nvmlDeviceGetCurrentClocksEventReasons(self.h))
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        names = [n for bit, n in self.REASONS.items() if self.reasons & bit]
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": names,
                "samples": len(self.samples)}


# ------------------------------------------------------------------ workloads

class Workload:
    """Device-resident rotating input sets plus host copies for e2e.

    A step is `launches_per_step` calls (16 chunk calls for the long-context
    workload, one call otherwise); every launch of a workload moves the
    same algorithmic bytes (`bytes_per_launch`)."""

    def __init__(self, name, rank):
        # decode calls with the independent-state promise (the previous
        # launch writes none of a call's state rows)
        self.early_state = name.endswith("_early")
        name = name[:-6] if self.early_state else name
        self.mx = name.endswith("_mx")  # MXFP8 cache store variant
        name = name[:-3] if self.mx else name
        self.ring = name.endswith("_ring")  # ring-buffer conv_state (decode)
        self.name, self.rank = name, rank
        self.launches_per_step = 1
        # prefill calls with the state-only dependency (the previous launch
        # writes none of a call's inputs but conv_state): set by the caller
        self.chain_overlap = False
        seed_shift = 97 * rank
        if name == "single":
            self.kind, self.batches = "prefill", [wl.single(seed=2000 + seed_shift)]
            self.desc = "single-sequence prefill T=8192, Hkv=8, D=128, W=4, zero state, contiguous cache (page 64)"
        elif name in ("wsweep2", "wsweep4", "wsweep8"):
            W = int(name[-1])
            self.kind = "prefill"
            self.batches = [wl.make_prefill([65536], Hkv=8, D=128, W=W, seed=5100 + W + seed_shift,
                                            state="zero", page_size=64, permute_pages=True,
                                            spare_pages=64)]
            self.desc = f"W-sweep prefill T=65536, W={W}, Hkv=8, D=128, zero state, permuted pages"
        elif name == "skew":
            self.kind = "prefill"
            lengths = [131072] + [16] * 1024
            self.batches = [wl.make_prefill(lengths, Hkv=8, D=128, W=4, seed=3500 + seed_shift,
                                            state="normal", page_size=64, permute_pages=True,
                                            spare_pages=64)]
            self.desc = ("skewed varlen prefill: one 131,072-token sequence + 1024 sequences of "
                         "16 tokens, Hkv=8, D=128, W=4, N(0,1) state, permuted pages")
        elif name == "many":
            self.kind = "prefill"
            g = torch.Generator().manual_seed(3600 + seed_shift)
            lengths = torch.randint(32, 97, (1900,), generator=g).tolist()
            self.batches = [wl.make_prefill(lengths, Hkv=8, D=128, W=4, seed=3601 + seed_shift,
                                            state="normal", page_size=64, permute_pages=True,
                                            spare_pages=64)]
            self.desc = ("many-sequence varlen prefill: 1900 sequences of 32..96 tokens, "
                         "Hkv=8, D=128, W=4, N(0,1) state, permuted pages")
        elif name == "varlen":
            self.kind, self.batches = "prefill", [wl.varlen(seed=3000 + seed_shift)]
            self.desc = "varlen prefill 32 seqs U[512,8192], Hkv=8, D=128, W=4, N(0,1) state, permuted pages"
        elif name == "long":
            self.kind = "long"
            self.long = wl.long_context(seed=5000 + seed_shift)
            self.launches_per_step = self.long.num_chunks
            self.desc = ("long-context chunked prefill: one 1,048,576-token sequence as 16 calls "
                         "of 65,536 tokens, state carried, Hkv=8, D=128, W=4, zero initial "
                         "state, paged cache (page 64, seeded permutation)")
        elif name in ("decode", "decode_ring"):
            self.kind = "decode"
            self.dec = wl.decode(seed=4000 + seed_shift)
            self.desc = "decode 1024 seqs x 1 token, Hkv=8, D=128, W=4, N(0,1) state, 4096-page cache"
            if name == "decode_ring":
                self.desc += "; ring-buffer state (one state row written per sequence)"
            if self.early_state:
                self.desc += "; independent-state promise (state rows requested before the wait)"
        else:
            raise SystemExit(f"unknown workload {name}")

    # -- device setup
    def setup(self, dev):
        from short_conv_kv_b200 import binding
        self.binding = binding
        self.calls_args = []
        if self.kind == "prefill":
            b = self.batches[0]
            self.W, self.Hkv, self.D = b.W, b.Hkv, b.D
            self.tokens_per_launch, self.seqs_per_step = b.num_tokens, b.num_seqs
            self.bytes_per_launch = algorithmic_bytes(b.num_tokens, b.num_seqs, b.W, b.Hkv, b.D,
                                                      mx=self.mx)
            shared = dict(conv_w_k=b.conv_w_k.to(dev), conv_w_v=b.conv_w_v.to(dev),
                          gamma_k=b.gamma_k.to(dev), gamma_v=b.gamma_v.to(dev))
            R = max(1, math.ceil(3 * L2_BYTES / self.bytes_per_launch))
            self.rotation = R
            for r in range(R):
                self.calls_args.append(dict(
                    k=b.k.to(dev), v=b.v.to(dev), cu_seqlens=b.cu_seqlens.to(dev),
                    conv_state=b.conv_state.to(dev), slot_mapping=b.slot_mapping.to(dev),
                    k_cache=b.empty_cache().to(dev), v_cache=b.empty_cache().to(dev),
                    eps=b.eps, **shared))
        elif self.kind == "long":
            s = self.long
            self.W, self.Hkv, self.D = s.W, s.Hkv, s.D
            self.tokens_per_launch, self.seqs_per_step = s.chunk, 1
            self.bytes_per_launch = algorithmic_bytes(s.chunk, 1, s.W, s.Hkv, s.D, mx=self.mx)
            shared = dict(conv_w_k=s.conv_w_k.to(dev), conv_w_v=s.conv_w_v.to(dev),
                          gamma_k=s.gamma_k.to(dev), gamma_v=s.gamma_v.to(dev), eps=s.eps,
                          conv_state=s.initial_state().to(dev),
                          k_cache=s.empty_cache().to(dev), v_cache=s.empty_cache().to(dev))
            self.rotation = s.num_chunks
            for c in range(s.num_chunks):
                k, v, sm, cu = s.chunk_inputs(c)
                self.calls_args.append(dict(k=k.to(dev), v=v.to(dev), cu_seqlens=cu.to(dev),
                                            slot_mapping=sm.to(dev), **shared))
        else:
            s = self.dec
            self.W, self.Hkv, self.D = s.W, s.Hkv, s.D
            self.tokens_per_launch, self.seqs_per_step = s.batch, s.batch
            self.bytes_per_launch = algorithmic_bytes(s.batch, s.batch, s.W, s.Hkv, s.D,
                                                      mx=self.mx, ring=self.ring)
            shared = dict(conv_w_k=s.conv_w_k.to(dev), conv_w_v=s.conv_w_v.to(dev),
                          gamma_k=s.gamma_k.to(dev), gamma_v=s.gamma_v.to(dev), eps=s.eps,
                          k_cache=s.empty_cache().to(dev), v_cache=s.empty_cache().to(dev))
            R = max(2, math.ceil(3 * L2_BYTES / self.bytes_per_launch))
            self.rotation = R
            states = [s.conv_state.to(dev) for _ in range(min(R, 16))]
            for r in range(R):
                k, v, sm = s.step_inputs(r % 64)
                a = dict(k=k.to(dev), v=v.to(dev), slot_mapping=sm.to(dev),
                         conv_state=states[r % len(states)], **shared)
                if self.ring:
                    pos = s.start_len.astype(np.int64) + (r % 64)
                    a["state_positions"] = torch.from_numpy(pos).to(dev)
                self.calls_args.append(a)
        self.tokens_per_step = self.tokens_per_launch * self.launches_per_step
        self.bytes_per_step = self.bytes_per_launch * self.launches_per_step

        if self.mx:
            # MXFP8 store: uint8 E4M3 data + E8M0 scale caches in place of
            # the bf16 caches (one set per distinct bf16 cache)
            made = {}
            for a in self.calls_args:
                for key in ("k_cache", "v_cache"):
                    c = a.pop(key)
                    if id(c) not in made:
                        P_, S_, H_, D_ = c.shape
                        made[id(c)] = (
                            torch.full((P_, S_, H_, D_), 0xFF, dtype=torch.uint8, device=dev),
                            torch.full((P_, S_, H_, D_ // 32), 0xFF, dtype=torch.uint8, device=dev))
                    a[key[0] + "_data"], a[key[0] + "_scale"] = made[id(c)]
            self.desc += "; MXFP8 cache store (E4M3 + E8M0 per 32 channels)"

    def prepared(self, i, stream):
        a = self.calls_args[i % len(self.calls_args)]
        if self.mx and self.kind == "decode":
            return self.binding.prepare_decode_mxfp8(
                a["k"], a["v"], a["conv_w_k"], a["conv_w_v"], a["gamma_k"], a["gamma_v"],
                a["eps"], a["conv_state"], a["slot_mapping"], a["k_data"], a["k_scale"],
                a["v_data"], a["v_scale"], stream=stream, independent_state=self.early_state)
        if self.mx:
            return self.binding.prepare_prefill_varlen_mxfp8(
                a["k"], a["v"], a["cu_seqlens"], a["conv_w_k"], a["conv_w_v"], a["gamma_k"],
                a["gamma_v"], a["eps"], a["conv_state"], a["slot_mapping"], a["k_data"],
                a["k_scale"], a["v_data"], a["v_scale"], stream=stream,
                state_only_dependency=self.chain_overlap)
        if self.kind == "decode":
            return self.binding.prepare_decode(
                a["k"], a["v"], a["conv_w_k"], a["conv_w_v"], a["gamma_k"], a["gamma_v"],
                a["eps"], a["conv_state"], a["slot_mapping"], a["k_cache"], a["v_cache"],
                stream=stream, state_positions=a.get("state_positions"),
                independent_state=self.early_state)
        return self.binding.prepare_prefill_varlen(
            a["k"], a["v"], a["cu_seqlens"], a["conv_w_k"], a["conv_w_v"], a["gamma_k"],
            a["gamma_v"], a["eps"], a["conv_state"], a["slot_mapping"], a["k_cache"],
            a["v_cache"], stream=stream, state_only_dependency=self.chain_overlap)

    def kernel_tag(self):
        tag = {"prefill": "prefill_tma_kernel", "long": "prefill_tma_kernel",
               "decode": "decode_tma_kernel"}[self.kind]
        return tag + ("_mx" if self.mx else "")


# ------------------------------------------------------------------ unfused chain

def time_unfused(work, n, Wu, dev):
    """The same step as the library's four unfused stage kernels (conv ->
    y, rmsnorm -> z, scatter, state update; bf16 intermediates in HBM) over
    the same rotating buffers, n calls in one CUDA graph replay (the fused
    kernel's timing method); returns ms per call.  Context for the
    fused-versus-unfused claim ("SGLang and Miles announce day-0 Inkling
    support", aib.vote English news item, paragraph 2)."""
    from short_conv_kv_b200 import binding
    stream = torch.cuda.Stream(device=dev)
    T = work.tokens_per_launch
    C = work.Hkv * work.D
    y = torch.empty(T, 2 * C, dtype=torch.bfloat16, device=dev)
    z = torch.empty_like(y)
    m = len(work.calls_args)
    if work.kind == "decode":
        cu = torch.arange(T + 1, dtype=torch.int32, device=dev)

    def chain(i, s):
        a = work.calls_args[i % m]
        return binding.prepare_unfused(
            a["k"], a["v"], a["cu_seqlens"] if work.kind != "decode" else cu, a["conv_w_k"],
            a["conv_w_v"], a["gamma_k"], a["gamma_v"], a["eps"], a["conv_state"],
            a["slot_mapping"], a["k_cache"], a["v_cache"], y, z, stream=s)

    with torch.cuda.stream(stream):
        for i in range(Wu):
            chain(i, stream)()
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        cap = torch.cuda.current_stream()
        runs = [chain(i, cap) for i in range(n)]
        for r in runs:
            r()
    g.replay()
    torch.cuda.synchronize()
    s_ev, e_ev = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda._sleep(SLEEP_CYCLES)  # (current stream) the host submits meanwhile
    stream.wait_stream(torch.cuda.current_stream())
    s_ev.record(stream)
    with torch.cuda.stream(stream):
        g.replay()
    e_ev.record(stream)
    e_ev.synchronize()
    del g
    return s_ev.elapsed_time(e_ev) / n


# ------------------------------------------------------------------ our arm

def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group(
            "nccl", timeout=datetime.timedelta(seconds=120),
            device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(x, world):
    """Slowest rank's value (NCCL needs a device tensor, gloo a host one)."""
    if world == 1:
        return x
    on_gpu = torch.distributed.get_backend() == "nccl"
    t = torch.tensor([x], dtype=torch.float64, device="cuda" if on_gpu else "cpu")
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def time_graph(work, K, Wu, dev, world, local, profile_range=False):
    """Warm-up W eager steps, then K steps (K x launches_per_step calls)
    captured in one CUDA graph (kernel nodes back to back, nothing between
    them) and replayed once as the timed region.  A sleep kernel queued in
    front of the start event keeps the GPU busy while the host submits the
    replay, so the region holds the launches (and the short gaps between
    consecutive launches) only.  With profile_range the timed replay is
    bracketed by cudaProfilerStart/Stop, for a profiler that captures the
    whole replay as one range."""
    lps = work.launches_per_step
    stream = torch.cuda.Stream(device=dev)
    with torch.cuda.stream(stream):
        for i in range(Wu * lps):
            work.prepared(i, stream)()
    stream.synchronize()

    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        cap = torch.cuda.current_stream()
        calls = [work.prepared(i, cap) for i in range(K * lps)]
        for c in calls:
            c()
    # one untimed replay uploads the graph and warms it
    g.replay()
    torch.cuda.synchronize()

    outer_s = torch.cuda.Event(enable_timing=True)
    outer_e = torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        with torch.cuda.stream(stream):
            torch.cuda._sleep(SLEEP_CYCLES)
        if profile_range:
            torch.cuda.profiler.start()
        outer_s.record(stream)
        with torch.cuda.stream(stream):
            g.replay()
        outer_e.record(stream)
        outer_e.synchronize()
        if profile_range:
            torch.cuda.profiler.stop()
    torch.cuda.synchronize()
    barrier(world)
    total_ms = outer_s.elapsed_time(outer_e)
    del g
    return total_ms, clk.summary()


def time_e2e(work, steps, dev):
    """Same metric end to end through the public API: every step copies its
    inputs from pinned host memory, runs the step, and reads the written
    caches and the state back into pinned host memory.  Steps are pipelined
    over two buffer sets on three streams (upload, compute, download), so
    step i+1's upload overlaps step i's download on the full-duplex link."""
    from short_conv_kv_b200 import binding
    a0 = work.calls_args[0]
    in_keys = ["k", "v", "slot_mapping"] + (["cu_seqlens"] if "cu_seqlens" in a0 else []) + \
        (["state_positions"] if "state_positions" in a0 else [])
    NB = 2
    host_in = [{k: a0[k].cpu().pin_memory() for k in in_keys} for _ in range(NB)]
    dev_in = [{k: torch.empty_like(a0[k], device=dev) for k in in_keys} for _ in range(NB)]
    dev_out = [{k: a0[k].clone() for k in ("k_cache", "v_cache", "conv_state")} for _ in range(NB)]
    # The step's result is the cache rows it wrote plus the new state.  When
    # the paged cache is much larger than the rows written, those rows are
    # gathered on the device first, so only the result crosses the link.
    C = work.Hkv * work.D
    slots = a0["slot_mapping"]
    slots = slots[slots >= 0]
    n_slots = a0["k_cache"].shape[0] * a0["k_cache"].shape[1]
    gather = n_slots > 2 * slots.numel()
    out_shapes = {"k_rows": (slots.numel(), C), "v_rows": (slots.numel(), C)} if gather else \
        {"k_rows": tuple(a0["k_cache"].shape), "v_rows": tuple(a0["v_cache"].shape)}
    out_shapes["conv_state"] = tuple(a0["conv_state"].shape)
    host_out = [{k: torch.empty(shp, dtype=torch.bfloat16, pin_memory=True)
                 for k, shp in out_shapes.items()} for _ in range(NB)]
    stage = [{k: torch.empty(out_shapes[k], dtype=torch.bfloat16, device=dev)
              for k in ("k_rows", "v_rows")} for _ in range(NB)] if gather else None
    h2d = sum(t.numel() * t.element_size() for t in host_in[0].values())
    d2h = sum(t.numel() * t.element_size() for t in host_out[0].values())
    s_up, s_cmp, s_dn = (torch.cuda.Stream(device=dev) for _ in range(3))
    up_done = [torch.cuda.Event() for _ in range(NB)]
    cmp_done = [torch.cuda.Event() for _ in range(NB)]
    dn_done = [torch.cuda.Event() for _ in range(NB)]
    for e in cmp_done + dn_done:
        e.record(s_cmp)

    def step(i):
        b = i % NB
        di, do = dev_in[b], dev_out[b]
        with torch.cuda.stream(s_up):
            s_up.wait_event(cmp_done[b])          # the kernel that read dev_in[b] is done
            for k in in_keys:
                di[k].copy_(host_in[b][k], non_blocking=True)
            up_done[b].record(s_up)
        with torch.cuda.stream(s_cmp):
            s_cmp.wait_event(up_done[b])
            s_cmp.wait_event(dn_done[b])          # dev_out[b] has been read back
            if work.kind == "decode":
                binding.decode(di["k"], di["v"], a0["conv_w_k"], a0["conv_w_v"], a0["gamma_k"],
                               a0["gamma_v"], a0["eps"], do["conv_state"], di["slot_mapping"],
                               do["k_cache"], do["v_cache"], stream=s_cmp,
                               state_positions=di.get("state_positions"))
            else:
                binding.prefill_varlen(di["k"], di["v"], di["cu_seqlens"], a0["conv_w_k"],
                                       a0["conv_w_v"], a0["gamma_k"], a0["gamma_v"], a0["eps"],
                                       do["conv_state"], di["slot_mapping"], do["k_cache"],
                                       do["v_cache"], stream=s_cmp)
            if gather:
                torch.index_select(do["k_cache"].view(-1, C), 0, slots, out=stage[b]["k_rows"])
                torch.index_select(do["v_cache"].view(-1, C), 0, slots, out=stage[b]["v_rows"])
            cmp_done[b].record(s_cmp)
        with torch.cuda.stream(s_dn):
            s_dn.wait_event(cmp_done[b])
            src = {"k_rows": stage[b]["k_rows"] if gather else do["k_cache"],
                   "v_rows": stage[b]["v_rows"] if gather else do["v_cache"],
                   "conv_state": do["conv_state"]}
            for k in out_shapes:
                host_out[b][k].copy_(src[k], non_blocking=True)
            dn_done[b].record(s_dn)

    for i in range(2):
        step(i)
    torch.cuda.synchronize()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(s_up)
    s_cmp.wait_stream(s_up)
    s_dn.wait_stream(s_up)
    for i in range(steps):
        step(i)
    s_up.wait_stream(s_dn)
    end.record(s_up)
    end.synchronize()
    ms = start.elapsed_time(end) / steps
    return ms, h2d, d2h


def _compact(slot_mapping, page_size, Hkv, D):
    """Dense slots 0..n-1 and a cache just large enough for them: the oracle
    copies its cache arguments, so timing it against a multi-GB paged cache
    would time the copy.  Placement is a layout detail; the work per token is
    the same."""
    n = int(slot_mapping.shape[0])
    pages = max(1, -(-n // page_size))
    cache = np.full((pages, page_size, Hkv, D), wl.SENTINEL_BITS, np.uint16)
    return np.arange(n, dtype=np.int64), cache


def cpu_oracle_baseline(work, budget_s=12.0):
    """The oracle as it stands (single-threaded C, test infrastructure) on a
    bounded sample of the same workload: whole batches, repeated until about
    `budget_s` seconds of CPU work."""
    import oracle
    lib = oracle.load()
    if work.kind == "prefill":
        b = work.batches[0]
        sm, cache = _compact(b.slot_mapping, b.page_size, b.Hkv, b.D)
        args = (wl.bits(b.k), wl.bits(b.v), b.cu_seqlens.numpy(), wl.bits(b.conv_w_k),
                wl.bits(b.conv_w_v), b.gamma_k.numpy(), b.gamma_v.numpy(), b.eps,
                wl.bits(b.conv_state), sm, cache, cache.copy())
        tokens, sample = b.num_tokens, "whole batch"
        run = lambda: oracle.prefill_varlen(*args, want_z=False, lib=lib)
    elif work.kind == "long":
        s = work.long
        k, v, sm, cu = s.chunk_inputs(0)
        sm, cache = _compact(sm, s.page_size, s.Hkv, s.D)
        args = (wl.bits(k), wl.bits(v), cu.numpy(), wl.bits(s.conv_w_k), wl.bits(s.conv_w_v),
                s.gamma_k.numpy(), s.gamma_v.numpy(), s.eps, wl.bits(s.initial_state()), sm,
                cache, cache.copy())
        tokens, sample = k.shape[0], "first 65,536-token chunk"
        run = lambda: oracle.prefill_varlen(*args, want_z=False, lib=lib)
    else:
        s = work.dec
        k, v, sm = s.step_inputs(0)
        sm, cache = _compact(sm, s.page_size, s.Hkv, s.D)
        args = (wl.bits(k), wl.bits(v), wl.bits(s.conv_w_k), wl.bits(s.conv_w_v), s.gamma_k.numpy(),
                s.gamma_v.numpy(), s.eps, wl.bits(s.conv_state), sm, cache, cache.copy())
        tokens, sample = s.batch, "decode step 0 (1024 sequences)"
        run = lambda: oracle.decode(*args, want_z=False, lib=lib)
    reps, t_tot = 0, 0.0
    while t_tot < budget_s and reps < 50:
        t0 = time.perf_counter()
        run()
        t_tot += time.perf_counter() - t0
        reps += 1
    return {"value": tokens * reps / t_tot, "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": f"{sample} x {reps} runs ({t_tot:.1f} s, single thread, dense slots; "
                      f"host has {os.cpu_count()} cores)"}


# Workloads timed beside the headline line (the other full-size
# configurations): name -> label of the `configs` entry.
SIDE_CONFIGS = [
    ("single", "single-sequence prefill T=8192"),
    ("varlen", "varlen prefill, 32 sequences"),
    ("decode", "decode step, 1024 sequences"),
    ("decode_early", "decode step, 1024 sequences, calls with the independent-state promise "
                     "(the launch before each writes none of its state rows)"),
    ("wsweep2", "65,536-token prefill, W=2"),
    ("wsweep8", "65,536-token prefill, W=8"),
]
SIDE_MIN_MS = 20.0     # timed region per side workload, at least
SIDE_MAX_LAUNCHES = 2500


def time_isolated_launch(work, dev, reps=7):
    """Median time of one launch with nothing before or after it on the GPU
    (a sleep kernel ahead of the start event hides the host's launch
    latency; CUDA events around the single launch): the time a call takes
    when nothing overlaps it, set against the chain's time per launch."""
    stream = torch.cuda.Stream(device=dev)
    times = []
    for i in range(reps):
        call = work.prepared(i, stream)
        s_ev, e_ev = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        with torch.cuda.stream(stream):
            torch.cuda._sleep(SLEEP_CYCLES // 20)  # ~0.1 ms
        s_ev.record(stream)
        call()
        e_ev.record(stream)
        e_ev.synchronize()
        times.append(s_ev.elapsed_time(e_ev))
    return statistics.median(times)


def line_roofline(work, kern_ms, peaks, peak_src, traffic):
    achieved = work.bytes_per_launch / (kern_ms / 1e3) / 1e9
    return {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": achieved / peaks["hbm_gbs"], "traffic": traffic,
            "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs copy bandwidth)",
            "frac_of_8tbs": achieved / 8000.0,
            "algorithmic_bytes_per_launch": work.bytes_per_launch,
            "kernel_ms_per_launch": kern_ms}


def time_side_config(name, label, K, Wu, dev, world, local, peaks, peak_src):
    """One full-size side workload timed like the headline (graph replay,
    rotating buffers), over max(K, enough launches for SIDE_MIN_MS) launches."""
    work = Workload(name, 0)
    work.setup(dev)
    # a short eager probe sets the number of launches of the timed region
    stream = torch.cuda.Stream(device=dev)
    s_ev, e_ev = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        for i in range(3):
            work.prepared(i, stream)()
        s_ev.record(stream)
        for i in range(10):
            work.prepared(i, stream)()
        e_ev.record(stream)
    e_ev.synchronize()
    est = max(s_ev.elapsed_time(e_ev) / 10, 1e-3)
    n = int(min(SIDE_MAX_LAUNCHES, max(K, math.ceil(SIDE_MIN_MS / est))))
    total_ms, clocks = time_graph(work, n, Wu, dev, world, local)
    total_ms = max_over_ranks(total_ms, world)
    kern_ms = total_ms / n
    r = line_roofline(work, kern_ms, peaks, peak_src,
                      profile_traffic(f"{work.kernel_tag()}_{name}"))
    out = {"label": label, "workload": work.desc, "launches": n,
           "ms_per_launch": kern_ms, "tokens_per_s": world * work.tokens_per_launch / (kern_ms / 1e3),
           "algorithmic_bytes_per_launch": work.bytes_per_launch,
           "achieved_gbs": r["achieved"], "frac": r["frac"], "frac_of_8tbs": r["frac_of_8tbs"],
           "traffic": r["traffic"], "clocks": clocks}
    del work
    torch.cuda.empty_cache()
    return out, n


def run_ours(args):
    world, rank, local = dist_setup(args)
    dev = torch.device("cuda", local)
    work = Workload(args.workload, rank)
    # consecutive chunks of one sequence are the case the state-only
    # dependency is for: the long-context workload promises it by default
    work.chain_overlap = work.kind != "decode" and (
        args.chain_overlap or (work.kind == "long" and not args.no_chain_overlap))
    work.early_state = (work.early_state or args.early_state) and work.kind == "decode"
    work.setup(dev)
    K, Wu = args.steps, args.warmup
    lps = work.launches_per_step
    total_ms, clocks = time_graph(work, K, Wu, dev, world, local,
                                  profile_range=args.profile_range)
    total_ms = max_over_ranks(total_ms, world)
    if args.profile_range:
        # the profiled run only needs its timed region; nothing else runs
        if rank == 0:
            print(json.dumps({"profile_range": work.desc, "steps": K,
                              "launches": K * lps, "ms": total_ms}), flush=True)
        if world > 1:
            torch.distributed.destroy_process_group()
        return
    ms_per_step = total_ms / K
    kern_ms = total_ms / (K * lps)  # average launch duration
    chain = None
    if lps > 1:
        iso_ms = max_over_ranks(time_isolated_launch(work, dev), world)
        chain = {"launches_per_step": lps, "ms_per_step": ms_per_step,
                 "isolated_launch_ms": iso_ms,
                 "step_vs_launches_alone": ms_per_step / (lps * iso_ms),
                 "state_only_dependency": work.chain_overlap,
                 "note": "the step's launches back to back (state carried) against as many "
                         "launches each timed alone on an idle GPU"}
        if work.chain_overlap:
            # the same chain with every CTA waiting for the previous launch
            work.chain_overlap = False
            t2, _ = time_graph(work, K, Wu, dev, world, local)
            work.chain_overlap = True
            t2 = max_over_ranks(t2, world)
            chain["without_state_only_dependency"] = {
                "ms_per_step": t2 / K, "ms_per_launch": t2 / (K * lps)}
    value = world * work.tokens_per_step * K / (total_ms / 1e3)
    launches = K * lps
    e2e = None
    if not work.mx:  # the end-to-end leg is measured on the bf16 store
        e2e_ms, h2d, d2h = time_e2e(work, args.e2e_steps, dev)
        e2e_ms = max_over_ranks(e2e_ms, world)
        e2e = {"value": world * work.tokens_per_launch / (e2e_ms / 1e3), "unit": "tokens/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
               "method": ("pinned host buffers; per call: upload of the inputs, the step, and "
                          "download of the written cache rows + new state, pipelined over two "
                          "buffer sets on three streams" +
                          ("; a step here is one 65,536-token call of the chunked sequence "
                           "(state carried from call to call)" if work.kind == "long" else ""))}
    unfused = None
    if not work.mx and not work.ring and not args.no_unfused:
        Ku = min(launches, 50)
        un_ms = max_over_ranks(time_unfused(work, Ku, Wu, dev), world)
        T, C = work.tokens_per_launch, work.Hkv * work.D
        un_bytes = work.bytes_per_launch + T * 2 * C * 2 * 4  # + y and z, each written and read
        unfused = {"ms_per_launch": un_ms, "launches": Ku, "fused_speedup": un_ms / kern_ms,
                   "algorithmic_bytes_per_launch": un_bytes,
                   "achieved_gbs": un_bytes / (un_ms / 1e3) / 1e9,
                   "kind": "the library's unfused stage kernels: conv -> y, rmsnorm -> z, "
                           "scatter, state update (4 launches, bf16 intermediates in HBM), "
                           "one CUDA graph replay"}
    peaks, peak_src = measured_peaks()
    configs = None
    side_launches = 0
    if not args.no_configs and args.workload == "long":
        configs = {}
        del work.calls_args  # free the headline's buffers first
        torch.cuda.empty_cache()
        for name, label in SIDE_CONFIGS:
            configs[name], n = time_side_config(name, label, K, Wu, dev, world, local, peaks,
                                                peak_src)
            side_launches += n
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_oracle_baseline(work)
    if rank == 0:
        line = {
            "metric": "fused ShortConv-KV tokens/s and achieved HBM GB/s (% of B200 peak)",
            "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K, "warmup": Wu,
            "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": work.desc,
                       "storage": ("bf16 in, MXFP8 cache, bf16 state, fp32 math" if work.mx
                                   else "bf16 in, bf16 cache/state, fp32 math"),
                       "tokens_per_step_per_gpu": work.tokens_per_step,
                       "launches_per_step": lps,
                       "tokens_per_launch": work.tokens_per_launch,
                       "seqs_per_step_per_gpu": work.seqs_per_step, "W": work.W,
                       "num_kv_heads": work.Hkv, "head_dim": work.D,
                       "parallelism": f"{world} independent replicas (sequence sharding, no collective)",
                       "l2": f"inputs rotate over {work.rotation} buffer sets "
                             f"({work.rotation * work.bytes_per_launch / 1e6:.0f} MB) > L2",
                       "timing": "K steps in one CUDA graph replay, CUDA events around the replay",
                       "calls": ("prefill calls promise the state-only dependency (the previous "
                                 "launch writes none of a call's inputs but conv_state)"
                                 if work.chain_overlap else "default calls")},
            "roofline": line_roofline(work, kern_ms, peaks, peak_src,
                                      profile_traffic(f"{work.kernel_tag()}_{args.workload}")),
            "configs": configs,
            "chain": chain,
            "cpu_baseline": cpu,
            "unfused_chain": unfused,
            "e2e": e2e,
            "gpu_launches": launches,
            "gpu_launches_side_configs": side_launches,
            "clocks": clocks,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


# ------------------------------------------------------------------ reference arm

def run_reference(args):
    """Time the CPU oracle (as it stands) on this arm's workload; rank 0 only."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    lib = oracle.load()
    work = Workload(args.workload, 0)
    K, Wu = args.steps, args.warmup
    # per-step sample: the whole batch if K+W steps fit the time budget,
    # else a prefix of the batch's tokens (same shapes and statistics)
    if work.kind == "prefill":
        b = work.batches[0]
    elif work.kind == "long":
        s = work.long
        k, v, sm, cu = s.chunk_inputs(0)
        b = wl.Batch(W=s.W, Hkv=s.Hkv, D=s.D, eps=s.eps, k=k, v=v, cu_seqlens=cu,
                     conv_w_k=s.conv_w_k, conv_w_v=s.conv_w_v, gamma_k=s.gamma_k,
                     gamma_v=s.gamma_v, conv_state=s.initial_state(), slot_mapping=sm,
                     num_pages=s.num_pages, page_size=s.page_size)
    else:
        s = work.dec
        k, v, sm = s.step_inputs(0)
        b = wl.Batch(W=s.W, Hkv=s.Hkv, D=s.D, eps=s.eps, k=k, v=v,
                     cu_seqlens=torch.arange(s.batch + 1, dtype=torch.int32),
                     conv_w_k=s.conv_w_k, conv_w_v=s.conv_w_v, gamma_k=s.gamma_k,
                     gamma_v=s.gamma_v, conv_state=s.conv_state, slot_mapping=sm,
                     num_pages=s.num_pages, page_size=s.page_size)
    kb, vb = wl.bits(b.k), wl.bits(b.v)
    cu = b.cu_seqlens.numpy()
    T = b.num_tokens
    common = (wl.bits(b.conv_w_k), wl.bits(b.conv_w_v), b.gamma_k.numpy(), b.gamma_v.numpy(), b.eps)
    state = wl.bits(b.conv_state)
    dense, cache = _compact(b.slot_mapping, b.page_size, b.Hkv, b.D)

    def one(ntok):
        # the first sequences' tokens up to ntok (cut inside a sequence if needed)
        cut = np.minimum(cu, ntok)
        return oracle.prefill_varlen(kb[:ntok], vb[:ntok], cut.astype(np.int32), *common[:4],
                                     common[4], state, dense[:ntok], cache, cache,
                                     want_z=False, lib=lib)

    t0 = time.perf_counter()
    one(T)
    full_s = time.perf_counter() - t0
    budget = 150.0
    ntok = T if (K + Wu) * full_s <= budget else max(32, int(T * budget / ((K + Wu) * full_s)))
    for _ in range(Wu):
        one(ntok)
    t0 = time.perf_counter()
    for _ in range(K):
        one(ntok)
    dt = time.perf_counter() - t0
    value = ntok * K / dt
    line = {
        "impl": "reference",
        "metric": "fused ShortConv-KV tokens/s and achieved HBM GB/s (% of B200 peak)",
        "value": value, "unit": "tokens/s", "n_gpus": 1, "steps": K, "warmup": Wu,
        "ms_per_step": dt / K * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64 (oracle)", "data": "synthetic",
        "config": {"workload": work.desc},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                         "sample": f"first {ntok} of {T} tokens per step, dense slots, single thread; "
                                   f"host has {os.cpu_count()} cores"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="long",
                    choices=["long", "single", "varlen", "skew", "decode", "decode_ring", "wsweep2",
                             "wsweep4", "wsweep8", "many",
                             "single_mx", "varlen_mx", "decode_mx", "long_mx", "wsweep2_mx",
                             "wsweep4_mx", "wsweep8_mx", "decode_early", "decode_mx_early",
                             "decode_ring_early"])
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-unfused", action="store_true",
                    help="skip timing the unfused four-kernel chain (context only)")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip timing the side workloads of the `configs` key")
    ap.add_argument("--chain-overlap", action="store_true",
                    help="prefill calls promise the state-only dependency (consecutive "
                         "launches overlap; see include/sconv_kv.h); on by default for the "
                         "long-context workload")
    ap.add_argument("--no-chain-overlap", action="store_true",
                    help="the long-context workload's calls without that promise")
    ap.add_argument("--early-state", action="store_true",
                    help="decode calls promise an independent state (each launch's state "
                         "rows are not written by the launch before it; see "
                         "include/sconv_kv.h)")
    ap.add_argument("--profile-range", action="store_true",
                    help="bracket the timed replay with cudaProfilerStart/Stop and run nothing "
                         "else (for a range capture of the DRAM counters)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
