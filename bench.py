#!/usr/bin/env python
"""Benchmark of the quantized hybrid layer-stage on B200.

Workload: the full 27B-shape stage, 64 layers (48 gated-DeltaNet + 16 GQA
attention, layer i attention iff i % 4 == 3), hidden 5120, FFN 17408, all
weights GGUF Q4_0 (12.85 GB streamed per pass), seeded synthetic weights
(seed 4) and N(0,1) hidden states.  One step = one plain-decode pass at
n_tok = 1 (stage_forward + stage_commit(1)) with context growing from 4096 (KV
caches prefilled with N(0,1) f16 rows, DeltaNet states N(0, 0.01)).  The
prefill leg runs 128 chunks of 16 tokens over a 2048-token prompt from
position 0.  The weights are far larger than L2 (126 MB), so no flush is needed
between steps.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

N > 1 runs N independent replicas (one per GPU, launched by torchrun): the
stage is a sequential chain of layers with no data-parallel split of one
sequence, so each GPU serves its own sequence; ranks synchronise only around
the timed region and report the max time.  Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import hashlib
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

import synth  # noqa: E402
from synth import FULL, Q4_0, Q8_0  # noqa: E402

METRIC = "stage tok/s & weight-stream HBM GB/s vs ~8 TB/s (64-layer Q4_0, n_tok 1/16)"
SEED = 4
CTX0 = 4096
PROMPT = 2048
CHUNK = 16
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0


# --------------------------------------------------------------------------
# distributed plumbing (replicas only)

def dist_setup(n_gpus: int):
    """(rank, world, local_rank, pg_initialised); one process per GPU under torchrun."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if world <= 1:
        return 0, 1, 0, False
    import datetime

    import torch
    import torch.distributed as dist
    backend = "nccl" if torch.cuda.is_available() else "gloo"
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if torch.cuda.is_available():
        torch.cuda.set_device(local)
    dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=600))
    return dist.get_rank(), dist.get_world_size(), local, True


def barrier(active: bool):
    if active:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, active: bool) -> float:
    if not active:
        return float(x)
    import torch
    import torch.distributed as dist
    dev = "cuda" if torch.cuda.is_available() and dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def dist_teardown(active: bool):
    if active:
        import torch.distributed as dist
        dist.destroy_process_group()


# --------------------------------------------------------------------------
# workload

def gen_tensors(shape, qtype, seed, begin, end, threads=None) -> dict:
    """Seeded weights of layers [begin, end), generated layer-parallel (independent streams)."""
    from concurrent.futures import ThreadPoolExecutor
    threads = threads or min(16, os.cpu_count() or 1)
    out = {}
    with ThreadPoolExecutor(threads) as ex:
        for t in ex.map(lambda l: synth.layer_tensors(shape, qtype, seed, l), range(begin, end)):
            out.update(t)
    return out


def layer_bytes(shape, qtype, layer: int) -> int:
    """GGUF bytes of one layer's quantised matrices (what one pass streams)."""
    bb = synth.BLOCK_BYTES[qtype]
    H, F = shape.hidden, shape.ffn
    mats = [(F, H), (F, H), (H, F)]
    if shape.is_attention(layer):
        mats += [(shape.attn_in_rows, H), (H, shape.attn_o)]
    else:
        mats += [(shape.dn_in_rows, H), (H, shape.dn_o)]
    return sum(r * c // 32 * bb for r, c in mats)


def pass_bytes(shape, qtype, layers, ctx: int, n_tok: int = 1) -> dict:
    """Algorithmic bytes of one pass: weights once, KV rows 0..ctx read per
    attention layer, DeltaNet state read once and written once per token."""
    w = sum(layer_bytes(shape, qtype, l) for l in layers)
    n_att = sum(1 for l in layers if shape.is_attention(l))
    n_dn = len(layers) - n_att
    kv = n_att * 2 * shape.att_kv_heads * (ctx + n_tok) * shape.att_dim * 2
    state = n_dn * shape.dn_v_heads * shape.dn_dim * shape.dn_dim * 4 * (1 + n_tok)
    return {"weights": w, "kv": kv, "state": state, "total": w + kv + state}


def launches_per_pass(shape, layers, persistent: bool = False) -> int:
    """Kernels the stage launches per pass: one persistent kernel, or input +
    per layer (in-proj, mixer kernel(s), out-proj, gate/up, down)."""
    if persistent:
        return 1
    n = 1
    for l in layers:
        n += 6 if shape.is_attention(l) else 5
    return n


def measured_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return json.load(f)
    return {}


def kernel_sources_sha() -> str:
    """Hash of the GEMV's sources with comments and blank lines dropped (what
    the compiler sees), to tell whether committed ncu counters still apply."""
    import re
    h = hashlib.sha256()
    for f in ("qgemv.cuh", "qpack.cuh", "qact.cuh", "common.cuh"):
        with open(os.path.join(ROOT, "quantized_hybrid_layer_b200", "csrc", f)) as fh:
            for line in fh:
                code = re.sub(r"//.*", "", line).rstrip()
                if code:
                    h.update(code.encode() + b"\n")
    return h.hexdigest()


def committed_traffic():
    """DRAM bytes per launch of the GEMV from the committed ncu summary, if the
    kernel sources are unchanged since it was taken; else None."""
    p = os.path.join(ROOT, "profiles", "qgemv_dram.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    if d.get("sources_sha256") != kernel_sources_sha():
        return None
    return d.get("traffic_bytes_per_launch")


class ClockSampler:
    """SM clocks and clock-event (throttle) reasons sampled while the timed
    region runs: NVML polled every 10 ms from a host thread (the timed regions
    last tens of milliseconds), nvidia-smi at its 200 ms period as the fallback
    where NVML is unavailable.  Only reads; changes no GPU setting."""

    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.thread = None
        self.samples = []
        self.max_mhz = None
        self.err = None

    def _nvml_loop(self, stop):
        import pynvml as nv
        h = self._handle(nv)
        self.max_mhz = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
        bits = {"hw_slowdown": nv.nvmlClocksEventReasonHwSlowdown,
                "hw_thermal_slowdown": nv.nvmlClocksEventReasonHwThermalSlowdown,
                "sw_thermal_slowdown": nv.nvmlClocksEventReasonSwThermalSlowdown,
                "sw_power_cap": nv.nvmlClocksEventReasonSwPowerCap}
        while True:
            mhz = float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
            r = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
            self.samples.append((mhz, {n for n, b in bits.items() if r & b}))
            if stop.wait(0.01):
                break

    def _handle(self, nv):
        """NVML handle of CUDA device self.idx, matched by UUID (CUDA and NVML
        number the GPUs differently when CUDA_VISIBLE_DEVICES is set)."""
        try:
            import torch
            uuid = str(torch.cuda.get_device_properties(self.idx).uuid)
            return nv.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
        except Exception:
            return nv.nvmlDeviceGetHandleByIndex(self.idx)

    def start(self):
        import threading
        try:
            import pynvml as nv
            nv.nvmlInit()
            self._handle(nv)
            self.stop_ev = threading.Event()
            self.thread = threading.Thread(target=self._nvml_loop, args=(self.stop_ev,), daemon=True)
            self.thread.start()
            return
        except Exception as e:   # no NVML: fall back to nvidia-smi
            self.err = str(e)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self) -> dict:
        if self.thread is not None:
            self.stop_ev.set()
            self.thread.join(timeout=5)
            sm = [m for m, _ in self.samples]
            reasons = set().union(*[r for _, r in self.samples]) if self.samples else set()
            return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": self.max_mhz,
                    "reasons": sorted(reasons), "samples": len(sm), "source": "nvml, 10 ms"}
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["clock sampling unavailable"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], [], set()
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for name, v in zip(self.NAMES, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm), "source": "nvidia-smi, 200 ms"}


def workload_config(args, shape) -> dict:
    return {
        "workload": (f"{args.layers}-layer hybrid layer-stage (gated DeltaNet : attention 3:1), hidden "
                     f"{shape.hidden}, FFN {shape.ffn}, {args.qtype.upper()} weights, plain decode n_tok=1 "
                     f"from context {CTX0}; prefill 16-token chunks over a {PROMPT}-token prompt"),
        "layers": args.layers, "qtype": args.qtype, "n_tok": 1, "ctx_start": CTX0,
        "prefill_prompt": PROMPT, "prefill_chunk": CHUNK,
        "l2": "no flush: 12.85 GB of weights streamed per pass, far above the 126 MB L2",
        "parallelism": f"replicas x{args.gpus}",
    }


# --------------------------------------------------------------------------
# the oracle as a timed CPU baseline (test infrastructure, imported only here)

def oracle_decode_sample(shape, qtype, tensors, layers, n_layers_sample=None):
    """Time the oracle on one decode token (pos 4096) through the given layers;
    returns seconds per full token (scaled when only a sample of layers runs)."""
    import oracle
    sample = layers if n_layers_sample is None else layers[:n_layers_sample]
    st = oracle.OracleStage(shape, qtype, tensors, sample[0], sample[-1] + 1, CTX0 + 64)
    for l in sample:
        if shape.is_attention(l):
            K, V = synth.kv_prefill(shape, SEED, l, CTX0, CTX0 + 64)
            st.set_kv(l, K, V)
        else:
            st.set_dn_state(l, synth.dn_state(shape, SEED, l))
    st.set_kv_len(CTX0)
    h = synth.hidden(shape, SEED, 10_000, 1)
    t0 = time.perf_counter()
    st.forward(h, CTX0)
    dt = time.perf_counter() - t0
    return dt * len(layers) / len(sample), oracle.threads()


# --------------------------------------------------------------------------

def run_reference(args, rank, world, pg):
    """The oracle on the host cores: each step is one decode token through one
    layer of the stage (cycling through the 64 layers), so K steps are K/64
    tokens of the same workload."""
    shape = FULL
    qtype = Q4_0 if args.qtype == "q4_0" else Q8_0
    if rank != 0:
        return None
    import oracle
    layers = list(range(args.layers))
    tensors = gen_tensors(shape, qtype, SEED, 0, args.layers)
    max_ctx = CTX0 + (args.steps + args.warmup) // len(layers) + 64
    st = oracle.OracleStage(shape, qtype, tensors, 0, args.layers, max_ctx)
    for l in layers:
        if shape.is_attention(l):
            K, V = synth.kv_prefill(shape, SEED, l, CTX0, max_ctx)
            st.set_kv(l, K, V)
        else:
            st.set_dn_state(l, synth.dn_state(shape, SEED, l))
    st.set_kv_len(CTX0)

    def one_layer_step(i, h):
        # the token in flight passes layer l at the committed position; the
        # position advances once it has left the last layer
        l = layers[i % len(layers)]
        st.begin, st.end = l, l + 1
        out = st.forward(h, st.kv_len)
        st.commit(1)
        if l != layers[-1]:
            st.kv_len -= 1
        return out

    h = synth.hidden(shape, SEED, 0, 1).astype(np.float64)
    i = 0
    for _ in range(args.warmup):
        h = one_layer_step(i, h)
        i += 1
        if i % len(layers) == 0:
            h = synth.hidden(shape, SEED, i, 1).astype(np.float64)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        h = one_layer_step(i, h)
        i += 1
        if i % len(layers) == 0:
            h = synth.hidden(shape, SEED, i, 1).astype(np.float64)
    dt = time.perf_counter() - t0
    tokens = args.steps / len(layers)
    tok_s = tokens / dt
    cores = oracle.threads()
    cfg = workload_config(args, shape)
    return {
        "impl": "reference", "metric": METRIC, "value": tok_s, "unit": "tok/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": cfg,
        "cpu_baseline": {"value": tok_s, "unit": "tok/s", "cores": cores, "kind": "oracle",
                         "sample": f"{args.steps} steps of one decode token through one layer each "
                                   f"({tokens:g} tokens of the {args.layers}-layer stage from context {CTX0})"},
        "e2e": {"value": tok_s, "unit": "tok/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def run_ours(args, rank, world, local, pg):
    import torch

    import quantized_hybrid_layer_b200 as q
    q.lib()                                           # fails loudly without the CUDA library
    shape = FULL
    qtype = Q4_0 if args.qtype == "q4_0" else Q8_0
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.Stream(device=dev)
    layers = list(range(args.layers))
    max_ctx = ((CTX0 + 2 * (args.steps + args.warmup) + 64 + 63) // 64) * 64
    max_ctx = max(max_ctx, PROMPT + 64)

    tensors = gen_tensors(shape, qtype, SEED, 0, args.layers)
    cfg = q.config_from_shape(shape, qtype, max_ctx)
    with torch.cuda.stream(stream):
        st = q.stage_load(cfg, tensors, 0, args.layers, stream=stream)
        st.set_pass_mode(q.PASS_PERSISTENT if args.pass_mode == "persistent" else q.PASS_KERNELS)
        persistent = st.pass_persistent(1)
        for l in layers:
            if shape.is_attention(l):
                K, V = synth.kv_prefill(shape, SEED, l, CTX0, max_ctx)
                st.set_kv(l, K, V)
            else:
                st.set_dn_state(l, synth.dn_state(shape, SEED, l))
        st.set_kv_len(CTX0)

        H = shape.hidden
        n_steps = args.warmup + args.steps
        hid = torch.from_numpy(synth.normal_f32(synth.rng_for(SEED, rank, 77), (n_steps, H))).to(dev)
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

        # ---- decode, inputs resident in HBM ----
        for i in range(args.warmup):
            st.forward(hid[i:i + 1], st.committed_len)
            st.commit(1)
        st.sync()
        clocks = ClockSampler(local)
        barrier(pg)
        torch.cuda.synchronize()
        clocks.start()
        ev0.record(stream)
        for i in range(args.warmup, n_steps):
            st.forward(hid[i:i + 1], st.committed_len)
            st.commit(1)
        ev1.record(stream)
        torch.cuda.synchronize()
        barrier(pg)
        clk = clocks.stop()
        st.sync()
        dt = max_over_ranks(ev0.elapsed_time(ev1) / 1e3, pg)
        ctx_mid = CTX0 + args.warmup + args.steps // 2
        pb = pass_bytes(shape, qtype, layers, ctx_mid)
        tok_s = args.steps / dt
        value = tok_s * world

        # ---- end to end through the C ABI's host-buffer call (stage_forward_host):
        # every step copies its input from page-locked host memory, runs the
        # pass and copies the result back, all inside the timed region ----
        e2e = None
        if not args.no_e2e:
            host_in = torch.from_numpy(synth.normal_f32(synth.rng_for(SEED, rank, 78), (n_steps, H))).pin_memory()
            host_out = torch.empty((n_steps, H), dtype=torch.float32).pin_memory()
            for i in range(args.warmup):
                st.forward_host_buffers(host_in[i:i + 1], host_out[i:i + 1], st.committed_len, sync=False)
                st.commit(1)
            torch.cuda.synchronize()
            barrier(pg)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for i in range(args.warmup, n_steps):
                st.forward_host_buffers(host_in[i:i + 1], host_out[i:i + 1], st.committed_len, sync=False)
                st.commit(1)
            e1.record(stream)
            torch.cuda.synchronize()
            barrier(pg)
            st.sync()
            dte = max_over_ranks(e0.elapsed_time(e1) / 1e3, pg)
            e2e = {"value": args.steps / dte * world, "unit": "tok/s", "h2d_bytes_per_step": H * 4,
                   "d2h_bytes_per_step": H * 4, "call": "stage_forward_host (page-locked host buffers)"}

        # ---- prefill: 16-token chunks over a 2048-token prompt from position 0 ----
        prefill = None
        if not args.no_prefill:
            st.reset()
            n_chunks = min(PROMPT // CHUNK, args.prefill_chunks) if args.prefill_chunks > 0 else PROMPT // CHUNK
            ph = torch.from_numpy(synth.normal_f32(synth.rng_for(SEED, rank, 79), (n_chunks, CHUNK, H))).to(dev)
            st.prefill(ph[0].clone(), 0, chunked=True)      # builds the 16-token prefill graph
            st.reset()
            torch.cuda.synchronize()
            barrier(pg)
            p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            p0.record(stream)
            for c in range(n_chunks):
                st.prefill(ph[c], c * CHUNK, chunked=True)
            p1.record(stream)
            torch.cuda.synchronize()
            barrier(pg)
            st.sync()
            dtp = max_over_ranks(p0.elapsed_time(p1) / 1e3, pg)
            pbp = pass_bytes(shape, qtype, layers, PROMPT // 2, CHUNK)
            prefill = {"tok_s": n_chunks * CHUNK / dtp * world, "ms_per_chunk": dtp / n_chunks * 1e3,
                       "weight_gbs": pbp["weights"] * n_chunks / dtp / 1e9, "chunks": n_chunks,
                       "call": "stage_prefill, chunked DeltaNet form"}

        weight_bytes_packed = st.weight_bytes
        st.free()

    # ---- the dominant kernel alone: the dequant-GEMV on the stage's largest projection ----
    roof = None
    peaks = measured_peaks()
    hbm_peak = peaks.get("hbm_gbs")
    peak_src = "measured" if hbm_peak else "fallback"
    hbm_peak = hbm_peak or FALLBACK_HBM_GBS
    if not args.no_kernel_roofline:
        roof = gemv_roofline(q, torch, dev, stream, shape, qtype, hbm_peak, peak_src)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        sec_per_tok, cores = oracle_decode_sample(shape, qtype, tensors, layers)
        cpu = {"value": 1.0 / sec_per_tok, "unit": "tok/s", "cores": cores, "kind": "oracle",
               "sample": f"one decode token at position {CTX0} through all {args.layers} layers (f64 oracle)"}

    if rank != 0:
        return None
    weight_gbs = pb["weights"] * args.steps / dt / 1e9
    res = {
        "metric": METRIC, "value": value, "unit": "tok/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": workload_config(args, shape),
        "weight_gbs": weight_gbs, "weight_frac_of_8tbs": weight_gbs / NOMINAL_HBM_GBS,
        f"weight_frac_of_{peak_src}_copy_peak": weight_gbs / hbm_peak,
        "total_gbs": pb["total"] * args.steps / dt / 1e9,
        "bytes_per_pass": pb, "packed_weight_bytes": weight_bytes_packed,
        "prefill": prefill,
        "roofline": roof,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": (launches_per_pass(shape, layers, persistent) + 1) * args.steps,
        "pass_mode": "persistent" if persistent else "kernels",
        "clocks": clk,
    }
    return res


def gemv_roofline(q, torch, dev, stream, shape, qtype, hbm_peak, peak_src):
    """Time the GEMV kernel alone (same kernel, grid and block as in the pass, n_tok 1)
    on the stage's largest projection, gate+up as one [2*FFN, hidden] matrix, over
    copies whose total exceeds L2, with CUDA events on its stream."""
    rows, cols = 2 * shape.ffn, shape.hidden
    nbytes = q.qhl_packed_bytes(qtype, rows, cols)
    copies = max(8, int(np.ceil(2.0e9 / nbytes)))
    item = 18432 if qtype == Q4_0 else 34816     # packed item: 128 rows x 256 columns
    qb = 16384 if qtype == Q4_0 else 32768       # quants first, then the block scales
    mats = []
    with torch.cuda.stream(stream):
        g = torch.Generator(device=dev)
        g.manual_seed(SEED)
        for _ in range(copies):
            P = torch.randint(0, 256, (nbytes,), dtype=torch.uint8, device=dev, generator=g)
            P.view(-1, item)[:, qb:] = 0x20       # every f16 scale = 0x2020 (about 0.008)
            mats.append(P)
        x = torch.randn((1, cols), device=dev, generator=g)
        y = torch.empty((1, rows), device=dev)
        for P in mats[:4]:
            q.qhl_qgemv(qtype, rows, cols, P, x, y, stream=stream)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        reps = 3
        e0.record(stream)
        for _ in range(reps):
            for P in mats:
                q.qhl_qgemv(qtype, rows, cols, P, x, y, stream=stream)
        e1.record(stream)
        torch.cuda.synchronize()
    per_launch = e0.elapsed_time(e1) / 1e3 / (reps * len(mats))
    algo = rows * cols // 32 * synth.BLOCK_BYTES[qtype]
    achieved = algo / per_launch / 1e9
    del mats
    return {"kernel": "qgemv_kernel (dequant-GEMV, n_tok 1)", "shape": f"[{rows} x {cols}] {'Q4_0' if qtype == Q4_0 else 'Q8_0'}",
            "bound": "hbm", "achieved": achieved, "peak": hbm_peak, "peak_source": f"{peak_src} copy bandwidth (burst)",
            "unit": "GB/s", "frac": achieved / hbm_peak, "traffic": committed_traffic(),
            "algorithmic_bytes_per_launch": algo, "us_per_launch": per_launch * 1e6}


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=256)
    ap.add_argument("--warmup", type=int, default=8)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--layers", type=int, default=64)
    ap.add_argument("--qtype", choices=("q4_0", "q8_0"), default="q4_0")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-prefill", action="store_true")
    ap.add_argument("--prefill-chunks", type=int, default=0,
                    help="time only the first N 16-token chunks of the prompt (0: all; for short profiling runs)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-kernel-roofline", action="store_true")
    ap.add_argument("--pass-mode", choices=("kernels", "persistent"), default="kernels",
                    help="decode pass as a chain of kernels (CUDA graph) or as one persistent kernel")
    ap.add_argument("--only-kernel-roofline", action="store_true",
                    help="time only the dominant kernel alone (the GEMV roofline leg) and print it")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    rank, world, local, pg = dist_setup(args.gpus)
    try:
        if args.only_kernel_roofline:
            import torch

            import quantized_hybrid_layer_b200 as q
            q.lib()
            dev = torch.device("cuda", local)
            torch.cuda.set_device(dev)
            peaks = measured_peaks()
            hbm = peaks.get("hbm_gbs")
            roof = gemv_roofline(q, torch, dev, torch.cuda.Stream(device=dev), FULL,
                                 Q4_0 if args.qtype == "q4_0" else Q8_0, hbm or FALLBACK_HBM_GBS,
                                 "measured" if hbm else "fallback")
            if rank == 0:
                print(json.dumps({"roofline": roof}), flush=True)
            return
        if args.impl == "reference":
            res = run_reference(args, rank, world, pg)
        else:
            res = run_ours(args, rank, world, local, pg)
        if rank == 0 and res is not None:
            print(json.dumps(res), flush=True)
    finally:
        dist_teardown(pg)


if __name__ == "__main__":
    main()
