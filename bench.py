#!/usr/bin/env python
"""Throughput of the ALBERT phoneme-encoder forward pass on B200 (one JSON line).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

A step is one whole forward pass (embedding + LN, 128->768 projection, 12
executions of the shared layer, 768->512 projection) over one synthetic batch:
by default 256 sequences padded to T=128 with lengths uniform in [16, 128],
packed by length inside the library.  `value` counts valid tokens per second
over all ranks; every rank runs its own batch (sequences are independent:
weak scaling, no collective on the data path).  L2 is flushed (512 MiB write)
between timed steps; step times are CUDA-event times of the forward alone,
max over ranks.

`--impl reference` times the fp64 CPU oracle on the host cores instead (each
step: one sequence of the same workload), rank 0 only.

`--all-configs` prints one line per workload of the suite instead: b8_T128,
b64_T128_normal, b32_T512_long (packed), b256_T128 packed and padded, and the
batch-1 latency case b1_T64 as stream launches and as a CUDA-graph replay.

Tensor-peak fractions divide by the measured burst bf16 peak: the kernels are
timed for tens of microseconds inside steps of a few milliseconds, not in the
seconds-long loop the sustained figure describes (reported beside it).
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

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "encoder tokens/sec (BF16, 1×B200) and % of dense BF16 tensor peak"
UNIT = "tokens/s"
# Used only when MEASURED_PEAKS.json is absent: an earlier measurement on the
# same kind of B200 (STREAM-style copy; cuBLAS bf16 GEMM as a burst).
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}


# ------------------------------------------------------------- accounting ----

def flops_per_class(lengths, arch, rows):
    """Algorithmic FLOPs of one launch of each kernel class.  `rows` = rows the
    GEMMs process (valid tokens when packed); attention counts valid keys only."""
    H, E, F, O = arch["hidden"], arch["emb"], arch["ffn"], arch["out_dim"]
    s2 = float(sum(int(l) ** 2 for l in lengths))
    return {
        "gemm_in_proj": 2.0 * rows * E * H,
        # the embedding and the input projection in one kernel (its products are the in-projection's)
        "embed_proj": 2.0 * rows * E * H,
        "gemm_qkv": 2.0 * rows * H * 3 * H,
        "attention": 4.0 * s2 * H,
        "gemm_out_proj_ln": 2.0 * rows * H * H,
        "gemm_ffn_up_gelu": 2.0 * rows * H * F,
        "gemm_ffn_down_ln": 2.0 * rows * F * H,
        "gemm_final_proj": 2.0 * rows * H * O,
        # the whole forward after the embedding in one persistent kernel (batches of at most 128 rows)
        "small_batch_forward": forward_flops(lengths, arch)[0],
    }


def forward_flops(lengths, arch):
    """(whole forward, its GEMMs) in algorithmic FLOPs over the valid tokens."""
    H, E, F, O = arch["hidden"], arch["emb"], arch["ffn"], arch["out_dim"]
    n_tok = float(sum(int(l) for l in lengths))
    s2 = float(sum(int(l) ** 2 for l in lengths))
    gemm = 2.0 * n_tok * (E * H + arch["n_exec"] * (H * 3 * H + H * H + H * F + F * H) + H * O)
    return gemm + arch["n_exec"] * 4.0 * s2 * H, gemm


# DRAM traffic per launch of a kernel class, from ncu captures summarised in
# profiles/dram_traffic_<workload>.txt.  A line there records the digest of the
# kernel's sources at capture time; the figure is reported only while the
# sources are unchanged.
TRAFFIC_GLOB = os.path.join(os.path.dirname(os.path.abspath(__file__)), "profiles", "dram_traffic_*.txt")
CLASS_SOURCES = {
    "gemm": ["gemm_tcgen05.cu", "sm100_ptx.cuh", "kernels.h"],
    "attention": ["attention_tc.cu", "sm100_ptx.cuh", "kernels.h"],            # longest sequence <= 128
    "attention_long": ["attention_tc_long.cu", "sm100_ptx.cuh", "kernels.h"],  # 128 < longest <= 512
    "quant": ["fp8.cu", "sm100_ptx.cuh", "kernels.h"],
    "small": ["forward_small.cu", "sm100_ptx.cuh", "kernels.h"],
    "embed_proj": ["embed_proj.cu", "sm100_ptx.cuh", "kernels.h"],
}


def source_set(cls: str, seq_len: int = 128) -> str:
    if cls.startswith("gemm_"):
        return "gemm"
    if cls == "quant_e4m3":
        return "quant"
    if cls == "small_batch_forward":
        return "small"
    if cls == "embed_proj":
        return "embed_proj"
    return "attention" if seq_len <= 128 else "attention_long"


def sources_digest(cls: str, seq_len: int = 128) -> str:
    import hashlib
    csrc = os.path.join(os.path.dirname(os.path.abspath(__file__)), "transformer_encoder_albert_b200", "csrc")
    h = hashlib.sha256()
    for f in CLASS_SOURCES[source_set(cls, seq_len)]:
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def load_traffic(cls: str, workload: str, seq_len: int = 128):
    """(bytes per launch, note) for a class, or (None, reason)."""
    import glob
    files = sorted(glob.glob(TRAFFIC_GLOB))
    if not files:
        return None, "no ncu capture summarised"
    want = sources_digest(cls, seq_len)
    for path in files:
        with open(path) as fh:
            for ln in fh.read().splitlines():
                kv = dict(x.split("=", 1) for x in ln.split() if "=" in x)
                if kv.get("class") == cls and kv.get("workload") == workload:
                    if kv.get("sources") != want:
                        return None, "kernel changed since the ncu capture"
                    return float(kv["dram_bytes_per_launch"]), "ncu capture, " + os.path.basename(path)
    return None, "class not in the ncu capture"


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ---------------------------------------------------------------- clocks -----

class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.lines = []
        self.t = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu_id}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.t = threading.Thread(target=self._read, daemon=True)
        self.t.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            if self.t is not None:
                self.t.join(timeout=2)

    def summary(self, t0, t1):
        rows = []
        for ts, line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 8:
                continue
            rows.append((ts, parts))
        inside = [p for ts, p in rows if t0 <= ts <= t1] or [p for _, p in rows]
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(p[0]) for p in inside if num(p[0]) is not None]
        mx = [num(p[1]) for p in inside if num(p[1]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for p in inside for i in range(4) if p[4 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(inside)}


def nvidia_smi_id(torch, local: int) -> str:
    """nvidia-smi --id for the CUDA device `local`: its UUID, else its index."""
    try:
        uu = torch.cuda.get_device_properties(local).uuid
        raw = getattr(uu, "bytes", None)
        if raw is not None and len(raw) == 16:
            h = bytes(raw).hex()
            return f"GPU-{h[:8]}-{h[8:12]}-{h[12:16]}-{h[16:20]}-{h[20:]}"
        u = str(uu)
        if u and not u.startswith("<"):
            return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        pass
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        return vis.split(",")[local].strip()
    return str(local)


# -------------------------------------------------------------- oracle arm ---

def oracle_throughput(weights, ids, mask, L, arch, budget_s=None, steps=None, warmup=0):
    """Time the fp64 CPU oracle, one sequence per step (round robin over the batch)."""
    import oracle
    oracle.set_threads(os.cpu_count() or 1)
    m = oracle.Model(weights, arch)
    order = list(range(len(L)))
    tok, secs, done, i = 0, 0.0, 0, 0
    for _ in range(warmup):
        b = order[i % len(order)]; i += 1
        m.encode(ids[b, :L[b]], mask[b, :L[b]])
    while True:
        b = order[i % len(order)]; i += 1
        t0 = time.perf_counter()
        m.encode(ids[b, :L[b]], mask[b, :L[b]])
        secs += time.perf_counter() - t0
        tok += int(L[b])
        done += 1
        if steps is not None and done >= steps:
            break
        if budget_s is not None and secs >= budget_s:
            break
    return tok / secs, done, tok, secs, oracle.num_threads()


def workload_label(wl, args) -> str:
    """config.workload of both arms: the workload and whether the GEMMs run on the
    packed valid rows or on all B*T padded rows."""
    return wl.name + ("_padded" if args.padded else "_packed")


def run_reference(args):
    import synth
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    wl = synth.WORKLOADS[args.workload]
    w = synth.make_weights(seed=1234, bf16=True)
    ids, mask, L = synth.make_batch(wl)
    value, done, tok, secs, cores = oracle_throughput(w, ids, mask, L, synth.ARCH, steps=args.steps,
                                                      warmup=args.warmup)
    sample = f"{done} whole sequences of the {wl.name} batch ({tok} valid tokens), one per step"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000.0 * secs / max(done, 1),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded N(0,0.02) weights rounded to bf16, seeded ids and lengths)",
        "config": {"workload": workload_label(wl, args), "batch": wl.B, "seq_len": wl.T, "lengths": wl.describe()},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------- multi-rank ----

def measure_length_regulation(torch, synth, tea, L, flush, peaks, peaks_src, stream, steps):
    """Length regulation (the step after the encoder) on the same batch: its tokens
    packed, 50 duration channels, 512-wide bf16 features.  HBM-bound: algorithmic
    bytes = logits + features read, durations / frame starts / frames written."""
    import numpy as np
    n = int(np.sum(L))
    cu = torch.tensor(np.concatenate([[0], np.cumsum(L)]), dtype=torch.int32, device="cuda")
    C, D = synth.DURATION_CHANNELS, 512
    z = torch.tensor(synth.make_duration_logits(n, C), device="cuda")
    f = torch.tensor(synth.make_features(n, D), device="cuda").to(torch.bfloat16)
    st, dur, start, cuf, frames = tea.length_regulate(z, f, cu, speed=1.0, max_frames=16 * n)
    if st != 0:
        raise SystemExit(f"length regulation status {st}")
    A = int(cuf[-1].item())
    ms = []
    P = tea._ptr
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    scratch = torch.empty(int(tea.lib().albert_length_regulate_scratch_bytes(n)), dtype=torch.uint8, device="cuda")
    for k in range(steps + 3):
        flush.zero_()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        tea.lib().albert_length_regulate(P(z), C, 1.0, P(f), D, P(cu), len(L), n, P(dur), P(start), P(cuf),
                                         P(frames), frames.shape[0], P(scratch), P(status), tea._stream_ptr())
        e1.record(stream)
        torch.cuda.synchronize()
        if k >= 3:
            ms.append(e0.elapsed_time(e1))
    t = sum(ms) / len(ms)
    nbytes = n * C * 4 + n * D * 2 + n * 8 + A * D * 2 + 8 * (len(L) + 1)
    hbm = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    achieved = nbytes / (t / 1000.0) / 1e9
    return {"tokens": n, "frames": A, "channels": C, "width": D, "ms": t, "tokens_per_s": n / (t / 1000.0),
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
                         "bytes_per_launch": nbytes, "peak_source": f"{peaks_src} hbm_gbs"},
            "launches": 3, "l2": "flushed before each timed launch"}


def rank_batch_seed(base_seed: int, rank: int) -> int:
    """Each rank encodes its own batch of the workload (weak scaling)."""
    return base_seed + 1000 * rank


def max_over_ranks(x: float, dist=None, device="cpu") -> float:
    """Max of a per-rank float over all ranks (the job's time is its slowest rank's)."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(x)
    import torch
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float, dist=None, device="cpu") -> float:
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(x)
    import torch
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def job_throughput(local_tokens: float, local_ms: float, dist=None, device="cpu") -> float:
    """All ranks' tokens divided by the slowest rank's time (tokens/s)."""
    return sum_over_ranks(local_tokens, dist, device) / (max_over_ranks(local_ms, dist, device) / 1000.0)


# ---------------------------------------------------------------- GPU arm ----

def run_gpu(args):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        if world == 1 and args.gpus > 1:
            raise SystemExit("--gpus N > 1 needs torchrun with N processes")
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    ctx = {"world": world, "rank": rank, "local": local, "dist": dist, "dev": torch.device("cuda", local)}
    if args.all_configs:
        runs = [("b8_T128", False, False), ("b64_T128_normal", False, False), ("b32_T512_long", False, False),
                ("b256_T128", False, False), ("b256_T128", True, False), ("b1_T64_latency", False, False),
                ("b1_T64_latency", False, True)]
    else:
        runs = [(args.workload, args.padded, args.graph)]
    for name, padded, graph in runs:
        line = measure_workload(args, ctx, name, padded, graph, extras=not args.all_configs)
        if rank == 0 and line is not None:
            print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def measure_workload(args, ctx, name, padded, graph_mode, extras):
    """One JSON line for one workload: device-timed forwards, live roofline of the
    dominant kernel class, per-class breakdown, end-to-end host-buffer figure and
    the oracle's CPU throughput.  extras: also the length-regulation leg."""
    import numpy as np
    import torch

    import synth
    import transformer_encoder_albert_b200 as tea

    world, rank, local, dist, dev = ctx["world"], ctx["rank"], ctx["local"], ctx["dist"], ctx["dev"]

    def barrier():
        if world > 1:
            dist.barrier()

    max_r = lambda x: max_over_ranks(x, dist, dev)
    sum_r = lambda x: sum_over_ranks(x, dist, dev)

    arch = synth.ARCH
    wl = synth.WORKLOADS[name]
    label = wl.name + ("_padded" if padded else "_packed")
    w = synth.make_weights(seed=1234, bf16=True)
    ids, mask, L = synth.make_batch(wl, seed=rank_batch_seed(wl.seed, rank))
    n_tok = int(L.sum())
    ids_d = torch.as_tensor(ids).cuda()
    mask_d = torch.as_tensor(mask).cuda()
    enc = tea.Encoder(w, arch, dtype=args.dtype, max_tokens=wl.B * wl.T, pack=not padded)
    enc.set_small_batch_kernel(args.small_batch == "on")
    out = torch.empty(wl.B, wl.T, arch["out_dim"], device="cuda", dtype=torch.bfloat16)
    stream = torch.cuda.current_stream()
    rows = n_tok if not padded else wl.B * wl.T
    per_launch = flops_per_class(L, arch, rows)
    fwd_flops, gemm_flops = forward_flops(L, arch)

    if args.ncu_forwards:
        # untimed forwards only, for a profiler's launch list or kernel capture
        for _ in range(args.ncu_forwards):
            enc.forward(ids_d, mask_d, out)
        torch.cuda.synchronize()
        st = enc.status()
        enc.close()
        if st != 0:
            raise SystemExit(f"device status {st}")
        return {"ncu_forwards": args.ncu_forwards, "workload": wl.name, "tokens": n_tok}

    # which kernel dominates: a short all-class profile before the timed region, after
    # one untimed forward (a kernel's first launch loads its module, which the event
    # pair around that launch would count)
    enc.forward(ids_d, mask_d, out)
    torch.cuda.synchronize()
    enc.profile(None)
    for _ in range(3):
        enc.forward(ids_d, mask_d, out)
    prof0 = enc.profile_read()
    enc.profile([])
    enc.profile_reset()
    dominant = max(prof0, key=lambda k: prof0[k][1])

    for _ in range(args.warmup):
        enc.forward(ids_d, mask_d, out)
    if enc.status() != 0:
        raise SystemExit(f"device status {enc.status()}")
    flush = torch.empty(512 * 1024 * 1024, dtype=torch.uint8, device="cuda")

    sampler = ClockSampler(nvidia_smi_id(torch, local))
    sampler.start()
    time.sleep(0.5)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    # Only the dominant class is timed live, one of its launches per step (a
    # middle one): an event pair between launches breaks their chaining, so
    # fewer pairs disturb the step less.
    per_step = max(1, round(prof0[dominant][0] / 3))
    enc.profile([dominant])
    enc.profile_stride(per_step, per_step // 2)
    graph = None
    if graph_mode:
        # One forward captured in a CUDA graph (the chained launches become
        # programmatic edges); its dominant-class events are re-recorded by every
        # replay and read after it.
        enc.profile_retain(True)
        graph = torch.cuda.CUDAGraph()
        torch.cuda.synchronize()
        with torch.cuda.graph(graph):
            enc.forward(ids_d, mask_d, out)
        for _ in range(args.warmup):
            flush.zero_()
            graph.replay()
        torch.cuda.synchronize()
        enc.profile_reset()
    barrier()
    torch.cuda.synchronize()
    t_wall0 = time.time()
    dom = None
    for k in range(args.steps):
        flush.zero_()
        starts[k].record(stream)
        if graph is not None:
            graph.replay()
        else:
            enc.forward(ids_d, mask_d, out)
        ends[k].record(stream)
        if graph is not None:
            dom = enc.profile_read()[dominant]  # waits for this replay, adds its times
    torch.cuda.synchronize()
    barrier()
    t_wall1 = time.time()
    sampler.stop()
    st = enc.status()
    if st != 0:
        raise SystemExit(f"device status {tea.STATUS_NAMES.get(st, st)}")
    step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    launches = enc.last_forward_launches()  # kernels of one timed forward (the captured one for a graph)
    if graph is None:
        dom = enc.profile_read()[dominant]
    enc.profile_retain(False)
    enc.profile_stride(1, 0)
    enc.profile([])
    enc.profile_reset()
    del graph
    total_ms = max_r(sum(step_ms))
    tokens_all = sum_r(float(n_tok * args.steps))
    value = tokens_all / (total_ms / 1000.0)
    ms_per_step = total_ms / args.steps

    # graph mode: the same steps as stream launches, for comparison (the graph
    # loop reads the profiler after every replay, so the GPU idles between steps)
    stream_ms = None
    if graph_mode:
        sms = []
        for _ in range(min(args.steps, 20)):
            flush.zero_()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            enc.forward(ids_d, mask_d, out)
            e1.record(stream)
            torch.cuda.synchronize()
            sms.append(e0.elapsed_time(e1))
        stream_ms = max_r(sum(sms) / len(sms))

    # per-kernel breakdown: a profiled replay of a few steps (all classes); the
    # event pair around every launch breaks their programmatic chaining, so these
    # class times sum to more than the timed step
    enc.profile(None)
    n_prof = min(args.steps, 10)
    for _ in range(n_prof):
        flush.zero_()
        enc.forward(ids_d, mask_d, out)
    prof = enc.profile_read()
    enc.profile([])
    gemm_classes = [c for c in prof if c.startswith("gemm_")]
    gemm_ms = sum(prof[c][1] for c in gemm_classes) / n_prof
    breakdown = {c: {"launches_per_step": prof[c][0] / n_prof, "ms_per_step": prof[c][1] / n_prof}
                 for c in prof if prof[c][0]}

    # end to end through the public C calls with pinned host buffers: every step
    # copies its ids/mask to the device and its output back to the host.  The
    # pipelined call overlaps a step's output copy with the next step's forward;
    # the synchronous call is measured too, for reference.
    ids_h = torch.as_tensor(ids).pin_memory()
    mask_h = torch.as_tensor(mask).pin_memory()
    outs_h = [torch.empty(wl.B, wl.T, arch["out_dim"], dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    n_e2e = args.steps

    def timed_host_loop(pipelined: bool) -> float:
        e_s = torch.cuda.Event(enable_timing=True)
        e_e = torch.cuda.Event(enable_timing=True)
        barrier()
        torch.cuda.synchronize()
        e_s.record(stream)
        for k in range(n_e2e):
            if pipelined:
                rc = enc.forward_host_async(ids_h, mask_h, outs_h[k & 1])
            else:
                rc = enc.forward_host(ids_h, mask_h, outs_h[0])
            if rc != 0:
                raise SystemExit(f"host path status {rc}")
        if pipelined and enc.forward_host_wait() != 0:
            raise SystemExit("host path status")
        e_e.record(stream)  # all host copies have completed when this is recorded
        torch.cuda.synchronize()
        return max_r(e_s.elapsed_time(e_e))

    # the same through the packed host call: only the valid rows' ids travel in and
    # only the valid rows' outputs travel back
    packed_h = torch.as_tensor(np.concatenate([ids[b, :L[b]] for b in range(wl.B)])).pin_memory()
    cu_h = torch.as_tensor(np.concatenate([[0], np.cumsum(L)]).astype(np.int32)).pin_memory()
    pouts_h = [torch.empty(n_tok, arch["out_dim"], dtype=torch.bfloat16).pin_memory() for _ in range(2)]

    def timed_packed_loop() -> float:
        e_s = torch.cuda.Event(enable_timing=True)
        e_e = torch.cuda.Event(enable_timing=True)
        barrier()
        torch.cuda.synchronize()
        e_s.record(stream)
        for k in range(n_e2e):
            if enc.forward_varlen_host_async(packed_h, cu_h, int(L.max()), pouts_h[k & 1]) != 0:
                raise SystemExit("packed host path status")
        if enc.forward_host_wait() != 0:
            raise SystemExit("packed host path status")
        e_e.record(stream)
        torch.cuda.synchronize()
        return max_r(e_s.elapsed_time(e_e))

    timed_host_loop(True)  # warm-up: allocates the second staging slot
    e2e_ms = timed_host_loop(True)
    e2e_packed_value = None
    if not padded and wl.T <= 512:
        timed_packed_loop()
        e2e_packed_value = sum_r(float(n_tok * n_e2e)) / (timed_packed_loop() / 1000.0)
    e2e_value = sum_r(float(n_tok * n_e2e)) / (e2e_ms / 1000.0)
    e2e_sync_value = sum_r(float(n_tok * n_e2e)) / (timed_host_loop(False) / 1000.0)
    out_h = outs_h[0]

    peaks, peaks_src = load_peaks()
    peak = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    peak_sus = peaks.get("bf16_tflops_sustained")
    peak_note = f"{peaks_src} bf16_tflops (burst)"
    fp8_classes = ("gemm_qkv", "gemm_out_proj_ln", "gemm_ffn_up_gelu", "gemm_ffn_down_ln")
    if args.dtype == "fp8":
        # E4M3 products: the measured bf16 peak times the nominal dense fp8 / bf16 ratio (2)
        peak, peak_sus = 2.0 * peak, (2.0 * peak_sus if peak_sus else None)
        peak_note = f"{peaks_src} bf16_tflops (burst) x 2, the nominal dense E4M3 / bf16 ratio"
    lenreg = (measure_length_regulation(torch, synth, tea, L, flush, peaks, peaks_src, stream, args.steps)
              if extras else None)
    dom_ms = dom[1] / max(dom[0], 1)
    achieved = per_launch.get(dominant, 0.0) / (dom_ms / 1000.0) / 1e12
    if dominant == "quant_e4m3":
        # HBM-bound: bf16 rows read, E4M3 codes and a scale per row written.  Per
        # execution the quantized inputs are Q|K|V's, the out-projection's and FFN
        # up's (768 wide) and FFN down's (2048 wide), in that order; the timed
        # launch is launch per_step // 2 of each forward
        k_timed = 2048 if (per_step // 2) % 4 == 3 else 768
        qbytes = rows * k_timed * 3.0 + rows * 4
        hbm = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
        roofline_hbm = {"kernel": dominant, "bound": "hbm", "achieved": qbytes / (dom_ms / 1000.0) / 1e9,
                        "peak": hbm, "unit": "GB/s", "bytes_per_launch": qbytes,
                        "peak_source": f"{peaks_src} hbm_gbs"}
        roofline_hbm["frac"] = roofline_hbm["achieved"] / hbm
    else:
        roofline_hbm = None
    # E4M3 runs have their own capture (workload label + "_e4m3")
    traffic, traffic_note = load_traffic(dominant, label + ("_e4m3" if args.dtype == "fp8" else ""), wl.T)
    bound = "tensor"
    dom_peak = peak if (args.dtype == "bf16" or dominant in fp8_classes) else peak / 2.0
    roofline = {"kernel": dominant, "bound": bound, "achieved": achieved, "peak": dom_peak,
                "unit": "TFLOP/s", "frac": achieved / dom_peak, "traffic": traffic, "traffic_source": traffic_note,
                "peak_source": f"{peak_note} (the kernel runs {dom_ms * 1000:.0f} us inside a {ms_per_step:.3f} ms step)",
                "frac_of_sustained": (achieved / peak_sus) if peak_sus else None,
                "launches_timed": dom[0], "launches_timed_note": f"1 of {per_step} per step", "avg_launch_ms": dom_ms,
                "flops_per_launch": per_launch.get(dominant, 0.0)}
    if roofline_hbm is not None:
        roofline_hbm.update({"launches_timed": dom[0], "avg_launch_ms": dom_ms, "traffic": traffic,
                             "traffic_source": traffic_note})
        roofline = roofline_hbm
    clocks = sampler.summary(t_wall0, t_wall1)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if args.dtype == "bf16" else "e4m3 (the four layer GEMMs) + bf16",
        "data": "synthetic (seeded N(0,0.02) weights rounded to bf16, seeded ids and lengths)",
        "config": {"workload": label, "batch": wl.B,
                   "seq_len": wl.T, "lengths": wl.describe(), "valid_tokens_per_step_per_gpu": n_tok,
                   "padded_slot_tokens_per_step_per_gpu": wl.B * wl.T,
                   "pack": not padded, "parallelism": f"replicas x{world}",
                   "launch": "cuda_graph" if graph_mode else "stream",
                   "small_batch_kernel": args.small_batch,
                   "l2": "flushed between timed steps (512 MiB write)"},
        "padded_slot_tokens_per_s": sum_r(float(wl.B * wl.T * args.steps)) / (total_ms / 1000.0),
        "tensor_peak_frac": {"whole_encoder": fwd_flops / (ms_per_step / 1000.0) / 1e12 / peak,
                             "gemm_path": (gemm_flops / (gemm_ms / 1000.0) / 1e12 / peak) if gemm_ms > 0 else None,
                             "gemm_path_source": "per-class profiled replay (an event pair around every launch "
                                                 "breaks their chaining: a lower bound)" if gemm_ms > 0 else
                                                 "no separate GEMM launches (one persistent kernel)",
                             "peak_tflops": peak, "peak_source": peak_note,
                             "whole_encoder_of_sustained": (fwd_flops / (ms_per_step / 1000.0) / 1e12 / peak_sus)
                             if peak_sus else None},
        "roofline": roofline,
        "kernels": breakdown,
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": int(ids_h.numel() * 8 + mask_h.numel()),
                "d2h_bytes_per_step": int(out_h.numel() * 2),
                "api": "albert_forward_host_async (output copy of a step overlaps the next forward)",
                "synchronous_api_value": e2e_sync_value,
                "packed_api_value": e2e_packed_value,
                "packed_api": ("albert_forward_varlen_host_async (packed ids in, valid rows out: "
                               f"{int(packed_h.numel() * 8 + cu_h.numel() * 4)} B in, "
                               f"{int(n_tok * arch['out_dim'] * 2)} B out per step)")},
        "stream_launch_ms_per_step": stream_ms,
        "gpu_launches": launches * args.steps,
        "clocks": clocks,
    }
    if lenreg is not None:
        line["length_regulation"] = lenreg
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        budget = args.cpu_seconds if extras else min(args.cpu_seconds, 5.0)
        v, done, tok, secs, cores = oracle_throughput(w, ids, mask, L, arch, budget_s=budget)
        line["cpu_baseline"] = {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle",
                                "sample": f"{done} whole sequences of the same batch ({tok} valid tokens, "
                                          f"{secs:.1f} s of fp64 CPU work)"}
    enc.close()
    return line


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default="b256_T128")
    ap.add_argument("--padded", action="store_true", help="run the GEMMs on all B*T padded rows")
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--graph", action="store_true",
                    help="time replays of the forward captured in a CUDA graph instead of stream launches")
    ap.add_argument("--ncu-forwards", type=int, default=0,
                    help="run this many untimed forwards and exit (for ncu captures); no JSON metric line")
    ap.add_argument("--dtype", default="bf16", choices=["bf16", "fp8"],
                    help="fp8: the four layer GEMMs on E4M3 operands with per-row scales")
    ap.add_argument("--small-batch", default="on", choices=["on", "off"],
                    help="off: batches of at most 128 token rows also take the per-layer kernels")
    ap.add_argument("--all-configs", action="store_true",
                    help="one JSON line per workload of the suite (packed and padded b256, b1_T64 stream and graph)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
