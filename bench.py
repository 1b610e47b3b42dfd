#!/usr/bin/env python
"""Benchmark of the sm_100a Mamba-2 SSD hot path (prefill + cached decode).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Workload (per rank; ranks process independent batches, so scaling is weak):
  * prefill, the headline: the 2.7B-layer shape -- b=8 sequences x T=4096 tokens,
    H=80 heads, P=64, N=128, G=1, chunk 256, bf16 x/B/C, fp32 dt/A/D, h0 ~ N(0, 0.1).
    One step = one ssd_prefill call over that batch.  value = TFLOP/s of the chunked
    decomposition that ran (128-token chunks on the fused tensor-core path,
    chunk_executed); tokens/s does not depend on the decomposition.
  * cached decode at the 2.7B shape: 64 layers x (80 x 64 x 128) fp32 state + width-4
    conv over 5376 channels, batch 1 (and 32), state from the prefill's final state,
    run as graph launches of on-device steps; reported under "decode".
Inputs are seeded synthetic draws (ssd_inputs); the per-step prefill inputs (740 MB)
exceed the 126 MB L2, so no flush is needed between steps.

Prints ONE JSON line on rank 0.  gpu_launches counts our kernel launches inside the timed
region that `value` measures (three per step at the headline shape: the status reset, the
segment state pass for the pairs of the ragged last wave, the fused prefill);
gpu_launches_all_timed_regions adds those of the per-kernel timing, decode, raw-dt and
other-configuration regions.  --impl reference times the CPU oracle (the only
reference this method has: an fp64 C implementation of the recurrence) on bounded
samples of the same workload, in the same unit.
"""
from __future__ import annotations

import argparse
import hashlib
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

METRIC = "SSD prefill TFLOP/s + tokens/s; decode steps/s + HBM GB/s; % of roofline"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# nominal B200 figures, for context beside the measured ones: HBM3e per the HGX spec sheet
NOMINAL_HBM_GBS = 7700.0

# prefill workload (the 2.7B-layer configuration)
PB, PT, PH, PP, PN, PG, PL = 8, 4096, 80, 64, 128, 1, 256
# The fused tensor-core path (bf16, P = 64, N = 128) evaluates the chunked form with
# 128-token chunks whatever chunk length is requested (the same function; fewer FLOPs than
# L = 256).  TFLOP/s counts the FLOPs of the decomposition that ran; the L = 256 count is
# reported beside it.
EXEC_L_FUSED = 128
# decode workload (the 2.7B-shaped cache)
DL, DH, DP, DN, DG, DK = 64, 80, 64, 128, 1, 4


def peaks():
    if os.path.exists(PEAKS_FILE):
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return p, "measured"
    return FALLBACK_PEAKS, "fallback"


# ----------------------------------------------------------------------------- work counts
def prefill_flops(b, T, H, P, N, G, L):
    """Algorithmic FLOPs of the chunked dual form: per chunk and group the causal C.B^T
    triangle (diagonal included); per chunk and head the masked product with X (same
    triangle), the chunk state and the state-to-output term; plus the O(P N) scan."""
    nc_full, rem = divmod(T, L)
    lens = [L] * nc_full + ([rem] if rem else [])
    tri = sum(l * (l + 1) // 2 for l in lens)
    f = 2.0 * b * G * tri * N            # C.B^T, causal triangle, once per group
    f += 2.0 * b * H * tri * P           # (C.B^T o L) X
    f += 2.0 * b * H * T * P * N         # chunk states
    f += 2.0 * b * H * T * N * P         # state-to-output
    f += 2.0 * b * H * len(lens) * P * N  # inter-chunk recurrence
    return f


def prefill_bytes(b, T, H, P, N, G, io_bytes=2, with_h0=True):
    """Algorithmic HBM bytes: x, B, C, dt in, y out, h0 in, h_final out."""
    tok = b * T
    by = tok * H * P * io_bytes * 2 + tok * G * N * io_bytes * 2 + tok * H * 4
    by += b * H * P * N * 4 * (2 if with_h0 else 1) + 2 * H * 4
    return float(by)


def decode_bytes_per_step(layers, b, H, P, N, G, k=4, io_bytes=2):
    """State read+write, conv state read+write, step inputs, conv weights, A/D, y."""
    Dc = H * P + 2 * G * N
    st = 2.0 * layers * b * H * P * N * 4
    cv = 2.0 * layers * b * Dc * (k - 1) * 4
    inp = layers * b * (Dc * io_bytes + H * 4)
    w = layers * (Dc * k * 4 + Dc * 4 + 2 * H * 4)
    y = layers * b * H * P * io_bytes
    return st + cv + inp + w + y


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.idx = gpu_index
        self.proc = None
        self.lines = []
        self.windows = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except (OSError, ValueError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def mark(self, t0, t1):
        self.windows.append((t0, t1))

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ts, line in self.lines:
            if self.windows and not any(a - 0.15 <= ts <= b + 0.15 for a, b in self.windows):
                continue
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------------------- ranks
class Ranks:
    """One process per GPU, launched by torchrun: rank and world size from the launcher's
    environment, a barrier, and the max over ranks of a device-timed duration.  Ranks run
    independent batches (the prefill's (sequence, head) problems never interact), so the
    only collectives are the timing barrier and this max.  backend "nccl" on GPUs; the
    CPU tests use "gloo" with the same code."""

    def __init__(self, backend="nccl", device=None, timeout_s=120):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.device = device
        self.dist = None
        if self.world > 1:
            from datetime import timedelta
            import torch.distributed as dist
            kw = {"device_id": device} if backend == "nccl" else {}
            dist.init_process_group(backend, timeout=timedelta(seconds=timeout_s), **kw)
            self.dist = dist

    def barrier(self):
        if self.dist is not None:
            self.dist.barrier()

    def max(self, v):
        if self.dist is None:
            return float(v)
        import torch
        t = torch.tensor([float(v)], dtype=torch.float64, device=self.device)
        self.dist.all_reduce(t, op=self.dist.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.dist is not None:
            self.dist.destroy_process_group()
            self.dist = None


def rank_seed(rank, base=2):
    """Seed of a rank's synthetic batch: every rank draws its own sequences."""
    return base + 1000 * rank


def job_rate(units_per_rank, world, ms_max):
    """Whole-job throughput: the units all ranks processed over the slowest rank's time."""
    return units_per_rank * world / (ms_max * 1e-3)


# ----------------------------------------------------------------------------- helpers
def sha_prefix(path, upto=None):
    """sha256[:12] of a source file, or of its text before the first line that starts with
    `upto` (the part a kernel's code depends on, when later sections hold other kernels)."""
    with open(path, "rb") as f:
        data = f.read()
    if upto:
        i = data.find(b"\n" + upto.encode())
        if i >= 0:
            data = data[:i + 1]
    return hashlib.sha256(data).hexdigest()[:12]


# the fused prefill kernel and the helpers it uses end where the segment state pass begins
KERNEL_SOURCE_END = {"ssd_prefill_fused": "// ------------------------------------------------------------------ segment state pass"}


def dram_traffic(kernel):
    """Per-launch DRAM bytes of `kernel` from profiles/dram_traffic.txt, only if the kernel's
    source (the file up to KERNEL_SOURCE_END, else the whole file) is unchanged since the ncu
    capture (else None)."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    if not os.path.exists(path):
        return None
    for line in open(path):
        if line.startswith("#") or not line.strip():
            continue
        parts = line.split()
        if len(parts) >= 4 and parts[0] == kernel:
            src, sha, per_launch = parts[1], parts[2], float(parts[3])
            full = os.path.join(ROOT, src)
            if os.path.exists(full) and sha_prefix(full, KERNEL_SOURCE_END.get(kernel)) == sha:
                return per_launch
    return None


def oracle_prefill_sample(case, heads, seqs=(0,)):
    """Time the fp64 oracle recurrence on a (sequence x head) subset; returns seconds."""
    import oracle
    hpg = case.H // case.G
    x = case.x[list(seqs)][:, :, heads]
    dt = case.dt[list(seqs)][:, :, heads]
    B = case.B[list(seqs)][:, :, [h // hpg for h in heads]]
    C = case.C[list(seqs)][:, :, [h // hpg for h in heads]]
    h0 = None if case.h0 is None else case.h0[list(seqs)][:, heads]
    oracle.ssd_recurrence(x[:, :64], dt[:, :64], case.A[heads], B[:, :64], C[:, :64], case.D[heads], h0)
    t0 = time.perf_counter()
    oracle.ssd_recurrence(x, dt, case.A[heads], B, C, case.D[heads], h0)
    return time.perf_counter() - t0, oracle.max_threads()


def cpu_baseline(case, flops_per_tokhead, target_s=10.0):
    """The oracle as it stands on the host cores, on a bounded sample of the workload:
    8 heads of sequence 0 first, then as many (sequence, head) pairs as fit ~target_s."""
    t8, cores = oracle_prefill_sample(case, list(range(8)))
    pairs = int(min(case.b * case.H, max(8, 8 * target_s / max(t8, 1e-3))))
    seqs = max(1, min(case.b, pairs // case.H))
    heads = list(range(min(case.H, pairs if seqs == 1 else case.H)))
    t, cores = oracle_prefill_sample(case, heads, tuple(range(seqs)))
    n = seqs * len(heads)
    return {"value": flops_per_tokhead * case.T * n / t / 1e12, "unit": "TFLOP/s", "cores": cores,
            "kind": "oracle", "seconds": t,
            "sample": "fp64 oracle recurrence on %d sequence(s) x %d heads x %d tokens of this workload (%.1f s), "
                      "scaled by the algorithmic FLOPs per token-head" % (seqs, len(heads), case.T, t)}


# ----------------------------------------------------------------------------- reference arm
def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from ssd_inputs import make_config
    case = make_config("mamba2_2p7b_layer")
    flops_per_tokhead = prefill_flops(PB, PT, PH, PP, PN, PG, EXEC_L_FUSED) / (PB * PT * PH)
    heads = list(range(8))
    times = []
    for i in range(args.warmup + args.steps):
        dt_s, cores = oracle_prefill_sample(case, heads)
        if i >= args.warmup:
            times.append(dt_s)
    t = statistics.median(times)
    tokheads = PT * len(heads)
    value = flops_per_tokhead * tokheads / t / 1e12
    sample = "fp64 oracle recurrence, sequence 0 x heads 0-7 x 4096 tokens of the 2.7B-layer prefill per step"
    line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "impl": "reference", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": t * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": "mamba2_2p7b_layer_prefill", "b": PB, "T": PT, "H": PH, "P": PP, "N": PN,
                       "G": PG, "chunk": PL},
            "tokens_per_s": tokheads / PH / t,
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- our arm
def main():
    global PB
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--decode-steps", type=int, default=4096,
                    help="timed on-device decode steps per batch size (the cached-decode configuration's 4096)")
    ap.add_argument("--decode-batches", default="1,32")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--skip-loop-compare", action="store_true",
                    help="skip the decode loop and recompute comparisons")
    ap.add_argument("--skip-other-prefill", action="store_true",
                    help="skip the 130M-layer and long-context prefill timings")
    ap.add_argument("--prefill-batch", type=int, default=PB,
                    help="sequences per prefill step (default: the 2.7B-layer configuration's 8); "
                         "smaller values are for profiling captures only")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)

    import torch
    import state_space_model_04_b200 as ssd
    from ssd_inputs import make_config

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    ranks = Ranks("nccl", dev)
    world, rank = ranks.world, ranks.rank
    barrier, max_over_ranks = ranks.barrier, ranks.max

    pk, pk_kind = peaks()
    stream = torch.cuda.current_stream()

    # ---------------- prefill inputs (seeded per rank: independent batches)
    PB = args.prefill_batch
    case = make_config("mamba2_2p7b_layer", seed=rank_seed(rank), b=PB)
    def bf(bits):
        return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16)
    host = {"x": bf(case.x_bits), "B": bf(case.B_bits), "C": bf(case.C_bits),
            "dt": torch.from_numpy(case.dt), "A": torch.from_numpy(case.A), "D": torch.from_numpy(case.D),
            "h0": torch.from_numpy(case.h0)}
    pinned = {k: v.pin_memory() for k, v in host.items()}
    d = {k: v.to(dev) for k, v in host.items()}
    y = torch.empty_like(d["x"])
    hf = torch.empty_like(d["h0"])
    ws = torch.empty(ssd.prefill_workspace_size(PB, PT, PH, PP, PN, PG, PL, ssd.SSD_BF16), dtype=torch.uint8, device=dev)

    def prefill_step():
        ssd.prefill(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], chunk=PL, h0=d["h0"], y=y, h_final=hf,
                    workspace=ws)

    clocks = ClockSampler(local)
    clocks.start()
    for _ in range(args.warmup):
        prefill_step()
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    n0 = ssd.launch_count()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    w0 = time.time()
    e0.record(stream)
    step_ev = []  # an event after every step: per-step times (best and median) ride along
    for _ in range(args.steps):
        prefill_step()
        step_ev.append(torch.cuda.Event(enable_timing=True))
        step_ev[-1].record(stream)
    e1.record(stream)
    torch.cuda.synchronize()
    clocks.mark(w0, time.time())
    launches = ssd.launch_count() - n0
    headline_launches = launches  # our kernels inside the timed region that `value` measures
    barrier()
    ms = max_over_ranks(e0.elapsed_time(e1) / args.steps)
    step_ms = sorted((e0 if i == 0 else step_ev[i - 1]).elapsed_time(step_ev[i]) for i in range(args.steps))
    step_stats = {"best": max_over_ranks(step_ms[0]), "median": max_over_ranks(step_ms[len(step_ms) // 2]),
                  "steps": args.steps}
    # The same steps once more with an event pair around every kernel launch: the per-kernel
    # averages behind the roofline.  A separate region, because the events between the
    # launches keep each grid from starting before the one ahead of it ends.
    n0 = ssd.launch_count()
    ssd.profile_begin()
    e0p, e1p = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    w0 = time.time()
    e0p.record(stream)
    for _ in range(args.steps):
        prefill_step()
    e1p.record(stream)
    torch.cuda.synchronize()
    clocks.mark(w0, time.time())
    kt = ssd.profile_end()
    launches += ssd.launch_count() - n0
    barrier()
    ms_profiled = max_over_ranks(e0p.elapsed_time(e1p) / args.steps)
    # dominant kernel: the one with the largest summed event time in the timed region
    dom = max(kt.items(), key=lambda kv: kv[1][1])
    dom_name, (dom_n, dom_ms) = dom
    exec_L = EXEC_L_FUSED if "ssd_prefill_fused" in kt else PL
    flops = prefill_flops(PB, PT, PH, PP, PN, PG, exec_L)
    pbytes = prefill_bytes(PB, PT, PH, PP, PN, PG)
    tflops = job_rate(flops, world, ms) / 1e12
    tokens_s = job_rate(PB * PT, world, ms)
    dom_avg_ms = dom_ms / max(dom_n, 1)
    per_kernel_bytes = {
        # fused or not, the algorithmic bytes of one launch of the dominant prefill kernel
        "ssd_prefill_fused": pbytes,
        "simt_chunk_output": pbytes - PB * PH * PP * PN * 4 + PB * ((PT + PL - 1) // PL) * PH * PP * PN * 4,
    }
    alg = per_kernel_bytes.get(dom_name, pbytes)
    achieved = alg / (dom_avg_ms * 1e-3) / 1e9
    hbm_peak = pk["hbm_gbs"]
    roofline = {"kernel": dom_name, "bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                "frac": achieved / hbm_peak, "traffic": dram_traffic(dom_name),
                "peak_source": pk_kind + " (hbm_gbs, burst copy)", "avg_launch_ms": dom_avg_ms,
                "tensor_tflops": flops / (dom_avg_ms * 1e-3) / 1e12 if dom_name == "ssd_prefill_fused" else None,
                "tensor_frac_of_bf16_peak": (flops / (dom_avg_ms * 1e-3) / 1e12 / pk["bf16_tflops"])
                if dom_name == "ssd_prefill_fused" else None,
                "tensor_frac_of_bf16_sustained": (flops / (dom_avg_ms * 1e-3) / 1e12 / pk.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
                if dom_name == "ssd_prefill_fused" else None,
                "frac_of_nominal_hbm": achieved / NOMINAL_HBM_GBS, "nominal_hbm_gbs": NOMINAL_HBM_GBS,
                "kernels": {k: {"launches": v[0], "avg_ms": v[1] / max(v[0], 1)} for k, v in kt.items()},
                "kernel_times_from": "a second timed region of the same %d steps with an event pair around "
                                     "every launch (%.4f ms per step there)" % (args.steps, ms_profiled)}

    # ---------------- the same step from the raw time step (dt pre-processing fused into the
    # kernels: clamp(softplus(dt_raw + dt_bias), 0, inf)); dt_raw is chosen so that the
    # step sizes equal the headline's, so the work is the same.
    dt_bias = torch.full((PH,), 0.5, device=dev)
    dt_raw = torch.log(torch.expm1(d["dt"].double())).float() - 0.5
    for _ in range(3):
        ssd.prefill(d["x"], dt_raw, d["A"], d["B"], d["C"], d["D"], chunk=PL, h0=d["h0"], y=y, h_final=hf,
                    workspace=ws, dt_raw=True, dt_bias=dt_bias)
    torch.cuda.synchronize()
    barrier()
    n_raw = max(3, min(args.steps, 10))
    n0 = ssd.launch_count()
    e0r, e1r = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0r.record(stream)
    for _ in range(n_raw):
        ssd.prefill(d["x"], dt_raw, d["A"], d["B"], d["C"], d["D"], chunk=PL, h0=d["h0"], y=y, h_final=hf,
                    workspace=ws, dt_raw=True, dt_bias=dt_bias)
    e1r.record(stream)
    torch.cuda.synchronize()
    launches += ssd.launch_count() - n0
    barrier()
    ms_raw = max_over_ranks(e0r.elapsed_time(e1r) / n_raw)
    dt_raw_entry = {"ms_per_step": ms_raw, "vs_preprocessed_dt": ms_raw / ms,
                    "note": "softplus(dt_raw + dt_bias) formed inside the kernels (raw dt prefetched; the fused "
                            "kernel forms each block's dt one iteration before the block uses it); "
                            "no separate pass"}
    del dt_raw
    prefill_step()  # leave y / h_final as the headline step computes them
    torch.cuda.synchronize()

    # ---------------- e2e through the public API with host buffers.  Every step copies its
    # inputs from pinned host memory to the device and its outputs (y, h_final) back; steps
    # are pipelined as a serving loop runs them: copy-in, compute and copy-out on three
    # streams over two device buffer sets, so step i's copies overlap steps i-1 and i+1.
    sets = [d, {k: torch.empty_like(v) for k, v in d.items()}]
    ys, hfs = [y, torch.empty_like(y)], [hf, torch.empty_like(hf)]
    wss = [ws, torch.empty_like(ws)]
    out_y = [torch.empty(y.shape, dtype=y.dtype).pin_memory() for _ in range(2)]
    out_h = [torch.empty(hf.shape, dtype=hf.dtype).pin_memory() for _ in range(2)]
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    in_done = [torch.cuda.Event() for _ in range(2)]
    comp_done = [torch.cuda.Event() for _ in range(2)]
    out_done = [torch.cuda.Event() for _ in range(2)]

    def e2e_step(i):
        j = i & 1
        s_in.wait_event(comp_done[j])            # step i-2 has finished reading set j
        with torch.cuda.stream(s_in):
            for k in sets[j]:
                sets[j][k].copy_(pinned[k], non_blocking=True)
        in_done[j].record(s_in)
        stream.wait_event(in_done[j])
        stream.wait_event(out_done[j])           # step i-2's outputs have left the device
        t = sets[j]
        ssd.prefill(t["x"], t["dt"], t["A"], t["B"], t["C"], t["D"], chunk=PL, h0=t["h0"], y=ys[j],
                    h_final=hfs[j], workspace=wss[j], stream=stream)
        comp_done[j].record(stream)
        s_out.wait_event(comp_done[j])
        with torch.cuda.stream(s_out):
            out_y[j].copy_(ys[j], non_blocking=True)
            out_h[j].copy_(hfs[j], non_blocking=True)
        out_done[j].record(s_out)

    def e2e_run(n):
        # the region starts on the compute stream; the copy streams join it, and it ends
        # once the last step's outputs are in host memory
        start = torch.cuda.Event(enable_timing=True)
        end = torch.cuda.Event(enable_timing=True)
        start.record(stream)
        s_in.wait_event(start)
        s_out.wait_event(start)
        for i in range(n):
            e2e_step(i)
        stream.wait_event(out_done[(n - 1) & 1])
        end.record(stream)
        return start, end

    e2e_run(args.warmup)
    torch.cuda.synchronize()
    barrier()
    w0 = time.time()
    e2s, e2e_ = e2e_run(args.steps)
    torch.cuda.synchronize()
    clocks.mark(w0, time.time())
    barrier()
    ms_e2e = max_over_ranks(e2s.elapsed_time(e2e_) / args.steps)
    ok_e2e = bool(torch.equal(out_y[(args.steps - 1) & 1].to(dev), y)) if args.steps else True
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = y.numel() * y.element_size() + hf.numel() * hf.element_size()
    e2e = {"value": job_rate(flops, world, ms_e2e) / 1e12, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
           "d2h_bytes_per_step": d2h, "ms_per_step": ms_e2e, "pipelined": "copy-in / compute / copy-out streams",
           "output_matches_device_run": ok_e2e}

    # ---------------- cached decode (state from this prefill's final state)
    decode = {}
    for db in [int(v) for v in args.decode_batches.split(",") if v]:
        box = [0]
        decode["b%d" % db] = bench_decode(ssd, torch, dev, stream, case, hf, db, args, clocks, barrier,
                                          max_over_ranks, world, pk, box)
        launches += box[0]

    # ---------------- the other prefill configurations
    other = {}
    if not args.skip_other_prefill:
        box = [0]
        other = bench_prefill_configs(ssd, torch, dev, stream, args, clocks, barrier, max_over_ranks, world, pk, box)
        launches += box[0]

    clk = clocks.stop()

    cpu = None
    ablation = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(case, flops / (PB * PT * PH))
        ablation = decay_precision_ablation(ssd, torch, dev)

    if rank == 0:
        # the headline keys, then the roofline and a decode summary, so that a reader who
        # keeps only the start of the line still has them; the details follow
        decode_summary = {k: {"steps": v["steps"], "steps_per_s": v["steps_per_s"], "hbm_gbs_alg": v["hbm_gbs_alg"],
                              "hbm_frac": v["hbm_frac"]} for k, v in decode.items()}
        line = {"metric": METRIC, "value": tflops, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                "config": {"workload": "mamba2_2p7b_layer_prefill", "b": PB, "T": PT, "H": PH, "P": PP, "N": PN,
                           "G": PG, "chunk": PL, "global_batch": PB * world, "seq_len": PT,
                           "parallelism": "dp%d" % world,
                           "l2": "inputs larger than L2 (%.0f MB per step vs 126 MB)" % (pbytes / 1e6)},
                "roofline": roofline, "decode_summary": decode_summary, "e2e": e2e, "cpu_baseline": cpu,
                "gpu_launches": int(headline_launches),
                "tokens_per_s": tokens_s, "step_ms": step_stats, "flops_per_step": flops, "chunk_executed": exec_L,
                "bytes_per_step": pbytes,
                "hbm_gbs_alg": pbytes * world / (ms * 1e-3) / 1e9,
                "tensor_frac": tflops / world / pk["bf16_tflops"],
                "gpu_launches_all_timed_regions": int(launches),
                "prefill_split": {"whole_units": ssd.prefill_whole_units(PB, PT, PH, PP, PN, PG, PL, ssd.SSD_BF16),
                                  "segments": ssd.prefill_segments(PB, PT, PH, PP, PN, PG, PL, ssd.SSD_BF16)},
                "clocks": clk, "decode": decode, "prefill_configs": other, "prefill_dt_raw": dt_raw_entry,
                "decay_precision_ablation": ablation}
        print(json.dumps(line), flush=True)
    ranks.close()
    return 0


def decay_precision_ablation(ssd, torch, dev):
    """The analogue of the paper's decay-precision table without a model: the 130M-layer
    prefill (b=1, T=4096, H=24, one pass) with the decay in fp32 (the product), with every
    exponentiated decay factor rounded to bf16, and with the log-space prefix sums rounded
    to bf16 before exponentiation; max |error| of y and h_final against the fp64 oracle,
    also divided by max |reference|.  Not timed."""
    import oracle
    from ssd_inputs import make_config
    c = make_config("mamba2_130m_layer")
    def bf(bits):
        return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(dev)
    x, Bm, Cm = bf(c.x_bits), bf(c.B_bits), bf(c.C_bits)
    dt, A, D = (torch.from_numpy(v).to(dev) for v in (c.dt, c.A, c.D))
    y_ref, h_ref = oracle.ssd_recurrence(c.x, c.dt, c.A, c.B, c.C, c.D, None)
    out = {}
    ssd.debug_force_prefill_segments(1)
    try:
        for mode, name in ((0, "fp32_log_space_decay"), (1, "bf16_exp_outputs"), (2, "bf16_log_space_prefix_sums")):
            ssd.debug_decay_precision(mode)
            y, hf = ssd.prefill(x, dt, A, Bm, Cm, D, chunk=256)
            torch.cuda.synchronize()
            yd = np.abs(y.float().cpu().numpy() - y_ref)
            hd = np.abs(hf.cpu().numpy() - h_ref)
            out[name] = {"y_max_abs": float(yd.max()), "y_rel": float(yd.max() / np.abs(y_ref).max()),
                         "h_max_abs": float(hd.max()), "h_rel": float(hd.max() / np.abs(h_ref).max())}
    finally:
        ssd.debug_decay_precision(0)
        ssd.debug_force_prefill_segments(0)
    out["workload"] = "mamba2_130m_layer prefill, one pass, bf16 io"
    return out


def bench_prefill_configs(ssd, torch, dev, stream, args, clocks, barrier, max_over_ranks, world, pk, box):
    """The other prefill configurations: the tiny fp32 case (b=1, T=512, H=4, N=64; the fp32
    three-kernel fp32-FMA path, launch-latency bound), the 130M-layer shape (b=1, T=4096, H=24) and the
    long-context shape (b=1, T=65536, H=80, G=8), inputs resident in HBM, each step timed
    alone with CUDA events on the launching stream after a write that evicts L2, max over
    ranks; the per-kernel times come from a second pass with events around every launch.  The fused tensor-core path
    evaluates 128-token chunks whatever chunk length is requested: the long-context entry is
    timed once on it (chunk_executed = 128), and its chunk-length sweep L in {64, 128, 256}
    is timed literally on the fp32-FMA path (literal_chunk_sweep).  The bf16
    shapes have few (sequence, head) pairs for 148 SMs, so their sequences are split into
    segments (state pass, a prefix pass when there are many segments, fused pass); the
    segment count is reported."""
    from ssd_inputs import make_config
    out = {}
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)  # larger than the 126 MB L2
    for name, label in (("tiny_f32", "tiny_f32"), ("mamba2_130m_layer", "mamba2_130m_layer"),
                        ("long_context_L256", "long_context")):
        c = make_config(name)
        io = ssd.SSD_F32 if c.dtype == "f32" else ssd.SSD_BF16
        b, T, H, P, N, G = c.b, c.T, c.H, c.P, c.N, c.G
        def io_t(bits, vals):
            if io == ssd.SSD_F32:
                return torch.from_numpy(np.ascontiguousarray(vals, np.float32)).to(dev)
            return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(dev)
        x, Bm, Cm = io_t(c.x_bits, c.x), io_t(c.B_bits, c.B), io_t(c.C_bits, c.C)
        dt, A, D = (torch.from_numpy(v).to(dev) for v in (c.dt, c.A, c.D))
        y = torch.empty_like(x)
        hfin = torch.empty(b, H, P, N, device=dev)
        ws = torch.empty(ssd.prefill_workspace_size(b, T, H, P, N, G, 256, io), dtype=torch.uint8, device=dev)
        def step():
            ssd.prefill(x, dt, A, Bm, Cm, D, chunk=256, y=y, h_final=hfin, workspace=ws)
        for _ in range(args.warmup):
            step()
        torch.cuda.synchronize()
        barrier()
        n_steps = max(3, min(args.steps, 10))
        # each step timed alone, after a 256 MB write that evicts its inputs from L2
        n0 = ssd.launch_count()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n_steps)]
        w0 = time.time()
        for ev in evs:
            flush.fill_(1)
            ev[0].record(stream)
            step()
            ev[1].record(stream)
        torch.cuda.synchronize()
        clocks.mark(w0, time.time())
        box[0] += ssd.launch_count() - n0
        barrier()
        ms = max_over_ranks(sum(a.elapsed_time(b_) for a, b_ in evs) / n_steps)
        # per-kernel times from the same steps with an event pair around every launch
        n0 = ssd.launch_count()
        ssd.profile_begin()
        for _ in range(n_steps):
            flush.fill_(1)
            step()
        torch.cuda.synchronize()
        kt = ssd.profile_end()
        box[0] += ssd.launch_count() - n0
        byt = prefill_bytes(b, T, H, P, N, G, io_bytes=4 if io == ssd.SSD_F32 else 2, with_h0=False)
        gbs = byt * world / (ms * 1e-3) / 1e9
        entry = {"b": b, "T": T, "H": H, "G": G, "ms_per_step": ms, "tokens_per_s": job_rate(b * T, world, ms),
                 "bytes_per_step": byt, "hbm_gbs_alg": gbs, "hbm_frac": gbs / world / pk["hbm_gbs"],
                 "dtype": c.dtype,
                 "chunk_executed": EXEC_L_FUSED if io == ssd.SSD_BF16 else 256,
                 "tflops_executed": job_rate(prefill_flops(b, T, H, P, N, G, EXEC_L_FUSED if io == ssd.SSD_BF16 else 256),
                                             world, ms) / 1e12,
                 "kernels": {k: {"launches": v[0] // n_steps, "avg_ms": v[1] / max(v[0], 1)} for k, v in kt.items()},
                 "segments": ssd.prefill_segments(b, T, H, P, N, G, 256, io),
                 "l2": "256 MB written before every timed step"}
        if label == "long_context":
            entry["literal_chunk_sweep"] = literal_chunk_sweep(ssd, torch, x, dt, A, Bm, Cm, D, y, hfin, flush,
                                                               stream, barrier, max_over_ranks, world, box,
                                                               (b, T, H, P, N, G))
        out[label] = entry
        del x, Bm, Cm, dt, A, D, y, hfin, ws
        torch.cuda.empty_cache()
    return out


def literal_chunk_sweep(ssd, torch, x, dt, A, Bm, Cm, D, y, hfin, flush, stream, barrier, max_over_ranks, world,
                        box, shape):
    """The long-context prefill with chunks of exactly L tokens for L in {64, 128, 256}: the
    fp32-FMA path (ssd_debug_force_fma_prefill) evaluates the chunked form with the chunk
    length given, so this is the pages' chunk-size trade-off (arithmetic intensity of the
    dual form against the length of the sequential recurrence) measured on kernels that
    honour L.  The tensor-core kernel always evaluates 128-token chunks (its timing is the
    entry's ms_per_step).  Each L: one warm-up call, then two calls timed alone after an
    L2-evicting write; ms per call and TFLOP/s at that L's operation count."""
    b, T, H, P, N, G = shape
    out = {"path": "fp32 FMA (SIMT), bf16 io, literal chunk length"}
    ssd.debug_force_fma_prefill(True)
    try:
        for L in (64, 128, 256):
            ws = torch.empty(ssd.prefill_workspace_size(b, T, H, P, N, G, L, ssd.SSD_BF16), dtype=torch.uint8,
                             device=x.device)
            def step():
                ssd.prefill(x, dt, A, Bm, Cm, D, chunk=L, y=y, h_final=hfin, workspace=ws)
            step()
            torch.cuda.synchronize()
            barrier()
            n0 = ssd.launch_count()
            evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(2)]
            for ev in evs:
                flush.fill_(1)
                ev[0].record(stream)
                step()
                ev[1].record(stream)
            torch.cuda.synchronize()
            box[0] += ssd.launch_count() - n0
            ms = max_over_ranks(sum(a.elapsed_time(c) for a, c in evs) / len(evs))
            out["L%d" % L] = {"ms_per_step": ms,
                              "tflops": job_rate(prefill_flops(b, T, H, P, N, G, L), world, ms) / 1e12}
            del ws
            torch.cuda.empty_cache()
    finally:
        ssd.debug_force_fma_prefill(False)
    return out


def bench_decode(ssd, torch, dev, stream, case, hf, b, args, clocks, barrier, max_over_ranks, world, pk, box):
    from ssd_inputs import make_decode_params
    Dc = DH * DP + 2 * DG * DN
    A, D, conv_w, conv_b, dt_bias = make_decode_params(DL, DH, DP, DN, DG, DK, seed=3)
    A, D, conv_w, conv_b = (torch.from_numpy(v).to(dev) for v in (A, D, conv_w, conv_b))
    # state: the prefill's final state of sequence r mod 8, every layer
    h = hf[torch.arange(b, device=dev) % hf.shape[0]].unsqueeze(0).expand(DL, b, DH, DP, DN).contiguous()
    # conv window: the last k-1 tokens of that sequence's [x | B | C]
    rows = []
    for r in range(b):
        s = r % case.b
        xs = case.x[s, -3:].reshape(3, -1)
        bs = case.B[s, -3:].reshape(3, -1)
        cs_ = case.C[s, -3:].reshape(3, -1)
        rows.append(np.concatenate([xs, bs, cs_], 1).T)
    cst = torch.from_numpy(np.stack(rows)).to(dev).unsqueeze(0).expand(DL, b, Dc, 3).contiguous()
    ring = 256 if b == 1 else 32
    from ssd_inputs import make_decode_ring_device
    xbc, dt = make_decode_ring_device(ring, DL, b, DH, DP, DN, DG, dt_bias, seed=77, device=dev)
    steps_per_launch = min(args.decode_steps, 512 if b == 1 else 64)
    plan = ssd.DecodePlan(h, cst, xbc, dt, A, D, conv_w, conv_b, n_steps=steps_per_launch, G=DG)
    plan.launch()
    torch.cuda.synchronize()
    launches_timed = max(1, args.decode_steps // steps_per_launch)
    barrier()
    n0 = ssd.launch_count()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    w0 = time.time()
    ev[0].record(stream)
    for _ in range(launches_timed):
        plan.launch()
    ev[1].record(stream)
    torch.cuda.synchronize()
    clocks.mark(w0, time.time())
    box[0] = ssd.launch_count() - n0
    barrier()
    ms = max_over_ranks(ev[0].elapsed_time(ev[1]))
    steps = launches_timed * steps_per_launch
    sps = job_rate(steps, world, ms)
    byt = decode_bytes_per_step(DL, b, DH, DP, DN, DG)
    gbs = byt * sps / 1e9
    loops = {}
    if b == 1 and not args.skip_loop_compare:
        loops = bench_decode_loops(ssd, torch, dev, stream, h, cst, xbc, dt, A, D, conv_w, conv_b, ring,
                                   ms / steps, barrier, max_over_ranks, box)
    ok = bool(torch.isfinite(h).all().item())
    plan.close()
    del h, cst, xbc, dt
    torch.cuda.empty_cache()
    return {"batch": b, "layers": DL, "steps": steps, "steps_per_launch": steps_per_launch,
            "steps_per_s": sps, "tokens_per_s": sps * b, "ms_per_step": ms / steps,
            "bytes_per_step": byt, "hbm_gbs_alg": gbs, "hbm_frac": gbs / world / pk["hbm_gbs"],
            "hbm_frac_of_nominal": gbs / world / NOMINAL_HBM_GBS,
            "kernel": "decode_step (graph of %d steps)" % steps_per_launch, "state_finite": ok,
            "loop_compare": loops}


def bench_decode_loops(ssd, torch, dev, stream, h, cst, xbc, dt, A, D, conv_w, conv_b, ring, graph_ms_per_step,
                       barrier, max_over_ranks, box):
    """The comparisons the pages make for the cached decode, on our kernels at batch 1 and
    the 2.7B-shaped 64-layer cache ([CF-SSD] O(1) caching and compiled-loop sections):
      * the on-device loop (one CUDA graph of many steps) against the same steps launched one
        call at a time, and against a host loop that waits for each step before the next
        (the host round trip per token a non-compiled loop pays);
      * the cached step against recomputing the whole 4096-token context: one prefill of
        b = 1, T = 4096 over the 80 heads, times 64 layers, per generated token.
    All timed with CUDA events on the launching stream."""
    n = 128
    y = torch.empty(DL, 1, DH, DP, dtype=xbc.dtype, device=dev)
    ws = torch.empty(ssd.decode_workspace_size(DL, 1, DG), dtype=torch.uint8, device=dev)

    def step(t):
        ssd.decode_step(h, cst, xbc[t % ring], dt[t % ring], A, D, conv_w, conv_b, G=DG, y=y, workspace=ws)

    for t in range(8):
        step(t)
    torch.cuda.synchronize()
    barrier()
    res = {}
    for mode in ("launch_per_step", "host_sync_per_step"):
        n0 = ssd.launch_count()
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        ev[0].record(stream)
        for t in range(n):
            step(t)
            if mode == "host_sync_per_step":
                torch.cuda.synchronize()
        ev[1].record(stream)
        torch.cuda.synchronize()
        box[0] += ssd.launch_count() - n0
        barrier()
        res[mode] = max_over_ranks(ev[0].elapsed_time(ev[1])) / n
    # recompute: prefill of the full context for one sequence, all heads, one layer; x64 layers
    from ssd_inputs import make_config
    c = make_config("mamba2_2p7b_layer", b=1, seed=11)
    def bf(bits):
        return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(dev)
    px, pB, pC = bf(c.x_bits), bf(c.B_bits), bf(c.C_bits)
    pdt, pA, pD = (torch.from_numpy(v).to(dev) for v in (c.dt, c.A, c.D))
    py = torch.empty_like(px)
    pws = torch.empty(ssd.prefill_workspace_size(1, c.T, c.H, c.P, c.N, c.G, 256, ssd.SSD_BF16), dtype=torch.uint8,
                      device=dev)
    for _ in range(3):
        ssd.prefill(px, pdt, pA, pB, pC, pD, chunk=256, y=py, workspace=pws)
    torch.cuda.synchronize()
    barrier()
    n0 = ssd.launch_count()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    ev[0].record(stream)
    for _ in range(10):
        ssd.prefill(px, pdt, pA, pB, pC, pD, chunk=256, y=py, workspace=pws)
    ev[1].record(stream)
    torch.cuda.synchronize()
    box[0] += ssd.launch_count() - n0
    barrier()
    prefill_ms = max_over_ranks(ev[0].elapsed_time(ev[1])) / 10
    recompute_ms = prefill_ms * DL
    return {"steps": n, "graph_ms_per_step": graph_ms_per_step,
            "launch_per_step_ms": res["launch_per_step"], "host_sync_per_step_ms": res["host_sync_per_step"],
            "graph_vs_host_sync": res["host_sync_per_step"] / graph_ms_per_step,
            "graph_vs_launch_per_step": res["launch_per_step"] / graph_ms_per_step,
            "recompute_context": c.T, "recompute_prefill_ms_per_layer": prefill_ms,
            "recompute_ms_per_token": recompute_ms,
            "cached_vs_recompute_speedup": recompute_ms / graph_ms_per_step}


if __name__ == "__main__":
    sys.exit(main())
