#!/usr/bin/env python
"""Throughput of the gated delta-rule hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl gdr|reference]

One JSON line on rank 0.  A "step" is one chunked prefill over one batch of
the largest workload, the varlen mixed batch (32 sequences of 1024..16384
tokens packed by cu_seqlens, 32 heads, d_k = d_v = 128, bf16 q/k/v, fp32
beta/log_a/state, per-sequence initial states): the intra-chunk kernel (with
the chunk-local cumulative decay fused in) and the sequential state pass, two
launches (four when the pass is segmented).  ``value`` is prefill tokens/s
over all ranks (each rank runs its own batch: weak scaling, no collective on
the data path).  ``--workload`` picks another prefill workload for the main
line.  The same run also measures:

* ``decode``: the decode step on 256 sequences x 14 heads x 64 x 64 fp32 states,
  state bytes streamed per second (four state sets rotated so that the 235 MB
  working set exceeds the 126 MB L2);
* ``spec_decode``: speculative decoding on the same sequences: a draft of 4
  tokens that keeps the state after each token, then the accept (rollback)
  step, each timed alone and as one verify cycle;
* ``preprocess``: the input activations (conv-4, L2 norm of q and k, beta and
  log-decay gates) from raw projections of the graft layer's shape, alone and
  followed by the prefill;
* ``roofline``: the step's dominant kernel, timed alone with CUDA events;
* ``e2e``: the same prefill through the public API with pinned host buffers,
  host<->device copies inside the timed region;
* ``cpu_baseline``: the fp64 oracle on the host cores, a bounded sample of the
  same workload; ``cpu_baselines``: the same for the graft layer, the long
  Gated DeltaNet prefill and the decode step;
* ``extra``: the other prefill workloads (tiny fp32, the Qwen2.5-0.5B graft
  layer, the 65K-token scalar gate with snapshots), each with its own
  roofline block; the graft layer also with the output epilogue (RMSNorm and
  output gate) and the long prefill also with its snapshots offloaded to
  pinned host memory.

``--impl reference`` times the fp64 CPU oracle alone (rank 0; other ranks exit).
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads as wl  # noqa: E402

METRIC = "gated-delta prefill tokens/s + decode state GB/s, 1×B200 (% of roofline)"
CHUNK = 64
L2_BYTES = 126 * 2 ** 20


# ---------------------------------------------------------------------------
# algorithmic counts (per unit of work)
# ---------------------------------------------------------------------------
def prefill_flops_per_token_head(d_k: int, d_v: int) -> int:
    """Causal halves counted once: K K^T, Q K^T and T (b K) (C d_k each),
    T (b V) and P Delta (C d_v each), W S^T, Q S^T and Delta^T K (2 d_k d_v each)."""
    return 3 * CHUNK * d_k + 2 * CHUNK * d_v + 6 * d_k * d_v


def prefill_bytes_per_token_head(d_k: int, d_v: int, elem: int, scalar: bool) -> int:
    """q, k, v read and o written once, plus beta and log_a (fp32)."""
    return 2 * d_k * elem + 2 * d_v * elem + 4 + (4 if scalar else 4 * d_k)


def prefill_state_bytes(n_seqs: int, H: int, d_k: int, d_v: int, has_init: bool, n_snap: int) -> int:
    per = d_k * d_v * 4 * H
    return per * n_seqs * (2 if has_init else 1) + per * n_snap


def decode_bytes_per_head_state(d_k: int, d_v: int, elem: int, scalar: bool) -> int:
    """state read + written (fp32), q, k, v, beta, log_a read, o (fp32) written."""
    return 2 * 4 * d_k * d_v + (2 * d_k + d_v) * elem + 4 + (4 if scalar else 4 * d_k) + 4 * d_v


def draft_bytes_per_head_state(d_k: int, d_v: int, elem: int, scalar: bool, K: int) -> int:
    """state read once (fp32); per draft token the kept state written (fp32),
    q, k, v, beta, log_a read and o (fp32) written."""
    tok = (2 * d_k + d_v) * elem + 4 + (4 if scalar else 4 * d_k) + 4 * d_v
    return 4 * d_k * d_v + K * (4 * d_k * d_v + tok)


def preprocess_bytes_per_token_head(d: int, elem: int, scalar: bool) -> int:
    """raw x_q, x_k, x_v, beta_raw and a_raw read; q, k, v, beta and log a
    written (conv taps and biases are per head, not per token)."""
    return 2 * (3 * d * elem + 4 + (4 if scalar else 4 * d))


def peaks() -> dict:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        p = json.load(open(path))
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.proc = None
        self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", str(gpu_index)], stdout=self.file, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self, t0: datetime.datetime, t1: datetime.datetime):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.file.flush()
        rows = []
        for line in open(self.file.name):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f")
                rows.append((ts, float(parts[1]), float(parts[2]), parts[4:8]))
            except ValueError:
                continue
        os.unlink(self.file.name)
        if not rows:
            return None
        inside = [r for r in rows if t0 <= r[0] <= t1]
        window = inside or sorted(rows, key=lambda r: abs((r[0] - t0).total_seconds()))[:3]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in window for i, s in enumerate(r[3]) if s.lower() == "active"})
        return {"sm_mhz": statistics.median(r[1] for r in window),
                "sm_max_mhz": max(r[2] for r in window), "reasons": reasons,
                "samples": len(window), "samples_inside_timed_region": len(inside)}


class NvmlClockSampler:
    """SM clock and clock-event reasons read through NVML (read-only queries)
    by a thread every ~2 ms between start() and stop(), so that even a timed
    region of a few milliseconds holds samples.  Falls back to None when NVML
    is unavailable (the nvidia-smi sampler above then covers the run)."""
    REASONS = (("hw_slowdown", 0x8), ("sw_thermal_slowdown", 0x20),
               ("hw_thermal_slowdown", 0x40), ("hw_power_brake_slowdown", 0x80),
               ("sw_power_cap", 0x4))

    def __init__(self, cuda_index: int):
        import threading
        self.rows, self.ok, self._stop = [], False, threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            try:
                pr = torch.cuda.get_device_properties(cuda_index)
                bus = f"{pr.pci_domain_id:08x}:{pr.pci_bus_id:02x}:{pr.pci_device_id:02x}.0"
                self.h = pynvml.nvmlDeviceGetHandleByPciBusId(bus.encode())
            except Exception:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(cuda_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.ok = False
        self.thread = threading.Thread(target=self._run, daemon=True)

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.rows.append((time.perf_counter(), mhz, rs))
            except Exception:
                pass
            time.sleep(0.002)

    def start(self):
        if self.ok:
            self.thread.start()
        return self

    def stop(self, t0: float, t1: float):
        if not self.ok:
            return None
        self._stop.set()
        self.thread.join(timeout=5)
        inside = [r for r in self.rows if t0 <= r[0] <= t1]
        # a timed region shorter than the sampling interval: the samples
        # nearest to it
        window = inside or sorted(self.rows, key=lambda r: abs(r[0] - t0))[:3]
        if not window:
            return None
        reasons = sorted({n for r in window for n, bit in self.REASONS if r[2] & bit})
        return {"sm_mhz": statistics.median(r[1] for r in window), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(window),
                "samples_inside_timed_region": len(inside), "source": "nvml, every ~2 ms"}


# ---------------------------------------------------------------------------
# distributed plumbing (one process per GPU, torchrun)
# ---------------------------------------------------------------------------
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(x: float, world: int) -> float:
    """Slowest rank's value (timing is taken as the max over ranks)."""
    if world == 1:
        return x
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def rank_seed(base_seed: int, set_index: int, rank: int) -> int:
    """Seed of input set `set_index` on `rank`: every rank draws its own batch
    (weak scaling: the units all ranks process add up)."""
    return base_seed + 7919 * set_index + 100003 * rank


def job_throughput(units_per_rank: int, world: int, steps: int, max_ms: float) -> float:
    """Whole-job units per second: all ranks' units over the slowest rank's time."""
    return world * units_per_rank * steps / (max_ms * 1e-3)


def timed(fn, n, stream):
    """Average device time (ms) of n calls of fn, CUDA events on `stream`."""
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    start.record(stream)
    for i in range(n):
        fn(i)
    end.record(stream)
    torch.cuda.synchronize()
    return start.elapsed_time(end) / n


# ---------------------------------------------------------------------------
# prefill workloads on the GPU
# ---------------------------------------------------------------------------
class PrefillSets:
    """R independent input sets (rotated every step), outputs and workspaces."""

    def __init__(self, gdr, w: wl.PrefillWorkload, n_sets: int, rank: int):
        """n_sets = 0: one set when its buffers alone exceed L2, else enough
        sets (at most 4) that the rotation's footprint exceeds L2 where
        possible."""
        self.w = w
        self.sets = []
        i = 0
        while i < (n_sets or 4):
            wi = wl.shrink(w, seed=rank_seed(w.seed, i, rank))
            inp = wl.make_prefill_inputs(wi, device="cuda", draw_device="cuda")
            T, H, dk = inp["q"].shape
            dv = inp["v"].shape[-1]
            n = len(inp["lengths"])
            ns = gdr.snapshot_count(wl.cu_seqlens_of(inp["lengths"]), w.snap_interval) if w.snap_interval else 0
            out = torch.empty(T, H, dv, dtype=inp["q"].dtype, device="cuda")
            fin = torch.empty(n, H, dv, dk, device="cuda")
            snaps = torch.empty(max(ns, 1), H, dv, dk, device="cuda") if w.snap_interval else None
            ws = torch.empty(gdr.workspace_size(n, H, dk, dv, T, w.scalar_decay), dtype=torch.uint8,
                             device="cuda")
            prep = gdr.PreparedPrefill(inp["q"], inp["k"], inp["v"], inp["beta"], inp["log_a"],
                                       inp["cu_seqlens"], out=out, final_state=fin, workspace=ws,
                                       scalar_decay=w.scalar_decay, scale=w.scale,
                                       init_state=inp["init_state"], snap_interval=w.snap_interval,
                                       snapshots=snaps)
            self.sets.append(dict(inp=inp, prep=prep, n_snap=ns, T=T, H=H, dk=dk, dv=dv, n=n))
            i += 1
            one = sum(t.numel() * t.element_size() for t in prep._keep if torch.is_tensor(t))
            if not n_sets and one * i > 2 * L2_BYTES:
                break
        s0 = self.sets[0]
        self.T, self.H, self.dk, self.dv, self.n = s0["T"], s0["H"], s0["dk"], s0["dv"], s0["n"]
        elem = 2 if w.qkv_dtype == torch.bfloat16 else 4
        self.units = self.T * self.H
        self.flops = prefill_flops_per_token_head(self.dk, self.dv) * self.units
        self.bytes = (prefill_bytes_per_token_head(self.dk, self.dv, elem, w.scalar_decay) * self.units
                      + prefill_state_bytes(self.n, self.H, self.dk, self.dv, w.init_std > 0,
                                            s0["n_snap"]))
        self.footprint = sum(sum(t.numel() * t.element_size() for t in s["prep"]._keep
                                 if torch.is_tensor(t)) for s in self.sets)
        self.l2 = (f"{len(self.sets)} rotating input set(s), {self.footprint / 2**20:.0f} MiB "
                   f"{'>' if self.footprint > L2_BYTES else '<='} 126 MiB L2")

    def step(self, i, stages=(0, 1)):
        self.sets[i % len(self.sets)]["prep"].run(stages)


STAGES = ("intra_chunk", "state_pass")


def stage_times(ps: PrefillSets, n: int, stream) -> list:
    """Device time of each prefill stage launched alone (ms)."""
    for i in range(len(ps.sets)):
        ps.step(i)
    out = []
    for s in range(len(STAGES)):
        out.append(timed(lambda i: ps.step(i, (s, s)), n, stream))
    return out


def roofline_obj(bytes_, flops, t_ms, pk, traffic=None):
    gbs = bytes_ / (t_ms * 1e-3) / 1e9
    return {"bound": "hbm", "achieved": round(gbs, 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
            "frac": round(gbs / pk["hbm_gbs"], 4), "traffic": traffic,
            "tensor_tflops": round(flops / (t_ms * 1e-3) / 1e12, 2),
            "tensor_frac": round(flops / (t_ms * 1e-3) / 1e12 / pk["bf16_tflops"], 4),
            "peak_source": pk["source"]}


def recorded_traffic(kernel: str, workload: str):
    """dram bytes per launch from the committed ncu summary, if it still
    matches the kernel's current source."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    try:
        rows = json.load(open(path))
    except Exception:
        return None
    for r in rows:
        if r.get("kernel") == kernel and r.get("workload") == workload:
            src = os.path.join(ROOT, r["source"])
            sha = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
            if sha == r.get("source_sha"):
                return r.get("dram_bytes_per_launch")
    return None


# ---------------------------------------------------------------------------
# arms
# ---------------------------------------------------------------------------
def oracle_cores() -> int:
    return int(os.environ.get("OMP_NUM_THREADS", os.cpu_count()))


def _host_inputs(inp: dict, heads) -> dict:
    """The sampled heads of a prefill batch, on the host (same bits)."""
    out = {}
    for k_ in ("q", "k", "v", "beta", "log_a"):
        out[k_] = inp[k_][:, heads].cpu()
    out["init_state"] = None if inp["init_state"] is None else inp["init_state"][:, heads].cpu()
    out["cu_seqlens"] = inp["cu_seqlens"].cpu()
    return out


def oracle_prefill_sample(w: wl.PrefillWorkload, inp: dict, budget_s: float, steps: int = 0):
    """Time the fp64 oracle on a bounded sample of workload ``w``: all of its
    sequences, on as many heads as fit the time budget (one head's cost is
    measured first).  Returns (tokens/s scaled to all heads, sample text,
    seconds per pass)."""
    import oracle
    H = inp["q"].shape[1]
    T = inp["q"].shape[0]

    def run(heads):
        x = _host_inputs(inp, heads)
        t0 = time.perf_counter()
        oracle.prefill(x["q"], x["k"], x["v"], x["beta"], x["log_a"], x["cu_seqlens"],
                       scalar_decay=w.scalar_decay, scale=w.scale, init_state=x["init_state"],
                       snap_interval=w.snap_interval)
        return time.perf_counter() - t0

    t1 = run([0])
    n_heads = max(1, min(H, int(budget_s / max(t1, 1e-6))))
    heads = list(range(n_heads))
    passes = max(1, steps) if steps else max(1, min(20, int(budget_s / max(t1 * n_heads, 1e-6))))
    dt = sum(run(heads) for _ in range(passes)) / passes
    value = T * n_heads / H / dt
    sample = (f"{passes} pass(es) over heads 0..{n_heads - 1} of {H}, all {T} tokens of "
              f"{len(inp['lengths'])} sequence(s) of {w.name}, fp64; tokens/s = tokens x "
              f"sampled heads / {H} / seconds")
    return value, sample, dt


def run_reference(args):
    """The fp64 CPU oracle as the reference arm (rank 0 only), on the main
    line's workload, metric and unit.  The sample: every sequence and token of
    the workload, on as many heads as fit the time budget (drawn with the
    workload's shapes and distributions for that many heads; the oracle's
    cost does not depend on the values)."""
    world, rank, _ = dist_env()
    if rank != 0:
        return
    import oracle
    w = {**wl.PREFILL_WORKLOADS, **wl.PROFILE_CASES}[args.workload]
    H = w.n_heads

    def sample(n_heads):
        return wl.make_prefill_inputs(wl.shrink(w, n_heads=n_heads))

    def run(x):
        t0 = time.perf_counter()
        oracle.prefill(x["q"], x["k"], x["v"], x["beta"], x["log_a"], x["cu_seqlens"],
                       scalar_decay=w.scalar_decay, scale=w.scale, init_state=x["init_state"],
                       snap_interval=w.snap_interval)
        return time.perf_counter() - t0

    budget = 8.0
    t1 = run(sample(1))
    n = max(1, min(H, int(budget / max(t1, 1e-6))))
    x = sample(n)
    for _ in range(max(0, args.warmup - 3)):
        run(x)
    passes = max(1, min(args.steps, int(3 * budget / max(t1 * n, 1e-6))))
    dt = sum(run(x) for _ in range(passes)) / passes
    T = x["q"].shape[0]
    value = T * n / H / dt
    sample_text = (f"{passes} pass(es) over {n} of {H} heads (drawn with the workload's shapes "
                   f"and distributions), all {T} tokens of {len(x['lengths'])} sequence(s) of "
                   f"{w.name}, fp64; tokens/s = tokens x {n} / {H} / seconds")
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 1), "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(dt * 1e3, 3), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, "n_seqs": len(x["lengths"]), "tokens": T,
                       "heads": H, "d_k": w.d_k, "d_v": w.d_v,
                       "parallelism": "none (host cores)"},
            "cpu_baseline": {"value": round(value, 1), "unit": "tokens/s", "cores": oracle_cores(),
                             "kind": "oracle", "sample": sample_text},
            "e2e": {"value": round(value, 1), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def cpu_baseline_prefill(w: wl.PrefillWorkload, inp: dict, budget_s: float) -> dict:
    value, sample, _ = oracle_prefill_sample(w, inp, budget_s)
    return {"value": round(value, 1), "unit": "tokens/s", "cores": oracle_cores(),
            "kind": "oracle", "sample": sample}


def cpu_baseline_decode(budget_s: float) -> dict:
    """The oracle's decode step on a sample of the decode workload's
    sequences: state GB/s counted with the same bytes per head-state and step
    as the GPU line."""
    import oracle
    w = wl.DECODE
    inp = wl.make_decode_inputs(w, steps=4)
    B = w.batch
    state = inp["state"].double().numpy()
    elem = 2 if w.qkv_dtype == torch.bfloat16 else 4
    per = decode_bytes_per_head_state(w.d_k, w.d_v, elem, w.scalar_decay)
    b, n_steps, t_total = 16, 0, 0.0
    while True:
        t0 = time.perf_counter()
        oracle.decode_step(state[:b], inp["q"][0][:b], inp["k"][0][:b], inp["v"][0][:b],
                           inp["beta"][0][:b], inp["log_a"][0][:b], scalar_decay=w.scalar_decay)
        dt = time.perf_counter() - t0
        if dt * B / b * 2 < budget_s and b < B:
            b = min(B, 2 * b)
            continue
        n_steps, t_total = 1, dt
        while t_total < budget_s and n_steps < 64:
            t0 = time.perf_counter()
            oracle.decode_step(state[:b], inp["q"][n_steps % 4][:b], inp["k"][n_steps % 4][:b],
                               inp["v"][n_steps % 4][:b], inp["beta"][n_steps % 4][:b],
                               inp["log_a"][n_steps % 4][:b], scalar_decay=w.scalar_decay)
            t_total += time.perf_counter() - t0
            n_steps += 1
        break
    units = b * w.n_heads * n_steps
    gbs = per * units / t_total / 1e9
    return {"value": round(gbs, 4), "unit": "GB/s (state bytes per head-state and step)",
            "cores": oracle_cores(), "kind": "oracle",
            "sample": f"{n_steps} decode step(s) of {b} of {B} sequences x {w.n_heads} heads "
                      f"of {w.name}, fp64, {per} B per head-state and step"}


def dominant_roofline(ps: "PrefillSets", st_ms: list, pk: dict) -> dict:
    """Roofline block of the step's dominant kernel (the slower stage, timed
    alone): the whole step's algorithmic bytes over that kernel's time."""
    dom = max(range(len(STAGES)), key=lambda s_: st_ms[s_])
    roof = roofline_obj(ps.bytes, ps.flops, st_ms[dom], pk,
                        recorded_traffic(STAGES[dom], ps.w.name))
    roof["kernel"] = STAGES[dom]
    roof["kernel_ms"] = round(st_ms[dom], 4)
    roof["algorithmic_bytes_per_step"] = ps.bytes
    roof["algorithmic_flops_per_step"] = ps.flops
    return roof


def run_gdr(args):
    world, rank, local = dist_env()
    if world > 1:
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    torch.cuda.set_device(local)
    import gated_delta_rule_150_b200 as gdr
    gdr.lib()                                   # raises if the CUDA library is missing
    stream = torch.cuda.current_stream()
    pk = peaks()

    # ---- main workload (default: the varlen batch, inputs larger than L2) ----
    w_main = {**wl.PREFILL_WORKLOADS, **wl.PROFILE_CASES}[args.workload]
    ps = PrefillSets(gdr, w_main, args.sets or 0, rank)
    for i in range(args.warmup):
        ps.step(i)
    torch.cuda.synchronize()
    sampler = ClockSampler(local)
    nvml = NvmlClockSampler(local).start()
    time.sleep(0.3)
    barrier(world)
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t_wall0, t_perf0 = datetime.datetime.now(), time.perf_counter()
    start.record(stream)
    for i in range(args.steps):
        ps.step(i)
    end.record(stream)
    torch.cuda.synchronize()
    t_wall1, t_perf1 = datetime.datetime.now(), time.perf_counter()
    barrier(world)
    clocks_nvml = nvml.stop(t_perf0, t_perf1)
    clocks_smi = sampler.stop(t_wall0, t_wall1)
    clocks = clocks_nvml or clocks_smi
    ms_local = start.elapsed_time(end)
    ms_total = max_over_ranks(ms_local, world)
    ms_step = ms_total / args.steps
    value = job_throughput(ps.T, world, args.steps, ms_total)
    launches_per_step = gdr.kernel_count(ps.n, ps.H, ps.dk, ps.dv, ps.T, ps.w.scalar_decay)

    # ---- the prefill stages alone -> dominant kernel roofline -------------------
    st_ms = stage_times(ps, max(10, min(args.steps, 200)), stream)
    roof = dominant_roofline(ps, st_ms, pk)
    stage_report = {STAGES[s_]: round(st_ms[s_], 4) for s_ in range(len(STAGES))}
    la, cu0 = ps.sets[0]["inp"]["log_a"], ps.sets[0]["inp"]["cu_seqlens"]
    g_out = torch.empty_like(la)
    gdr.cumdecay(la, cu0, out=g_out, d_k=ps.dk, scalar_decay=ps.w.scalar_decay)   # warm-up
    stage_report["cumdecay_standalone"] = round(
        timed(lambda i: gdr.cumdecay(la, cu0, out=g_out, d_k=ps.dk,
                                     scalar_decay=ps.w.scalar_decay), 10, stream), 4)
    path_roof = roofline_obj(ps.bytes, ps.flops, ms_step, pk)
    main_inp = ps.sets[0]["inp"]
    config = {"workload": w_main.name, "n_seqs": ps.n, "tokens": ps.T, "heads": ps.H,
              "d_k": ps.dk, "d_v": ps.dv, "parallelism": "replicas" if world > 1 else "none",
              "l2": ps.l2}
    del g_out

    extra, decode, spec, pre = {}, None, None, None
    if not args.no_extra:
        decode = bench_decode(gdr, stream, pk, args)
        spec = bench_spec_decode(gdr, stream, pk, args)
        pre = bench_preprocess(gdr, stream, pk, args)
        for w in (wl.TINY_KDA, wl.GRAFT_LAYER, wl.GDN_LONG, wl.VARLEN):
            if w.name != w_main.name:
                extra[w.name] = bench_prefill_workload(gdr, w, stream, pk, rank, args)
    e2e = None if args.no_e2e else bench_e2e(gdr, w_main, stream, args)

    cpu, cpus = None, None
    if rank == 0 and world == 1 and not args.no_cpu:
        cpu = cpu_baseline_prefill(w_main, main_inp, 8.0)
        cpus = {"decode_" + wl.DECODE.name: cpu_baseline_decode(4.0)}
        for w in (wl.GRAFT_LAYER, wl.GDN_LONG):
            if w.name != w_main.name:
                inp = wl.make_prefill_inputs(w, device="cuda", draw_device="cuda")
                cpus[w.name] = cpu_baseline_prefill(w, inp, 4.0)
                del inp
    del ps, main_inp
    torch.cuda.empty_cache()
    if rank != 0:
        if world > 1:
            torch.distributed.destroy_process_group()
        return
    line = {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": config,
        "roofline": roof,
        "path_roofline": path_roof,
        "kernel_ms": stage_report,
        "decode": decode,
        "spec_decode": spec,
        "preprocess": pre,
        "e2e": e2e,
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
        "cpu_baseline": cpu,
        "cpu_baselines": cpus,
        "extra": extra,
        "gpu": torch.cuda.get_device_name(),
    }
    print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


def bench_prefill_workload(gdr, w, stream, pk, rank, args):
    """One prefill workload: whole step, its two stages alone, the dominant
    kernel's roofline; the graft layer also with the output epilogue, the long
    Gated DeltaNet prefill also with its snapshots in pinned host memory."""
    ps = PrefillSets(gdr, w, 0, rank)
    n = 3 if ps.T > 100000 else (10 if ps.T > 20000 else 20)
    for i in range(2):
        ps.step(i)
    ms = timed(lambda i: ps.step(i), n, stream)
    st = stage_times(ps, n, stream)
    res = {"tokens_per_s": round(ps.T / (ms * 1e-3), 1), "ms_per_step": round(ms, 4),
           "kernel_ms": {k_: round(v_, 4) for k_, v_ in zip(STAGES, st)},
           "roofline": dominant_roofline(ps, st, pk),
           "path_roofline": roofline_obj(ps.bytes, ps.flops, ms, pk), "tokens": ps.T,
           "sequences": ps.n, "l2": ps.l2, "steps": n}
    if w is wl.GRAFT_LAYER or w is wl.TINY_KDA:
        res["graph_replay"] = bench_graph(ps, stream, ms, n)
    if w is wl.GRAFT_LAYER:
        res["output_epilogue"] = bench_epilogue(gdr, ps, stream, ms, n)
    if w.snap_interval:
        res["snapshot_offload"] = bench_offload(gdr, ps, stream, ms, n)
    del ps
    torch.cuda.empty_cache()
    return res


def bench_graph(ps, stream, ms_eager, n):
    """The same steps replayed from CUDA graphs (one captured per input set:
    the prefill's launches and their programmatic-launch edges recorded once,
    so a step costs one graph launch on the host)."""
    try:
        graphs = []
        for i in range(len(ps.sets)):
            ps.step(i)                                  # outside capture first
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                ps.step(i)
            graphs.append(g)
        for i in range(2):
            graphs[i % len(graphs)].replay()
        ms = timed(lambda i: graphs[i % len(graphs)].replay(), n, stream)
        del graphs
        return {"ms_per_step": round(ms, 4), "eager_ms_per_step": round(ms_eager, 4),
                "graphs": len(ps.sets)}
    except Exception as e:                              # reported, not fatal
        return {"error": str(e)[:200]}


def bench_epilogue(gdr, ps, stream, ms_plain, n):
    """The same prefill with the RMSNorm and output gate fused into the
    output store (gate_raw [T, H, d_v] bf16 and norm weight [d_v])."""
    gated = []
    for i, s_ in enumerate(ps.sets):
        inp = s_["inp"]
        g = wl.make_output_gate(s_["T"], s_["H"], s_["dv"], inp["q"].dtype, seed=5000 + i,
                                device="cuda", draw_device="cuda")
        p = s_["prep"]
        gated.append((g, gdr.PreparedPrefill(
            inp["q"], inp["k"], inp["v"], inp["beta"], inp["log_a"], inp["cu_seqlens"],
            out=p.out, final_state=p.final_state, workspace=p.workspace,
            scalar_decay=ps.w.scalar_decay, scale=ps.w.scale, init_state=inp["init_state"],
            snap_interval=ps.w.snap_interval, snapshots=p.snapshots, gate_raw=g["gate_raw"],
            norm_weight=g["norm_weight"])))
    for i in range(2):
        gated[i % len(gated)][1].run()
    ms = timed(lambda i: gated[i % len(gated)][1].run(), n, stream)
    gate_bytes = gated[0][0]["gate_raw"].numel() * gated[0][0]["gate_raw"].element_size()
    return {"ms_per_step": round(ms, 4), "plain_ms_per_step": round(ms_plain, 4),
            "overhead_frac": round(ms / ms_plain - 1.0, 4), "gate_bytes_per_step": gate_bytes}


def bench_offload(gdr, ps, stream, ms_plain, n):
    """The same prefill with its snapshots offloaded to pinned host memory:
    (a) written by the state-pass kernel straight into host memory; (b) written
    to device memory and copied on a second stream while the next prefill runs
    (two device snapshot buffers alternate, so a prefill never overwrites a
    buffer being copied)."""
    s0 = ps.sets[0]
    inp, p = s0["inp"], s0["prep"]
    shape = tuple(p.snapshots.shape)
    hosts = [torch.empty(shape, dtype=torch.float32).pin_memory() for _ in range(2)]

    def prepared(snaps):
        return gdr.PreparedPrefill(
            inp["q"], inp["k"], inp["v"], inp["beta"], inp["log_a"], inp["cu_seqlens"],
            out=p.out, final_state=p.final_state, workspace=p.workspace,
            scalar_decay=ps.w.scalar_decay, scale=ps.w.scale, init_state=inp["init_state"],
            snap_interval=ps.w.snap_interval, snapshots=snaps)

    direct = [prepared(h) for h in hosts]
    devs = [p.snapshots, torch.empty_like(p.snapshots)]
    viadev = [prepared(d_) for d_ in devs]
    copy_stream = torch.cuda.Stream()
    events = [torch.cuda.Event() for _ in range(2)]

    def run_direct(i):
        direct[i % 2].run()

    def run_copy(i):
        viadev[i % 2].run()
        gdr.snapshot_offload(devs[i % 2], hosts[i % 2], copy_stream, events[i % 2], stream)

    for i in range(2):
        run_direct(i)
        run_copy(i)
    ms_direct = timed(run_direct, n, stream)
    torch.cuda.synchronize()
    ms_copy = timed(run_copy, n, stream)
    torch.cuda.synchronize()
    same = bool(torch.equal(hosts[(n - 1) % 2], devs[(n - 1) % 2].cpu()))
    nbytes = hosts[0].numel() * 4
    return {"device_snapshots_ms_per_step": round(ms_plain, 4), "host_bytes_per_step": nbytes,
            "copy_stream": {"ms_per_step": round(ms_copy, 4),
                            "overhead_frac": round(ms_copy / ms_plain - 1.0, 4),
                            "host_copy_equals_device": same},
            "direct_host_stores": {"ms_per_step": round(ms_direct, 4),
                                   "overhead_frac": round(ms_direct / ms_plain - 1.0, 4)}}


def bench_decode(gdr, stream, pk, args):
    """Decode step on the decode workload: 1024 steps, four rotating state sets."""
    w = wl.DECODE
    steps = w.steps
    inp = wl.make_decode_inputs(w, steps=steps, device="cuda", draw_device="cuda")
    states = [inp["state"].clone() for _ in range(4)]
    o = torch.empty(w.batch, w.n_heads, w.d_v, device="cuda")

    def step(i):
        t = i % steps
        gdr.decode_step(states[i % 4], inp["q"][t], inp["k"][t], inp["v"][t], inp["beta"][t],
                        inp["log_a"][t], scalar_decay=w.scalar_decay, scale=w.scale, out=o)

    for i in range(8):
        step(i)
    ms = timed(step, steps, stream)
    elem = 2 if w.qkv_dtype == torch.bfloat16 else 4
    per = decode_bytes_per_head_state(w.d_k, w.d_v, elem, w.scalar_decay)
    units = w.batch * w.n_heads
    gbs = per * units / (ms * 1e-3) / 1e9
    res = {"workload": w.name, "gbs": round(gbs, 1), "ms_per_step": round(ms, 5),
           "bytes_per_head_state": per, "head_states_per_step": units,
           "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": pk["hbm_gbs"],
                        "unit": "GB/s", "frac": round(gbs / pk["hbm_gbs"], 4),
                        "traffic": recorded_traffic("decode_step", w.name)},
           "l2": "4 rotating state sets, 235 MB > 126 MB L2", "steps": steps}
    del inp, states
    torch.cuda.empty_cache()
    return res


def bench_spec_decode(gdr, stream, pk, args):
    """Draft (K kept states) and accept on the draft workload, four rotating
    state sets; the kept states (235 MB per draft) exceed L2 on their own."""
    w = wl.SPEC_DRAFT
    d = w.decode
    K, B, H = w.draft_tokens, d.batch, d.n_heads
    inp = wl.make_draft_inputs(w, device="cuda", draw_device="cuda")
    states = [inp["state"].clone() for _ in range(4)]
    o = torch.empty(B, K, H, d.d_v, device="cuda")
    ts = torch.empty(B, K, H, d.d_v, d.d_k, device="cuda")

    def draft(i):
        r = i % w.rounds
        gdr.decode_draft(states[i % 4], inp["q"][r], inp["k"][r], inp["v"][r], inp["beta"][r],
                         inp["log_a"][r], scalar_decay=d.scalar_decay, scale=d.scale, out=o,
                         token_states=ts)

    def accept(i):
        gdr.decode_accept(states[i % 4], ts, inp["n_accept"][i % w.rounds])

    def cycle(i):
        draft(i)
        accept(i)

    for i in range(8):
        cycle(i)
    n = 256
    ms_d = timed(draft, n, stream)
    ms_a = timed(accept, n, stream)
    ms_c = timed(cycle, n, stream)
    elem = 2 if d.qkv_dtype == torch.bfloat16 else 4
    units = B * H
    per = draft_bytes_per_head_state(d.d_k, d.d_v, elem, d.scalar_decay, K)
    gbs_d = per * units / (ms_d * 1e-3) / 1e9
    # accept: n_accept read per sequence; a state copied (read + write) per
    # head of every sequence that accepted at least one token
    acc_frac = float((inp["n_accept"] > 0).float().mean())
    acc_bytes = 4 * B + acc_frac * units * 8 * d.d_k * d.d_v
    gbs_a = acc_bytes / (ms_a * 1e-3) / 1e9
    accepted = float(inp["n_accept"].float().mean()) * B
    res = {"workload": w.name, "draft_tokens": K,
           "draft": {"ms": round(ms_d, 5), "gbs": round(gbs_d, 1),
                     "bytes_per_head_state": per,
                     "roofline": {"bound": "hbm", "achieved": round(gbs_d, 1),
                                  "peak": pk["hbm_gbs"], "unit": "GB/s",
                                  "frac": round(gbs_d / pk["hbm_gbs"], 4),
                                  "traffic": recorded_traffic("decode_draft", w.name)}},
           "accept": {"ms": round(ms_a, 5), "gbs": round(gbs_a, 1),
                      "accepting_fraction": round(acc_frac, 4)},
           "cycle_ms": round(ms_c, 5),
           "accepted_tokens_per_s": round(accepted / (ms_c * 1e-3), 1),
           "l2": "4 rotating state sets; kept states 235 MB per draft > 126 MB L2",
           "cycles": n}
    del inp, states, ts
    torch.cuda.empty_cache()
    return res


def bench_preprocess(gdr, stream, pk, args):
    """Input activations on the graft layer's shape, four rotating input and
    output sets (4 x 148 MB > L2); then the same followed by the prefill."""
    w = wl.PREPROCESS
    names = ("xq", "xk", "xv", "conv_q", "conv_k", "conv_v", "beta_raw", "a_raw", "a_bias",
             "cu_seqlens")
    sets = []
    for i in range(4):
        inp = wl.make_preprocess_inputs(wl.shrink(w, seed=w.seed + 10 * i), device="cuda",
                                        draw_device="cuda")
        T, H, d = inp["xq"].shape
        act = {n: torch.empty(T, H, d, dtype=inp["xq"].dtype, device="cuda") for n in ("q", "k", "v")}
        act["beta"] = torch.empty(T, H, device="cuda")
        act["log_a"] = torch.empty(inp["a_raw"].shape, device="cuda")
        ws = torch.empty(gdr.workspace_size(1, H, d, d, T), dtype=torch.uint8, device="cuda")
        prep = gdr.PreparedPrefill(act["q"], act["k"], act["v"], act["beta"], act["log_a"],
                                   inp["cu_seqlens"], out=torch.empty_like(act["v"]),
                                   final_state=torch.empty(1, H, d, d, device="cuda"),
                                   workspace=ws)
        sets.append((inp, act, prep))

    def pre(i):
        inp, act, _ = sets[i % 4]
        gdr.preprocess(*(inp[n] for n in names), out=act)

    def layer(i):
        pre(i)
        sets[i % 4][2].run()

    def plain(i):
        sets[i % 4][2].run()

    def fused(i):
        inp, _, prep = sets[i % 4]
        gdr.prefill_from_projections(*(inp[n_] for n_ in names), out=prep.out,
                                     final_state=prep.final_state, workspace=prep.workspace)

    for i in range(8):
        layer(i)
        fused(i)
    n = 200
    ms_p = timed(pre, n, stream)
    ms_l = timed(layer, n, stream)
    ms_plain = timed(plain, n, stream)
    ms_f = timed(fused, n, stream)
    T, H, d = sets[0][0]["xq"].shape
    elem = 2 if w.qkv_dtype == torch.bfloat16 else 4
    per = preprocess_bytes_per_token_head(d, elem, w.scalar_decay)
    gbs = per * T * H / (ms_p * 1e-3) / 1e9
    res = {"workload": w.name, "ms": round(ms_p, 5), "gbs": round(gbs, 1),
           "bytes_per_token_head": per,
           "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": pk["hbm_gbs"],
                        "unit": "GB/s", "frac": round(gbs / pk["hbm_gbs"], 4),
                        "traffic": recorded_traffic("preprocess", w.name)},
           "with_prefill": {"ms_per_step": round(ms_l, 5),
                            "tokens_per_s": round(T / (ms_l * 1e-3), 1)},
           "fused_prefill_from_projections": {
               "ms_per_step": round(ms_f, 5), "tokens_per_s": round(T / (ms_f * 1e-3), 1),
               "plain_prefill_ms": round(ms_plain, 5),
               "over_plain_prefill": round(ms_f / ms_plain - 1.0, 4)},
           "l2": "4 rotating input and output sets, 4 x 148 MB > 126 MB L2", "steps": n}
    del sets
    torch.cuda.empty_cache()
    return res


def bench_e2e(gdr, w, stream, args):
    """The main workload's prefill through the public API from pinned host
    buffers, every step: H2D of the inputs, the prefill, D2H of o and the
    final states.  Timed twice: all on one stream, and pipelined over three
    streams (step i+1's H2D and step i-1's D2H overlap step i's prefill; two
    device buffer sets alternate, ordered by events) -- ``value`` is the
    pipelined figure, each step still moving all of its bytes."""
    dev0 = wl.make_prefill_inputs(w, device="cuda", draw_device="cuda")
    names = [k_ for k_ in ("q", "k", "v", "beta", "log_a", "cu_seqlens", "init_state")
             if dev0.get(k_) is not None]
    pinned = {k_: dev0[k_].cpu().pin_memory() for k_ in names}
    T, H, dk = pinned["q"].shape
    dv = pinned["v"].shape[-1]
    n = pinned["cu_seqlens"].numel() - 1
    ws = torch.empty(gdr.workspace_size(n, H, dk, dv, T, w.scalar_decay), dtype=torch.uint8,
                     device="cuda")
    ns = gdr.snapshot_count(pinned["cu_seqlens"], w.snap_interval) if w.snap_interval else 0
    bufs = []
    for b in range(2):
        dev = dev0 if b == 0 else {k_: torch.empty_like(dev0[k_]) for k_ in names}
        dev = {k_: dev[k_] for k_ in names}
        out = torch.empty(T, H, dv, dtype=pinned["q"].dtype, device="cuda")
        fin = torch.empty(n, H, dv, dk, device="cuda")
        snaps = torch.empty(max(ns, 1), H, dv, dk, device="cuda") if w.snap_interval else None
        prep = gdr.PreparedPrefill(dev["q"], dev["k"], dev["v"], dev["beta"], dev["log_a"],
                                   dev["cu_seqlens"], out=out, final_state=fin, workspace=ws,
                                   scalar_decay=w.scalar_decay, scale=w.scale,
                                   init_state=dev.get("init_state"),
                                   snap_interval=w.snap_interval, snapshots=snaps)
        out_h = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        fin_h = torch.empty(fin.shape, dtype=fin.dtype).pin_memory()
        bufs.append(dict(dev=dev, out=out, fin=fin, prep=prep, out_h=out_h, fin_h=fin_h,
                         loaded=torch.cuda.Event(), done=torch.cuda.Event(),
                         read=torch.cuda.Event()))
    del dev0

    def serial(i):
        b = bufs[0]
        for k_ in names:
            b["dev"][k_].copy_(pinned[k_], non_blocking=True)
        b["prep"].run()
        b["out_h"].copy_(b["out"], non_blocking=True)
        b["fin_h"].copy_(b["fin"], non_blocking=True)

    h2d, d2h = torch.cuda.Stream(), torch.cuda.Stream()

    def pipelined(i):
        b = bufs[i % 2]
        with torch.cuda.stream(h2d):
            if i >= 2:
                h2d.wait_event(b["done"])            # prefill i-2 has read these inputs
            for k_ in names:
                b["dev"][k_].copy_(pinned[k_], non_blocking=True)
            b["loaded"].record(h2d)
        stream.wait_event(b["loaded"])
        if i >= 2:
            stream.wait_event(b["read"])             # D2H of step i-2 has read o, final
        b["prep"].run(stream=stream)
        b["done"].record(stream)
        with torch.cuda.stream(d2h):
            d2h.wait_event(b["done"])
            b["out_h"].copy_(b["out"], non_blocking=True)
            b["fin_h"].copy_(b["fin"], non_blocking=True)
            b["read"].record(d2h)

    def timed_streams(fn, n_steps):
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        start.record(stream)
        h2d.wait_event(start)
        d2h.wait_event(start)
        for i in range(n_steps):
            fn(i)
        stream.wait_stream(h2d)
        stream.wait_stream(d2h)
        end.record(stream)
        torch.cuda.synchronize()
        return start.elapsed_time(end) / n_steps

    for i in range(3):
        serial(i)
    for i in range(4):
        pipelined(i)
    torch.cuda.synchronize()
    n_steps = max(5, min(args.steps, 20))
    ms_serial = timed_streams(serial, n_steps)
    ms = timed_streams(pipelined, n_steps)
    h2d_bytes = sum(t.numel() * t.element_size() for t in pinned.values())
    b0 = bufs[0]
    d2h_bytes = b0["out_h"].numel() * b0["out_h"].element_size() + \
        b0["fin_h"].numel() * b0["fin_h"].element_size()
    res = {"value": round(T / (ms * 1e-3), 1), "unit": "tokens/s", "h2d_bytes_per_step": h2d_bytes,
           "d2h_bytes_per_step": d2h_bytes, "ms_per_step": round(ms, 4),
           "serial_one_stream": {"ms_per_step": round(ms_serial, 4),
                                 "tokens_per_s": round(T / (ms_serial * 1e-3), 1)},
           "steps": n_steps, "workload": w.name,
           "pipelining": "H2D, prefill and D2H on three streams, two buffer sets"}
    del pinned, bufs, ws
    torch.cuda.empty_cache()
    return res


def main():
    p = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=2000)
    p.add_argument("--warmup", type=int, default=20)
    p.add_argument("--impl", choices=["gdr", "reference"], default="gdr")
    p.add_argument("--no-extra", action="store_true", help="skip decode and the other workloads")
    p.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline")
    p.add_argument("--no-e2e", action="store_true",
                   help="skip the end-to-end measurement (for profiling runs)")
    p.add_argument("--only-decode", action="store_true",
                   help="run only the decode measurement (for profiling)")
    p.add_argument("--only-spec", action="store_true",
                   help="run only the speculative-decoding measurement (for profiling)")
    p.add_argument("--only-preprocess", action="store_true",
                   help="run only the input-activation measurement (for profiling)")
    p.add_argument("--workload", default=wl.VARLEN.name,
                   choices=sorted(wl.PREFILL_WORKLOADS) + sorted(wl.PROFILE_CASES),
                   help="prefill workload of the main line (default: the varlen batch, the "
                        "largest workload)")
    p.add_argument("--sets", type=int, default=0,
                   help="rotating input sets of the main line (default: enough to exceed L2)")
    args = p.parse_args()
    if args.warmup < 3:
        p.error("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    elif args.only_decode:
        import gated_delta_rule_150_b200 as gdr
        gdr.lib()
        print(json.dumps(bench_decode(gdr, torch.cuda.current_stream(), peaks(), args)), flush=True)
    elif args.only_preprocess:
        import gated_delta_rule_150_b200 as gdr
        gdr.lib()
        print(json.dumps(bench_preprocess(gdr, torch.cuda.current_stream(), peaks(), args)),
              flush=True)
    elif args.only_spec:
        import gated_delta_rule_150_b200 as gdr
        gdr.lib()
        print(json.dumps(bench_spec_decode(gdr, torch.cuda.current_stream(), peaks(), args)),
              flush=True)
    else:
        run_gdr(args)


if __name__ == "__main__":
    main()
