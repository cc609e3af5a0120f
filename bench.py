#!/usr/bin/env python
"""Benchmark: one decode-attention layer step of KV-parallel (sequence-sharded) attention.

A step = append one new token per request (helix_kv_append) + per-shard partial attention over the
whole history (helix_attn_partial) + the LSE-rescaling combine (helix_attn_combine), on synthetic
seeded inputs already resident in HBM. Default workload: B=8 requests, 128 query heads, 8 KV heads,
d=128, 1,048,576-token bf16 history per request, 8 KV-parallel shards with round-robin-16 placement.

Prints ONE JSON line (rank 0): the headline workload's fields first; after its timed region the
NVFP4 and MLA workloads at the same context are timed the same way and reported under
``per_workload`` (each with its own roofline, clocks and end-to-end figure). ``--impl reference``
times the fp64 CPU oracle instead, on a bounded sample of the same workload, scaled to the same unit.

Multi-GPU (torchrun, N ranks): by default every rank runs its own independent batch (replicas, weak
scaling); the step time is the max over ranks. ``--kvp-ranks`` instead makes rank r KVP shard r of
one batch (the pages' setting): each step appends on the owning rank, runs the partial over the
local shard and exchanges the partials (the owner's combine reads them from the other GPUs).
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import workloads as wl  # noqa: E402

METRIC = "us per decode-attention layer step & achieved HBM TB/s (B=8, 1M ctx, 1 GPU)"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS_SUSTAINED = 1400.0
SPEC_HBM_GBS = 8000.0  # B200 HBM3e data-sheet bandwidth, for context beside the measured peaks
# workloads timed after the headline one and reported under per_workload
DEFAULT_ALSO = {"gqa_s1m": ["gqa_nvfp4_s1m", "mla_s1m"]}


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=40)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="helix", choices=["helix", "reference"])
    ap.add_argument("--workload", default="gqa_s1m", choices=sorted(wl.WORKLOADS))
    ap.add_argument("--also", default="auto",
                    help="comma-separated workloads timed after the headline one and reported "
                         "under 'per_workload' ('auto': NVFP4 and MLA after gqa_s1m; '' = none)")
    ap.add_argument("--min-timed-ms", type=float, default=300.0,
                    help="per_workload entries time at least this long (more steps if needed) so "
                         "that the clock record has several samples")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--graph", action="store_true",
                    help="also time the steps launched from CUDA graphs (reported under 'graph')")
    ap.add_argument("--hopb-groups", type=int, default=4,
                    help="request groups of the two-stream HOP-B analogue, timed after the main "
                         "steps and reported under 'hopb' (0 = skip)")
    ap.add_argument("--kvp-ranks", action="store_true",
                    help="under torchrun: rank r is KVP shard r of one batch; time append + "
                         "partial + exchange/combine per step (reported under 'kvp')")
    ap.add_argument("--kvp-exchange", default="peer", choices=["peer", "gather"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-read-probe", action="store_true",
                    help="skip the pure-read bandwidth probe reported beside the roofline")
    ap.add_argument("--cpu-sample-tokens", type=int, default=None,
                    help="history tokens per sampled head group for the CPU oracle (default: "
                         "about 2^18 tokens' worth of GQA work, see cpu_sample_plan)")
    ap.add_argument("--cpu-sample-groups", type=int, default=2)
    ap.add_argument("--cpu-baseline-samples", type=int, default=20,
                    help="samples the cpu_baseline leg times (each as one reference-arm step)")
    ap.add_argument("--wait-limit-s", type=float, default=300.0,
                    help="limit of every host wait on the GPU (helix_stream_wait)")
    ap.add_argument("--context", type=int, default=None,
                    help="override the history length (fixed lengths), e.g. for small profiling runs")
    return ap.parse_args(argv)


# ------------------------------------------------------------------------------------------------
# distributed plumbing


def dist_init(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist

        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist

    t = torch.tensor([x], dtype=torch.float64,
                     device="cuda" if dist.get_backend() == "nccl" else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------------------------------------------
# clocks during the timed region

# NVML clock-event reason bits (nvml.h, nvmlClocksEventReason*)
_REASON_BITS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
                "hw_thermal_slowdown": 0x40}


class ClockSampler:
    """SM clock and throttle reasons sampled while a timed region runs. NVML (nvidia-ml-py) is
    read every 5 ms from a thread; without it, ``nvidia-smi -lms 100`` writes to a scratch file
    (HELIX_CLOCKS_DIR, else the system temp directory). Both only read the GPU's state."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, interval_s: float = 0.005):
        self.gpu = gpu_index
        self.interval = interval_s
        self.proc = None
        self.thread = None
        self.samples = []
        self.max_mhz = None
        out_dir = os.environ.get("HELIX_CLOCKS_DIR") or tempfile.gettempdir()
        self.path = os.path.join(out_dir, f"helix_clocks_rank{gpu_index}.csv")
        self.nvml = None
        try:
            import pynvml

            pynvml.nvmlInit()
            # the physical index of the visible device
            vis = os.environ.get("CUDA_VISIBLE_DEVICES")
            phys = int(vis.split(",")[gpu_index]) if vis and vis.split(",")[0].isdigit() else gpu_index
            self.handle = pynvml.nvmlDeviceGetHandleByIndex(phys)
            self.nvml = pynvml
        except Exception:
            self.nvml = None

    def _poll(self):
        nv = self.nvml
        get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self._stop.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(self.handle, nv.NVML_CLOCK_SM)
                bits = get_reasons(self.handle)
                self.samples.append((float(sm), int(bits)))
            except Exception:
                pass
            self._stop.wait(self.interval)

    def start(self):
        self.samples = []
        if self.nvml is not None:
            try:
                self.max_mhz = float(self.nvml.nvmlDeviceGetMaxClockInfo(self.handle,
                                                                         self.nvml.NVML_CLOCK_SM))
            except Exception:
                self.max_mhz = None
            self._stop = threading.Event()
            self.thread = threading.Thread(target=self._poll, daemon=True)
            self.thread.start()
            return
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", str(self.gpu)], stdout=self.fh, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
            return
        # nvidia-smi takes a while to print its first line: wait for it (bounded)
        t_end = time.time() + 5.0
        while time.time() < t_end and self.proc.poll() is None:
            self.fh.flush()
            if os.path.getsize(self.path) > 0:
                break
            time.sleep(0.02)

    def stop(self):
        if self.thread is not None:
            self._stop.set()
            self.thread.join(timeout=5)
            self.thread = None
            if not self.samples:
                return None
            reasons = sorted(n for n, bit in _REASON_BITS.items()
                             if any(b & bit for _, b in self.samples))
            return {"sm_mhz": statistics.median(s for s, _ in self.samples),
                    "sm_max_mhz": self.max_mhz, "reasons": reasons,
                    "samples": len(self.samples), "source": "nvml, 5 ms"}
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.fh.close()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm), "source": "nvidia-smi, 100 ms"}


def read_probe_gbs(dev, gib: int = 4, reps: int = 5):
    """HBM read bandwidth of a plain torch reduction over a buffer far larger than L2, best of
    `reps` (CUDA events): a pure-read figure taken in the same run, for context beside the measured
    copy peak. It is not one of this library's kernels and runs outside the timed region."""
    try:
        x = torch.ones(gib << 28, dtype=torch.float32, device=dev)
        best = None
        for _ in range(reps + 1):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            torch.sum(x)
            e1.record()
            torch.cuda.synchronize()
            ms = e0.elapsed_time(e1)
            best = ms if best is None else min(best, ms)
        gbs = x.numel() * 4 / (best * 1e-3) / 1e9
        del x
        torch.cuda.empty_cache()
        return {"gbs": gbs, "how": f"torch.sum over a {gib} GiB fp32 buffer, best of {reps}"}
    except RuntimeError:
        return None


def measured_peaks():
    """(HBM GB/s, bf16 TFLOP/s sustained, source). The sustained tensor figure applies because the
    partial kernel is timed inside a long step."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), float(d["bf16_tflops_sustained"]), "measured"
    return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS_SUSTAINED, "fallback"


def profile_traffic(kernel: str, workload: str):
    """dram read+write bytes per launch from a committed ncu summary, when one exists for this
    workload and the kernel source is unchanged since the counters were taken; otherwise None."""
    import hashlib

    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    e = json.load(open(p)).get(f"{kernel}:{workload}")
    if e is None:
        return None
    src = os.path.join(ROOT, e["source"])
    if not os.path.exists(src):
        return None
    sha = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    return e["dram_bytes_per_launch"] if sha == e["source_sha256_16"] else None


# ------------------------------------------------------------------------------------------------
# CPU oracle: one sampling recipe for the reference arm and the cpu_baseline leg


def cpu_sample_plan(w: wl.Workload, groups: int, tokens: int | None):
    """The bounded sample both CPU legs time: ``groups`` seeded (request, KV head) groups of
    ``tokens`` history tokens each. By default the token count gives about the work of 2^18 tokens
    of the GQA workloads (16 heads x (128 + 128) wide), so an MLA sample is shorter."""
    lens = wl.seq_lens(w)
    if tokens is None:
        per_pair = w.G * (w.d + w.dv)
        tokens = int(2 ** round(np.log2((1 << 18) * 16 * 256 / per_pair)))
    T = max(1, min(tokens, min(lens)))
    rng = np.random.default_rng(w.seed)
    n_groups = w.B * w.Hkv
    if groups >= n_groups:
        picks = [(b, h) for b in range(w.B) for h in range(w.Hkv)]
    else:
        picks = [(int(rng.integers(w.B)), int(rng.integers(w.Hkv))) for _ in range(64)]
    total_pairs = sum(lens) * w.Hkv
    return {"T": T, "groups": min(groups, n_groups), "picks": picks, "total_pairs": total_pairs,
            "sample_pairs": min(groups, n_groups) * T, "lens": lens}


def _oracle_inputs(w, b, h, T):
    import oracle

    if w.kind == "mla":
        K = oracle.attention._f64(wl.kv_range_bf16(w, "c", b, 0, 0, T))
        return K, K[:, : w.dv]
    if w.kv_dtype == "nvfp4":
        return (oracle.nvfp4_dequant(*wl.kv_range_nvfp4(w, "k", b, h, 0, T)),
                oracle.nvfp4_dequant(*wl.kv_range_nvfp4(w, "v", b, h, 0, T)))
    return (oracle.attention._f64(wl.kv_range_bf16(w, "k", b, h, 0, T)),
            oracle.attention._f64(wl.kv_range_bf16(w, "v", b, h, 0, T)))


def cpu_oracle_time(w: wl.Workload, plan, sample_index: int, q=None):
    """Time the fp64 oracle (per-shard partials + combine) on sample ``sample_index`` of the plan
    (its groups taken in turn from the seeded pick list); input generation is not timed. Returns
    (seconds, us per full step scaled linearly from the sample)."""
    import oracle

    q = wl.query(w) if q is None else q
    g = plan["groups"]
    picks = [plan["picks"][(sample_index * g + i) % len(plan["picks"])] for i in range(g)]
    elapsed = 0.0
    for b, h in picks:
        K, V = _oracle_inputs(w, b, h, plan["T"])
        qg = q[b, h * w.G:(h + 1) * w.G]
        t0 = time.perf_counter()
        sets = oracle.shard_tokens(plan["T"], w.kvp, w.layout, w.rr_block, w.contig_chunk)
        parts = [oracle.attend(qg, K[idx], V[idx], w.softmax_scale) for idx in sets]
        oracle.combine(np.stack([p[0] for p in parts]), np.stack([p[1] for p in parts]))
        elapsed += time.perf_counter() - t0
    return elapsed, elapsed / plan["sample_pairs"] * plan["total_pairs"] * 1e6


def sample_desc(w, plan):
    scale = plan["total_pairs"] / plan["sample_pairs"]
    return (f"{plan['groups']} (request, KV head) groups x {plan['T']} history tokens each "
            f"({plan['sample_pairs']} of {plan['total_pairs']} token-head pairs per step), "
            f"per-shard fp64 partials + combine; input generation not timed; "
            f"scaled linearly to a full step (x{scale:.4g})")


def tiny_full_oracle():
    """The tiny workload (4,096 tokens, 4 contiguous shards) timed in full, not extrapolated: all
    host cores, then one thread (BLAS limited to 1)."""
    from threadpoolctl import threadpool_limits

    import oracle

    w = wl.WORKLOADS["tiny_gqa"]
    lens = wl.seq_lens(w)
    q = wl.query(w)
    ins = {(b, h): _oracle_inputs(w, b, h, lens[b]) for b in range(w.B) for h in range(w.Hkv)}

    def run():
        t0 = time.perf_counter()
        for (b, h), (K, V) in ins.items():
            qg = q[b, h * w.G:(h + 1) * w.G]
            sets = oracle.shard_tokens(lens[b], w.kvp, w.layout, w.rr_block, w.contig_chunk)
            parts = [oracle.attend(qg, K[idx], V[idx], w.softmax_scale) for idx in sets]
            oracle.combine(np.stack([p[0] for p in parts]), np.stack([p[1] for p in parts]))
        return time.perf_counter() - t0

    run()
    multi = min(run() for _ in range(5))
    with threadpool_limits(limits=1):
        run()
        single = min(run() for _ in range(5))
    return {"workload": "tiny_gqa", "us_per_step": multi * 1e6, "cores": cores(),
            "us_per_step_1thread": single * 1e6, "extrapolated": False,
            "how": "whole step (every head group, every shard, combine), best of 5"}


def cores():
    return len(os.sched_getaffinity(0))


def cpu_baseline(w, args):
    """The cpu_baseline leg: the same samples the reference arm times per step, here
    ``--cpu-baseline-samples`` of them, reported as the mean of the per-sample scaled times."""
    plan = cpu_sample_plan(w, args.cpu_sample_groups, args.cpu_sample_tokens)
    q = wl.query(w)
    vals = [cpu_oracle_time(w, plan, i, q)[1] for i in range(args.cpu_baseline_samples)]
    return {"value": float(np.mean(vals)), "unit": "us/step", "cores": cores(), "kind": "oracle",
            "sample": sample_desc(w, plan) + f"; mean of {len(vals)} samples",
            "extrapolated": True, "scale": plan["total_pairs"] / plan["sample_pairs"],
            "spread": [float(min(vals)), float(max(vals))], "tiny_full": tiny_full_oracle()}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    w = wl.WORKLOADS[args.workload]
    plan = cpu_sample_plan(w, args.cpu_sample_groups, args.cpu_sample_tokens)
    q = wl.query(w)
    for i in range(args.warmup):
        cpu_oracle_time(w, plan, i, q)
    vals = [cpu_oracle_time(w, plan, i, q)[1] for i in range(args.steps)]
    value = float(np.mean(vals))
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "us/step",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": value / 1e3, "higher_is_better": False, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(w, plan["lens"]),
        "parallelism": "one process on the host cores (rank 0)",
        "cpu_baseline": {"value": value, "unit": "us/step", "cores": cores(), "kind": "oracle",
                         "sample": sample_desc(w, plan) + "; one sample per step",
                         "extrapolated": True,
                         "scale": plan["total_pairs"] / plan["sample_pairs"]},
        "e2e": {"value": value, "unit": "us/step", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def config_of(w, lens):
    return {"workload": w.name, "kind": w.kind, "kv_dtype": w.kv_dtype, "B": w.B, "Hq": w.Hq,
            "Hkv": w.Hkv, "d": w.d, "dv": w.dv, "S_mean": float(np.mean(lens)),
            "S_min": int(min(lens)), "S_max": int(max(lens)), "kvp": w.kvp, "layout": w.layout,
            "rr_block": w.rr_block, "page_tokens": w.page_tokens,
            "l2": "inputs larger than L2 (the KV history is re-read in full every step)"}


# ------------------------------------------------------------------------------------------------
# GPU arm


class Step:
    """One workload's state resident in HBM and the calls of one decode step."""

    def __init__(self, hx, w, dev, n_steps):
        self.hx, self.dev = hx, dev
        lens = wl.seq_lens(w)
        S_cap = max(lens) + n_steps + 16
        if w.layout == "contig":  # size the contiguous shards for the history plus the new tokens
            w = w.with_(S_final=S_cap)
        self.w, self.lens = w, lens
        pt, n_pages = wl.page_table(w, S_cap)
        self.cache = hx.KVCache(hx.ATTN_MLA if w.kind == "mla" else hx.ATTN_GQA,
                                hx.KV_NVFP4 if w.kv_dtype == "nvfp4" else hx.KV_BF16,
                                hx.LAYOUT_RR if w.layout == "rr" else hx.LAYOUT_CONTIG,
                                w.kvp, w.B, w.Hkv, w.d, w.dv, pt.shape[2],
                                page_tokens=w.page_tokens, rr_block=w.rr_block,
                                contig_chunk=w.contig_chunk, page_table=pt, num_pages=n_pages,
                                device=dev)
        # the history (S_b - 1 tokens), then one new token per step
        hist = [L - 1 for L in lens]
        chunk = 65536
        for t0 in range(0, max(hist), chunk):
            n = min(chunk, max(hist) - t0)
            nv = torch.tensor([min(max(L - t0, 0), n) for L in hist], dtype=torch.int32,
                              device=dev)
            hx.append(self.cache, **wl.append_rows(w, t0, t0 + n, dev), n_valid=nv)
        torch.cuda.synchronize()
        assert self.cache.err_bits() == 0, "prefill reported a device error"
        # An NVFP4 cache takes the new token as bf16 rows and encodes it on the device
        # (helix_kv_append_quantize), as a decode loop over an FP4 cache does.
        self.quant = w.kv_dtype == "nvfp4"
        if self.quant:
            rows = {"k_new": torch.stack([wl.kv_tokens(w, "k", b, 0, n_steps, dev)
                                          for b in range(w.B)]),
                    "v_new": torch.stack([wl.kv_tokens(w, "v", b, 0, n_steps, dev)
                                          for b in range(w.B)])}
        else:
            rows = wl.append_rows(w, 0, n_steps, dev)
        # [step][B][1][...]: each step's slice is dense
        self.rows = {k: v.transpose(0, 1).unsqueeze(2).contiguous() for k, v in rows.items()}
        self.q = wl.query(w, dev)
        self.o_part = torch.empty(w.kvp, w.B, w.Hq, w.dv, dtype=torch.float32, device=dev)
        self.lse_part = torch.empty(w.kvp, w.B, w.Hq, dtype=torch.float32, device=dev)
        self.out = torch.empty(w.B, w.Hq, w.dv, dtype=torch.bfloat16, device=dev)
        self.lse_out = torch.empty(w.B, w.Hq, dtype=torch.float32, device=dev)
        self.ws = self.cache.workspace(w.Hq)
        self.stream = torch.cuda.current_stream()
        self.si = 0  # next unused new-token row

    def append(self, a):
        if self.quant:
            self.hx.append_quantize(self.cache, a["k_new"], a["v_new"])
        else:
            self.hx.append(self.cache, a["k_new"], a.get("v_new"), a.get("k_scale"),
                           a.get("v_scale"))

    def attend(self, q=None):
        # partial attention and the combine: one launch for GQA (helix_attn_partial_combine)
        self.hx.partial_combine(self.cache, self.q if q is None else q, self.w.softmax_scale,
                                self.o_part, self.lse_part, self.out, self.lse_out,
                                workspace=self.ws)

    def one(self, ev=None):
        self.append({k: v[self.si] for k, v in self.rows.items()})
        self.si += 1
        if ev is not None:
            ev[0].record(self.stream)
        self.attend()
        if ev is not None:
            ev[1].record(self.stream)

    def launches_per_step(self):
        # append (one kernel) + the fused partial/combine (GQA) or partial + combine (MLA)
        return 3 if self.w.kind == "mla" else 2


def wait(hx, args, stream=None):
    """Bounded host wait for the GPU (helix_stream_wait); raises HelixError on timeout."""
    hx.wait(stream, limit_s=args.wait_limit_s)


def time_steps(hx, st: Step, K, W, args, world, local):
    """W untimed steps, then exactly K timed steps between barriers; per-step events around the
    partial (+ combine). Returns (ms per step max over ranks, per-step partial ms, clocks)."""
    for _ in range(W):
        st.one()
    wait(hx, args)
    clocks = ClockSampler(local)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(K)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    wait(hx, args)
    clocks.start()
    torch.cuda.nvtx.range_push("timed_steps")  # lets a profiler's launch list select this region
    start.record(st.stream)
    for i in range(K):
        st.one(evs[i])
    stop.record(st.stream)
    torch.cuda.nvtx.range_pop()
    wait(hx, args)
    clk = clocks.stop()
    barrier(world)
    ms_step = max_over_ranks(start.elapsed_time(stop) / K, world)
    assert st.cache.err_bits() == 0, "a timed step reported a device error"
    return ms_step, [a.elapsed_time(b) for a, b in evs], clk


def time_e2e(hx, st: Step, K, args, world):
    """The same step through the public calls with host buffers: q and the new token copied in
    from pinned memory, O copied back, every step, inside the timed region."""
    q_h = st.q.cpu().pin_memory()
    rows_h = {k: v.cpu().pin_memory() for k, v in st.rows.items()}
    out_h = torch.empty(st.out.shape, dtype=st.out.dtype).pin_memory()
    q_d = torch.empty_like(st.q)
    tok_d = {k: torch.empty_like(v[0]) for k, v in st.rows.items()}
    h2d = st.q.numel() * st.q.element_size() + sum(
        v[0].numel() * v.element_size() for v in st.rows.values())
    d2h = st.out.numel() * st.out.element_size()
    barrier(world)
    wait(hx, args)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(st.stream)
    for _ in range(K):
        q_d.copy_(q_h, non_blocking=True)
        for k_ in tok_d:
            tok_d[k_].copy_(rows_h[k_][st.si], non_blocking=True)
        st.si += 1
        st.append(tok_d)
        st.attend(q_d)
        out_h.copy_(st.out, non_blocking=True)
    e1.record(st.stream)
    wait(hx, args)
    barrier(world)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / K, world)
    return {"value": e2e_ms * 1e3, "unit": "us/step", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h}


def time_graph(hx, st: Step, K, W, args, world, dev):
    graphs = []
    cap_stream = torch.cuda.Stream(dev)
    for _ in range(K):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=cap_stream):
            st.one()
        graphs.append(g)
    wait(hx, args)
    for g in graphs[:min(W, K)]:  # warm-up replays
        g.replay()
    barrier(world)
    wait(hx, args)
    g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    g0.record()
    for g in graphs:
        g.replay()
    g1.record()
    wait(hx, args)
    barrier(world)
    graph_ms = max_over_ranks(g0.elapsed_time(g1) / K, world)
    del graphs
    assert st.cache.err_bits() == 0, "a graph-launched step reported a device error"
    return {"us_per_step": graph_ms * 1e3, "steps": K,
            "how": "each step captured once in a CUDA graph, then replayed back to back"}


def time_hopb(hx, st: Step, K, W, args, world, dev, serial_ms):
    """HOP-B analogue: the combine of request group g on a second stream overlaps the partial of
    group g+1 (and, for bf16 caches, the appends too); same inputs, timed like the main steps."""
    ov = hx.Overlap(args.hopb_groups, dev)
    w = st.w

    def hopb_step():
        a = {k: v[st.si] for k, v in st.rows.items()}
        st.si += 1
        if st.quant:  # the device-encoding append is not part of the overlapped call
            st.append(a)
            hx.overlapped(st.cache, st.q, w.softmax_scale, ov, st.o_part, st.lse_part, st.out,
                          st.lse_out, workspace=st.ws)
        else:  # append, partial and combine of request groups over two streams
            hx.decode_overlapped(st.cache, st.q, w.softmax_scale, ov, a["k_new"], a.get("v_new"),
                                 o_partial=st.o_part, lse=st.lse_part, out=st.out,
                                 lse_out=st.lse_out, workspace=st.ws)

    for _ in range(W):
        hopb_step()
    barrier(world)
    wait(hx, args)
    h0, h1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    h0.record(st.stream)
    for _ in range(K):
        hopb_step()
    h1.record(st.stream)
    wait(hx, args)
    barrier(world)
    hopb_ms = max_over_ranks(h0.elapsed_time(h1) / K, world)
    n_groups = min(args.hopb_groups, w.B)
    per = -(-w.B // n_groups)
    groups = -(-w.B // per)
    assert st.cache.err_bits() == 0, "a HOP-B step reported a device error"
    return {"groups": groups, "us_per_step": hopb_ms * 1e3, "serial_us_per_step": serial_ms * 1e3,
            "speedup": serial_ms / hopb_ms, "gpu_launches": K * 3 * groups}


def roofline(w, lens_at, part_ms, read_probe):
    """The dominant kernel's roofline: algorithmic bytes (and flops) per launch over its mean
    event-timed duration, against the measured peaks; the binding roof is the one with the longer
    ideal time."""
    part_bytes = float(np.mean([wl.partial_bytes(w, L) for L in lens_at])) + wl.combine_bytes(w)
    peak, tflops_peak, peak_kind = measured_peaks()
    achieved_gbs = part_bytes / (part_ms * 1e-3) / 1e9
    kname = ("mla_partial_kernel + combine_kernel" if w.kind == "mla" else
             "gqa_partial_nvfp4_kernel (fused combine)" if w.kv_dtype == "nvfp4" else
             f"gqa_partial_kernel<{w.d}> (fused combine)")
    flops = float(np.mean([wl.partial_flops(w, L) for L in lens_at]))
    achieved_tf = flops / (part_ms * 1e-3) / 1e12
    hbm = {"achieved": achieved_gbs, "peak": peak, "unit": "GB/s", "frac": achieved_gbs / peak}
    tensor = {"achieved": achieved_tf, "peak": tflops_peak, "unit": "TFLOP/s",
              "frac": achieved_tf / tflops_peak}
    tensor_bound = flops / (tflops_peak * 1e12) > part_bytes / (peak * 1e9)
    hbm["frac_of_spec"] = achieved_gbs / SPEC_HBM_GBS
    if read_probe is not None:
        hbm["frac_of_read_probe"] = achieved_gbs / read_probe["gbs"]
    return dict(tensor if tensor_bound else hbm, bound="tensor" if tensor_bound else "hbm",
                peak_source=peak_kind, kernel=kname, bytes_per_launch=part_bytes,
                flops_per_launch=flops, other=(hbm if tensor_bound else tensor),
                traffic=profile_traffic("partial", w.name))


def measure(hx, w, args, K, W, world, local, dev, extras: bool, read_probe=None):
    """Build a workload's state, time its steps (and, when ``extras``, the graph and HOP-B forms)
    and return the fields of its JSON record."""
    n_steps = (K + W + (K if not args.no_e2e else 0) +
               ((W + K) if (extras and args.graph) else 0) +
               ((W + K) if (extras and args.hopb_groups > 0) else 0))
    st = Step(hx, w, dev, n_steps)
    w = st.w
    lens_at = [[L + W + i for L in st.lens] for i in range(K)]  # lengths during timed step i
    ms_step, partial_ms, clk = time_steps(hx, st, K, W, args, world, local)
    rec = {"value": ms_step * 1e3, "unit": "us/step", "steps": K, "warmup": W,
           "ms_per_step": ms_step}
    part_ms = float(np.mean(partial_ms))
    step_bytes = float(np.mean([wl.step_bytes(w, L) for L in lens_at]))
    rec["achieved_hbm_tbs"] = step_bytes / (ms_step * 1e-3) / 1e12 * world
    rec["step_bytes"] = step_bytes
    rec["kernels_us"] = {"partial_and_combine": part_ms * 1e3,
                         "append_and_gaps": ms_step * 1e3 - part_ms * 1e3}
    rec["gpu_launches"] = st.launches_per_step() * K
    rec["roofline"] = roofline(w, lens_at, part_ms, read_probe)
    rec["clocks"] = clk
    rec["e2e"] = None if args.no_e2e else time_e2e(hx, st, K, args, world)
    if extras:
        rec["graph"] = time_graph(hx, st, K, W, args, world, dev) if args.graph else None
        rec["hopb"] = (time_hopb(hx, st, K, W, args, world, dev, ms_step)
                       if args.hopb_groups > 0 else None)
    rec["config"] = config_of(w, st.lens)
    rec["dtype"] = "bf16" if w.kv_dtype == "bf16" else "nvfp4"
    del st
    torch.cuda.empty_cache()
    return rec


def also_list(args):
    if args.also == "auto":
        return [] if args.context is not None else DEFAULT_ALSO.get(args.workload, [])
    return [a for a in args.also.split(",") if a]


def run_helix(args):
    rank, world, local = dist_init(args)
    import long_context_decode_helix_b200 as hx

    if args.kvp_ranks:
        return run_kvp(hx, args, rank, world, local)
    w = wl.WORKLOADS[args.workload]
    if args.context is not None:
        w = w.with_(S=args.context, S_min=None)
    dev = torch.device("cuda", local)
    K, W = args.steps, args.warmup
    head = measure(hx, w, args, K, W, world, local, dev, extras=True)

    per_workload = {}
    for name in also_list(args):
        wo = wl.WORKLOADS[name]
        # enough steps for a clock record of several samples: estimate the step from its bytes at
        # the headline's rate
        est_ms = head["ms_per_step"] * wl.step_bytes(wo, wl.seq_lens(wo)) / head["step_bytes"]
        Ko = max(K, int(np.ceil(args.min_timed_ms / max(est_ms, 1e-3))))
        rec = measure(hx, wo, args, Ko, W, world, local, dev, extras=False)
        per_workload[name] = rec

    read_probe = read_probe_gbs(dev) if rank == 0 and not args.no_read_probe else None
    if read_probe is not None:  # the roofline's context figure, taken after the timed regions
        for rec in [head, *per_workload.values()]:
            if rec["roofline"]["bound"] == "hbm":
                rec["roofline"]["frac_of_read_probe"] = (rec["roofline"]["achieved"] /
                                                         read_probe["gbs"])
            else:
                rec["roofline"]["other"]["frac_of_read_probe"] = (
                    rec["roofline"]["other"]["achieved"] / read_probe["gbs"])
    if rank == 0:
        line = {
            "metric": METRIC, "value": head["value"], "unit": "us/step", "n_gpus": world,
            "steps": K, "warmup": W, "ms_per_step": head["ms_per_step"],
            "higher_is_better": False, "scaling": "weak", "vs_baseline": None,
            "dtype": head["dtype"], "data": "synthetic", "config": head["config"],
            "parallelism": f"replicas x{world} (every rank its own batch)",
            "achieved_hbm_tbs": head["achieved_hbm_tbs"], "step_bytes": head["step_bytes"],
            "kernels_us": head["kernels_us"], "gpu_launches": head["gpu_launches"],
            "roofline": head["roofline"], "e2e": head["e2e"], "clocks": head["clocks"],
            "hopb": head.get("hopb"), "graph": head.get("graph"), "read_probe": read_probe,
        }
        if per_workload:
            line["per_workload"] = per_workload
        if not args.no_cpu_baseline and world == 1:
            line["cpu_baseline"] = cpu_baseline(w, args)
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()
    return 0


# ------------------------------------------------------------------------------------------------
# KV parallelism across ranks


def kvp_local_rows(w, t0, t1, rank, world, dev):
    """Append arguments for this rank's tokens among history positions [t0, t1) of every request
    (t0 a multiple of rr_block * world): [B, n_local, ...]."""
    from long_context_decode_helix_b200 import kvp

    rows = wl.append_rows(w, t0, t1, dev)
    idx = kvp.local_positions(t1, rank, world, w.rr_block)
    idx = (idx[idx >= t0] - t0).to(dev)
    return {k: v.index_select(1, idx).contiguous() for k, v in rows.items()}


def run_kvp(hx, args, rank, world, local):
    """Rank r holds KVP shard r of one batch in a kvp = 1 cache. A step: append the new token on its
    owner, partial attention over the local shard for every head, then the exchange of the partials
    and the combine of the heads this rank owns (``kvp.KVPExchange``)."""
    import torch.distributed as dist

    from long_context_decode_helix_b200 import kvp

    own_group = False
    if not dist.is_initialized():  # one rank: the exchange still runs through a process group
        import datetime
        import socket

        with socket.socket() as s_:
            s_.bind(("127.0.0.1", 0))
            port = s_.getsockname()[1]
        dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0,
                                world_size=1, timeout=datetime.timedelta(seconds=120))
        own_group = True
    w0 = wl.WORKLOADS[args.workload]
    if args.context is not None:
        w0 = w0.with_(S=args.context, S_min=None)
    if w0.kind != "gqa" or w0.kv_dtype != "bf16":
        raise SystemExit("--kvp-ranks runs the bf16 GQA workloads")
    dev = torch.device("cuda", local)
    K, W = args.steps, args.warmup
    lens = wl.seq_lens(w0)
    S_cap = max(lens) + K + W + 16
    # this rank's cache: kvp = 1, its own tokens only
    w = w0.with_(kvp=1)
    local_cap = -(-S_cap // (w0.rr_block * world)) * w0.rr_block + w0.rr_block
    pt, n_pages = wl.page_table(w, local_cap)
    cache = hx.KVCache(hx.ATTN_GQA, hx.KV_BF16, hx.LAYOUT_RR, 1, w.B, w.Hkv, w.d, w.dv,
                       pt.shape[2], page_table=pt, num_pages=n_pages, device=dev)
    hist = [L - 1 for L in lens]
    chunk = 65536  # a multiple of rr_block * world (world <= 16)
    for t0 in range(0, max(hist), chunk):
        t1 = min(t0 + chunk, max(hist))
        rows = kvp_local_rows(w0, t0, t1, rank, world, dev)
        # request b appends its local tokens among positions [t0, min(t1, hist_b))
        nv = torch.tensor([kvp.owned_count(min(max(L, t0), t1), rank, world, w0.rr_block) -
                           kvp.owned_count(t0, rank, world, w0.rr_block) for L in hist],
                          dtype=torch.int32, device=dev)
        hx.append(cache, **rows, n_valid=nv)
    wait(hx, args)
    assert cache.err_bits() == 0, "prefill reported a device error"
    new_rows = wl.append_rows(w0, 0, K + W, dev)
    step_rows = {k: v.transpose(0, 1).unsqueeze(2).contiguous() for k, v in new_rows.items()}
    q = wl.query(w0, dev)
    ws = cache.workspace(w.Hq)
    mode = args.kvp_exchange if world > 1 else "gather"
    ex = kvp.KVPExchange(w.B, w.Hq, w.dv, dev, mode=mode)
    dec = kvp.KVPDecodeRank(
        ex, lambda r, nv: hx.append(cache, **r, n_valid=nv),
        lambda q_, o, l: hx.partial(cache, q_, w.softmax_scale, o, l, workspace=ws), hist,
        w0.rr_block)
    stream = torch.cuda.current_stream()
    si = 0
    for _ in range(W):
        dec.step({k: v[si] for k, v in step_rows.items()}, q)
        si += 1
    wait(hx, args)
    barrier(world)
    exch = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            for _ in range(K)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t_wall = time.perf_counter()
    start.record(stream)
    for i in range(K):
        dec.append({k: v[si] for k, v in step_rows.items()})
        si += 1
        hx.partial(cache, q, w.softmax_scale, ex.o_partial, ex.lse, workspace=ws)
        exch[i][0].record(stream)
        ex.combine()
        exch[i][1].record(stream)
    stop.record(stream)
    wait(hx, args)
    t_wall = time.perf_counter() - t_wall
    barrier(world)
    assert cache.err_bits() == 0, "a timed step reported a device error"
    ms_step = max_over_ranks(start.elapsed_time(stop) / K, world)
    ex_ms = max_over_ranks(float(np.mean([a.elapsed_time(b) for a, b in exch])), world)
    h0, h1 = kvp.owned_heads(rank, world, w.Hq)
    if rank == 0:
        line = {
            "metric": METRIC, "value": ms_step * 1e3, "unit": "us/step", "n_gpus": world,
            "steps": K, "warmup": W, "ms_per_step": ms_step, "higher_is_better": False,
            "scaling": "strong", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": config_of(w0, lens),
            "parallelism": f"KVP x{world}: rank r holds shard r of one batch",
            "gpu_launches": 3 * K,  # append, partial, combine over the ranks' partials
            "kvp": {"ranks": world, "exchange": mode,
                    "exchange_us": ex_ms * 1e3, "exchange_share": ex_ms / ms_step,
                    "owner_read_bytes": world * w.B * (h1 - h0) * (w.dv + 1) * 4,
                    "host_wall_us_per_step": t_wall / K * 1e6,
                    "how": "events around the exchange + combine (two barriers, the owner's "
                           "combine over every rank's partial); the step includes the append "
                           "and the partial over the local shard"},
        }
        print(json.dumps(line), flush=True)
    ex.close()
    if world > 1 or own_group:
        dist.destroy_process_group()
    return 0


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    return run_helix(args)


if __name__ == "__main__":
    sys.exit(main())
