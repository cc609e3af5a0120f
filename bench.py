#!/usr/bin/env python
"""Benchmark: one decode-attention layer step of KV-parallel (sequence-sharded) attention.

A step = append one new token per request (helix_kv_append) + per-shard partial attention over the
whole history (helix_attn_partial) + the LSE-rescaling combine (helix_attn_combine), on synthetic
seeded inputs already resident in HBM. Default workload: B=8 requests, 128 query heads, 8 KV heads,
d=128, 1,048,576-token bf16 history per request, 8 KV-parallel shards with round-robin-16 placement.

Prints ONE JSON line (rank 0). ``--impl reference`` times the fp64 CPU oracle instead, on a bounded
sample of the same workload, scaled to the same unit.

Multi-GPU (torchrun, N ranks): every rank runs its own independent batch (replicas, weak scaling);
the step time is the max over ranks.
"""

from __future__ import annotations

import argparse
import json
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

import workloads as wl  # noqa: E402

METRIC = "us per decode-attention layer step & achieved HBM TB/s (B=8, 1M ctx, 1 GPU)"
FALLBACK_HBM_GBS = 6650.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=40)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="helix", choices=["helix", "reference"])
    ap.add_argument("--workload", default="gqa_s1m", choices=sorted(wl.WORKLOADS))
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--graph", action="store_true",
                    help="also time the steps launched from CUDA graphs (reported under 'graph')")
    ap.add_argument("--hopb-groups", type=int, default=4,
                    help="request groups of the two-stream HOP-B analogue, timed after the main "
                         "steps and reported under 'hopb' (0 = skip)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-read-probe", action="store_true",
                    help="skip the pure-read bandwidth probe reported beside the roofline")
    ap.add_argument("--cpu-sample-tokens", type=int, default=1 << 19,
                    help="history tokens per sampled head group for the CPU oracle")
    ap.add_argument("--cpu-sample-groups", type=int, default=4)
    ap.add_argument("--context", type=int, default=None,
                    help="override the history length (fixed lengths), e.g. for small profiling runs")
    return ap.parse_args()


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


class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.proc = None
        self.gpu = gpu_index
        # the raw samples go to a scratch file (HELIX_CLOCKS_DIR, else the system temp directory)
        out_dir = os.environ.get("HELIX_CLOCKS_DIR") or tempfile.gettempdir()
        self.path = os.path.join(out_dir, f"helix_clocks_rank{gpu_index}.csv")

    def start(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", str(self.gpu)], stdout=self.fh, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
            return
        # nvidia-smi takes a while to print its first line: wait for it (bounded), so that even a
        # short timed region falls inside the sampled window
        t_end = time.time() + 5.0
        while time.time() < t_end and self.proc.poll() is None:
            self.fh.flush()
            if os.path.getsize(self.path) > 0:
                break
            time.sleep(0.02)

    def stop(self):
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
                "samples": len(sm)}


FALLBACK_BF16_TFLOPS_SUSTAINED = 1400.0
SPEC_HBM_GBS = 8000.0  # B200 HBM3e data-sheet bandwidth, for context beside the measured peaks


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
# CPU oracle on a bounded sample


def cpu_oracle_sample(w: wl.Workload, tokens: int, groups: int):
    """Time the fp64 oracle (per-shard partials + combine) on `groups` head groups of `tokens`
    history tokens each; return (us per full step, description, cores)."""
    import oracle

    cores = len(os.sched_getaffinity(0))
    lens = wl.seq_lens(w)
    q = wl.query(w)
    total_pairs = sum(lens) * w.Hkv
    rng = np.random.default_rng(w.seed)
    picks = [(int(rng.integers(w.B)), int(rng.integers(w.Hkv))) for _ in range(groups)]
    T = min(tokens, min(lens))
    elapsed = 0.0
    for b, h in picks:
        if w.kind == "mla":
            K = oracle.attention._f64(wl.kv_range_bf16(w, "c", b, 0, 0, T))
            V = K[:, : w.dv]
        elif w.kv_dtype == "nvfp4":
            K = oracle.nvfp4_dequant(*wl.kv_range_nvfp4(w, "k", b, h, 0, T))
            V = oracle.nvfp4_dequant(*wl.kv_range_nvfp4(w, "v", b, h, 0, T))
        else:
            K = oracle.attention._f64(wl.kv_range_bf16(w, "k", b, h, 0, T))
            V = oracle.attention._f64(wl.kv_range_bf16(w, "v", b, h, 0, T))
        qg = q[b, h * w.G:(h + 1) * w.G]
        t0 = time.perf_counter()
        sets = oracle.shard_tokens(T, w.kvp, w.layout, w.rr_block, w.contig_chunk)
        parts = [oracle.attend(qg, K[idx], V[idx], w.softmax_scale) for idx in sets]
        oracle.combine(np.stack([p[0] for p in parts]), np.stack([p[1] for p in parts]))
        elapsed += time.perf_counter() - t0
    sample_pairs = groups * T
    us_per_step = elapsed / sample_pairs * total_pairs * 1e6
    desc = (f"{groups} (request, KV head) groups x {T} history tokens each "
            f"({sample_pairs} token-head pairs of {total_pairs} per step), per-shard fp64 "
            f"partials + combine; input generation not timed; scaled linearly to a full step")
    return us_per_step, desc, cores, elapsed


# ------------------------------------------------------------------------------------------------


def run_reference(args):
    rank, world, _ = int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")), 0
    if rank != 0:
        return 0
    w = wl.WORKLOADS[args.workload]
    lens = wl.seq_lens(w)
    tokens = max(4096, min(args.cpu_sample_tokens, 1 << 17))
    for _ in range(args.warmup):
        cpu_oracle_sample(w, 4096, 1)
    vals, descs, cores, spent = [], None, None, 0.0
    for _ in range(args.steps):
        v, descs, cores, el = cpu_oracle_sample(w, tokens, 1)
        vals.append(v)
        spent += el
    value = float(np.mean(vals))
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "us/step",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": value / 1e3, "higher_is_better": False, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(w, lens),
        "cpu_baseline": {"value": value, "unit": "us/step", "cores": cores, "kind": "oracle",
                         "sample": descs},
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


def run_helix(args):
    rank, world, local = dist_init(args)
    import long_context_decode_helix_b200 as hx

    w = wl.WORKLOADS[args.workload]
    if args.context is not None:
        w = w.with_(S=args.context, S_min=None)
    lens = wl.seq_lens(w)
    dev = torch.device("cuda", local)
    K, W = args.steps, args.warmup
    n_steps = (K + W + (K if not args.no_e2e else 0) + (W + K if args.graph else 0) +
               (W + K if args.hopb_groups > 0 else 0))
    S_cap = max(lens) + n_steps + 16
    if w.layout == "contig":  # size the contiguous shards for the history plus the new tokens
        w = w.with_(S_final=S_cap)

    # --- state resident in HBM: the history (S_b - 1 tokens), then one new token per step ---
    pt, n_pages = wl.page_table(w, S_cap)
    cache = hx.KVCache(hx.ATTN_MLA if w.kind == "mla" else hx.ATTN_GQA,
                       hx.KV_NVFP4 if w.kv_dtype == "nvfp4" else hx.KV_BF16,
                       hx.LAYOUT_RR if w.layout == "rr" else hx.LAYOUT_CONTIG,
                       w.kvp, w.B, w.Hkv, w.d, w.dv, pt.shape[2], page_tokens=w.page_tokens,
                       rr_block=w.rr_block, contig_chunk=w.contig_chunk, page_table=pt,
                       num_pages=n_pages, device=dev)
    hist = [L - 1 for L in lens]
    chunk = 65536
    for t0 in range(0, max(hist), chunk):
        n = min(chunk, max(hist) - t0)
        nv = torch.tensor([min(max(L - t0, 0), n) for L in hist], dtype=torch.int32, device=dev)
        hx.append(cache, **wl.append_rows(w, t0, t0 + n, dev), n_valid=nv)
    torch.cuda.synchronize()
    assert cache.err_bits() == 0, "prefill reported a device error"
    # the new token of every step, resident as [step][B][1][...] so each step's slice is dense
    # An NVFP4 cache takes the new token as bf16 rows and encodes it on the device
    # (helix_kv_append_quantize), as a decode loop over an FP4 cache does.
    quant = w.kv_dtype == "nvfp4"
    if quant:
        new_rows = {"k_new": torch.stack([wl.kv_tokens(w, "k", b, 0, n_steps, dev)
                                          for b in range(w.B)]),
                    "v_new": torch.stack([wl.kv_tokens(w, "v", b, 0, n_steps, dev)
                                          for b in range(w.B)])}
    else:
        new_rows = wl.append_rows(w, 0, n_steps, dev)
    step_rows = {k: v.transpose(0, 1).unsqueeze(2).contiguous() for k, v in new_rows.items()}

    def append_step(a):
        if quant:
            hx.append_quantize(cache, a["k_new"], a["v_new"])
        else:
            hx.append(cache, a["k_new"], a.get("v_new"), a.get("k_scale"), a.get("v_scale"))
    q = wl.query(w, dev)
    o_part = torch.empty(w.kvp, w.B, w.Hq, w.dv, dtype=torch.float32, device=dev)
    lse_part = torch.empty(w.kvp, w.B, w.Hq, dtype=torch.float32, device=dev)
    out = torch.empty(w.B, w.Hq, w.dv, dtype=torch.bfloat16, device=dev)
    lse_out = torch.empty(w.B, w.Hq, dtype=torch.float32, device=dev)
    ws = cache.workspace(w.Hq)
    stream = torch.cuda.current_stream()

    def one_step(i, ev=None):
        append_step({k: v[i] for k, v in step_rows.items()})
        if ev is not None:
            ev[0].record(stream)
        # partial attention and the combine: one launch for GQA (helix_attn_partial_combine)
        hx.partial_combine(cache, q, w.softmax_scale, o_part, lse_part, out, lse_out, workspace=ws)
        if ev is not None:
            ev[1].record(stream)

    si = 0
    for _ in range(W):
        one_step(si)
        si += 1
    torch.cuda.synchronize()

    clocks = ClockSampler(local)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(K)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    lens_at = [[L + si + i for L in lens] for i in range(K)]  # history length during timed step i
    barrier(world)
    torch.cuda.synchronize()
    clocks.start()
    torch.cuda.nvtx.range_push("timed_steps")
    start.record(stream)
    for i in range(K):
        one_step(si + i, evs[i])
    stop.record(stream)
    torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    si += K
    total_ms = start.elapsed_time(stop)
    ms_step = max_over_ranks(total_ms / K, world)
    partial_ms = [a.elapsed_time(b) for a, b in evs]
    assert cache.err_bits() == 0, "a timed step reported a device error"

    # --- end to end through host buffers: q and the new token in, O out, every step ---
    e2e = None
    if not args.no_e2e:
        q_h = q.cpu().pin_memory()
        rows_h = {k: v.cpu().pin_memory() for k, v in step_rows.items()}
        out_h = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        q_d = torch.empty_like(q)
        tok_d = {k: torch.empty_like(v[0]) for k, v in step_rows.items()}
        h2d = q.numel() * q.element_size() + sum(
            v[0].numel() * v.element_size() for v in step_rows.values())
        d2h = out.numel() * out.element_size()
        barrier(world)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(K):
            q_d.copy_(q_h, non_blocking=True)
            for k_ in tok_d:
                tok_d[k_].copy_(rows_h[k_][si + i], non_blocking=True)
            append_step(tok_d)
            hx.partial_combine(cache, q_d, w.softmax_scale, o_part, lse_part, out, lse_out,
                               workspace=ws)
            out_h.copy_(out, non_blocking=True)
        e1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        si += K
        e2e_ms = max_over_ranks(e0.elapsed_time(e1) / K, world)
        e2e = {"value": e2e_ms * 1e3, "unit": "us/step", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h}

    # --- optional: the same steps launched from CUDA graphs (one graph per step, captured outside
    # the timed region), the form a caller uses when the step is launch-bound (short contexts) ---
    graph = None
    if args.graph:
        graphs = []
        cap_stream = torch.cuda.Stream(dev)
        for i in range(K):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=cap_stream):
                one_step(si + i)
            graphs.append(g)
        torch.cuda.synchronize()
        for g in graphs[:min(W, K)]:  # warm-up replays
            g.replay()
        barrier(world)
        torch.cuda.synchronize()
        g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        g0.record()
        for g in graphs:
            g.replay()
        g1.record()
        torch.cuda.synchronize()
        barrier(world)
        graph_ms = max_over_ranks(g0.elapsed_time(g1) / K, world)
        si += K
        graph = {"us_per_step": graph_ms * 1e3, "steps": K,
                 "how": "each step captured once in a CUDA graph, then replayed back to back"}
        del graphs
        assert cache.err_bits() == 0, "a graph-launched step reported a device error"

    # --- HOP-B analogue: the combine of request group g on a second stream overlaps the partial of
    # group g+1; same append, same inputs, timed like the main steps ---
    hopb = None
    if args.hopb_groups > 0:
        ov = hx.Overlap(args.hopb_groups, dev)

        def hopb_step(i):
            a = {k: v[i] for k, v in step_rows.items()}
            if quant:  # the device-encoding append is not part of the overlapped call
                append_step(a)
                hx.overlapped(cache, q, w.softmax_scale, ov, o_part, lse_part, out, lse_out,
                              workspace=ws)
            else:  # append, partial and combine of request groups over two streams
                hx.decode_overlapped(cache, q, w.softmax_scale, ov, a["k_new"], a.get("v_new"),
                                     o_partial=o_part, lse=lse_part, out=out, lse_out=lse_out,
                                     workspace=ws)

        for _ in range(W):
            hopb_step(si)
            si += 1
        barrier(world)
        torch.cuda.synchronize()
        h0, h1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        h0.record(stream)
        for i in range(K):
            hopb_step(si + i)
        h1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        si += K
        hopb_ms = max_over_ranks(h0.elapsed_time(h1) / K, world)
        n_groups = min(args.hopb_groups, w.B)
        per = -(-w.B // n_groups)
        hopb = {"groups": -(-w.B // per), "us_per_step": hopb_ms * 1e3,
                "serial_us_per_step": ms_step * 1e3, "speedup": ms_step / hopb_ms,
                "gpu_launches": K * 3 * (-(-w.B // per))}
        assert cache.err_bits() == 0, "a HOP-B step reported a device error"

    read_probe = read_probe_gbs(dev) if rank == 0 and not args.no_read_probe else None
    if rank == 0:
        step_bytes = float(np.mean([wl.step_bytes(w, L) for L in lens_at]))
        # the timed kernel: the fused partial + combine (GQA); for MLA the two launches
        part_bytes = float(np.mean([wl.partial_bytes(w, L) for L in lens_at])) + wl.combine_bytes(w)
        part_ms = float(np.mean(partial_ms))
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
        # the binding roof is the one with the longer ideal time
        tensor_bound = flops / (tflops_peak * 1e12) > part_bytes / (peak * 1e9)
        # context for the HBM roofline: the data-sheet figure and a pure-read probe of this run
        hbm["frac_of_spec"] = achieved_gbs / SPEC_HBM_GBS
        if read_probe is not None:
            hbm["frac_of_read_probe"] = achieved_gbs / read_probe["gbs"]
        roof = dict(tensor if tensor_bound else hbm, bound="tensor" if tensor_bound else "hbm",
                    peak_source=peak_kind, kernel=kname, bytes_per_launch=part_bytes,
                    flops_per_launch=flops, other=(hbm if tensor_bound else tensor),
                    traffic=profile_traffic("partial", w.name))
        line = {
            "metric": METRIC, "value": ms_step * 1e3, "unit": "us/step", "n_gpus": world,
            "steps": K, "warmup": W, "ms_per_step": ms_step, "higher_is_better": False,
            "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if w.kv_dtype == "bf16" else "nvfp4", "data": "synthetic",
            "config": dict(config_of(w, lens), parallelism=f"replicas x{world}"),
            "achieved_hbm_tbs": step_bytes / (ms_step * 1e-3) / 1e12 * world,
            "step_bytes": step_bytes,
            "kernels_us": {"partial_and_combine": part_ms * 1e3,
                           "append_and_gaps": ms_step * 1e3 - part_ms * 1e3},
            "gpu_launches": (3 if w.kind == "mla" else 2) * K,
            "roofline": roof,
            "e2e": e2e,
            "clocks": clk,
            "hopb": hopb,
            "graph": graph,
            "read_probe": read_probe,
        }
        if not args.no_cpu_baseline and world == 1:
            v, desc, cores, _ = cpu_oracle_sample(w, args.cpu_sample_tokens, args.cpu_sample_groups)
            line["cpu_baseline"] = {"value": v, "unit": "us/step", "cores": cores,
                                    "kind": "oracle", "sample": desc}
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()
    return 0


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    return run_helix(args)


if __name__ == "__main__":
    sys.exit(main())
