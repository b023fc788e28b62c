#!/usr/bin/env python
"""Benchmark of the Julia-1 decision-model forward pass on B200.

One step = one full forward pass (serialised rows -> logits, probabilities,
choice / score / noul) over one batch of the throughput workload: 1024 packed
rows of 64..1024 tokens (2..20 options, head budget 512, strict), synthetic
ids and random-init weights.  Multi-GPU: one process per GPU, each rank runs
its own 1024 rows (rows are independent decisions; no collective on the data
path), value = all ranks' decisions / max over ranks of the device time.

Prints one JSON line on rank 0.  --impl reference times the CPU oracle on a
bounded sample of the same workload instead.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decisions/s batched and p50 ms/call, Julia-1 forward on 1 B200 (BF16)"
UNIT = "decisions/s"
D, FF, HFF, NH = 384, 1152, 1536, 6


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--rows", type=int, default=None,
                    help="rows per rank and step (default 1024 for throughput, 16 for long)")
    ap.add_argument("--workload", default="throughput", choices=["throughput", "long"],
                    help="throughput: 1024 rows of 64..1024 tokens; long: 16 rows of 8192 tokens")
    ap.add_argument("--latency-calls", type=int, default=1000)
    ap.add_argument("--router-reps", type=int, default=5, help="timed jd_route_host calls (0: skip)")
    ap.add_argument("--serve-seconds", type=float, default=2.0,
                    help="seconds per thread count of the concurrent-serving measurement (0: skip)")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile-steps", type=int, default=3)
    ap.add_argument("--fp8-steps", type=int, default=3, help="profiled steps of the FP8-mode leg (0: skip)")
    ap.add_argument("--long-rows", type=int, default=16,
                    help="rows of the long-context leg (8192 tokens each; 0: skip)")
    ap.add_argument("--json-out", default=None)
    return ap.parse_args()


# ----------------------------------------------------------------------------- workload


def workload(args, rank):
    from workloads import rows_config2, rows_config3
    if args.workload == "long":
        n = args.rows or 16
        rows = rows_config3(n, seed=103 + 1000 * rank)
        opts = dict(max_length=8192, head_budget=256, strict=False)
        desc = (f"long context: {n} rows x 8192 tokens, 20 options (capped to the 256-token head budget, "
                "non-strict), choice/score")
    else:
        rows = rows_config2(args.rows or 1024, seed=102 + 1000 * rank)
        opts = dict(max_length=1024, head_budget=512, strict=True)
        desc = (f"batched throughput: {args.rows or 1024} packed rows, lengths U[64,1024], 2..20 options of 1..48 ids, "
                "types uniform, head budget 512, strict")
    return rows, opts, desc


def algorithmic_cost(name, lens, n_markers, kper=None, n_unique_ids=None):
    """(bytes, flops) per launch of kernel `name` for rows of lengths `lens`
    (`kper`: options per row, needed for the marker attention; `n_unique_ids`:
    distinct token ids of the batch, whose FP32 embedding rows are the gather's
    compulsory reads -- a repeated id is an L2 hit, not a second HBM read)."""
    lens = np.asarray(lens, dtype=np.float64)
    T = lens.sum()
    M = float(n_markers)
    if name == "embed_ln":
        U = T if n_unique_ids is None else float(n_unique_ids)
        return T * 4 + U * 1536 + T * (1536 + 768), T * 3 * D
    if name in ("gemm_qkv_rope", "head0_gemm_in"):
        return T * (768 + 2304), T * 2 * D * 3 * D
    if name in ("gemm_wo_res_ln", "head0_gemm_out"):
        return T * (768 + 1536 + 1536 + 768), T * 2 * D * D
    if name == "gemm_wi_geglu":
        return T * (768 + 2304), T * 2 * D * 2 * FF
    if name == "gemm_wo2_res_ln":
        return T * (2304 + 1536 + 1536 + 768), T * 2 * FF * D
    if name == "head0_gemm_ffn1":
        return T * (768 + 3072), T * 2 * D * HFF
    if name == "head0_gemm_ffn2":
        return T * (3072 + 1536 + 1536 + 768), T * 2 * HFF * D
    if name in ("attn_global", "head0_attn"):
        return T * (3 * 768 + 768), 4.0 * 64 * NH * float((lens ** 2).sum())
    if name == "attn_local":
        vis = 0.0
        for L in lens.astype(np.int64):
            i = np.arange(L)
            vis += float((np.minimum(L - 1, i + 64) - np.maximum(0, i - 64) + 1).sum())
        return T * (3 * 768 + 768), 4.0 * 64 * NH * vis
    if name == "head1_gemm_kv":
        return T * (768 + 1536), T * 2 * D * 2 * D
    if name == "head1_gather":  # mask_pos, FP32 state row and BF16 normed row in, both out
        return M * (4 + 2 * (1536 + 768)), 0.0
    if name == "head1_marker_attn" and kper is not None:  # K,V of every row once; q in, o out
        return T * 1536 + M * (768 + 768), 4.0 * 64 * NH * float((np.asarray(kper, np.float64) * lens).sum())
    if name == "head":  # FP32 marker states and the scorer weights in; logits, probs and read-outs out
        nb = len(lens)
        return (M * (1536 + 4 + 4) + 4 * (D * D + 4 * D + 1) + 4 * (nb + 1) + nb * (4 + 16),
                M * (2 * D * D + 2 * D + 8 * D))
    return None


def read_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm=float(d["hbm_gbs"]), tc_burst=float(d["bf16_tflops"]),
                    tc_sust=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), src="measured")
    return dict(hbm=6650.0, tc_burst=1590.0, tc_sust=1400.0, src="fallback")


# The source file that defines each timed kernel (and its launcher); every kernel also
# depends on the shared device headers.
KERNEL_FILES = {"gemm": ("gemm.cu", "epilogue.cuh"), "attn_global": ("attention_tc.cu",),
                "head0_attn": ("attention_tc.cu",), "attn_local": ("attention.cu",),
                "head1_marker_attn": ("attention.cu",), "head": ("head.cu",)}
SHARED_FILES = ("common.cuh", "kernels.h")


def kernel_source_sha(kernel=None):
    """SHA-256 (first 16 hex digits) of the sources that decide what the GPU runs.
    kernel=None: every kernel and launcher (*.cu, *.cuh) and their shared
    declarations (kernels.h); the host-only serializer, router and API files
    launch nothing and are not part of it.  kernel=name: only the file that
    defines that kernel (gemm.cu for every GEMM, small.cu for the bandwidth
    kernels) and the shared device headers."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "encoder_decision_model_b200", "csrc")
    if kernel is None:
        files = [f for f in sorted(os.listdir(csrc)) if f.endswith((".cu", ".cuh")) or f == "kernels.h"]
    else:
        own = KERNEL_FILES.get("gemm" if "gemm" in kernel else kernel, ("small.cu",))
        files = sorted(set(own) | set(SHARED_FILES))
    for f in files:
        h.update(open(os.path.join(csrc, f), "rb").read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel, workload_tag):
    """DRAM bytes per token from a committed ncu summary, if its source hash
    matches the kernel's current sources (else None)."""
    pdir = os.path.join(ROOT, "profiles")
    if not os.path.isdir(pdir):
        return None
    sha = kernel_source_sha(kernel)
    for f in sorted(os.listdir(pdir)):
        if not f.endswith(".md"):
            continue
        txt = open(os.path.join(pdir, f)).read()
        for m in re.finditer(r"traffic\s+kernel=(\S+)\s+workload=(\S+)\s+dram_bytes_per_token=([0-9.eE+-]+)"
                             r"\s+source_sha=(\S+)", txt):
            if m.group(1) == kernel and m.group(2) == workload_tag and m.group(4) == sha:
                return float(m.group(3))
    return None


# ----------------------------------------------------------------------------- ranks


class Ranks:
    """The timing protocol's process-group steps: barrier, max and sum over
    ranks (NCCL on the GPU machine, gloo in the CPU tests; single process: no-ops)."""

    def __init__(self, world, device):
        self.world = world
        self.device = device

    def barrier(self):
        if self.world > 1:
            import torch.distributed as dist
            dist.barrier()

    def _reduce(self, x, op):
        if self.world == 1:
            return float(x)
        import torch
        import torch.distributed as dist
        t = torch.tensor([float(x)], dtype=torch.float64, device=self.device)
        dist.all_reduce(t, op=op)
        return float(t.item())

    def max(self, x):
        import torch.distributed as dist
        return self._reduce(x, dist.ReduceOp.MAX)

    def sum(self, x):
        import torch.distributed as dist
        return self._reduce(x, dist.ReduceOp.SUM)


def whole_job_rate(units_this_rank, seconds_this_rank, ranks):
    """Units processed by all ranks / the slowest rank's time."""
    return ranks.sum(units_this_rank) / ranks.max(seconds_this_rank)


# ----------------------------------------------------------------------------- clocks


class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.p = None

    def start(self):
        try:
            self.p = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                                       "--format=csv,noheader,nounits", "-lms", "100"], stdout=self.f,
                                      stderr=subprocess.DEVNULL)
        except OSError:
            self.p = None

    def stop(self):
        if self.p is None:
            return None
        self.p.terminate()
        try:
            self.p.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.p.kill()
        self.f.flush()
        rows = [l.split(",") for l in open(self.f.name).read().strip().splitlines() if l.strip()]
        os.unlink(self.f.name)
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            r = [x.strip() for x in r]
            try:
                sm.append(float(r[1]))
                mx = float(r[2])
            except (ValueError, IndexError):
                continue
            for n, v in zip(names, r[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return dict(sm_mhz=statistics.median(sm), sm_max_mhz=mx, reasons=sorted(reasons), samples=len(sm))


# ----------------------------------------------------------------------------- CPU oracle


def oracle_sample(rows, opts, seconds, min_rows=2):
    """Time the oracle as it stands on the first rows until `seconds` elapse."""
    from oracle import EncodeOptions, OracleModel, serialize_row, readouts
    from workloads import weights_path
    m = OracleModel(weights_path(0))
    eo = EncodeOptions(max_length=opts["max_length"], head_budget=opts["head_budget"], strict=opts["strict"])
    t0 = time.perf_counter()
    n = toks = 0
    for r in rows:
        e = serialize_row(r, eo)
        readouts(m.logits(e), e.qtype)
        n += 1
        toks += len(e.ids)
        if time.perf_counter() - t0 >= seconds and n >= min_rows:
            break
    return n, toks, time.perf_counter() - t0


def blas_threads():
    """Threads of the BLAS that runs NumPy's matmuls (the oracle's); other BLAS
    copies loaded by other packages do not run the oracle."""
    try:
        from threadpoolctl import threadpool_info
        info = [i for i in threadpool_info() if i.get("user_api") == "blas"]
        own = [i for i in info if "numpy" in (i.get("filepath") or "")] or info
        if own:
            return int(max(i.get("num_threads", 0) for i in own))
    except Exception:
        pass
    return os.cpu_count()


def oracle_four_threads(rows, opts, seconds):
    """The same oracle sample with BLAS held to 4 threads (the CPU runtimes on the
    pages quote 4-thread figures); None when threadpoolctl is missing."""
    try:
        from threadpoolctl import threadpool_limits
    except ImportError:
        return None
    with threadpool_limits(limits=4, user_api="blas"):
        n, toks, el = oracle_sample(rows, opts, seconds)
        cores = blas_threads()
    return {"value": n / el, "unit": UNIT, "cores": cores,
            "sample": f"first {n} rows ({toks} tokens), {el:.1f} s"}


# ----------------------------------------------------------------------------- reference arm


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    rows, opts, desc = workload(args, 0)
    per_step = 2 if args.workload == "throughput" else 1
    cores = blas_threads()
    for w in range(args.warmup):
        oracle_sample(rows[w * per_step:(w + 1) * per_step], opts, 0.0, per_step)
    n = toks = 0
    el = 0.0
    base = args.warmup * per_step
    for s in range(args.steps):
        sl = rows[(base + s * per_step) % len(rows):][:per_step]
        a, b, t = oracle_sample(sl, opts, 0.0, per_step)
        n += a
        toks += b
        el += t
    v = n / el
    sample = f"{n} rows ({toks} tokens) of the workload, {per_step} per step, float64 NumPy oracle"
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000 * el / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": desc, "rows_per_step": per_step},
            "cpu_baseline": {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- our arm


ROUTER_KERNELS = ("embed_ln", "attn_local", "attn_global", "head0_attn", "head1_gather", "head1_marker_attn",
                  "head")
ENCODER_GEMMS = ("gemm_qkv_rope", "gemm_wo_res_ln", "gemm_wi_geglu", "gemm_wo2_res_ln")


def _r(x, n=4):
    return None if x is None else float(f"{x:.{n}g}")


def kernel_fractions(prof, steps, lens, n_markers, kper, n_unique_ids, peaks):
    """Per kernel: launches and ms per step, and the fraction of the measured
    HBM copy bandwidth and of the sustained BF16 tensor rate its algorithmic
    bytes and FLOPs reach per launch (CUDA events on the launching stream)."""
    out = {}
    for name, (n, tot) in prof.items():
        d = dict(launches_per_step=n // max(1, steps), ms_per_step=_r(tot / max(1, steps)))
        c = algorithmic_cost(name, lens, n_markers, kper, n_unique_ids)
        if c is not None and n:
            a = tot / n / 1000.0
            d["hbm_frac"] = _r(c[0] / a / 1e9 / peaks["hbm"], 3)
            d["tensor_frac"] = _r(c[1] / a / 1e12 / peaks["tc_sust"], 3)
        out[name] = d
    return out


def upload_batch(jl, hb, dev):
    import torch
    up = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)
    keep = [up(hb.tokens), up(hb.cu_seqlens), up(hb.mask_pos), up(hb.opt_off), up(hb.row_type)]
    batch = jl.Model.device_batch(hb.n_rows, hb.n_tokens, hb.n_markers, hb.max_row_len, *keep)
    B, M = hb.n_rows, hb.n_markers
    outs = dict(logits=torch.empty(M, device=dev), probs=torch.empty(M, device=dev),
                choice=torch.empty(B, dtype=torch.int32, device=dev), score=torch.empty(B, device=dev),
                noul=torch.empty(B, device=dev), max_p=torch.empty(B, device=dev))
    return batch, outs, keep


def profile_batch(jl, wpath, local, hb, steps, peaks, warmup=2, precision=None):
    """Run one packed batch with per-kernel events; per-kernel fractions."""
    import torch
    dev = torch.device("cuda", local)
    prec = jl.JD_PREC_BF16 if precision is None else precision
    m = jl.Model(wpath, hb.n_tokens, hb.n_rows, hb.n_markers, precision=prec, device=local)
    batch, outs, keep = upload_batch(jl, hb, dev)
    st = torch.cuda.Stream(device=dev)
    for _ in range(warmup):
        m.jd_decide(batch, **outs, stream=st)
    torch.cuda.synchronize()
    m.jd_check_status()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(st)
    for _ in range(steps):
        m.jd_decide(batch, **outs, stream=st)
    e1.record(st)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    m.jd_set_profiling(True)
    for _ in range(steps):
        m.jd_decide(batch, **outs, stream=st)
    prof = m.jd_profile_report()
    m.jd_set_profiling(False)
    torch.cuda.synchronize()
    m.jd_check_status()
    m.close()
    lens = np.diff(hb.cu_seqlens)
    pk = kernel_fractions(prof, steps, lens, hb.n_markers, np.diff(hb.opt_off), len(np.unique(hb.tokens)), peaks)
    return ms, pk


def measure_long(jl, wpath, local, rows, steps, peaks):
    """A bounded leg of the long-context workload (rows of exactly 8192 tokens,
    20 options capped to the 256-token head budget, non-strict): decisions/s and
    the per-kernel fractions, the encoder GEMMs' share of the tensor peak first."""
    from workloads import rows_config3
    r = rows_config3(rows, seed=103)
    hb = jl.jd_serialize(r, jl.encode_opts(8192, 256, False))
    ms, pk = profile_batch(jl, wpath, local, hb, steps, peaks)
    return {"workload": f"long context: {rows} rows x 8192 tokens (20 options capped to the 256-token head "
                        "budget, non-strict), choice/score", "rows": int(hb.n_rows), "tokens": int(hb.n_tokens),
            "decisions_per_s": _r(hb.n_rows / (ms / 1000.0)), "ms_per_batch": _r(ms),
            "encoder_gemm_tensor_frac": {k: pk[k].get("tensor_frac") for k in ENCODER_GEMMS if k in pk},
            "encoder_gemm_hbm_frac": {k: pk[k].get("hbm_frac") for k in ENCODER_GEMMS if k in pk},
            "per_kernel": pk}


def measure_fp8(jl, wpath, local, hb, steps, peaks):
    """The same batch with the encoder QKV projections on E4M3 operands (JD_PREC_FP8):
    decisions/s and the QKV kernel against the FP8 dense peak, taken as twice the measured
    BF16 one (the tensor cores' nominal FP8 / BF16 ratio)."""
    ms, pk = profile_batch(jl, wpath, local, hb, steps, peaks, precision=jl.JD_PREC_FP8)
    q = dict(pk.get("gemm_qkv_rope", {}))
    if "tensor_frac" in q:
        q["tensor_frac_of_fp8_peak"] = _r(q["tensor_frac"] / 2.0, 3)
    return {"precision": "E4M3 encoder QKV projections, everything else as the BF16 line",
            "decisions_per_s": _r(hb.n_rows / (ms / 1000.0)), "ms_per_step": _r(ms), "gemm_qkv_rope": q,
            "fp8_peak_tflops": _r(2.0 * peaks["tc_sust"]), "per_kernel": pk}


def measure_latency(jl, wpath, local, calls, n_distinct=128):
    """Batch-1 latency of the 3-question request (choice/4, score/3, noul/2 on one
    200-token state) through jd_decide_host, host serialisation and copies included.
    `distinct`: a pool of `n_distinct` seeded requests of that recipe (questions
    8..24 ids, options 3..20 ids, so each has its own length), called in turn;
    eager launches and CUDA-graph mode side by side.  Graph mode keeps one graph
    per bucket of padded shapes; one untimed pass over the pool captures them, so
    the timed calls only replay (their capture count is reported).  `repeated`: one
    request called over and over in graph mode."""
    from workloads import rows_config1
    o1 = jl.encode_opts(1024, 512, True)
    pool = [rows_config1(seed=101 + k) for k in range(n_distinct)]
    lm = jl.Model(wpath, 2048, 8, 64, precision=jl.JD_PREC_BF16, device=local)

    def run(graph, reqs):
        lm.jd_set_graph_mode(graph)
        for k in range(max(20, len(reqs))):  # graph mode: every bucket of the pool captured before timing
            lm.jd_decide_host(reqs[k % len(reqs)], o1)
        c0, r0, _ = lm.jd_graph_stats()
        ts = []
        for k in range(calls):
            t = time.perf_counter()
            lm.jd_decide_host(reqs[k % len(reqs)], o1)
            ts.append(1000 * (time.perf_counter() - t))
        c1, r1, nb = lm.jd_graph_stats()
        out = {"p50_ms": _r(float(np.percentile(ts, 50))), "p99_ms": _r(float(np.percentile(ts, 99)))}
        if graph:
            out.update(captures_in_timed_calls=c1 - c0, replays_in_timed_calls=r1 - r0, buckets=nb)
        return out

    out = {"distinct_eager": run(False, pool), "distinct_graph": run(True, pool),
           "repeated_graph": run(True, pool[:1])}
    lm.jd_set_graph_mode(False)
    # per-kernel device time of one call (events around every launch; these calls synchronise)
    n_prof = 50
    lm.jd_set_profiling(True)
    for k in range(n_prof):
        lm.jd_decide_host(pool[k % len(pool)], o1)
    prof = lm.jd_profile_report()
    lm.jd_set_profiling(False)
    lm.close()
    out["per_kernel_us_per_call"] = {k: _r(1000.0 * ms / n_prof) for k, (n, ms) in
                                     sorted(prof.items(), key=lambda kv: -kv[1][1])}
    out["timed_launch_groups_per_call"] = int(sum(n for n, _ in prof.values()) // n_prof)
    out["device_us_per_call"] = _r(1000.0 * sum(ms for _, ms in prof.values()) / n_prof)
    best = min(("distinct_eager", "distinct_graph"), key=lambda k: out[k]["p50_ms"])
    out["reported"] = best
    out["workload"] = (f"{n_distinct} distinct 3-question requests (choice/4, score/3, noul/2) on a 200-token "
                       "state, called in turn through jd_decide_host (serialise + H2D + forward + D2H + sync)")
    return out


def measure_serving(jl, wpath, local, seconds, thread_counts=(1, 2, 4)):
    """Single 3-question requests (one 200-token state) served from 1, 2, 4 host
    threads, each with its own handle (jd_model_create_shared: one copy of the
    weights) and its own stream, CUDA-graph replay on; requests/s and latency."""
    import threading
    import torch
    from workloads import rows_config1
    r1 = rows_config1()
    o1 = jl.encode_opts(1024, 512, True)
    base = jl.Model(wpath, 2048, 8, 64, precision=jl.JD_PREC_BF16, device=local)
    out = []
    for n in thread_counts:
        handles = [jl.Model.shared(base, 2048, 8, 64) for _ in range(n)]
        lat = [[] for _ in range(n)]
        start = threading.Barrier(n + 1)

        def serve(k):
            torch.cuda.set_device(local)
            st = torch.cuda.Stream(device=local)
            h = handles[k]
            h.jd_set_graph_mode(True)
            for _ in range(10):
                h.jd_decide_host(r1, o1, stream=st)
            start.wait()
            t_end = time.perf_counter() + seconds
            while True:
                t = time.perf_counter()
                if t >= t_end:
                    break
                h.jd_decide_host(r1, o1, stream=st)
                lat[k].append(1000 * (time.perf_counter() - t))

        ths = [threading.Thread(target=serve, args=(k,)) for k in range(n)]
        for t in ths:
            t.start()
        start.wait()
        t0 = time.perf_counter()
        for t in ths:
            t.join()
        el = time.perf_counter() - t0
        allv = np.concatenate([np.asarray(v) for v in lat])
        out.append({"threads": n, "requests_per_s": _r(float(len(allv) / el)),
                    "p50_ms_per_call": _r(float(np.percentile(allv, 50))),
                    "p99_ms_per_call": _r(float(np.percentile(allv, 99)))})
        for h in handles:
            h.jd_check_status()
            h.close()
    base.close()
    return {"workload": "one 3-question request (choice/4, score/3, noul/2, 200-token state) repeated, "
                        "each thread its own shared handle and stream, CUDA-graph replay, host work included",
            "results": out}


def measure_router(jl, wpath, local, rank, ranks, reps, peaks):
    """Router workload: 512 independent requests, each a 256-id state, a question
    and 72 labels; round 1 scores groups of <=20 labels (4 rows per request), the
    survivors go to one final row per request.  decisions/s = requests / wall time
    of jd_route_device (rows of both rounds formed and packed on the device, forward
    rounds, survivor rule, copies), with jd_route_host (host serialisation per round)
    timed beside it and its outputs compared.
    Round 1 is also run alone with per-kernel events to give the HBM fraction of
    the attention, norm and gather kernels at this shape."""
    from workloads import Row, requests_config4
    reqs = requests_config4(512, seed=104 + 1000 * rank)
    opts = jl.encode_opts(1024, 512, True)
    m = jl.Model(wpath, 1 << 20, 2048, 2048 * 20, precision=jl.JD_PREC_BF16, device=local)

    def timed(call):
        for _ in range(2):
            o = call(reqs, opts)
        ranks.barrier()
        t0 = time.perf_counter()
        for _ in range(reps):
            o = call(reqs, opts)
        return o, ranks.max(time.perf_counter() - t0)

    out_h, el_h = timed(m.jd_route_host)
    out, el = timed(m.jd_route_device)
    same = all(np.array_equal(np.asarray(out[k]), np.asarray(out_h[k]))
               for k in ("winner", "winner_p", "final_candidates", "final_probs", "rows_per_round"))
    total = ranks.sum(float(len(reqs) * reps))
    m.jd_check_status()
    m.close()

    rows = [Row(state=q.state, question=q.question, options=q.labels[g:g + 20], qtype=0)
            for q in reqs for g in range(0, len(q.labels), 20)]
    hb = jl.jd_serialize(rows, opts)
    ms, r1 = profile_batch(jl, wpath, local, hb, 3, peaks)
    return {"workload": "512 requests x 72 labels of 3..12 ids on a 256-id state; groups of <=20, then one "
                        "final row of the survivors; head budget 512, max_length 1024, strict",
            "value": _r(total / el), "unit": "requests/s", "ms_per_call": _r(1000 * el / reps),
            "call": "jd_route_device (rounds formed, encoded and narrowed on the device; four counters read "
                    "back per round)",
            "host_rounds": {"value": _r(total / el_h), "ms_per_call": _r(1000 * el_h / reps),
                            "call": "jd_route_host (each round serialised on the host)",
                            "outputs_identical": bool(same)},
            "rows_per_round": [int(x) for x in out["rows_per_round"]],
            "round1": {"rows": int(hb.n_rows), "tokens": int(hb.n_tokens), "markers": int(hb.n_markers),
                       "ms_forward": _r(ms),
                       "hbm_bound_kernels": {k: r1[k] for k in ROUTER_KERNELS if k in r1}}}


def roofline_line(name, n, tot, cost, peaks, workload_tag, T):
    """The roofline object of one kernel from its event totals (n launches, tot ms)."""
    avg_s = tot / n / 1000.0
    byt, fl = cost
    t_hbm = byt / (peaks["hbm"] * 1e9)
    t_tc = fl / (peaks["tc_sust"] * 1e12)
    tr = recorded_traffic(name, workload_tag)
    if t_tc > t_hbm:
        ach = fl / avg_s / 1e12
        roof = {"bound": "tensor", "achieved": ach, "peak": peaks["tc_sust"], "unit": "TFLOP/s",
                "frac": ach / peaks["tc_sust"], "traffic": None if tr is None else tr * T,
                "kernel": name, "peak_source": f"{peaks['src']} sustained bf16 (cuBLAS)",
                "peak_burst": peaks["tc_burst"], "frac_of_burst": ach / peaks["tc_burst"]}
    else:
        ach = byt / avg_s / 1e9
        roof = {"bound": "hbm", "achieved": ach, "peak": peaks["hbm"], "unit": "GB/s",
                "frac": ach / peaks["hbm"], "traffic": None if tr is None else tr * T,
                "kernel": name, "peak_source": f"{peaks['src']} copy bandwidth"}
    roof["algorithmic_per_launch"] = {"bytes": byt, "flops": fl}
    roof["avg_launch_ms"] = avg_s * 1000.0
    roof["kernel_source_sha"] = kernel_source_sha(name)
    return roof


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
        dist.init_process_group("nccl", device_id=dev, timeout=timedelta(seconds=120))

    ranks = Ranks(world, dev)
    barrier, max_over_ranks, sum_over_ranks = ranks.barrier, ranks.max, ranks.sum

    from encoder_decision_model_b200.build import build
    if rank == 0:
        build()
    barrier()
    from encoder_decision_model_b200 import _lib as jl
    from workloads import weights_path

    if rank == 0:
        weights_path(0)
    barrier()
    rows, opts, desc = workload(args, rank)
    hb = jl.jd_serialize(rows, jl.encode_opts(**opts))
    T, B, M = hb.n_tokens, hb.n_rows, hb.n_markers
    lens = np.diff(hb.cu_seqlens)
    n_unique = len(np.unique(hb.tokens))

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        n, toks, el = oracle_sample(rows, opts, args.cpu_seconds)
        cpu = {"value": n / el, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
               "sample": f"first {n} rows ({toks} tokens) of this workload, float64 NumPy oracle, {el:.1f} s"}
        cpu["threads_4"] = oracle_four_threads(rows, opts, args.cpu_seconds)

    model = jl.Model(weights_path(0), T, B, M, precision=jl.JD_PREC_BF16, device=local)
    batch, outs, keep = upload_batch(jl, hb, dev)
    stream = torch.cuda.Stream(device=dev)

    def step():
        model.jd_decide(batch, **outs, stream=stream)

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            step()
        torch.cuda.synchronize()
        model.jd_check_status()
        launches_per_step = model.jd_last_launch_count()

        clocks = ClockSampler(local)
        barrier()
        torch.cuda.synchronize()
        clocks.start()
        time.sleep(0.3)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            step()
        e1.record(stream)
        torch.cuda.synchronize()
        barrier()
        ck = clocks.stop()
        ms = e0.elapsed_time(e1)
        ms_max = max_over_ranks(ms)
        model.jd_check_status()

        # per-kernel event timing on the launching stream (separate profiled steps)
        model.jd_set_profiling(True)
        for _ in range(args.profile_steps):
            step()
        prof = model.jd_profile_report()
        model.jd_set_profiling(False)
        torch.cuda.synchronize()

    decisions = sum_over_ranks(float(B * args.steps))
    tokens = sum_over_ranks(float(T * args.steps))
    value = decisions / (ms_max / 1000.0)

    # ---- end to end through the host entry point: serialise + H2D + forward + D2H
    e2e_steps = max(3, min(args.steps, 10))
    hopts = jl.encode_opts(**opts)
    model.jd_decide_host(rows, hopts)  # warm
    barrier()
    t0 = time.perf_counter()
    for _ in range(e2e_steps):
        model.jd_decide_host(rows, hopts)
    e2e_sync_s = max_over_ranks(time.perf_counter() - t0)
    e2e_sync_val = sum_over_ranks(float(B * e2e_steps)) / e2e_sync_s
    # the same calls with two in flight: the host serialises batch k + 1 while the device runs k
    barrier()
    t0 = time.perf_counter()
    inflight = []
    for _ in range(e2e_steps):
        inflight.append(model.jd_decide_host_submit(rows, hopts))
        if len(inflight) == 2:
            model.jd_decide_host_collect(inflight.pop(0))
    while inflight:
        model.jd_decide_host_collect(inflight.pop(0))
    e2e_s = max_over_ranks(time.perf_counter() - t0)
    e2e_val = sum_over_ranks(float(B * e2e_steps)) / e2e_s
    h2d = 4 * (T + (B + 1) + M + (B + 1) + B)
    d2h = 4 * (2 * M + 4 * B)
    model.close()

    peaks = read_peaks()
    # ---- batch-1 latency over distinct requests, eager and graph side by side
    lat = {}
    latency = None
    if rank == 0 and args.latency_calls > 0:
        latency = measure_latency(jl, weights_path(0), local, args.latency_calls)
        best = latency[latency["reported"]]
        lat = dict(p50_ms_per_call=best["p50_ms"], p99_ms_per_call=best["p99_ms"])

    serving = None
    if rank == 0 and args.serve_seconds > 0:
        serving = measure_serving(jl, weights_path(0), local, args.serve_seconds)

    # ---- router: 512 requests x 72 labels, both rounds and the host work between them
    router = None
    if args.router_reps > 0:
        router = measure_router(jl, weights_path(0), local, rank, ranks, args.router_reps, peaks)

    # ---- bounded long-context leg (rows of 8192 tokens)
    long_leg = None
    if rank == 0 and args.long_rows > 0 and args.workload == "throughput":
        long_leg = measure_long(jl, weights_path(0), local, args.long_rows, 3, peaks)

    # ---- the same batch in FP8 mode (E4M3 encoder QKV projections)
    fp8 = None
    if rank == 0 and args.fp8_steps > 0:
        fp8 = measure_fp8(jl, weights_path(0), local, hb, args.fp8_steps, peaks)

    # ---- roofline of the dominant kernel
    roof = None
    per_kernel = kernel_fractions(prof, args.profile_steps, lens, M, np.diff(hb.opt_off), n_unique, peaks) \
        if prof else {}
    if prof:
        top = max(prof, key=lambda k: prof[k][1])
        n, tot = prof[top]
        cost = algorithmic_cost(top, lens, M, np.diff(hb.opt_off), n_unique)
        if cost is not None:
            roof = roofline_line(top, n, tot, cost, peaks, args.workload, T)

    targets = {"peaks": {k: peaks[k] for k in ("hbm", "tc_sust", "tc_burst", "src")}}
    if long_leg:
        targets["long_encoder_gemm_tensor_frac"] = long_leg["encoder_gemm_tensor_frac"]
    if fp8:
        targets["fp8_qkv_tensor_frac_of_fp8_peak"] = fp8["gemm_qkv_rope"].get("tensor_frac_of_fp8_peak")
    if router:
        targets["router_round1_hbm_frac"] = {k: v.get("hbm_frac") for k, v in
                                             router["round1"]["hbm_bound_kernels"].items()}
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_max / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": desc, "global_batch": int(B * world), "rows_per_gpu": int(B),
                       "tokens_per_gpu_step": int(T), "markers_per_gpu_step": int(M),
                       "parallelism": f"dp{world} (independent rows per rank, no collective)",
                       "l2": "inputs larger than L2 (FP32 residual stream of one step alone is "
                             f"{T * 1536 / 1e6:.0f} MB)",
                       "weights": "random init N(0,0.02), seed 0"},
            "tokens_per_s": tokens / (ms_max / 1000.0),
            **lat,
            "roofline": roof, "cpu_baseline": cpu,
            "e2e": {"value": e2e_val, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "one_call_at_a_time": {"value": e2e_sync_val, "call": "jd_decide_host"},
                    "call": "jd_decide_host_submit / jd_decide_host_collect, two calls in flight (serialise + H2D "
                            "from pinned staging + forward + D2H + wait, the next call prepared meanwhile)"},
            "gpu_launches": int(launches_per_step * args.steps),
            "clocks": ck, "per_kernel": per_kernel, "latency": latency, "concurrent_serving": serving,
            "router": router, "long_context": long_leg, "fp8": fp8, "targets": targets}
    if rank == 0:
        s = json.dumps(line)
        print(s, flush=True)
        if args.json_out:
            open(args.json_out, "w").write(s + "\n")
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
