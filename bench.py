"""Throughput of the sparse paged attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload c3]
                    [--impl ours|reference] [--no-e2e] [--no-cpu-baseline]

A step is one pass of the whole path over one resident batch: KV-set build,
FP8 page decode (mixed cache only) and sparse sink attention. The default
workload is the ratio-4 CSA prefill (2 x 8192 tokens, 128 heads, d = 128,
W = 128, top-k 512, page 64): the configuration whose tensor-core target the
method states; its inputs (Q and O are 537 MB each) exceed the 126 MB L2, so
no flush is needed between steps. Decode workloads (c4, c5) write a 256 MB
buffer (more than the L2) between timed steps, outside the timed intervals.

Under torchrun every rank runs its own batch (independent requests, no
collective on the data path; weak scaling); rank 0 prints one JSON line.
``--impl reference`` times the CPU oracle (the only reference this path
has) on a bounded sample of the same workload, on the host cores.
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = ("attended query·head·KV pairs/s and TFLOP/s (prefill); decode tok/s, HBM GB/s")
UNIT = "query·head·KV pairs/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


def env_rank():
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("LOCAL_RANK", 0)),
            int(os.environ.get("WORLD_SIZE", 1)))


def job_totals(local_units, local_ms, world, device):
    """Whole-job figures over the ranks: the units every rank processed
    (ranks draw their own inputs, so their counts may differ) and the time
    of the slowest rank. Every rank makes the same two collective calls."""
    if world == 1:
        return float(local_units), float(local_ms)
    import torch
    import torch.distributed as dist
    u = torch.tensor([float(local_units)], dtype=torch.float64, device=device)
    dist.all_reduce(u, op=dist.ReduceOp.SUM)
    t = torch.tensor([float(local_ms)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(u.item()), float(t.item())


class ClockSampler:
    """nvidia-smi samples of the SM clock and throttle reasons."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.samples = []
        self.proc = None
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.samples.append((time.time(), [x.strip() for x in line.split(",")]))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        if self.thread is not None:
            self.thread.join(timeout=5)

    def summary(self, t0, t1):
        rows = [s for (t, s) in self.samples if t0 - 0.15 <= t <= t1 + 0.15] or \
               [s for (_, s) in self.samples[-3:]]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        sm = [float(r[0]) for r in rows if r[0].replace(".", "").isdigit()]
        mx = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[k] for r in rows for k in range(4)
                          if len(r) > 4 + k and r[4 + k].lower() == "active"})
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


def physical_gpu(local_rank):
    vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
    parts = [x for x in vis.split(",") if x.strip()]
    if parts and all(x.strip().isdigit() for x in parts) and local_rank < len(parts):
        return int(parts[local_rank])
    return local_rank


def algorithmic(w, nnz):
    """Per-step algorithmic work of the attention launch: FLOPs = 4 d per
    (query, head, key) triple (2d for QK^T, 2d for PV)."""
    triples = nnz * w.H
    flops = 4.0 * w.d * triples
    return triples, flops


def measured_traffic(w, args):
    """DRAM bytes per attention launch from the committed ncu capture, if it
    was taken on the kernel source as it is now (else None)."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "attn_dram_traffic.json")
    if not os.path.exists(path):
        return None
    rec = json.load(open(path))
    h = hashlib.sha256()
    for f in ("attn_fwd.cu", "attn_common.cuh", "spa_device.cuh"):
        h.update(open(os.path.join(ROOT, "sparse_paged_attention_build_b200", "csrc", f), "rb").read())
    fused = w.k_cmp_fp8 is not None and args.fp8_path == "fused"
    entry = rec.get(w.name + (":fused" if fused else ""))
    if entry is None or rec.get("kernel_sha256") != h.hexdigest() or args.shrink != 1:
        return None
    return entry["dram_bytes_per_launch"]


def algorithmic_bytes(w, indptr, indices, fused_fp8=False):
    """HBM bytes the attention launch must move at least once: Q, O, LSE,
    the CSR sets, the page tables and every distinct (request, key) K/V row
    (a compressed row read as FP8 codes and scales when the decode is fused
    into the gather)."""
    req_of_key = np.repeat(w.req.astype(np.int64), np.diff(indptr))
    keys = np.unique(req_of_key * (1 << 31) + indices.astype(np.int64))
    distinct = keys.size
    qo = 2 * w.N * w.H * w.d * 2
    if fused_fp8:
        n_cmp = int(((keys & ((1 << 31) - 1)) < (1 << 30)).sum())
        kv = (distinct - n_cmp) * 2 * w.d * 2 + n_cmp * 2 * (w.d + 4 * (w.d // 64))
    else:
        kv = distinct * 2 * w.d * 2
    other = w.N * w.H * 4 + indptr.nbytes + indices.nbytes + w.pt_raw.nbytes + \
        (0 if w.pt_cmp is None else w.pt_cmp.nbytes)
    return qo + kv + other, distinct


def run_reference(args, rank, world):
    """The oracle, as it stands, on a bounded sample of the workload."""
    if rank != 0:
        return 0
    import oracle
    from sparse_paged_attention_build_b200 import workloads
    w = workloads.make(args.workload)
    ip, idx = oracle.build_kv_sets(w.pos, w.W, w.ratio, w.topk)
    k_cmp, v_cmp = w.k_cmp, w.v_cmp
    if w.k_cmp_fp8 is not None:
        k_cmp = oracle.dequant_fp8_pages(w.k_cmp_fp8, w.k_cmp_scale, w.cmp_page_ids)
        v_cmp = oracle.dequant_fp8_pages(w.v_cmp_fp8, w.v_cmp_scale, w.cmp_page_ids)
    threads = os.cpu_count() or 1
    rng = np.random.default_rng(0)
    rows_per_step = args.ref_rows or max(threads, 16)
    times, triples = [], []
    for s in range(args.warmup + args.steps):
        rows = np.sort(rng.choice(w.N, size=min(w.N, rows_per_step), replace=False)).astype(np.int32)
        t0 = time.perf_counter()
        oracle.sparse_sink_attn(w.q, w.k_raw, w.v_raw, w.pt_raw, w.req, ip, idx, w.sink, w.scale,
                                k_cmp=k_cmp, v_cmp=v_cmp, pt_cmp=w.pt_cmp, rows=rows, threads=threads)
        dt = time.perf_counter() - t0
        if s >= args.warmup:
            times.append(dt)
            triples.append(int((ip[rows + 1] - ip[rows]).sum()) * w.H)
    value = float(sum(triples) / sum(times))
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * float(np.mean(times)),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": config_of(w, world, int(ip[-1]), args.fp8_path),
        "cpu_baseline": {"kind": "oracle", "value": value, "unit": UNIT, "cores": threads,
                         "cpu_model": cpu_model(),
                         "sample": f"{rows_per_step} random query tokens per step (of {w.N}), all heads, "
                                   f"FP64 C oracle with {threads} threads"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def sets_mode(w, args):
    """Where the step builds its key sets when --sets is auto: "inline"
    (inside the attention kernel, which measured faster than a separate
    build on every workload) wherever the kernel can (top-k rows of at most
    512 entries), else "csr"; otherwise as asked."""
    from sparse_paged_attention_build_b200.pipeline import inline_sets_supported
    if args.sets != "auto":
        return args.sets
    return "inline" if inline_sets_supported(w) else "csr"


SETS_TEXT = {"csr": "spa_build_kv_sets, then the attention reads the CSR sets",
             "inline": "built inside the attention kernel (the *_inline_sets call)"}


def config_of(w, world, nnz, fp8_path=None):
    from sparse_paged_attention_build_b200 import workloads
    c = {"workload": f"{w.name}: {workloads.DESCRIPTIONS[w.name]}", "n_queries": w.N, "heads": w.H,
         "head_dim": w.d, "window": w.W, "ratio": w.ratio, "topk": w.K,
         "page_size": w.raw_page_size, "parallelism": f"dp{world}",
         "l2": "inputs larger than L2 (no flush)" if w.kind == "prefill"
               else "256 MB buffer written between timed steps (L2 flush)"}
    if nnz is not None:
        c["kv_pairs_per_step"] = nnz
        c["mean_set_size"] = nnz / w.N
    if w.k_cmp_fp8 is not None:
        c["fp8_path"] = fp8_path
    return c


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default="c3", choices=["c1", "c2", "c3", "c4", "c5", "f1", "f2"],
                    help="c1..c5: the 128-head configurations; f1, f2: the 32-head, 512-wide DSV4-Flash shape")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--splits", type=int, default=0)
    ap.add_argument("--sets", default="auto", choices=["auto", "csr", "inline"],
                    help="csr: spa_build_kv_sets, then the attention reads the CSR sets; inline: the "
                         "sets built inside the attention kernel; auto: inline wherever the kernel can "
                         "(top-k rows of at most 512 entries)")
    ap.add_argument("--fp8-path", default="fused", choices=["fused", "decode"],
                    help="mixed FP8 cache: decode inside the attention gather, or decode the pages first")
    ap.add_argument("--op", default="path", choices=["path", "kv_write", "bwd", "unpack_d512"],
                    help="path: the attention hot path (the bench line); kv_write: the paged KV write alone; "
                         "bwd: the backward of the attention alone")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ref-rows", type=int, default=0)
    ap.add_argument("--no-decode", dest="decode_too", action="store_false",
                    help="prefill workloads: skip the ratio-128 decode measurement that rides along")
    ap.add_argument("--shrink", type=int, default=1,
                    help="divide requests/tokens (profiling cases only; not a bench line)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    rank, local_rank, world = env_rank()

    if args.impl == "reference":
        return run_reference(args, rank, world)
    if args.op == "kv_write":
        return run_kv_write(args, rank, local_rank, world)
    if args.op == "bwd":
        return run_bwd(args, rank, local_rank, world)
    if args.op == "unpack_d512":
        return run_unpack_d512(args, rank, local_rank, world)

    import torch
    import torch.distributed as dist
    from sparse_paged_attention_build_b200 import workloads
    from sparse_paged_attention_build_b200.pipeline import DeviceBatch
    import sparse_paged_attention_build_b200 as spa

    torch.cuda.set_device(local_rank)
    if world > 1:
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))

    def barrier():
        if world > 1:
            dist.barrier()

    w = workloads.make(args.workload, shrink=args.shrink, seed_offset=rank)
    res = measure_path(w, args, args.steps, args.warmup, args.splits, local_rank, world, barrier, dist)

    # The ratio-128 decode rides along in the default run, so that every
    # bench line carries both targets of the path: the prefill's tensor
    # roofline and the decode's HBM roofline. Same protocol (graph replay,
    # L2 flushed between steps, CUDA events on the launching stream).
    dec = None
    if args.decode_too and w.kind == "prefill" and args.shrink == 1:
        wd = workloads.make("c4", seed_offset=rank)
        dres = measure_path(wd, args, max(args.steps, 50), args.warmup, 0, local_rank, world, barrier, dist,
                            want_e2e=not args.no_e2e)
        dec = {"workload": f"{wd.name}: {workloads.DESCRIPTIONS[wd.name]}",
               "tok_per_s": dres["total_queries"] / (dres["elapsed_ms"] / 1e3),
               "ms_per_step": dres["elapsed_ms"] / dres["steps"],
               "attn_ms_per_launch": dres["attn_ms"], "hbm_gbs": dres["roofline"]["hbm_gbs"],
               "pairs_per_s": dres["value"], "roofline": dres["roofline"], "clocks": dres["clocks"],
               "num_splits": dres["num_splits"], "gpu_launches": dres["gpu_launches"],
               "device_status": dres["status"], "config": config_of(wd, world, dres["nnz"], args.fp8_path),
               "sets": SETS_TEXT[dres["sets"]], "e2e": dres["e2e"]}
        if dres["e2e"] is not None:
            # the same tokens per step, at the end-to-end rate of pairs
            dec["e2e"]["tok_per_s"] = dec["tok_per_s"] * dres["e2e"]["value"] / max(dres["value"], 1e-30)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w)

    if rank == 0:
        line = {
            "metric": METRIC, "value": res["value"], "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": res["elapsed_ms"] / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": config_of(w, world, res["nnz"], args.fp8_path),
            "tflops": res["tflops"],
            "roofline": res["roofline"],
            "clocks": res["clocks"], "e2e": res["e2e"], "gpu_launches": res["gpu_launches"],
            "device_status": res["status"], "sets": SETS_TEXT[res["sets"]],
        }
        if w.kind == "decode":
            line["tok_per_s"] = res["total_queries"] / (res["elapsed_ms"] / 1e3)
            if res["e2e"] is not None:
                line["e2e"]["tok_per_s"] = line["tok_per_s"] * res["e2e"]["value"] / max(res["value"], 1e-30)
        if dec is not None:
            line["decode"] = dec
        if cpu is not None:
            line["cpu_baseline"] = cpu
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def measure_path(w, args, steps, warmup, splits, local_rank, world, barrier, dist, want_e2e=None):
    """Time the hot path (sets, FP8 decode, attention) on one workload:
    graph replays, CUDA events on the launching stream, whole-job totals
    over the ranks; the roofline of the attention launch; clocks sampled
    during the timed region; the end-to-end figure through the public API."""
    import torch
    from sparse_paged_attention_build_b200.pipeline import DeviceBatch

    decode = w.kind == "decode"
    sets = sets_mode(w, args)
    b0 = DeviceBatch(w, num_splits=splits, fp8_path=args.fp8_path, sets=sets)
    stream = torch.cuda.current_stream()
    b0.build_sets()   # the CSR sets, for the counts below (inside the step only on the csr path)
    b0.step()
    torch.cuda.synchronize()
    nnz = b0.nnz()
    triples, flops = algorithmic(w, nnz)
    hbm_bytes, distinct_rows = algorithmic_bytes(w, b0.indptr.cpu().numpy(),
                                                 b0.indices[:nnz].cpu().numpy(), fused_fp8=b0.fused)
    # a decode batch fits in L2: write a buffer larger than L2 between
    # timed steps (outside the timed intervals)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda") if decode else None

    # The step is replayed from two CUDA graphs (set build + FP8 decode, then
    # attention) so that host-side launch cost does not enter the device
    # timings; the graphs launch exactly the library's kernels.
    # (With the sets built inside the attention kernel and no FP8 decode, the
    # first graph would be empty: the step is the attention alone.)
    has_front = not b0.inline_sets or (b0.fp8 and not b0.fused)
    g_front, g_attn = (torch.cuda.CUDAGraph() if has_front else None), torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream()
    cap.wait_stream(stream)
    with torch.cuda.stream(cap):
        if has_front:
            with torch.cuda.graph(g_front, stream=cap):
                if not b0.inline_sets:
                    b0.build_sets()
                b0.dequant()
        with torch.cuda.graph(g_attn, stream=cap):
            b0.attend()
    stream.wait_stream(cap)
    torch.cuda.synchronize()

    for s in range(warmup):
        if flush is not None:
            flush.zero_()
        if has_front:
            g_front.replay()
        g_attn.replay()
    torch.cuda.synchronize()

    sampler = ClockSampler(physical_gpu(local_rank))
    sampler.start()
    time.sleep(0.3)
    ev = [tuple(torch.cuda.Event(enable_timing=True) for _ in range(3)) for _ in range(steps)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    t_wall0 = time.time()
    start.record(stream)
    for s in range(steps):
        if flush is not None:
            flush.zero_()
        ev[s][0].record(stream)
        if has_front:
            g_front.replay()
        ev[s][1].record(stream)
        g_attn.replay()
        ev[s][2].record(stream)
    stop.record(stream)
    stop.synchronize()
    torch.cuda.synchronize()
    barrier()
    t_wall1 = time.time()
    time.sleep(0.25)
    sampler.stop()
    clocks = sampler.summary(t_wall0, t_wall1)

    if decode:   # the sum of the steps, without the flushes between them
        elapsed_ms = float(sum(e0.elapsed_time(e2) for e0, _, e2 in ev))
    else:
        elapsed_ms = start.elapsed_time(stop)
    attn_ms = float(np.mean([e1.elapsed_time(e2) for _, e1, e2 in ev]))
    total_triples, elapsed_ms = job_totals(triples * steps, elapsed_ms, world, "cuda")
    total_queries, _ = job_totals(w.N * steps, 0.0, world, "cuda")
    total_flops = total_triples * 4.0 * w.d
    status = b0.status_word()

    value = total_triples / (elapsed_ms / 1e3)
    pk, pk_kind = peaks()
    timed_s = elapsed_ms / 1e3
    burst = timed_s < 2.0
    peak_tf = pk["bf16_tflops"] if burst else pk.get("bf16_tflops_sustained", pk["bf16_tflops"])
    peak_gbs = pk["hbm_gbs"]
    achieved_tf = flops / (attn_ms / 1e3) / 1e12
    achieved_gbs = hbm_bytes / (attn_ms / 1e3) / 1e9
    # the bound is the roof the launch's arithmetic intensity reaches first
    tensor_bound = flops / hbm_bytes > (peak_tf * 1e12) / (peak_gbs * 1e9)
    traffic = measured_traffic(w, args)
    if tensor_bound:
        roofline = {"bound": "tensor", "achieved": achieved_tf, "peak": peak_tf, "unit": "TFLOP/s",
                    "frac": achieved_tf / peak_tf,
                    "peak_source": f"{pk_kind} {'burst' if burst else 'sustained'} bf16 GEMM"}
    else:
        roofline = {"bound": "hbm", "achieved": achieved_gbs, "peak": peak_gbs, "unit": "GB/s",
                    "frac": achieved_gbs / peak_gbs, "peak_source": f"{pk_kind} HBM copy"}
    kernel = ("sparse_sink_attn_d512_kernel" if w.d == 512
              else f"sparse_sink_attn_kernel<{w.d}, {'true' if b0.fused else 'false'}>")
    roofline.update({"kernel": kernel,
                     "traffic": traffic,
                     "algorithmic_bytes": hbm_bytes, "algorithmic_flops": flops,
                     "distinct_kv_rows": int(distinct_rows), "tflops": achieved_tf,
                     "hbm_gbs": achieved_gbs, "attn_ms_per_launch": attn_ms})
    kernels_per_step = b0.kernels_per_step()

    # end to end through the public API: pinned host inputs -> device ->
    # the three calls -> O and LSE back to the host, every step
    e2e = None
    if want_e2e if want_e2e is not None else not args.no_e2e:
        e2e = measure_e2e(w, b0, args, stream, world, barrier, dist)
    splits_used = b0.splits_used()
    del g_front, g_attn
    return {"value": value, "elapsed_ms": elapsed_ms, "attn_ms": attn_ms, "nnz": nnz,
            "tflops": total_flops / (elapsed_ms / 1e3) / 1e12, "roofline": roofline, "clocks": clocks,
            "e2e": e2e, "gpu_launches": kernels_per_step * steps, "status": status, "steps": steps,
            "total_queries": total_queries, "num_splits": splits_used, "sets": sets}


def run_kv_write(args, rank, local_rank, world):
    """The paged KV write alone: the workload's new tokens (every token of a
    prefill batch, the last token of each decode request) written into the
    raw window pools through the page table; HBM GB/s against the copy peak.
    The rows written are the ones the pools already hold, so the pools keep
    their contents."""
    import torch
    import torch.distributed as dist
    from sparse_paged_attention_build_b200 import workloads
    import sparse_paged_attention_build_b200 as spa
    torch.cuda.set_device(local_rank)
    if world > 1:
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    w = workloads.make(args.workload, shrink=args.shrink, seed_offset=rank)
    ps = w.raw_page_size
    rows = w.pt_raw[w.req, w.pos // ps].astype(np.int64) * ps + w.pos % ps
    k_new = w.k_raw.reshape(-1, w.d)[rows]
    v_new = w.v_raw.reshape(-1, w.d)[rows]
    dev = lambda a, dt=None: torch.from_numpy(np.ascontiguousarray(a)).cuda() if dt is None else \
        torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(dt)
    bf = torch.bfloat16
    kn, vn = dev(k_new, bf), dev(v_new, bf)
    kp, vp = dev(w.k_raw, bf), dev(w.v_raw, bf)
    req, pos, pt = dev(w.req), dev(w.pos), dev(w.pt_raw)
    st = spa.new_status()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    g = torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream()
    cap.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(cap):
        with torch.cuda.graph(g, stream=cap):
            spa.paged_kv_write(kn, vn, req, pos, pt, kp, vp, dev_status=st)
    torch.cuda.current_stream().wait_stream(cap)
    for _ in range(args.warmup):
        flush.zero_()
        g.replay()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for e0, e1 in evs:
        flush.zero_()   # new tokens and pools come from HBM
        e0.record()
        g.replay()
        e1.record()
    torch.cuda.synchronize()
    ms = float(np.median([e0.elapsed_time(e1) for e0, e1 in evs]))
    n = len(rows)
    bytes_step = n * 2 * (2 * w.d * 2) + 2 * n * 4 + w.pt_raw.nbytes   # rows read + written, req/pos, table
    total_bytes, ms = job_totals(bytes_step, ms, world, "cuda")
    pk, pk_kind = peaks()
    gbs = total_bytes / (ms / 1e3) / 1e9
    ok = np.array_equal(kp.view(torch.int16).cpu().numpy().view(np.uint16), w.k_raw) and spa.read_status(st) == 0
    if rank == 0:
        print(json.dumps({
            "metric": "paged KV write HBM GB/s", "value": gbs, "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": f"{w.name}: {workloads.DESCRIPTIONS[w.name]}", "tokens_written": int(n),
                       "l2": "256 MB buffer written between timed steps (L2 flush)"},
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs / pk["hbm_gbs"], "peak_source": f"{pk_kind} HBM copy",
                         "kernel": "paged_kv_write_kernel", "algorithmic_bytes": int(bytes_step)},
            "gpu_launches": args.steps, "pools_unchanged": bool(ok)}))
    if world > 1:
        dist.destroy_process_group()
    return 0


def run_bwd(args, rank, local_rank, world):
    """The backward of the attention alone (dq, dk/dv into the pool-shaped
    gradients, dsink), from the forward's O and LSE and a seeded dO. The
    sets and the forward run once, untimed; each timed step is one backward
    launch, graph-replayed, after an L2 flush. The gradients are added into
    (zeroing them is the caller's, once per accumulation, and is not timed).
    Algorithmic FLOPs per query.head.key pair: 5 products x 2d."""
    import torch
    import torch.distributed as dist
    from sparse_paged_attention_build_b200 import workloads
    from sparse_paged_attention_build_b200.pipeline import DeviceBatch
    import sparse_paged_attention_build_b200 as spa
    torch.cuda.set_device(local_rank)
    if world > 1:
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    w = workloads.make(args.workload, shrink=args.shrink, seed_offset=rank)
    if w.k_cmp_fp8 is not None:
        raise SystemExit("the backward takes BF16 pools; the mixed FP8 workload has none")
    b = DeviceBatch(w)
    b.build_sets()
    out, lse = spa.sparse_sink_attn_fwd(b.q, b.k_raw, b.v_raw, b.pt_raw, b.req, b.indptr, b.indices, b.sink,
                                        w.scale, k_cmp=b.k_cmp, v_cmp=b.v_cmp, pt_cmp=b.pt_cmp)
    dO = torch.from_numpy(workloads.make_dout(w).view(np.int16)).cuda().view(torch.bfloat16)
    torch.cuda.synchronize()
    pairs = int(b.indptr[-1].item()) * w.H
    # FP32 reduction bytes per call: each 64-key tile of a unit adds one
    # [64 keys x d] block into dK and one into dV (bulk reductions), and
    # every slice of a query adds its [H x d] block into dq
    set_sizes = np.diff(b.indptr.cpu().numpy().astype(np.int64))
    splits_used = args.splits if args.splits > 0 else spa.choose_splits(w.N, w.H, 0)
    red_dkdv = int(np.sum((set_sizes + 63) // 64)) * 2 * 64 * w.d * 4
    red_dq = int(splits_used) * w.N * w.H * w.d * 4
    st = spa.new_status()
    grads = spa.sparse_sink_attn_bwd(b.q, b.k_raw, b.v_raw, b.pt_raw, b.req, b.indptr, b.indices, b.sink,
                                     w.scale, out, lse, dO, k_cmp=b.k_cmp, v_cmp=b.v_cmp, pt_cmp=b.pt_cmp,
                                     num_splits=args.splits, dev_status=st)
    torch.cuda.synchronize()
    dq, dkr, dvr, dkc, dvc, dsk = grads
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    g = torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream()
    cap.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(cap):
        with torch.cuda.graph(g, stream=cap):
            spa.sparse_sink_attn_bwd(b.q, b.k_raw, b.v_raw, b.pt_raw, b.req, b.indptr, b.indices, b.sink,
                                     w.scale, out, lse, dO, k_cmp=b.k_cmp, v_cmp=b.v_cmp, pt_cmp=b.pt_cmp,
                                     dq=dq, dk_raw=dkr, dv_raw=dvr, dk_cmp=dkc, dv_cmp=dvc, dsink=dsk,
                                     num_splits=args.splits, dev_status=st)
    torch.cuda.current_stream().wait_stream(cap)
    for _ in range(args.warmup):
        flush.zero_()
        g.replay()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for e0, e1 in evs:
        flush.zero_()
        e0.record()
        g.replay()
        e1.record()
    torch.cuda.synchronize()
    times = [e0.elapsed_time(e1) for e0, e1 in evs]
    ms = float(np.median(times))
    total_pairs, ms = job_totals(pairs, ms, world, "cuda")
    flops = 10.0 * w.d * total_pairs
    tflops = flops / (ms / 1e3) / 1e12
    pk, pk_kind = peaks()
    ok = spa.read_status(st) == 0 and all(bool(torch.isfinite(t).all()) for t in grads if t is not None)
    if rank == 0:
        print(json.dumps({
            "metric": "backward query.head.KV pairs/s", "value": total_pairs / (ms / 1e3),
            "unit": "pairs/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "ms_min": float(np.min(times)), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "config": {"workload": f"{w.name}: {workloads.DESCRIPTIONS[w.name]}", "pairs": int(pairs),
                       "num_splits": args.splits, "l2": "256 MB buffer written between timed steps (L2 flush)",
                       "gradient zeroing": "not timed (the call adds into the gradients)",
                       "reduction_bytes": {"dk_dv": red_dkdv, "dq": red_dq, "total": red_dkdv + red_dq}},
            "roofline": {"bound": "tensor", "achieved": tflops, "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                         "frac": tflops / pk["bf16_tflops"], "peak_source": f"{pk_kind} BF16 burst",
                         "kernel": "sparse_sink_attn_bwd_kernel", "algorithmic_flops": flops},
            "gpu_launches": args.steps, "finite_and_status_ok": bool(ok)}))
    if world > 1:
        dist.destroy_process_group()
    return 0


def run_unpack_d512(args, rank, local_rank, world):
    """The packed 512-wide row decode alone: a seeded packed cache of
    8192 pages x 64 tokens (584 bytes per token; a 128-request, 4096-token
    context in 64-token pages), every page decoded to BF16; HBM GB/s
    against the copy peak. Algorithmic bytes per token: 584 read + 1024
    written."""
    import torch
    import torch.distributed as dist
    from sparse_paged_attention_build_b200 import workloads
    import sparse_paged_attention_build_b200 as spa
    torch.cuda.set_device(local_rank)
    if world > 1:
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    pages, ps = 8192 // max(1, args.shrink), 64
    src = torch.from_numpy(workloads.make_packed_d512(pages, ps, seed=rank)).cuda()
    ids = torch.arange(pages, dtype=torch.int32, device="cuda")
    dst = torch.empty((pages, ps, 512), dtype=torch.bfloat16, device="cuda")
    st = spa.new_status()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    g = torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream()
    cap.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(cap):
        with torch.cuda.graph(g, stream=cap):
            spa.unpack_d512_pages(src, ids, dst, dev_status=st)
    torch.cuda.current_stream().wait_stream(cap)
    for _ in range(args.warmup):
        flush.zero_()
        g.replay()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for e0, e1 in evs:
        flush.zero_()
        e0.record()
        g.replay()
        e1.record()
    torch.cuda.synchronize()
    ms = float(np.median([e0.elapsed_time(e1) for e0, e1 in evs]))
    tokens = pages * ps
    bytes_step = tokens * (584 + 1024) + pages * 4
    total_bytes, ms = job_totals(bytes_step, ms, world, "cuda")
    pk, pk_kind = peaks()
    gbs = total_bytes / (ms / 1e3) / 1e9
    if rank == 0:
        print(json.dumps({
            "metric": "packed D512 row decode HBM GB/s", "value": gbs, "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "e4m3+bf16 -> bf16", "data": "synthetic",
            "config": {"workload": f"packed 512-wide rows: {pages} pages x {ps} tokens x 584 bytes",
                       "l2": "256 MB buffer written between timed steps (L2 flush)"},
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs / pk["hbm_gbs"], "peak_source": f"{pk_kind} HBM copy",
                         "kernel": "unpack_d512_kernel", "algorithmic_bytes": int(bytes_step)},
            "gpu_launches": args.steps, "status_ok": spa.read_status(st) == 0}))
    if world > 1:
        dist.destroy_process_group()
    return 0


def measure_e2e(w, b0, args, stream, world, barrier, dist):
    import torch
    import sparse_paged_attention_build_b200 as spa

    def pinned(a, dtype=None):
        if a is None:
            return None
        t = torch.from_numpy(np.ascontiguousarray(a))
        if dtype is not None:
            t = t.view(dtype)
        return t.pin_memory()

    bf = torch.bfloat16
    host = {
        "q": pinned(w.q.view(np.int16), bf), "pos": pinned(w.pos), "req": pinned(w.req),
        "topk": pinned(w.topk), "pt_raw": pinned(w.pt_raw), "pt_cmp": pinned(w.pt_cmp),
        "sink": pinned(w.sink),
    }
    if w.kind == "prefill":
        host["k_raw"] = pinned(w.k_raw.view(np.int16), bf)
        host["v_raw"] = pinned(w.v_raw.view(np.int16), bf)
        if w.k_cmp is not None:
            host["k_cmp"] = pinned(w.k_cmp.view(np.int16), bf)
            host["v_cmp"] = pinned(w.v_cmp.view(np.int16), bf)
    if w.k_cmp_fp8 is not None and not b0.fused:
        host["cmp_page_ids"] = pinned(w.cmp_page_ids)
    dev = {k: getattr(b0, k) for k in host}
    h2d = sum(t.numel() * t.element_size() for t in host.values() if t is not None)
    out_h = torch.empty(b0.out.shape, dtype=bf).pin_memory()
    lse_h = torch.empty(b0.lse.shape, dtype=torch.float32).pin_memory()
    d2h = out_h.numel() * 2 + lse_h.numel() * 4
    steps = max(3, min(args.steps, 20))

    def one():
        for k, t in host.items():
            if t is not None:
                dev[k].copy_(t, non_blocking=True)
        b0.step()
        out_h.copy_(b0.out, non_blocking=True)
        lse_h.copy_(b0.lse, non_blocking=True)

    for _ in range(2):
        one()
    torch.cuda.synchronize()
    barrier()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record(stream)
    for _ in range(steps):
        one()
    e.record(stream)
    e.synchronize()
    ms = s.elapsed_time(e)
    total, ms = job_totals(b0.nnz() * w.H * steps, ms, world, "cuda")
    copies = ("per-step inputs host->device (q, positions, requests, top-k, page tables, sink"
              + (", the step's raw and compressed K/V" if w.kind == "prefill" else "")
              + "), O and LSE device->host"
              + ("; the paged KV caches stay resident on the device (decode)" if w.kind == "decode" else ""))
    return {"value": total / (ms / 1e3), "unit": UNIT,
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "ms_per_step": ms / steps, "steps": steps, "copies": copies}


def cpu_model():
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def cpu_baseline(w, budget_s=15.0, budget_1t_s=5.0):
    """The FP64 oracle on a bounded sample of the same workload: once with
    every host thread, once single-threaded."""
    import oracle
    threads = os.cpu_count() or 1
    ip, idx = oracle.build_kv_sets(w.pos, w.W, w.ratio, w.topk)
    k_cmp, v_cmp = w.k_cmp, w.v_cmp
    if w.k_cmp_fp8 is not None:
        k_cmp = oracle.dequant_fp8_pages(w.k_cmp_fp8, w.k_cmp_scale, w.cmp_page_ids)
        v_cmp = oracle.dequant_fp8_pages(w.v_cmp_fp8, w.v_cmp_scale, w.cmp_page_ids)
    rng = np.random.default_rng(1)

    def run(n, nthreads):
        rows = np.sort(rng.choice(w.N, size=min(n, w.N), replace=False)).astype(np.int32)
        t0 = time.perf_counter()
        oracle.sparse_sink_attn(w.q, w.k_raw, w.v_raw, w.pt_raw, w.req, ip, idx, w.sink, w.scale,
                                k_cmp=k_cmp, v_cmp=v_cmp, pt_cmp=w.pt_cmp, rows=rows, threads=nthreads)
        return time.perf_counter() - t0, int((ip[rows + 1] - ip[rows]).sum()) * w.H, rows.size

    dt, _, n = run(threads, threads)
    n2 = int(max(threads, min(w.N, n * budget_s / max(dt, 1e-3))))
    dt, tri, n2 = run(n2, threads)
    dt1, _, m = run(1, 1)
    m2 = int(max(1, min(w.N, m * budget_1t_s / max(dt1, 1e-3))))
    dt1, tri1, m2 = run(m2, 1)
    return {"kind": "oracle", "value": tri / dt, "unit": UNIT, "cores": threads,
            "cpu_model": cpu_model(), "value_1_thread": tri1 / dt1,
            "sample": f"{n2} random query tokens of {w.N} (all {w.H} heads), FP64 C oracle, "
                      f"{threads} threads, {dt:.1f} s; single-threaded: {m2} query tokens, {dt1:.1f} s"}


if __name__ == "__main__":
    sys.exit(main())
