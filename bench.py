"""Benchmark of the block-sparse decode step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...      # the fp64 CPU oracle, timed alone

One step = one pass of the whole hot path over one batch: incremental pooled-
key update of the newest block, gate scores, top-k block selection, split-KV
sparse decode and LSE combine (one ``seer_decode_step`` call: the fused
pool+gate+select kernel, the decode kernel and the combine kernel, chained by
programmatic dependent launch; the step is replayed as a CUDA graph).
Inputs are seeded synthetic tensors already resident in HBM; the timed loop
rotates over R independent replicas whose combined footprint exceeds four
times the L2, so every step reads its K/V, pooled keys and weights from HBM.
Prints one JSON line (rank 0).  With N > 1 (torchrun) every rank runs its own
replica of the workload (the step has no exchange: "replicas only", weak
scaling) and the time is the max over ranks.
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
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "sparse-decode tokens/s and µs/step at 32K ctx, 90% sparsity; HBM GB/s vs roofline"
UNIT = "tokens/s"
KERNELS_PER_STEP = 3   # gate+select (with the incremental pooled-key update), decode, combine
NOMINAL_HBM_GBS = 8000.0   # B200 HBM3e nominal, for the second roofline denominator
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0  # dense bf16 burst measured earlier on this machine's B200s


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return json.load(f), "measured"
    except (OSError, ValueError):
        return {"hbm_gbs": FALLBACK_HBM_GBS, "bf16_tflops": FALLBACK_BF16_TFLOPS}, "fallback"


def _code_only(src: str) -> str:
    """C++ source without its comments and with whitespace collapsed: what
    the compiler sees, so that a comment edit does not mark the kernel as
    changed."""
    import re
    src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
    src = re.sub(r"//[^\n]*", " ", src)
    return " ".join(src.split())


def decode_source_hash():
    """Hash of the decode kernel's code (its source and the two headers it
    takes its parameters and helpers from), comments and layout ignored."""
    h = hashlib.sha256()
    for name in ("sparse_decode.cu", "seer_common.cuh", "seer_kernels.cuh"):
        with open(os.path.join(ROOT, "block_sparse_attention_step_b200", "csrc", name)) as f:
            h.update(_code_only(f.read()).encode())
    return h.hexdigest()[:16]


def recorded_traffic(workload):
    """DRAM bytes per decode launch from the committed ncu summary, if it was
    taken on the current kernel source (else None)."""
    path = os.path.join(ROOT, "profiles", f"sparse_decode_{workload}.traffic.txt")
    try:
        kv = dict(line.split(":", 1) for line in open(path) if ":" in line)
    except OSError:
        return None
    kv = {k.strip(): v.strip() for k, v in kv.items()}
    if kv.get("source_hash") != decode_source_hash():
        return None
    try:
        return float(kv["dram_bytes_per_launch_full_size"])
    except (KeyError, ValueError):
        return None


# ------------------------------------------------------------------ clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, device_index):
        self.proc = None
        try:
            import torch
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            target = uuid if uuid.startswith("GPU-") else f"GPU-{uuid}"
        except Exception:
            target = str(device_index)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50", "-i", target], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, loaded, reasons = [], [], [], set()
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                s, m, pw = float(parts[1]), float(parts[2]), float(parts[3])
            except ValueError:
                continue
            sm.append(s)
            smax.append(m)
            if pw > 200:          # under load
                loaded.append(s)
            for name, val in zip(self.NAMES, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        use = loaded or sm
        return {"sm_mhz": statistics.median(use) if use else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm), "samples_under_load": len(loaded)}


# ------------------------------------------------------------------ CPU oracle

def oracle_rows_timed(w, data, rows, budget_s, k_per_seq, force_newest):
    """Time the fp64 oracle's whole step on (b, h) rows, one after another,
    until the row list or the time budget runs out.  Returns (seconds per
    row, rows timed, threads)."""
    import numpy as np
    from block_sparse_attention_step_b200 import workloads as W
    from oracle import seer_oracle as O
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        threads = 1
    scale = 1.0 / math.sqrt(w.head_dim)
    G = w.group
    spent, done = 0.0, 0
    for (b, h) in rows:
        L = int(data["seqlens"][b])
        q = data["q"][b, h * G:(h + 1) * G].double().cpu().numpy()
        Wg = data["w_gate"][h].double().cpu().numpy()
        K = W.gather_rows(data["k_pool"], data["page_table"], b, h, L, w.block_size, data.get("layout", "nhd")).double().numpy()
        V = W.gather_rows(data["v_pool"], data["page_table"], b, h, L, w.block_size, data.get("layout", "nhd")).double().numpy()
        t0 = time.perf_counter()
        O.decode_row(q, Wg, K, V, L, w.block_size, int(k_per_seq[b]), force_newest, scale, scale)
        spent += time.perf_counter() - t0
        done += 1
        if spent >= budget_s:
            break
    return spent / max(done, 1), done, threads


def cpu_k_per_seq(w, seqlens):
    from oracle import seer_oracle as O
    out = []
    for L in seqlens:
        nb = O.num_blocks(int(L), w.block_size)
        if w.budget_tokens:
            out.append(O.k_from_budget(nb, w.budget_tokens, w.block_size))
        else:
            out.append(O.k_from_sparsity(nb, w.sparsity_permille))
    return out


def run_reference(args):
    """The oracle alone on the host cores: each step is a bounded sample of
    the workload's (b, h) rows, scaled to tokens/s of the whole batch."""
    if int(os.environ.get("RANK", "0")) != 0:
        return 0
    import torch
    from block_sparse_attention_step_b200 import workloads as W
    w = W.WORKLOADS[args.workload]
    # rows of a batch-1 draw have the workload's per-row shape (L, G, bs, k)
    one = w.replace(batch=1) if w.seqlen_range is None else w.replace(batch=2)
    data = W.generate(one, args.seed, "cpu")
    kps = cpu_k_per_seq(one, data["seqlens"].tolist())
    rows = [(b, h) for b in range(one.batch) for h in range(one.kv_heads)]
    per_step = max(1, min(len(rows), args.ref_rows))
    times = []
    for i in range(args.warmup + args.steps):
        sample = [rows[(i * per_step + r) % len(rows)] for r in range(per_step)]
        sec, n, threads = oracle_rows_timed(one, data, sample, 1e9, kps, w.force_newest)
        if i >= args.warmup:
            times.append(sec)
    sec_row = sum(times) / len(times)
    if w.seqlen_range is not None:
        sec_row *= _ragged_row_scale(w, data)
    step_s = sec_row * w.batch * w.kv_heads
    value = w.batch / step_s
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_s * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": workload_config(w, None),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": f"{per_step} (b, kv-head) rows of a batch-{one.batch} draw per "
                                   f"step, fp64 numpy oracle, scaled to {w.batch}x{w.kv_heads} rows"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def _ragged_row_scale(w, data):
    """Oracle cost grows with L: scale the sampled rows' mean length to the
    workload's expected mean length."""
    lo, hi = w.seqlen_range
    sampled = float(data["seqlens"].double().mean())
    return ((lo + hi) / 2.0) / sampled


def workload_config(w, run, replicas=None, touched=None, layout=None):
    cfg = {"workload": w.name, "batch": w.batch, "q_heads": w.q_heads, "kv_heads": w.kv_heads,
           "head_dim": w.head_dim, "block_size": w.block_size,
           "seq_len": w.seqlen if w.seqlen else f"U[{w.seqlen_range[0]},{w.seqlen_range[1]}]",
           "selection": (f"budget {w.budget_tokens} tokens" if w.budget_tokens
                         else f"sparsity {w.sparsity_permille / 10:g}%"),
           "force_newest": w.force_newest, "paged": w.paged}
    if layout is not None:
        cfg["kv_layout"] = layout
    if run is not None:
        cfg["num_splits"] = run.num_splits
        cfg["k_max"] = run.k_max
    if replicas is not None:
        cfg["l2"] = (f"inputs larger than L2: {replicas} rotating replicas, "
                     f"{touched / 1e6:.0f} MB read per step, L2 126 MB")
    return cfg


# ------------------------------------------------------------------ our arm

def run_ours(args):
    import torch
    import torch.distributed as dist
    from block_sparse_attention_step_b200 import seer
    from block_sparse_attention_step_b200 import workloads as W
    from block_sparse_attention_step_b200.runner import StepBuffers

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    seer.library()
    w = W.WORKLOADS[args.workload]
    if args.sparsity is not None:
        w = w.replace(sparsity_permille=args.sparsity, budget_tokens=None)

    # replicas: enough that one rotation reads > 4x L2
    l2 = torch.cuda.get_device_properties(local).L2_cache_size
    probe = W.generate(w, args.seed + 1000 * rank, dev, layout=args.layout)
    run0 = StepBuffers(w, probe, num_splits=args.splits, mass=args.mass, unified=args.unified)
    run0.pool_full()
    torch.cuda.synchronize()
    sel_bytes, sel_tokens = selected_bytes(run0, probe, w)
    kbar_bytes = run0.kbar.numel() * 4
    touched = sel_bytes + kbar_bytes
    replicas = max(2, math.ceil(4 * l2 / max(touched, 1)))
    replicas = min(replicas, args.max_replicas)
    runs = [run0]
    for r in range(1, replicas):
        d = W.generate(w, args.seed + 1000 * rank + r, dev, layout=args.layout)
        # each replica sizes its index rows for its own sequences (ragged
        # replicas draw other lengths, so a shared k_max could clamp their k)
        rr = StepBuffers(w, d, num_splits=run0.num_splits, mass=args.mass, unified=args.unified)
        rr.pool_full()
        runs.append(rr)
    step_args = [r.args(update_kbar=1) for r in runs]
    # the per-stage step (3 kernels chained by PDL) or the single-launch step
    step_call = seer.seer_decode_step_fused if args.fused else seer.seer_decode_step
    stream = torch.cuda.current_stream(dev)
    torch.cuda.synchronize()

    def barrier():
        if world > 1:
            dist.barrier(device_ids=[local])

    # One step per replica captured as a CUDA graph (the step is two kernels
    # chained by programmatic dependent launch); replaying it keeps host launch
    # cost out of the device time.  --no-graph launches the C-ABI call directly.
    graphs = []
    if not args.no_graph:
        side = torch.cuda.Stream(dev)
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            for i in range(replicas):
                step_call(runs[i].dims, step_args[i], side)
        stream.wait_stream(side)
        torch.cuda.synchronize()
        for i in range(replicas):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                step_call(runs[i].dims, step_args[i], torch.cuda.current_stream())
            graphs.append(g)
        torch.cuda.synchronize()

    def one_step(i):
        if graphs:
            graphs[i % replicas].replay()
        else:
            step_call(runs[i % replicas].dims, step_args[i % replicas], stream)

    clocks = ClockSampler(local) if rank == 0 else None
    for i in range(args.warmup):
        one_step(i)
    torch.cuda.synchronize()

    # ---- timed region: exactly K steps
    barrier()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for i in range(args.steps):
        one_step(i)
    t1.record(stream)
    torch.cuda.synchronize()
    barrier()
    ms_total = t0.elapsed_time(t1)
    ms_max = max_over_ranks(ms_total, dev) if world > 1 else ms_total
    ms_step = ms_max / args.steps

    # ---- per-step spread (outside the timed region): an event pair per step
    pct = step_percentiles(one_step, min(args.steps, 400), stream)

    # ---- the dominant kernel alone (roofline), K more launches
    dec_us = decode_alone(runs, args.steps, stream, replicas)

    # ---- every stage through its standalone entry point (separate launches)
    stages = standalone_stages(runs, min(args.steps, 400), stream, replicas)

    # ---- end to end through the host entry point: q from pinned host memory
    # in, out to pinned host memory back, every step
    e2e = end_to_end(runs, args.steps, stream, replicas, w)
    clock_info = clocks.stop() if clocks else None
    status = [int(r.status.item()) for r in runs]
    recall = gate_recall_stats(run0, probe, w) if args.recall else None

    graphs.clear()   # release the graphs before the process group goes
    if world > 1:
        dist.barrier(device_ids=[local])
        dist.destroy_process_group()
    if rank != 0:
        return 0

    peaks, peak_kind = measured_peaks()
    dec_bytes = decode_bytes(run0, sel_bytes, w)
    achieved = dec_bytes / (dec_us * 1e-6) / 1e9
    line = {
        "metric": METRIC,
        "value": job_tokens_per_s(world, w.batch, ms_step),
        "unit": UNIT,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_step,
        "us_per_step": ms_step * 1e3,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded; random-init gate projection)",
        "config": dict(workload_config(w, run0, replicas, touched, args.layout),
                       block_mass=bool(args.mass),
                       selection_scope="one block set per sequence (all KV heads)"
                       if args.unified else "per KV head",
                       step_launch="single cooperative launch" if args.fused
                       else "per stage, PDL-chained"),
        "selected_kv_bytes_per_step": sel_bytes,
        "selected_tokens_per_step": sel_tokens,
        "step_hbm_gbs": (touched / (ms_step * 1e-3)) / 1e9,
        "selected_kv_gbs": (sel_bytes / (ms_step * 1e-3)) / 1e9,
        "stage_us": {"step": ms_step * 1e3, "sparse_decode_alone": dec_us,
                     "rest_of_step": ms_step * 1e3 - dec_us, "standalone": stages},
        "step_us_percentiles": pct,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"],
                     "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"],
                     "traffic": recorded_traffic(w.name), "kernel": "sparse_decode_kernel",
                     "bytes_per_launch": dec_bytes, "peak_source": f"{peak_kind} hbm_gbs",
                     "peak_nominal": NOMINAL_HBM_GBS,
                     "frac_nominal": achieved / NOMINAL_HBM_GBS},
        "e2e": e2e,
        "gpu_launches": (1 if args.fused else
                         KERNELS_PER_STEP + int(args.mass) + int(args.unified)) * args.steps,
        "clocks": clock_info,
        "device_status": status,
    }
    if recall is not None:
        line["gate_recall"] = recall
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, runs[0], args)
    print(json.dumps(line), flush=True)
    return 0


def gate_recall_stats(run0, data, w):
    """Gate recall on replica 0 (outside the timed region): a dense step with
    the block masses (every block selected) and the sparse step on the same
    inputs; the share of each (b, query head)'s dense attention mass that the
    sparse selection keeps."""
    import torch
    from block_sparse_attention_step_b200.runner import StepBuffers, gate_recall
    dense = StepBuffers(w, data, sparsity_permille=0, budget_tokens=0, mass=True)
    dense.step(update_kbar=2)
    run0.step(update_kbar=0)
    torch.cuda.synchronize()
    v = run0.workspace_views()
    rec = gate_recall(dense.block_mass, v["idx"], v["n_sel"], w.group).flatten().float()
    return {"mean": float(rec.mean()), "p10": float(torch.quantile(rec, 0.1)),
            "min": float(rec.min()),
            "what": "share of the dense attention mass in the blocks the gate selected, per "
                    "(sequence, query head) of replica 0 (random-init gate: a capability "
                    "check, not a quality number)",
            "device_status": [int(dense.status.item()), int(run0.status.item())]}


def prefill_flops(run, w):
    """Algorithmic FLOPs of the prefill attention: 4 D per (query token, head,
    attended key), the attended keys being the valid tokens of the query
    block's chosen blocks up to the query itself (counted from the selection
    the input actually produces)."""
    import torch
    idx, n_sel = run.selection()
    bs, G = w.block_size, w.group
    L = run.data["seqlens"].long()
    total = 0
    for b in range(w.batch):
        Lb = int(L[b])
        nb = -(-Lb // bs)
        sel = idx[b, :, :nb].long()                       # [Hkv][nb][k_max]
        live = torch.arange(sel.shape[-1], device=sel.device)[None, None] < n_sel[b, :, :nb, None]
        qi = torch.arange(nb, device=sel.device)[None, :, None]
        # full earlier blocks: every query token of block i sees all their valid keys
        start = sel.clamp(min=0) * bs
        valid = (Lb - start).clamp(min=0, max=bs)
        q_in = (Lb - qi * bs).clamp(min=0, max=bs)          # query tokens in block i
        earlier = (live & (sel < qi)) * valid * q_in
        # the diagonal block: token u of the block sees u + 1 keys
        diag = (live & (sel == qi)) * (q_in * (q_in + 1) // 2)
        total += int((earlier + diag).sum().item())
    return 4 * w.head_dim * G * total


def prefill_cpu_baseline(w, data, q, args):
    """The fp64 oracle's prefill (pooled keys, pooled-query gate, per-block
    selection, causal block-sparse attention) timed on (b, h) rows of the
    same inputs until the CPU budget runs out, scaled to the whole batch."""
    import random
    import numpy as np
    from block_sparse_attention_step_b200 import workloads as W
    from oracle import seer_oracle as O
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        threads = 1
    rows = [(b, h) for b in range(w.batch) for h in range(w.kv_heads)]
    random.Random(0).shuffle(rows)
    G, bs = w.group, w.block_size
    scale = 1.0 / math.sqrt(w.head_dim)
    if w.budget_tokens:
        k_of = lambda i: O.k_from_budget(i + 1, w.budget_tokens, bs)
    else:
        k_of = lambda i: O.k_from_sparsity(i + 1, w.sparsity_permille)
    spent, done = 0.0, 0
    for (b, h) in rows:
        L = int(data["seqlens"][b])
        Qg = q[b, :L, h * G:(h + 1) * G].double().cpu().numpy()
        Wg = data["w_gate"][h].double().cpu().numpy()
        K = W.gather_rows(data["k_pool"], data["page_table"], b, h, L, bs).double().numpy()
        V = W.gather_rows(data["v_pool"], data["page_table"], b, h, L, bs).double().numpy()
        t0 = time.perf_counter()
        O.prefill_row(Qg, Wg, K, V, L, bs, k_of, scale, scale)
        spent += time.perf_counter() - t0
        done += 1
        if spent >= args.cpu_budget:
            break
    sec_row = spent / max(done, 1)
    tokens = int(data["seqlens"].sum())
    return {"value": tokens / (sec_row * len(rows)), "unit": "tokens/s", "cores": threads,
            "kind": "oracle",
            "sample": f"{done} of {len(rows)} (b, kv-head) rows of this prompt batch, fp64 numpy "
                      f"oracle prefill (pooled keys, pooled-query gate, selection, causal "
                      f"attention), {sec_row:.1f} s/row, scaled to the whole batch"}


def run_prefill(args):
    """Prefill with query pooling on the headline shapes at batch 2 and a
    16K-token prompt: one JSON line (prompt tokens/s, tensor roofline)."""
    import torch
    from block_sparse_attention_step_b200 import workloads as W
    from block_sparse_attention_step_b200.runner import PrefillBuffers
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    w = W.WORKLOADS[W.HEADLINE].replace(batch=2, seqlen=16384)
    if args.sparsity is not None:
        w = w.replace(sparsity_permille=args.sparsity)
    runs = []
    for r in range(2):
        data = W.generate(w, args.seed + r, dev)
        q = W.prefill_queries(w, args.seed + r, data["nb_max"], dev)
        pr = PrefillBuffers(w, data, q)
        pr.run(pool_keys=True)
        runs.append(pr)
    torch.cuda.synchronize()
    flops = prefill_flops(runs[0], w)
    stream = torch.cuda.current_stream(dev)
    clocks = ClockSampler(0)

    def timed(pool):
        for i in range(args.warmup):
            runs[i % 2].run(pool_keys=pool)
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for i in range(args.steps):
            runs[i % 2].run(pool_keys=pool)
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / args.steps

    ms_full = timed(True)
    ms_attn_gate = timed(False)
    clock_info = clocks.stop()
    peaks, kind = measured_peaks()
    tflops = flops / (ms_attn_gate * 1e-3) / 1e12
    line = {
        "metric": "prefill prompt tokens/s (query-pooled block gate + causal block-sparse attention)",
        "value": w.batch * w.seqlen / (ms_full * 1e-3), "unit": "tokens/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_full,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded)",
        "config": {"workload": f"prefill_b{w.batch}_h{w.q_heads}_L{w.seqlen}_bs{w.block_size}_"
                               f"s{w.sparsity_permille // 10}", "batch": w.batch,
                   "seq_len": w.seqlen, "q_heads": w.q_heads, "kv_heads": w.kv_heads,
                   "block_size": w.block_size, "sparsity_permille": w.sparsity_permille,
                   "step": "seer_prefill with the full key pooling"},
        "stage_ms": {"prefill_with_pooling": ms_full, "gate_select_attention": ms_attn_gate},
        "roofline": {"bound": "tensor", "achieved": tflops, "peak": peaks["bf16_tflops"],
                     "unit": "TFLOP/s", "frac": tflops / peaks["bf16_tflops"], "traffic": None,
                     "kernel": "prefill gate+select and attention (algorithmic attention FLOPs "
                               "over both launches)", "flops_per_step": flops,
                     "peak_source": f"{kind} bf16_tflops (burst)"},
        "gpu_launches": 3 * args.steps,
        "clocks": clock_info,
        "device_status": [int(r.status.item()) for r in runs],
    }
    if not args.no_cpu_baseline:
        line["cpu_baseline"] = prefill_cpu_baseline(w, runs[0].data, runs[0].q, args)
    print(json.dumps(line), flush=True)
    return 0


def max_over_ranks(ms: float, device) -> float:
    """The slowest rank's time: every rank contributes its own elapsed time
    and all receive the maximum (the job is as fast as its slowest replica)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(ms)], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(world: int, batch: int, ms_step: float) -> float:
    """Whole-job decode throughput: every rank decodes `batch` sequences per
    step (weak scaling, one replica per GPU), at the slowest rank's pace."""
    return world * batch / (ms_step * 1e-3)


def selected_bytes(run, data, w):
    """Bytes of K and V the selection makes the decode kernel read (valid
    tokens of the selected blocks x D x 2 bytes x 2 tensors), from the
    selection this input actually produces."""
    import torch
    run.step(update_kbar=0)
    torch.cuda.synchronize()
    v = run.workspace_views()
    idx = v["idx"].long()
    n = v["n_sel"].long()
    L = data["seqlens"].long()
    bs = w.block_size
    pos = torch.arange(idx.shape[-1], device=idx.device)
    live = pos[None, None, :] < n[:, :, None]
    start = idx.clamp(min=0) * bs
    valid = (L[:, None, None] - start).clamp(min=0, max=bs) * live
    tokens = int(valid.sum().item())
    return tokens * w.head_dim * 2 * 2, tokens


def decode_bytes(run, sel_bytes, w):
    """Algorithmic bytes of one decode launch: selected K/V, q, the index
    rows, and the split partials written."""
    B, Hq, Hkv, S, D = w.batch, w.q_heads, w.kv_heads, run.num_splits, w.head_dim
    return (sel_bytes + B * Hq * D * 2 + B * Hkv * (run.k_max + 1) * 4 + B * Hq * S * (D + 1) * 4)


def step_percentiles(one_step, n, stream):
    """p10 / p50 / p90 of single-step device times, each step between its own
    pair of CUDA events (taken after the timed region; the pairs add a little
    per-step overhead, so p50 sits slightly above the timed mean)."""
    import torch
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(n)]
    for i, (a, b) in enumerate(evs):
        a.record(stream)
        one_step(i)
        b.record(stream)
    torch.cuda.synchronize()
    t = sorted(a.elapsed_time(b) * 1e3 for a, b in evs)
    pick = lambda f: t[min(len(t) - 1, int(f * len(t)))]
    return {"p10": pick(0.10), "p50": pick(0.50), "p90": pick(0.90), "n": n}


def standalone_stages(runs, n, stream, replicas):
    """Mean device time of each stage through its own C-ABI entry point
    (incremental pooling, gate scores, block select, combine), n launches each
    over the rotating replicas.  The step fuses pooling, gate and select into
    one kernel and chains the rest, so these do not add up to the step."""
    import torch
    from block_sparse_attention_step_b200 import seer
    views = [r.workspace_views() for r in runs]

    def timed(launch):
        for i in range(3):
            launch(i)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for i in range(n):
            launch(i)
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / n * 1e3

    def pool(i):
        r = runs[i % replicas]
        seer.seer_pool_keys(r.dims, r.data["k_pool"], r.page_table, r.data["seqlens"], 1, r.kbar,
                            r.status, stream)

    def gate(i):
        r, v = runs[i % replicas], views[i % replicas]
        seer.seer_gate_scores(r.dims, r.data["q"], r.data["w_gate"], r.kbar, r.data["seqlens"],
                              r.scale, v["scores"], r.status, stream)

    def select(i):
        r, v = runs[i % replicas], views[i % replicas]
        seer.seer_block_select(r.dims, v["scores"], r.data["seqlens"], r.k_per_seq,
                               r.force_newest, r.k_max, v["idx"], v["n_sel"], r.status, stream)

    def combine(i):
        r, v = runs[i % replicas], views[i % replicas]
        seer.seer_combine(r.dims, v["o_part"], v["lse_part"], r.num_splits, r.out, r.lse, stream)

    return {"pool_keys_incremental": timed(pool), "gate_scores": timed(gate),
            "block_select": timed(select), "combine": timed(combine)}


def decode_alone(runs, steps, stream, replicas):
    """Mean duration of the dominant kernel, sparse decode, launched alone K
    times over the rotating replicas (each replica's index rows are those its
    last step selected), CUDA events on the launching stream."""
    import torch
    from block_sparse_attention_step_b200 import seer
    views = [r.workspace_views() for r in runs]
    # the item counter the step uses too (zeroed once; each launch leaves it zero)
    counter = torch.zeros(2, dtype=torch.int32, device=runs[0].out.device)

    def launch(i):
        r, v = runs[i % replicas], views[i % replicas]
        d = r.data
        if r.block_lse is not None:
            seer.seer_sparse_decode_mass(r.dims, d["q"], d["k_pool"], d["v_pool"], r.page_table,
                                         d["seqlens"], v["idx"], v["n_sel"], r.k_max,
                                         r.num_splits, r.scale, v["o_part"], v["lse_part"],
                                         r.block_lse, r.status, stream, work_counter=counter)
        else:
            seer.seer_sparse_decode(r.dims, d["q"], d["k_pool"], d["v_pool"], r.page_table,
                                    d["seqlens"], v["idx"], v["n_sel"], r.k_max, r.num_splits,
                                    r.scale, v["o_part"], v["lse_part"], r.status, stream,
                                    work_counter=counter)
    for i in range(3):
        launch(i)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for i in range(steps):
        launch(i)
    b.record(stream)
    torch.cuda.synchronize()
    return a.elapsed_time(b) / steps * 1e3


def end_to_end(runs, steps, stream, replicas, w):
    import torch
    from block_sparse_attention_step_b200 import seer
    q_host = [r.data["q"].cpu().pin_memory() for r in runs]
    out_host = [torch.empty(r.out.shape, dtype=torch.bfloat16).pin_memory() for r in runs]
    q_dev = [torch.empty_like(r.data["q"]) for r in runs]
    args = [r.args(update_kbar=1, q=q_dev[i]) for i, r in enumerate(runs)]
    for i in range(3):
        seer.seer_decode_step_host(runs[i % replicas].dims, args[i % replicas], q_host[i % replicas],
                                   q_dev[i % replicas], out_host[i % replicas], stream)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for i in range(steps):
        k = i % replicas
        seer.seer_decode_step_host(runs[k].dims, args[k], q_host[k], q_dev[k], out_host[k], stream)
    b.record(stream)
    torch.cuda.synchronize()
    wall = time.perf_counter() - t0
    ms = a.elapsed_time(b) / steps
    qbytes = runs[0].data["q"].numel() * 2
    mapped = seer.seer_host_ptr_mapped(q_host[0]) and seer.seer_host_ptr_mapped(out_host[0])
    how = ("q read from pinned host memory by the gate kernel, out written to pinned host "
           "memory by the combine kernel (zero-copy, both over PCIe inside the step)"
           if mapped else "pinned q H2D copy, step, out D2H copy")
    return {"value": w.batch / (ms * 1e-3), "unit": UNIT, "h2d_bytes_per_step": qbytes,
            "d2h_bytes_per_step": runs[0].out.numel() * 2, "ms_per_step": ms,
            "host_wall_ms_per_step": wall / steps * 1e3,
            "path": f"seer_decode_step_host: {how}; device-timed"}


def cpu_baseline(w, run, args):
    rows = [(b, h) for b in range(w.batch) for h in range(w.kv_heads)]
    import random
    random.Random(0).shuffle(rows)
    k = run.k_per_seq.cpu().tolist()
    sec_row, n, threads = oracle_rows_timed(w, run.data, rows, args.cpu_budget, k, run.force_newest)
    step_s = sec_row * len(rows)
    out = {"value": w.batch / step_s, "unit": UNIT, "cores": threads, "kind": "oracle",
           "sample": f"{n} of {len(rows)} (b, kv-head) rows of this workload, fp64 numpy oracle "
                     f"(pool, gate, select, masked attention), {sec_row * 1e3:.1f} ms/row, scaled "
                     f"to the whole batch"}
    try:  # the same oracle held to one BLAS thread, on a shorter sample
        from threadpoolctl import threadpool_limits
        with threadpool_limits(limits=1):
            sec1, n1, _ = oracle_rows_timed(w, run.data, rows, args.cpu_budget / 3, k,
                                            run.force_newest)
        out["value_1core"] = w.batch / (sec1 * len(rows))
        out["sample_1core"] = f"{n1} rows, one BLAS thread, {sec1 * 1e3:.1f} ms/row"
    except ImportError:
        pass
    return out


def main(argv=None):
    p = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=2000)
    p.add_argument("--warmup", type=int, default=50)
    p.add_argument("--impl", choices=("ours", "reference"), default="ours")
    from block_sparse_attention_step_b200 import workloads as W
    p.add_argument("--workload", choices=sorted(W.WORKLOADS), default=W.HEADLINE)
    p.add_argument("--sparsity", type=int, default=None, help="override: sparsity in permille")
    p.add_argument("--splits", type=int, default=None)
    p.add_argument("--layout", choices=("nhd", "hnd"), default="nhd",
                   help="KV pool page layout: token-major [P][bs][Hkv][D] or head-major [P][Hkv][bs][D]")
    p.add_argument("--seed", type=int, default=1)
    p.add_argument("--max-replicas", type=int, default=8)
    p.add_argument("--cpu-budget", type=float, default=15.0, help="seconds of oracle time")
    p.add_argument("--ref-rows", type=int, default=4, help="oracle rows per reference step")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-graph", action="store_true", help="launch each step directly, no CUDA graph")
    p.add_argument("--mass", action="store_true",
                   help="also emit every block's attention mass (dense-mode gate target)")
    p.add_argument("--recall", action="store_true",
                   help="also report the gate recall (dense attention mass kept by the selection)")
    p.add_argument("--unified", action="store_true",
                   help="one block set per sequence shared by all KV heads (cross-head ranking)")
    p.add_argument("--fused", action="store_true",
                   help="the whole step as one cooperative launch (seer_decode_step_fused)")
    p.add_argument("--prefill", action="store_true",
                   help="measure the prefill path with query pooling instead of the decode step")
    args = p.parse_args(argv)
    if args.warmup < 3:
        p.error("--warmup must be at least 3")
    if args.impl == "reference":
        return run_reference(args)
    if args.prefill:
        return run_prefill(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
