"""Benchmark of the block-sparse decode step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...      # the fp64 CPU oracle, timed alone

One step = one pass of the whole hot path over one batch: incremental pooled-
key update of the newest block, gate scores, top-k block selection, split-KV
sparse decode and LSE combine (one ``seer_decode_step`` call: the fused
pool+gate+select kernel, the decode kernel and the combine kernel, chained by
programmatic dependent launch; the timed steps are replayed as CUDA graphs of
one whole rotation of the replicas each, so consecutive steps chain too).
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
    """SM clock, power and clock-event reasons sampled every 50 ms while the
    measurements run, through read-only NVML queries in a thread (nothing is
    set).  Falls back to ``nvidia-smi -lms 50 -f <file>`` (the tool writes
    each sample to the file itself, so nothing is lost when it is stopped)."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
    LOADED_W = 200.0    # power draw above which a sample counts as "under load"

    def __init__(self, device_index, period_s=0.05):
        import threading
        self.samples = []          # (sm_mhz, sm_max_mhz, power_w, frozenset(reasons))
        self.source = None
        self.proc = self.path = None
        self._stop = threading.Event()
        self._thread = None
        uuid = None
        try:
            import torch
            u = str(torch.cuda.get_device_properties(device_index).uuid)
            uuid = u if u.startswith("GPU-") else f"GPU-{u}"
        except Exception:
            pass
        try:
            import pynvml as nv
            nv.nvmlInit()
            h = (nv.nvmlDeviceGetHandleByUUID(uuid) if uuid else
                 nv.nvmlDeviceGetHandleByIndex(int(device_index)))
            smax = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
            bits = {"hw_slowdown": nv.nvmlClocksEventReasonHwSlowdown,
                    "hw_thermal_slowdown": nv.nvmlClocksEventReasonHwThermalSlowdown,
                    "sw_thermal_slowdown": nv.nvmlClocksEventReasonSwThermalSlowdown,
                    "sw_power_cap": nv.nvmlClocksEventReasonSwPowerCap}

            def loop():
                while not self._stop.is_set():
                    try:
                        sm = float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
                        pw = nv.nvmlDeviceGetPowerUsage(h) / 1000.0
                        r = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                        self.samples.append((sm, smax, pw,
                                             frozenset(k for k, b in bits.items() if r & b)))
                    except Exception:
                        pass
                    self._stop.wait(period_s)
            self._thread = threading.Thread(target=loop, daemon=True)
            self._thread.start()
            self.source = "nvml"
            return
        except Exception:
            pass
        try:
            import tempfile
            fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", str(int(period_s * 1000)), "-i", uuid or str(device_index),
                 "-f", self.path], stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
            self.source = "nvidia-smi"
        except OSError:
            self.proc = None

    def _read_smi_file(self):
        try:
            text = open(self.path).read()
        except OSError:
            return
        for line in text.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm, m, pw = float(parts[1]), float(parts[2]), float(parts[3])
            except ValueError:
                continue
            self.samples.append((sm, m, pw, frozenset(
                n for n, v in zip(self.NAMES, parts[5:9]) if v.lower() == "active")))

    def stop(self):
        if self._thread is not None:
            self._stop.set()
            self._thread.join(timeout=2)
        elif self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.proc.wait()
            self._read_smi_file()
            try:
                os.unlink(self.path)
            except OSError:
                pass
        else:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no clock source"],
                    "samples": 0}
        return self.summary(self.samples, self.source)

    @classmethod
    def summary(cls, samples, source):
        sm = [s[0] for s in samples]
        loaded = [s[0] for s in samples if s[2] > cls.LOADED_W]
        reasons = set()
        for s in samples:
            reasons |= s[3]
        use = loaded or sm
        return {"sm_mhz": statistics.median(use) if use else None,
                "sm_max_mhz": max(s[1] for s in samples) if samples else None,
                "reasons": sorted(reasons), "samples": len(sm),
                "samples_under_load": len(loaded),
                "power_w_max": max((s[2] for s in samples), default=None),
                "source": source}


# ------------------------------------------------------------------ CPU oracle
#
# The oracle is timed in parallel over the host cores: one spawned process
# per core, each held to one BLAS thread, each owning a share of the (b, h)
# rows balanced by sequence length.  A row's inputs reach its process once,
# as raw bf16 bits (q, K, V) and fp32 (W), before any timing; a timed pass
# then runs the oracle's whole step on every row -- the exact bf16 -> fp64
# conversion, pooled keys, gate scores, selection and masked attention (or
# the prefill path) -- and the pass's wall time is the slowest process's.


def _oracle_run_row(O, np, r):
    """The oracle's step on one row from its raw inputs (timed part)."""
    q = O.bf16_bits_to_f64(r["q"])
    Wg = np.asarray(r["W"], dtype=np.float64)
    K = O.bf16_bits_to_f64(r["K"])
    V = O.bf16_bits_to_f64(r["V"])
    if r["kind"] == "decode":
        return O.decode_row(q, Wg, K, V, r["L"], r["bs"], r["k"], r["force"], r["scale"],
                            r["scale"])
    bs = r["bs"]
    if r["budget"]:
        k_of = lambda i: O.k_from_budget(i + 1, r["budget"], bs)
    else:
        k_of = lambda i: O.k_from_sparsity(i + 1, r["permille"])
    return O.prefill_row(q, Wg, K, V, r["L"], bs, k_of, r["scale"], r["scale"])


def _oracle_worker(conn):
    """One host core's share of the oracle step (a spawned process).  Its
    BLAS is held to one thread: the variables are read when numpy loads its
    BLAS, which happens here, after they are set."""
    for var in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS",
                "BLIS_NUM_THREADS", "NUMEXPR_NUM_THREADS"):
        os.environ[var] = "1"
    import numpy as np
    try:
        from threadpoolctl import threadpool_limits
        threadpool_limits(1)
    except ImportError:
        pass
    from oracle import seer_oracle as O
    rows = conn.recv()
    while True:
        cmd = conn.recv()
        if cmd == "run":
            t0 = time.perf_counter()
            for r in rows:
                _oracle_run_row(O, np, r)
            conn.send(time.perf_counter() - t0)
        elif cmd == "results":
            conn.send([_oracle_run_row(O, np, r) for r in rows])
        else:
            break
    conn.close()


def host_cpu_info():
    model = None
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                model = line.split(":", 1)[1].strip()
                break
    except OSError:
        pass
    try:
        usable = len(os.sched_getaffinity(0))
    except AttributeError:
        usable = os.cpu_count() or 1
    return {"nproc": os.cpu_count(), "usable_cores": usable, "cpu_model": model}


class OraclePool:
    """Spawned oracle processes (spawn, so that none inherits a CUDA
    context), each with its share of rows; ``step()`` times one parallel pass
    over all of them."""

    def __init__(self, workers: int):
        import multiprocessing as mp
        ctx = mp.get_context("spawn")
        self.conns, self.procs = [], []
        for _ in range(max(1, int(workers))):
            a, b = ctx.Pipe()
            proc = ctx.Process(target=_oracle_worker, args=(b,), daemon=True)
            proc.start()
            self.conns.append(a)
            self.procs.append(proc)
        self.order = []

    def load(self, rows, cost):
        """Deal the rows out, longest first, each to the least-loaded process."""
        n = len(self.conns)
        load = [0.0] * n
        share = [[] for _ in range(n)]
        self.order = [[] for _ in range(n)]
        for i in sorted(range(len(rows)), key=lambda i: -cost[i]):
            j = min(range(n), key=lambda j: load[j])
            load[j] += cost[i]
            share[j].append(rows[i])
            self.order[j].append(i)
        for c, part in zip(self.conns, share):
            c.send(part)

    def step(self) -> float:
        t0 = time.perf_counter()
        for c in self.conns:
            c.send("run")
        for c in self.conns:
            c.recv()
        return time.perf_counter() - t0

    def results(self):
        """The oracle's outputs per row, in the order the rows were loaded."""
        for c in self.conns:
            c.send("results")
        out = {}
        for c, idx in zip(self.conns, self.order):
            for i, r in zip(idx, c.recv()):
                out[i] = r
        return [out[i] for i in range(len(out))]

    def close(self):
        for c in self.conns:
            try:
                c.send("stop")
            except (OSError, BrokenPipeError):
                pass
        for proc in self.procs:
            proc.join(timeout=10)
            if proc.is_alive():
                proc.kill()


def _bits(t):
    import torch
    return t.contiguous().view(torch.int16).cpu().numpy().view("uint16")


def oracle_decode_rows(w, data, rows, k_per_seq, force_newest):
    """Raw per-row inputs of the oracle's decode step (host copies, not timed)."""
    from block_sparse_attention_step_b200 import workloads as W
    G, bs = w.group, w.block_size
    layout = data.get("layout", "nhd")
    q = _bits(data["q"])
    wg = data["w_gate"].cpu().numpy()
    L_all = data["seqlens"].cpu().tolist()
    out = []
    for (b, h) in rows:
        L = int(L_all[b])
        out.append({"kind": "decode", "q": q[b, h * G:(h + 1) * G], "W": wg[h],
                    "K": _bits(W.gather_rows(data["k_pool"], data["page_table"], b, h, L, bs,
                                             layout)),
                    "V": _bits(W.gather_rows(data["v_pool"], data["page_table"], b, h, L, bs,
                                             layout)),
                    "L": L, "bs": bs, "k": int(k_per_seq[b]), "force": bool(force_newest),
                    "scale": 1.0 / math.sqrt(w.head_dim)})
    return out


def pick_rows(w, seqlens, max_bytes):
    """Every (b, h) row when their inputs fit in ``max_bytes`` of host
    copies, else the longest-first sample of rows that does (each row ships
    its K and V, L x D x 2 bytes each)."""
    rows = [(b, h) for b in range(w.batch) for h in range(w.kv_heads)]
    per = lambda r: 4 * w.head_dim * int(seqlens[r[0]])
    if sum(per(r) for r in rows) <= max_bytes:
        return rows, False
    import random
    rng = random.Random(0)
    rng.shuffle(rows)
    pick, total = [], 0
    for r in rows:
        if total + per(r) > max_bytes and pick:
            continue
        pick.append(r)
        total += per(r)
    return sorted(pick), True


def oracle_parallel_timing(w, data, k_per_seq, force_newest, rows, workers, steps,
                           warmup=1, budget_s=None):
    """Mean wall time of one parallel oracle pass over ``rows`` (after
    ``warmup`` passes), with the pool's processes and the rows' lengths."""
    seqlens = data["seqlens"].cpu().tolist()
    inputs = oracle_decode_rows(w, data, rows, k_per_seq, force_newest)
    pool = OraclePool(min(workers, len(rows)))
    try:
        pool.load(inputs, [float(seqlens[b]) for (b, _) in rows])
        del inputs
        for _ in range(warmup):
            pool.step()
        times = []
        spent = 0.0
        for _ in range(steps):
            t = pool.step()
            times.append(t)
            spent += t
            if budget_s is not None and spent >= budget_s and len(times) >= 1:
                break
        return times, len(pool.conns)
    finally:
        pool.close()


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


def row_share(w, seqlens, rows):
    """The whole batch's oracle work over the sample's: by row count for
    fixed lengths, by total length (the oracle's cost grows with L) for a
    ragged batch."""
    all_l = sum(int(seqlens[b]) for b in range(w.batch)) * w.kv_heads
    got = sum(int(seqlens[b]) for (b, _) in rows)
    return all_l / max(got, 1)


def run_reference(args):
    """The oracle alone on the host cores, on the same workload draw and the
    same rows as the CPU baseline of the GPU arm: each step is one parallel
    pass of the oracle's whole step over every (b, h) row of the batch (a
    longest-first sample of rows for batches whose inputs exceed the host
    copy budget, scaled by total length and marked as extrapolated)."""
    if int(os.environ.get("RANK", "0")) != 0:
        return 0
    import torch
    from block_sparse_attention_step_b200 import workloads as W
    w = resolve_workload(args)
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    data = W.generate(w, args.seed if args.seed is not None else w.seed, dev)
    seqlens = data["seqlens"].cpu().tolist()
    kps = cpu_k_per_seq(w, seqlens)
    rows, sampled = pick_rows(w, seqlens, args.cpu_max_bytes)
    info = host_cpu_info()
    workers = info["usable_cores"]
    inputs = oracle_decode_rows(w, data, rows, kps, w.force_newest)
    pool = OraclePool(min(workers, len(rows)))
    try:
        pool.load(inputs, [float(seqlens[b]) for (b, _) in rows])
        del inputs
        # the selection the oracle makes (for the config's byte count), untimed
        res = pool.results()
        for _ in range(args.warmup):
            pool.step()
        times = [pool.step() for _ in range(args.steps)]
        used = len(pool.conns)
    finally:
        pool.close()
    scale = row_share(w, seqlens, rows)
    step_s = statistics.mean(times) * scale
    value = w.batch / step_s
    sel_tokens = 0
    for (b, _), r in zip(rows, res):
        L = int(seqlens[b])
        sel_tokens += sum(min(w.block_size, L - int(j) * w.block_size) for j in r["indices"])
    sel_bytes = int(round(sel_tokens * scale)) * w.head_dim * 4
    kbar_bytes = w.batch * w.kv_heads * data["nb_max"] * w.head_dim * 4
    k_max = max(1, min(max(kps), data["nb_max"]))
    cfg = workload_config(w, reference_splits(w, data, k_max), k_max,
                          replica_count(sel_bytes + kbar_bytes, dev, args.max_replicas),
                          args.layout, args)
    sample = (f"{'a longest-first sample of ' if sampled else 'all '}{len(rows)} (b, kv-head) "
              f"rows of this workload draw (seed {args.seed if args.seed is not None else w.seed})"
              f" per step, fp64 numpy oracle (bf16->f64, pool, gate, select, masked attention), "
              f"{used} spawned processes with one BLAS thread each"
              + (f", scaled x{scale:.2f} by total length to the whole batch" if sampled else ""))
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_s * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded; random-init gate projection)", "config": cfg,
        "extrapolated": bool(sampled), "rows_per_step": len(rows),
        "cpu_baseline": dict({"value": value, "unit": UNIT, "cores": used, "kind": "oracle",
                              "sample": sample}, **info),
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def resolve_workload(args):
    from block_sparse_attention_step_b200 import workloads as W
    w = W.WORKLOADS[args.workload]
    if args.sparsity is not None:
        w = w.replace(sparsity_permille=args.sparsity, budget_tokens=None)
    if args.batch is not None:   # a smaller case of the same workload (profiler captures)
        w = w.replace(batch=args.batch)
    return w


def replica_count(touched, dev, max_replicas):
    """Replicas whose rotation reads more than 4x the L2 (at least 2)."""
    l2 = 126 * 1024 * 1024
    if str(dev).startswith("cuda"):
        import torch
        l2 = torch.cuda.get_device_properties(torch.device(dev)).L2_cache_size
    return min(max(2, math.ceil(4 * l2 / max(touched, 1))), max_replicas), touched


def reference_splits(w, data, k_max):
    """The split count the GPU arm launches with on this workload (a host
    helper of the library: no device work), so both lines name one config."""
    if w.num_splits:
        return w.num_splits
    from block_sparse_attention_step_b200 import seer
    d = seer.make_dims(w.batch, w.q_heads, w.kv_heads, w.head_dim, w.block_size,
                       data["nb_max"], data["num_pages"])
    return seer.seer_default_splits(d, k_max, 0)


def workload_config(w, num_splits, k_max, rep, layout, args):
    """The config object both arms print (the same keys and values for the
    same workload, split count and selection size)."""
    replicas, touched = rep
    rotation = replicas * touched
    l2_bytes = 126 * 1024 * 1024
    if rotation > 4 * l2_bytes:
        l2 = (f"inputs larger than L2: {replicas} rotating replicas, "
              f"{touched / 1e6:.0f} MB read per step, L2 126 MB")
    elif rotation > l2_bytes:
        l2 = (f"partly L2-resident: {replicas} rotating replicas, {touched / 1e6:.0f} MB read "
              f"per step, the rotation is less than 4x the 126 MB L2")
    else:
        l2 = (f"L2-hot: {replicas} replica(s), {touched / 1e6:.0f} MB read per step, the "
              f"rotation fits in the 126 MB L2")
    cfg = {"workload": w.name, "batch": w.batch, "q_heads": w.q_heads, "kv_heads": w.kv_heads,
           "head_dim": w.head_dim, "block_size": w.block_size,
           "seq_len": w.seqlen if w.seqlen else f"U[{w.seqlen_range[0]},{w.seqlen_range[1]}]",
           "selection": (f"budget {w.budget_tokens} tokens" if w.budget_tokens
                         else f"sparsity {w.sparsity_permille / 10:g}%"),
           "force_newest": w.force_newest, "paged": w.paged, "kv_layout": layout,
           "num_splits": int(num_splits), "k_max": int(k_max),
           "l2": l2,
           "block_mass": bool(args.mass),
           "selection_scope": ("one block set per sequence (all KV heads)" if args.unified
                               else "per KV head"),
           "step_launch": ("single cooperative launch" if args.fused
                           else "per stage, PDL-chained"),
           "timed_launches": ("direct C-ABI calls" if args.no_graph
                              else "one CUDA graph per step" if args.graph_per_step
                              else "one CUDA graph per rotation of the replicas (PDL between "
                                   "steps inside it)")}
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
    w = resolve_workload(args)
    seed0 = (args.seed if args.seed is not None else w.seed) + 1000 * rank

    # replicas: enough that one rotation reads > 4x L2
    probe = W.generate(w, seed0, dev, layout=args.layout)
    run0 = StepBuffers(w, probe, num_splits=args.splits, mass=args.mass, unified=args.unified)
    run0.pool_full()
    torch.cuda.synchronize()
    sel_bytes, sel_tokens = selected_bytes(run0, probe, w)
    kbar_bytes = run0.kbar.numel() * 4
    touched = sel_bytes + kbar_bytes
    rep = replica_count(touched, dev, args.max_replicas)
    replicas = rep[0]
    runs = [run0]
    for r in range(1, replicas):
        d = W.generate(w, seed0 + r, dev, layout=args.layout)
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

    # CUDA graphs keep host launch cost out of the device time: one graph per
    # replica holding its step (single steps: warm-up and the per-step
    # spread), and one graph holding a whole rotation, the replicas' steps one
    # after another, so that inside it every step's first kernel is chained to
    # the previous step's last by programmatic dependent launch just as on a
    # stream (between two graph launches it is not).  --no-graph launches the
    # C-ABI call directly; --graph-per-step replays the per-replica graphs only.
    graphs, rotation = [], None
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
        if not args.graph_per_step:
            rotation = torch.cuda.CUDAGraph()
            with torch.cuda.graph(rotation):
                for i in range(replicas):
                    step_call(runs[i].dims, step_args[i], torch.cuda.current_stream())
        torch.cuda.synchronize()

    def one_step(i):
        if graphs:
            graphs[i % replicas].replay()
        else:
            step_call(runs[i % replicas].dims, step_args[i % replicas], stream)

    def steps_from_zero(k):
        """Exactly k steps, replicas in turn from replica 0."""
        i = 0
        if rotation is not None:
            for _ in range(k // replicas):
                rotation.replay()
            i = k - k % replicas
        for j in range(i, k):
            one_step(j)

    clocks = ClockSampler(local) if rank == 0 else None
    for i in range(args.warmup):
        one_step(i)
    torch.cuda.synchronize()

    # ---- timed region: exactly K steps
    barrier()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    steps_from_zero(args.steps)
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
        "config": workload_config(w, run0.num_splits, run0.k_max, rep, args.layout, args),
        "selected_kv_bytes_per_step": sel_bytes,
        "selected_tokens_per_step": sel_tokens,
        "step_hbm_gbs": (touched / (ms_step * 1e-3)) / 1e9,
        "selected_kv_gbs": (sel_bytes / (ms_step * 1e-3)) / 1e9,
        "stage_us": {"step": ms_step * 1e3, "sparse_decode_alone": dec_us,
                     "rest_of_step": ms_step * 1e3 - dec_us, "standalone": stages},
        "step_us_percentiles": pct,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"],
                     "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"],
                     # the records are taken on each workload's own selection and batch
                     "traffic": (recorded_traffic(w.name)
                                 if args.sparsity is None and args.batch is None else None),
                     "kernel": "sparse_decode_kernel",
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
        line["cpu_baseline"] = cpu_baseline(w, runs[0].data, args, seed0)
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
    selection, causal block-sparse attention) on every (b, h) row of the
    prompt batch, one spawned process per usable core with one BLAS thread
    each, one timed parallel pass."""
    from block_sparse_attention_step_b200 import workloads as W
    rows = [(b, h) for b in range(w.batch) for h in range(w.kv_heads)]
    G, bs = w.group, w.block_size
    info = host_cpu_info()
    seqlens = data["seqlens"].cpu().tolist()
    wg = data["w_gate"].cpu().numpy()
    inputs = []
    for (b, h) in rows:
        L = int(seqlens[b])
        inputs.append({"kind": "prefill", "q": _bits(q[b, :L, h * G:(h + 1) * G]), "W": wg[h],
                       "K": _bits(W.gather_rows(data["k_pool"], data["page_table"], b, h, L, bs)),
                       "V": _bits(W.gather_rows(data["v_pool"], data["page_table"], b, h, L, bs)),
                       "L": L, "bs": bs, "budget": w.budget_tokens or 0,
                       "permille": w.sparsity_permille or 0,
                       "scale": 1.0 / math.sqrt(w.head_dim)})
    pool = OraclePool(min(info["usable_cores"], len(rows)))
    try:
        pool.load(inputs, [float(seqlens[b]) for (b, _) in rows])
        del inputs
        t = pool.step()
        used = len(pool.conns)
    finally:
        pool.close()
    tokens = int(sum(seqlens))
    return dict({"value": tokens / t, "unit": "tokens/s", "cores": used, "kind": "oracle",
                 "sample": f"all {len(rows)} (b, kv-head) rows of this prompt batch in one "
                           f"parallel pass ({t:.1f} s), fp64 numpy oracle prefill (pooled keys, "
                           f"pooled-query gate, selection, causal attention), {used} spawned "
                           f"processes with one BLAS thread each"}, **info)


def run_prefill(args):
    """Prefill with query pooling on the headline shapes at batch 2 and a
    16K-token prompt: one JSON line (prompt tokens/s, tensor roofline)."""
    import torch
    from block_sparse_attention_step_b200 import workloads as W
    from block_sparse_attention_step_b200.runner import PrefillBuffers
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    w = W.WORKLOADS[W.HEADLINE].replace(batch=args.prefill_batch, seqlen=args.prefill_seqlen)
    if args.sparsity is not None:
        w = w.replace(sparsity_permille=args.sparsity)
    runs = []
    for r in range(2):
        seed = (args.seed if args.seed is not None else w.seed) + r
        data = W.generate(w, seed, dev)
        q = W.prefill_queries(w, seed, data["nb_max"], dev)
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
    # the dominant kernel alone: the attention over the selection in place
    for i in range(args.warmup):
        runs[i % 2].attention()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for i in range(args.steps):
        runs[i % 2].attention()
    b.record(stream)
    torch.cuda.synchronize()
    ms_attn = a.elapsed_time(b) / args.steps
    clock_info = clocks.stop()
    peaks, kind = measured_peaks()
    tflops = flops / (ms_attn * 1e-3) / 1e12
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
        "stage_ms": {"prefill_with_pooling": ms_full, "gate_select_attention": ms_attn_gate,
                     "attention_alone": ms_attn},
        "roofline": {"bound": "tensor", "achieved": tflops, "peak": peaks["bf16_tflops"],
                     "unit": "TFLOP/s", "frac": tflops / peaks["bf16_tflops"], "traffic": None,
                     "kernel": "prefill_attention_kernel (tcgen05), launched alone through "
                               "seer_prefill_attention on the selection in place",
                     "flops_per_launch": flops,
                     "flops_note": "4 D per (query token, query head, attended key): real heads "
                                   "only (a group of odd size also computes one padded head "
                                   "per head pair that is not counted)",
                     "gate_select_attention_tflops": flops / (ms_attn_gate * 1e-3) / 1e12,
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


def cpu_baseline(w, data, args, seed):
    """The oracle on the host cores, on replica 0's draw (the reference arm's
    draw): every (b, h) row of the batch per parallel pass where the inputs
    fit the host copy budget, one spawned process per usable core with one
    BLAS thread each; then the same oracle on one core over a few rows."""
    seqlens = data["seqlens"].cpu().tolist()
    kps = cpu_k_per_seq(w, seqlens)
    info = host_cpu_info()
    rows, sampled = pick_rows(w, seqlens, args.cpu_max_bytes)
    times, used = oracle_parallel_timing(w, data, kps, w.force_newest, rows,
                                         info["usable_cores"], steps=5, warmup=1,
                                         budget_s=args.cpu_budget)
    step_s = statistics.mean(times) * row_share(w, seqlens, rows)
    out = dict({"value": w.batch / step_s, "unit": UNIT, "cores": used, "kind": "oracle",
                "sample": (f"{'a longest-first sample of ' if sampled else 'all '}{len(rows)} "
                           f"(b, kv-head) rows of this workload draw (seed {seed}) per pass, "
                           f"{len(times)} timed passes, fp64 numpy oracle (bf16->f64, pool, "
                           f"gate, select, masked attention), {used} spawned processes with "
                           f"one BLAS thread each"
                           + (", scaled by total length to the whole batch" if sampled else "")),
                "ms_per_step": step_s * 1e3, "extrapolated": bool(sampled)}, **info)
    # one core: the longest rows that make about a tenth of the batch
    few = sorted(rows, key=lambda r: -int(seqlens[r[0]]))[:max(1, len(rows) // 10)]
    t1, _ = oracle_parallel_timing(w, data, kps, w.force_newest, few, 1, steps=2, warmup=1)
    step1 = statistics.mean(t1) * row_share(w, seqlens, few)
    out["value_1core"] = w.batch / step1
    out["sample_1core"] = (f"{len(few)} rows in one process with one BLAS thread, "
                           f"{statistics.mean(t1) / len(few) * 1e3:.1f} ms/row, scaled by total "
                           f"length to the whole batch")
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
    p.add_argument("--batch", type=int, default=None,
                   help="override: batch size (a smaller case of the workload, e.g. for a capture)")
    p.add_argument("--splits", type=int, default=None)
    p.add_argument("--layout", choices=("nhd", "hnd"), default="nhd",
                   help="KV pool page layout: token-major [P][bs][Hkv][D] or head-major [P][Hkv][bs][D]")
    p.add_argument("--seed", type=int, default=None,
                   help="seed of replica 0 (default: the workload's recorded seed)")
    p.add_argument("--max-replicas", type=int, default=24)
    p.add_argument("--cpu-budget", type=float, default=15.0,
                   help="seconds of timed oracle passes for the CPU baseline (at least one)")
    p.add_argument("--cpu-max-bytes", type=float, default=4e9,
                   help="host bytes of oracle inputs (K and V rows); a batch above it is sampled")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-graph", action="store_true", help="launch each step directly, no CUDA graph")
    p.add_argument("--graph-per-step", action="store_true",
                   help="replay one graph per step (no whole-rotation graph)")
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
    p.add_argument("--prefill-batch", type=int, default=2)
    p.add_argument("--prefill-seqlen", type=int, default=16384)
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
