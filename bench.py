#!/usr/bin/env python
"""Benchmark of the DSA decode step on B200: lightning indexer + TopK + sparse
MLA attention over a 16 x 128K-context batch (one query per sequence).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--ragged] [--nseq S] [--L CTX]
                    [--no-cpu-baseline] [--no-e2e] [--no-next-rows] [--clocks-csv PATH]
    python bench.py --profile [--workload NAME] [--nseq S] [--L CTX] [--warmup W] [--steps K]
    python bench.py --profile-next ROW [--nseq S] [--L CTX] [--warmup W] [--steps K]

Workloads: long_decode_16x128k (default: the headline), batched_decode_64x32k,
paged_mtp_decode_128seq, causal_prefill_16k, tiny_decode_4k; --ragged draws
the long-decode context lengths from U[1024, L] (sequence 0 at 2048 and 1 at
2049); --nseq / --L resize a workload.

One step = one dsa_forward call over the batch (fused FP8 indexer + exact TopK,
sparse MLA, split combine), inputs resident in HBM.  Every timed step is
bracketed by CUDA events on the launching stream.  No L2 flush runs between
steps of the decode workloads: each step streams the whole index-K cache (268
MB at 16 x 128K, more than twice the 126 MB L2) through L2, which evicts the
previous step's data.  (A flush by writing a buffer would leave ~126 MB of
dirty lines that the next step pays to write back.)  Smaller workloads, and
the attention-only stage, evict L2 before each timed call by reading a 256 MiB
buffer, outside the timed interval.  With N > 1 (torchrun) every rank runs its
own replica batch (the path has no exchange step) and the time is the max over
ranks.

Printed: one JSON line (rank 0).  `roofline` is for the dominant kernel (the
fused indexer), timed alone over the same workload; `stages` gives each
stage's time and its fraction of the binding roofline; `e2e` repeats the step
through the C ABI from pinned host buffers (query-side inputs in, outputs
out; the caches are resident state), steps pipelined over two buffer sets
so that each step's copies overlap its neighbours' kernels; `cpu_baseline` is the fp64 oracle timed
on a bounded sample on this host, on all cores and on one.  `next_rows` (one
GPU, decode workloads) times the rows after the decode path alone: the
indexer's q/k/w producer for the batch's tokens, attention over an FP8
latent cache, the distillation loss (sparse and dense stage) and the
masked-MHA short prefill of 4096 tokens, each with its algorithmic bytes and
FLOPs as fractions of the measured peaks.

--profile runs warm-up + K forward steps with no timing and checks the
device status: the command the ncu captures run; --profile-next does the same
for one of the next rows (after W forward steps that produce its indices).
"""
from __future__ import annotations

import argparse
import faulthandler
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from long_context_decode_indexer_b200 import dsa  # noqa: E402
from long_context_decode_indexer_b200.batch import upload, workspace  # noqa: E402
from long_context_decode_indexer_b200.synth import (CONFIGS, make_inputs, make_mha_inputs,  # noqa: E402
                                                     make_project_inputs)

METRIC = "DSA decode queries/s at 128K ctx (indexer+TopK+sparse MLA); % of HBM/TC roofline"
WORKLOADS = {c["name"]: cid for cid, c in CONFIGS.items()}
DEFAULT_WORKLOAD = CONFIGS[3]["name"]
L2_BYTES = 126 * 1024 * 1024
STAGE_ITERS = 200  # iterations of each stage-alone timing loop (more clock samples)


# DRAM traffic of the fused indexer from one ncu capture of the 16 x 65536
# decode case (dram__bytes_read.sum + dram__bytes_write.sum per launch over
# the scored positions), valid only while the indexer's sources hash to the
# captured build.
K1_SOURCES = ("long_context_decode_indexer_b200/csrc/indexer.cu",
              "long_context_decode_indexer_b200/csrc/select.cuh",
              "long_context_decode_indexer_b200/csrc/ptx.cuh",
              "long_context_decode_indexer_b200/csrc/kernels.h")
# kernels.h holds every kernel's parameters: only its indexer part (up to
# this line) belongs to k1
K1_HEADER_END = "// ------------------------------------------------------ sparse MLA attention"
K1_PROFILED = {"sha256_16": "d9af3af125c4e33f", "bytes_per_position": 131.944580078125}


def k1_sources_hash() -> str:
    """Hash of the indexer kernel's sources (the k1 part of kernels.h)."""
    import hashlib
    h = hashlib.sha256()
    for f in K1_SOURCES:
        with open(os.path.join(ROOT, f), "rb") as fh:
            data = fh.read()
        if f.endswith("kernels.h"):
            data = data[:data.index(K1_HEADER_END.encode())]
        h.update(data)
    return h.hexdigest()[:16]


def k1_traffic(inp):
    if k1_sources_hash() != K1_PROFILED["sha256_16"]:
        return None
    n = inp.q_n.astype(np.int64)
    return float(K1_PROFILED["bytes_per_position"] * n[n > inp.topk].sum())


def peaks():
    """(HBM GB/s, bf16 TFLOP/s burst, bf16 TFLOP/s sustained, source)."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return (float(d["hbm_gbs"]), float(d["bf16_tflops"]),
                float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), "measured")
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


# ----------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clock, max clock, power and clock-event reasons while the
    timed loops run: NVML polled every ~1 ms from a thread (read-only), plus,
    when `csv_path` is given, an nvidia-smi CSV record (every 200 ms)."""
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}
    SMI_FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                  "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                  "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int, csv_path: str = None):
        self.dev = device_index
        self.csv_path = csv_path
        self.samples = []
        self.active = False
        self.stop = False
        self.smi = None
        self.nvml = None

    def __enter__(self):
        import threading
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nvml = pynvml
            self.handle = pynvml.nvmlDeviceGetHandleByIndex(self.dev)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nvml = None
        if self.nvml is not None:
            self.thread = threading.Thread(target=self._poll, daemon=True)
            self.thread.start()
        try:
            if not self.csv_path:
                raise RuntimeError("no clock record requested")
            os.makedirs(os.path.dirname(os.path.abspath(self.csv_path)), exist_ok=True)
            self.fh = open(self.csv_path, "w")
            self.smi = subprocess.Popen(
                ["stdbuf", "-oL", "nvidia-smi", "-i", str(self.dev), "--query-gpu=" + self.SMI_FIELDS,
                 "--format=csv", "-lms", "200"], stdout=self.fh, stderr=subprocess.DEVNULL)
        except Exception:
            self.smi = None
        return self

    def _poll(self):
        p = self.nvml
        while not self.stop:
            if self.active:
                try:
                    mhz = p.nvmlDeviceGetClockInfo(self.handle, p.NVML_CLOCK_SM)
                    rs = p.nvmlDeviceGetCurrentClocksEventReasons(self.handle)
                    self.samples.append((mhz, rs))
                except Exception:
                    pass
            time.sleep(0.001)

    def __exit__(self, *exc):
        self.stop = True
        if self.nvml is not None:
            self.thread.join(timeout=2)
        if self.smi is not None:
            self.smi.terminate()
            try:
                self.smi.wait(timeout=5)
            except Exception:
                self.smi.kill()
            self.fh.close()

    def summary(self):
        if self.nvml is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["no samples"]}
        reasons = sorted({name for _, r in self.samples for bit, name in self.REASONS.items() if r & bit})
        return {"sm_mhz": statistics.median(m for m, _ in self.samples),
                "sm_max_mhz": self.max_mhz, "reasons": reasons, "samples": len(self.samples)}


# ----------------------------------------------------------------- helpers
def dist_init(backend: str = "nccl"):
    """Rank, world and local rank from the torchrun environment; one process
    per GPU over NCCL (gloo runs the same host logic on CPU, in tests)."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    elif backend == "nccl":
        torch.cuda.set_device(0)
    return world, rank, local


def workload_inputs(args, seed_offset: int = 0):
    """The workload's seeded batch (resized by --nseq / --L, ragged lengths
    with --ragged)."""
    cid = WORKLOADS[args.workload]
    kw = {}
    if getattr(args, "nseq", None) is not None and CONFIGS[cid]["kind"] != "prefill":
        kw["nseq"] = args.nseq
    if getattr(args, "L", None) is not None:
        kw["L"] = args.L
    if getattr(args, "ragged", False):
        kw["ragged"] = True
    return make_inputs(cid, seed_offset=seed_offset, **kw)


def replica_inputs(cid: int, rank: int):
    """Each rank runs its own replica batch (the path has no exchange step):
    the same workload shape, its own seeded draw."""
    return make_inputs(cid, seed_offset=rank * 101)


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    """The job's time is the slowest rank's (a device-timed value per rank)."""
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_rate(units_per_rank: int, steps: int, world: int, t_max: float) -> float:
    """Whole-job throughput: every rank's units over the slowest rank's time."""
    return units_per_rank * steps * world / t_max


def workload_name(inp, ragged=False):
    return inp.name + ("_ragged" if ragged else "")


def workload_config(inp, world, ragged=False, flush=False):
    """The `config` object of the JSON line (the same for both arms)."""
    l2 = ("inputs larger than L2: each step streams the %.0f MB index-K cache; no flush "
          "between steps (attention-only stage: L2 evicted by a 256 MiB read before each call)"
          % (algorithmic_bytes(inp)["indexer"] / 1e6)) if not flush else \
         "L2 evicted by a 256 MiB read before every timed call (outside the timed interval)"
    return {"workload": workload_name(inp, ragged), "nq": inp.nq, "context": int(inp.q_n.max()),
            "context_min": int(inp.q_n.min()), "topk": inp.topk, "h_idx": inp.h_idx,
            "d_idx": inp.d_idx, "heads": inp.h, "d_qk": inp.d_qk, "d_v": inp.d_v,
            "queries_per_sequence": inp.q_per_seq, "paged": inp.page_table is not None,
            "parallelism": "replicas" if world > 1 else "single", "l2": l2}


def algorithmic_bytes(inp):
    """Bytes and FLOPs the three steps must move / compute at minimum (per
    batch).  The index-K rows of a sequence are read once however many of
    its queries score them; a query whose history fits in k reads none."""
    n = inp.q_n.astype(np.int64)
    k = inp.topk
    scored = n > k
    kI = 0
    for s in range(inp.nseq):
        m = (inp.q_seq == s) & scored
        if m.any():
            kI += int(n[m].max()) * inp.d_idx                    # rows streamed once per sequence
    idx_in = int(scored.sum()) * (inp.h_idx * inp.d_idx + inp.h_idx * 2)   # q^I + w
    idx_out = inp.nq * k * 4                                     # selected positions
    sel = np.minimum(n, k)
    rows = 0
    for s in range(inp.nseq):                                    # distinct latent rows per sequence
        m = inp.q_seq == s
        if m.any():
            rows += int(sel[m].max()) if inp.kind != "prefill" else int(n[m].max())
    if inp.kind != "prefill":
        rows = int(sel.sum())                                    # every query gathers its own rows
    gather = rows * inp.d_qk * 2
    att_io = inp.nq * inp.h * (inp.d_qk * 2 + inp.d_v * 2 + 4) + inp.nq * k * 4
    flops_idx = 2 * int(n[scored].sum()) * inp.h_idx * inp.d_idx
    flops_att = 2 * int(sel.sum()) * inp.h * (inp.d_qk + inp.d_v)
    return dict(indexer=kI + idx_in + idx_out, attention=gather + att_io,
                flops_indexer=flops_idx, flops_attention=flops_att)


def stage_fraction(bytes_, flops, t, hbm_gbs, tflops):
    """max(t_bytes, t_flops) / t: the stage's fraction of its binding roofline."""
    t_b = bytes_ / (hbm_gbs * 1e9)
    t_f = flops / (tflops * 1e12) if flops else 0.0
    return max(t_b, t_f) / t, ("hbm" if t_b >= t_f else "tensor")


def count_our_launches(fn) -> int:
    """Kernels of libdsa_b200 that one call of fn launches (torch profiler)."""
    try:
        from torch.profiler import ProfilerActivity, profile
        torch.cuda.synchronize()
        with profile(activities=[ProfilerActivity.CUDA]) as prof:
            fn()
            torch.cuda.synchronize()
        names = [e.name for e in prof.events() if str(e.device_type).endswith("CUDA")]
        return sum(1 for nm in names if "dsa::" in nm)
    except Exception:
        return -1


# -------------------------------------------------------------- our arm
def run_ours(args, world, rank):
    t_gen = time.time()
    inp = workload_inputs(args, seed_offset=rank * 101)
    db = upload(inp)
    torch.cuda.synchronize()
    gen_s = time.time() - t_gen
    p = db.params()
    kv = db.kvdesc()
    paged = db.page_table is not None
    prefill = inp.kind == "prefill"
    st = torch.cuda.current_stream()
    ws = workspace(dsa.workspace_size(p, kv, dsa.OP_FORWARD))
    ws_idx = workspace(dsa.workspace_size(p, kv, dsa.OP_INDEXER_TOPK))
    mla_op = dsa.OP_SPARSE_MLA_PREFILL if prefill else dsa.OP_SPARSE_MLA_DECODE
    ws_mla = workspace(dsa.workspace_size(p, kv, mla_op))
    mla_fn = dsa.sparse_mla_prefill if prefill else dsa.sparse_mla_decode
    out = torch.empty((inp.nq, inp.h, inp.d_v), dtype=torch.int16, device="cuda")
    lse = torch.empty((inp.nq, inp.h), dtype=torch.float32, device="cuda")
    idx = torch.empty((inp.nq, inp.topk), dtype=torch.int32, device="cuda")
    evict_buf = torch.ones(2 * L2_BYTES // 4, dtype=torch.int32, device="cuda")
    alg = algorithmic_bytes(inp)
    flush = alg["indexer"] < 2 * L2_BYTES   # the step's own stream does not evict L2

    def evict():
        # read (not write) a buffer twice the size of L2: evicts the cache
        # without leaving dirty lines behind
        evict_buf.max()

    def step():
        dsa.forward(p, kv, db.q_idx, db.w, db.kidx, db.k_scale, db.q, db.kv, db.kv_row_stride,
                    out, lse, idx, ws, stream=st, paged=paged)

    def timed(fn, k, before=None):
        """Sum over k runs of the device time of fn (`before` runs ahead of
        each run, outside the timed interval)."""
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(k)]
        for a, b in evs:
            if before is not None:
                before()
            a.record(st)
            fn()
            b.record(st)
        torch.cuda.synchronize()
        return sum(a.elapsed_time(b) for a, b in evs) / 1e3

    if args.profile_next:
        for _ in range(max(args.warmup, 1)):  # the indices the next rows read
            step()
        runs = {r[0]: r for r in next_row_runners(inp, db, p, kv, idx, st)}
        name, fn, _, _, _, wss = runs[args.profile_next]
        for _ in range(args.warmup + args.steps):
            fn()
        status = max((dsa.check_status(w_) for w_ in wss), key=abs)
        print(json.dumps({"profile": name, "steps": args.warmup + args.steps, "device_status": status}))
        return None, inp
    if args.profile:
        for _ in range(args.warmup + args.steps):
            step()
        status = dsa.check_status(ws)
        print(json.dumps({"profile": workload_name(inp, args.ragged), "nq": inp.nq,
                          "max_n": inp.max_n, "steps": args.warmup + args.steps,
                          "device_status": status}))
        return None, inp

    phase("warm-up")
    for _ in range(args.warmup):
        step()
    assert dsa.check_status(ws) == dsa.DSA_OK, dsa.last_error()
    phase("timed steps")
    launches_per_step = count_our_launches(step)
    barrier(world)
    torch.cuda.synchronize()
    stage_iters = max(args.steps, STAGE_ITERS)
    with ClockSampler(torch.cuda.current_device(), args.clocks_csv) as clk:
        clk.active = True
        t_total = timed(step, args.steps, before=evict if flush else None)
        torch.cuda.synchronize()
        barrier(world)
        # stage timings (same workload, same stream) for the roofline
        t_idx = timed(lambda: dsa.indexer_topk(p, kv, db.q_idx, db.w, db.kidx, db.k_scale, idx,
                                               None, ws_idx, stream=st), stage_iters,
                      before=evict if flush else None)
        t_mla = timed(lambda: mla_fn(p, kv, db.q, db.kv, db.kv_row_stride, idx, out, lse, ws_mla,
                                     stream=st), stage_iters, before=evict)
    status = dsa.check_status(ws)
    t_max = max_over_ranks(t_total, world)

    next_rows = None
    phase("next rows")
    if not args.no_next_rows and world == 1 and not prefill and not paged:
        next_rows = measure_next_rows(next_row_runners(inp, db, p, kv, idx, st), timed, evict, *peaks()[:2])

    e2e = None
    phase("end to end")
    if not args.no_e2e:
        e2e = run_e2e(args, world, inp, db, p, idx, out, lse, ws_idx, ws_mla, mla_fn, timed)
    for w_ in (ws, ws_idx, ws_mla):
        assert dsa.check_status(w_) == dsa.DSA_OK, dsa.last_error()

    hbm, bf16, bf16_sus, peak_kind = peaks()
    us_idx = t_idx / stage_iters * 1e6
    us_mla = t_mla / stage_iters * 1e6
    idx_gbs = alg["indexer"] / (us_idx * 1e-6) / 1e9
    mla_gbs = alg["attention"] / (us_mla * 1e-6) / 1e9
    mla_tflops = alg["flops_attention"] / (us_mla * 1e-6) / 1e12
    idx_tflops = alg["flops_indexer"] / (us_idx * 1e-6) / 1e12
    step_s = t_total / args.steps
    step_gbs = (alg["indexer"] + alg["attention"]) / step_s / 1e9
    mla_frac, mla_bound = stage_fraction(alg["attention"], alg["flops_attention"], us_mla * 1e-6,
                                         hbm, bf16)
    mla_frac_sus, _ = stage_fraction(alg["attention"], alg["flops_attention"], us_mla * 1e-6,
                                     hbm, bf16_sus)
    # FP8 dense peak: the recipe's nominal FP8 / bf16 ratio (2x) times the
    # measured bf16 burst peak
    fp8 = 2.0 * bf16
    idx_frac, idx_bound = stage_fraction(alg["indexer"], alg["flops_indexer"], us_idx * 1e-6, hbm, fp8)
    total_q = inp.nq * args.steps * world
    qps = job_rate(inp.nq, args.steps, world, t_max)
    if idx_bound == "hbm":
        roof = {"bound": "hbm", "achieved": idx_gbs, "peak": hbm, "unit": "GB/s",
                "frac": idx_gbs / hbm}
    else:
        roof = {"bound": "tensor", "achieved": idx_tflops, "peak": fp8, "unit": "TFLOP/s",
                "frac": idx_tflops / fp8}
    roof.update({"traffic": k1_traffic(inp) if not prefill else None,
                 "kernel": "k1_indexer (fused indexer + TopK)", "peak_source": peak_kind,
                 "kernel_sources_sha16": k1_sources_hash()})
    res = {
        "metric": METRIC,
        "value": qps,
        "unit": "queries/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": t_max / args.steps * 1e3,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "e4m3+bf16",
        "data": "synthetic",
        "impl": "ours",
        "tokens_per_s": qps,
        "config": workload_config(inp, world, args.ragged, flush),
        "roofline": roof,
        "stages": {
            "indexer_topk_us": us_idx,
            "indexer_topk_gbs": idx_gbs,
            "indexer_topk_tflops_fp8": idx_tflops,
            "indexer_topk_bound": idx_bound,
            "indexer_topk_frac": idx_frac,
            "indexer_topk_frac_nominal_8tbs": idx_gbs / 8000.0,
            "sparse_mla_us": us_mla,
            "sparse_mla_gbs": mla_gbs,
            "sparse_mla_tflops": mla_tflops,
            "sparse_mla_bound": mla_bound,
            "sparse_mla_frac": mla_frac,
            "sparse_mla_frac_sustained_bf16": mla_frac_sus,
            "sparse_mla_frac_hbm": mla_gbs / hbm,
            "sparse_mla_frac_bf16": mla_tflops / bf16,
            "step_us": step_s * 1e6,
            "step_gbs": step_gbs,
            "step_frac_hbm": step_gbs / hbm,
            "algorithmic_bytes_per_step": alg["indexer"] + alg["attention"],
            "flops_per_step": alg["flops_indexer"] + alg["flops_attention"],
            "fp8_peak_tflops": fp8,
            "fp8_peak_source": "2 x measured bf16 burst (nominal FP8/bf16 ratio)",
            "stage_iters": stage_iters,
        },
        "gpu_launches": launches_per_step * args.steps if launches_per_step >= 0 else None,
        "gpu_launches_per_step": launches_per_step,
        "device_status": status,
        "input_gen_s": gen_s,
        "clocks": clk.summary(),
    }
    if next_rows is not None:
        res["next_rows"] = next_rows
    if e2e is not None:
        e2e["value"] = total_q / e2e.pop("t")
        e2e["eager_value"] = total_q / e2e.pop("t_eager")
        t_graph = e2e.pop("t_graph")
        e2e["graph_value"] = total_q / t_graph if t_graph else None
        res["e2e"] = e2e
    return res, inp


def next_row_runners(inp, db, p, kv, idx, st):
    """The rows after the decode path, on this batch or (masked MHA) the
    short-prefill shape: a list of (name, run, algorithmic bytes, FLOPs,
    extra keys, workspaces).  The indexer's q/k/w producer for this batch's
    tokens; attention over an FP8 latent cache (this batch's selected rows,
    the cache cast to e4m3 on the device with unit row scales); the
    distillation loss, sparse stage over the selected sets and dense stage
    over every visible position; the masked-MHA short prefill of 4096 tokens
    (128 heads, 192 / 128 wide) under the indexer's TopK."""
    runs = []
    d = lambda a, dt=None: (torch.from_numpy(np.ascontiguousarray(a)).view(dt) if dt is not None
                            else torch.from_numpy(np.ascontiguousarray(a))).cuda()
    # f1: the producer for nq tokens (decode: one token per query)
    phase("set up the next rows")
    nt = inp.nq
    pi = make_project_inputs(np.arange(nt, dtype=np.int32), np.arange(nt, dtype=np.int32))
    pp = dsa.make_project_params(nt=nt, hidden=pi.x.shape[1], q_lora_rank=pi.q_lora.shape[1],
                                 h_idx=pi.h_idx, d_idx=pi.d_idx, rope_dim=pi.rope_dim)
    pkeep = [d(pi.q_seq), d(np.zeros(nt, np.int64))]  # referenced as long as the runner lives
    pkv = dsa.make_kv(q_seq=pkeep[0], q_n=None, seq_row0=pkeep[1], cache_rows=nt)
    pws = workspace(dsa.project_workspace_size(pp))
    H, dI = pi.h_idx, pi.d_idx
    pargs = [d(pi.x, torch.int16), d(pi.q_lora, torch.int16), d(pi.w_qb, torch.int16),
             d(pi.w_k, torch.int16), d(pi.w_proj, torch.int16), d(pi.ln_gamma), d(pi.ln_beta),
             d(pi.positions), torch.empty((nt, H, dI), dtype=torch.uint8, device="cuda"),
             torch.empty((nt, H), dtype=torch.float32, device="cuda"),
             torch.empty((nt, H), dtype=torch.int16, device="cuda"),
             torch.empty((nt, dI), dtype=torch.uint8, device="cuda"),
             torch.empty((nt,), dtype=torch.float32, device="cuda")]
    wsz = pi.w_qb.size + pi.w_k.size + pi.w_proj.size
    runs.append(("f1_indexer_project",
                 lambda: dsa.indexer_project(pp, pkv, *pargs, pws),
                 2 * wsz + 2 * (pi.x.size + pi.q_lora.size), 2 * nt * wsz,
                 {"tokens": nt, "bound": "hbm", "_keep": (pkeep, pargs)}, [pws]))

    # f4: attention over an FP8 latent cache (the same selected rows)
    kv8 = db.kv.view(torch.bfloat16).to(torch.float8_e4m3fn).view(torch.uint8)
    ksc = torch.ones(kv8.shape[0], dtype=torch.float32, device="cuda")
    ws8 = workspace(dsa.workspace_size(p, kv, dsa.OP_SPARSE_MLA_DECODE))
    out = torch.empty((inp.nq, inp.h, inp.d_v), dtype=torch.int16, device="cuda")
    lse = torch.empty((inp.nq, inp.h), dtype=torch.float32, device="cuda")
    sel = np.minimum(inp.q_n.astype(np.int64), inp.topk)
    rows = int(sel.sum())
    att_io = inp.nq * inp.h * (inp.d_qk * 2 + inp.d_v * 2 + 4) + inp.nq * inp.topk * 4
    runs.append(("f4_sparse_mla_fp8",
                 lambda: dsa.sparse_mla_decode_fp8(p, kv, db.q, kv8, kv8.stride(0), ksc, idx, out, lse, ws8),
                 rows * (inp.d_qk + 4) + att_io, 2 * rows * inp.h * (inp.d_qk + inp.d_v),
                 {"rows": rows, "_keep": (kv8, ksc, out, lse)}, [ws8]))

    # f3: distillation loss, sparse stage (the selected sets) and dense stage
    ld = max(inp.max_n, 1)
    scores = torch.zeros((inp.nq, ld), dtype=torch.float32, device="cuda")
    wsc = workspace(dsa.workspace_size(p, kv, dsa.OP_INDEXER_SCORES))
    dsa.indexer_scores(p, kv, db.q_idx, db.w, db.kidx, db.k_scale, scores, ld, wsc)
    kl = torch.empty((inp.nq,), dtype=torch.float32, device="cuda")
    for name, ix, op in (("f3_index_kl_sparse", idx, dsa.OP_INDEX_KL_SPARSE),
                         ("f3_index_kl_dense", None, dsa.OP_INDEX_KL_DENSE)):
        wsk = workspace(dsa.workspace_size(p, kv, op))
        r = rows if ix is not None else int(inp.q_n.astype(np.int64).sum())
        # two passes of Q . K^T over the set; the rows read once from HBM
        runs.append((name,
                     (lambda ix=ix, wsk=wsk: dsa.index_kl(p, kv, db.q, db.kv, db.kv_row_stride, scores, ld, ix,
                                                          kl, None, wsk)),
                     r * inp.d_qk * 2 + r * 4 + (inp.nq * ld * 4 if ix is None else 0),
                     2 * 2 * r * inp.h * inp.d_qk, {"rows": r, "_keep": (scores, kl)}, [wsk, wsc]))

    # f2: masked-MHA short prefill, 4096 tokens, the indexer's TopK as the mask
    L = 4096
    pin = make_inputs(4, L=L, with_attention=False)
    pdb = upload(pin)
    ipar, ikv = pdb.params(), pdb.kvdesc()
    pidx = torch.empty((L, pin.topk), dtype=torch.int32, device="cuda")
    wsi = workspace(dsa.workspace_size(ipar, ikv, dsa.OP_INDEXER_TOPK))
    dsa.indexer_topk(ipar, ikv, pdb.q_idx, pdb.w, pdb.kidx, pdb.k_scale, pidx, None, wsi)
    m = make_mha_inputs(L)
    mkeep = [d(m.q, torch.int16), d(m.k, torch.int16), d(m.v, torch.int16), d(m.q_seq), d(m.q_n),
             d(m.seq_row0)]
    hq, dq, dv = m.q.shape[1], m.q.shape[2], m.v.shape[2]
    pm = dsa.make_params(nq=L, h_idx=1, d_idx=64, h=hq, topk=pin.topk, max_n=L, q_per_seq=L, scale=m.scale,
                         d_qk=dq, d_v=dv)
    kvm = dsa.make_kv(q_seq=mkeep[3], q_n=mkeep[4], seq_row0=mkeep[5], cache_rows=L)
    wsm = workspace(dsa.workspace_size(pm, kvm, dsa.OP_MASKED_MHA))
    mout = torch.empty((L, hq, dv), dtype=torch.int16, device="cuda")
    mlse = torch.empty((L, hq), dtype=torch.float32, device="cuda")
    runs.append(("f2_masked_mha_prefill_4k",
                 lambda: dsa.masked_mha_prefill(pm, kvm, mkeep[0], mkeep[1], mkeep[2], pidx, mout, mlse, wsm),
                 2 * L * hq * (2 * dq + 2 * dv),                            # q, k, v, out
                 2 * hq * float(m.q_n.astype(np.int64).sum()) * (dq + dv),  # causal dense
                 {"tokens": L, "bound": "tensor", "_keep": (mkeep, pdb, pidx, mout, mlse)}, [wsm, wsi]))
    return runs


def measure_next_rows(runs, timed, evict, hbm, bf16, iters=20):
    """Each next row timed alone, L2 evicted before every run: replayed as a
    CUDA graph (device time: the library's host-side set-up, e.g. tensor-map
    encoding, runs once at capture) and as eager calls (device time plus
    whatever host time the calls leave the GPU idle).  The algorithmic bytes
    and FLOPs are given as fractions of the measured peaks at the graph
    time."""
    res = {}
    for name, fn, bytes_, flops, extra, wss in runs:
        phase(name)
        fn()
        t_eager = timed(fn, iters, before=evict) / iters
        for w_ in wss:
            assert dsa.check_status(w_) == dsa.DSA_OK, dsa.last_error()
        t, launch = t_eager, "eager"
        try:
            g = torch.cuda.CUDAGraph()
            side = torch.cuda.Stream()
            side.wait_stream(torch.cuda.current_stream())
            with torch.cuda.stream(side):
                fn()
            torch.cuda.current_stream().wait_stream(side)
            torch.cuda.synchronize()
            with torch.cuda.graph(g):
                fn()
            g.replay()
            torch.cuda.synchronize()
            t = timed(g.replay, iters, before=evict) / iters
            launch = "cuda_graph"
            del g
        except RuntimeError as exc:
            print("next row %s: graph capture failed (%s); eager time reported" % (name, exc),
                  file=sys.stderr)
        for w_ in wss:
            assert dsa.check_status(w_) == dsa.DSA_OK, dsa.last_error()
        r = {"us": t * 1e6, "us_eager": t_eager * 1e6, "launch": launch,
             "gbs": bytes_ / t / 1e9, "tflops": flops / t / 1e12,
             "frac_hbm": bytes_ / t / 1e9 / hbm, "frac_bf16": flops / t / 1e12 / bf16,
             "algorithmic_bytes": bytes_, "flops": flops}
        r.update({k: v for k, v in extra.items() if not k.startswith("_")})
        res[name] = r
    return res


E2E_SLOTS = 2        # device buffer sets: step k uses slot k % 2
E2E_GRAPH_STEPS = 8  # steps recorded in one CUDA graph (pipelined inside it)


def run_e2e(args, world, inp, db, p, idx, out, lse, ws_idx, ws_mla, mla_fn, timed):
    """The step end to end through the C ABI from pinned host buffers: every
    step uploads its query-side inputs and downloads its indices, attention
    output and LSE (the caches are resident state).  Steps are pipelined over
    two buffer sets and three streams, as a server runs independent batches:
    the uploads of step k + 1 (copy engine, host to device) and the downloads
    of step k - 1 (device to host) run while step k computes."""
    st = torch.cuda.current_stream()
    h_qidx = torch.from_numpy(inp.q_idx).pin_memory()
    h_w = torch.from_numpy(inp.w.view(np.int16)).pin_memory()
    h_q = torch.from_numpy(inp.q.view(np.int16)).pin_memory()
    h_qn = torch.from_numpy(inp.q_n).pin_memory()
    h_qseq = torch.from_numpy(inp.q_seq).pin_memory()
    slots = []
    for j in range(E2E_SLOTS):
        sl = {"d_qidx": torch.empty_like(db.q_idx), "d_w": torch.empty_like(db.w), "d_q": torch.empty_like(db.q),
              "d_qn": torch.empty_like(db.q_n), "d_qseq": torch.empty_like(db.q_seq),
              "idx": torch.empty_like(idx), "out": torch.empty_like(out), "lse": torch.empty_like(lse),
              "h_out": torch.empty(out.shape, dtype=out.dtype).pin_memory(),
              "h_lse": torch.empty(lse.shape, dtype=lse.dtype).pin_memory(),
              "h_idx": torch.empty(idx.shape, dtype=idx.dtype).pin_memory()}
        sl["kv"] = dsa.make_kv(q_seq=sl["d_qseq"], q_n=sl["d_qn"], seq_row0=db.seq_row0,
                               page_table=db.page_table, page_size=inp.page_size, cache_rows=db.kidx.shape[0])
        slots.append(sl)
    h2d = sum(t.numel() * t.element_size() for t in (h_qidx, h_w, h_q, h_qn, h_qseq))
    d2h = sum(slots[0][k].numel() * slots[0][k].element_size() for k in ("h_out", "h_lse", "h_idx"))

    ref_out = out.clone()  # the device-resident path's result, for the check below
    up_stream, down_stream = torch.cuda.Stream(), torch.cuda.Stream()

    def run_steps(n):
        """n consecutive steps; `cur` is the capture stream while a graph is
        recorded (the side streams fork from it and join it at the end)."""
        cur = torch.cuda.current_stream()
        up_stream.wait_stream(cur)
        down_stream.wait_stream(cur)
        # fresh events: a wait on one not yet recorded is a no-op, and no wait
        # reaches an event recorded outside the run (or outside a capture)
        for sl in slots:
            sl["up"], sl["comp"], sl["down"] = torch.cuda.Event(), torch.cuda.Event(), torch.cuda.Event()
        for k in range(n):
            sl = slots[k % E2E_SLOTS]
            with torch.cuda.stream(up_stream):
                up_stream.wait_event(sl["comp"])      # step k - 2 is done with the inputs
                for d, h in (("d_qidx", h_qidx), ("d_w", h_w), ("d_q", h_q), ("d_qn", h_qn), ("d_qseq", h_qseq)):
                    sl[d].copy_(h, non_blocking=True)
                sl["up"].record(up_stream)
            cur.wait_event(sl["up"])
            cur.wait_event(sl["down"])                # step k - 2's results are on the host
            dsa.indexer_topk(p, sl["kv"], sl["d_qidx"], sl["d_w"], db.kidx, db.k_scale, sl["idx"], None, ws_idx)
            mla_fn(p, sl["kv"], sl["d_q"], db.kv, db.kv_row_stride, sl["idx"], sl["out"], sl["lse"], ws_mla)
            sl["comp"].record(cur)
            with torch.cuda.stream(down_stream):
                down_stream.wait_event(sl["comp"])
                sl["h_idx"].copy_(sl["idx"], non_blocking=True)
                sl["h_out"].copy_(sl["out"], non_blocking=True)
                sl["h_lse"].copy_(sl["lse"], non_blocking=True)
                sl["down"].record(down_stream)
        cur.wait_stream(up_stream)
        cur.wait_stream(down_stream)

    run_steps(max(args.warmup, E2E_SLOTS))
    torch.cuda.synchronize()
    barrier(world)
    t_eager = max_over_ranks(timed(lambda: run_steps(args.steps), 1), world)
    # E2E_GRAPH_STEPS pipelined steps recorded once as a CUDA graph and
    # replayed: one host launch per group of steps, as a decode loop would
    # run it; the time per step is the replays' time over the steps they ran.
    try:
        graph = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream()
        side.wait_stream(st)
        with torch.cuda.stream(side):
            run_steps(E2E_SLOTS)
        st.wait_stream(side)
        torch.cuda.synchronize()
        with torch.cuda.graph(graph):
            run_steps(E2E_GRAPH_STEPS)
        for _ in range(max(1, args.warmup // E2E_GRAPH_STEPS)):
            graph.replay()
        torch.cuda.synchronize()
        barrier(world)
        reps = max(1, args.steps // E2E_GRAPH_STEPS)
        t_graph = max_over_ranks(timed(graph.replay, reps), world) / (reps * E2E_GRAPH_STEPS) * args.steps
        del graph
    except RuntimeError as exc:  # capture refused: report the eager loop
        print("e2e graph capture failed (%s); reporting the eager loop" % exc, file=sys.stderr)
        t_graph = None
    # the faster of the two launch modes (both reported); on the boxes
    # measured the copies set the pace and the eager loop overlapped them better
    t, launch = (t_graph, "cuda_graph") if t_graph is not None and t_graph <= t_eager else (t_eager, "eager")
    torch.cuda.synchronize()
    same = all(bool(torch.equal(sl["h_out"], ref_out.cpu())) for sl in slots)  # host copies == device result
    return {"t": t, "t_eager": t_eager, "t_graph": t_graph, "unit": "queries/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "launch": launch,
            "copies": "pipelined: uploads of the next step and downloads of the previous one run "
                      "during each step's kernels (two buffer sets, three streams)",
            "graph_steps": E2E_GRAPH_STEPS,
            "matches_device_result": same}


# --------------------------------------------------------- oracle timing
def _oracle_queries(inp, sel, nthreads):
    import oracle
    t0 = time.time()
    oracle.forward(inp.q_idx[sel], inp.w[sel], inp.kidx, inp.q[sel], inp.kv, inp.q_seq[sel],
                   inp.q_n[sel], k=inp.topk, scale=inp.scale, seq_row0=inp.seq_row0,
                   page_table=inp.page_table, page_size=inp.page_size, k_scale=inp.k_scale,
                   nthreads=nthreads)
    return time.time() - t0


def oracle_sample(inp, n_queries, nthreads=0, seed=0):
    """Time the fp64 oracle (score -> TopK -> attention) on n_queries queries
    of the batch (the first ones; a seeded random subset for a prefill, whose
    queries differ in length); returns (queries/s, threads, seconds, sel)."""
    import oracle
    n_queries = min(n_queries, inp.nq)
    if inp.kind == "prefill":
        sel = np.sort(np.random.default_rng(1000 + seed).choice(inp.nq, n_queries, replace=False))
    else:
        sel = np.arange(n_queries)
    dt = _oracle_queries(inp, sel, nthreads)
    threads = oracle.max_threads() if nthreads == 0 else nthreads
    return len(sel) / dt, threads, dt, sel


def cpu_baseline(inp, target_s=12.0):
    """Bounded samples of the oracle on this host: as many queries as ~target_s
    allows on all cores, and one query on one core."""
    qps1, cores, dt1, _ = oracle_sample(inp, 1)
    n = max(1, min(inp.nq, int(target_s / max(dt1, 1e-3))))
    if n > 1:
        qps, cores, dt, sel = oracle_sample(inp, n)
    else:
        qps, dt = qps1, dt1
    qps_1c, _, dt_1c, _ = oracle_sample(inp, 1, nthreads=1)
    kind = "a seeded random subset" if inp.kind == "prefill" else "the first"
    return {"value": qps, "unit": "queries/s", "cores": cores, "kind": "oracle",
            "sample": "%s %d of %d queries of %s (full context), fp64 C oracle, %.1f s on %d threads; "
                      "1 query on 1 thread: %.1f s" % (kind, n, inp.nq, inp.name, dt, cores, dt_1c),
            "value_1core": qps_1c, "cpu": cpu_model()}


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def run_reference(args, world, rank):
    """The oracle as the reference arm: rank 0 alone; every step is a bounded
    sample (one query of the workload)."""
    if rank != 0:
        return None
    inp = workload_inputs(args)
    import oracle
    oracle.build()
    for _ in range(min(args.warmup, 1)):
        oracle_sample(inp, 1)
    times = []
    cores = 0
    for i in range(args.steps):
        _, cores, dt, _ = oracle_sample(inp, 1, seed=i)
        times.append(dt)
    qps = args.steps / sum(times)
    return {
        "metric": METRIC, "value": qps, "unit": "queries/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": sum(times) / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "impl": "reference",
        "config": workload_config(inp, world, getattr(args, "ragged", False)),
        "cpu_baseline": {"value": qps, "unit": "queries/s", "cores": cores, "kind": "oracle",
                         "sample": "1 query of %s per step (full context), fp64 C oracle"
                                   % inp.name},
        "e2e": {"value": qps, "unit": "queries/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default=DEFAULT_WORKLOAD)
    ap.add_argument("--ragged", action="store_true",
                    help="decode context lengths ~ U[1024, L] (sequence 0 at 2048, 1 at 2049)")
    ap.add_argument("--nseq", type=int, default=None, help="resize: number of sequences")
    ap.add_argument("--L", type=int, default=None, help="resize: context length (median for paged)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-next-rows", action="store_true",
                    help="skip the next rows' timings (producer, FP8 attention, distillation loss, masked MHA)")
    ap.add_argument("--profile", action="store_true",
                    help="run warm-up + steps forward calls untimed (for profiler captures)")
    ap.add_argument("--profile-next", default=None,
                    choices=["f1_indexer_project", "f2_masked_mha_prefill_4k", "f3_index_kl_sparse",
                             "f3_index_kl_dense", "f4_sparse_mla_fp8"],
                    help="run warm-up forward steps, then warm-up + steps calls of one next row untimed")
    ap.add_argument("--clocks-csv", default=None,
                    help="also record nvidia-smi clock samples (CSV) during the timed loops")
    args = ap.parse_args(argv)
    if not args.profile and not args.profile_next:
        args.warmup = max(args.warmup, 3)
    return args


def phase(name: str):
    """A progress line on stderr (where a crash happened, with faulthandler's
    traceback)."""
    print("bench: %s" % name, file=sys.stderr, flush=True)


def main():
    faulthandler.enable()
    args = parse_args()
    world, rank, _ = dist_init() if args.impl == "ours" else (
        int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")), 0)
    if args.impl == "reference":
        res = run_reference(args, world, rank)
        if res is not None:
            print(json.dumps(res))
        return
    res, inp = run_ours(args, world, rank)
    if rank == 0 and res is not None:
        if world == 1 and not args.no_cpu_baseline:
            phase("cpu baseline")
            res["cpu_baseline"] = cpu_baseline(inp)
        print(json.dumps(res))
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
