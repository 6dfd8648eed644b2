#!/usr/bin/env python
"""Benchmark of the DSA decode step on B200: lightning indexer + TopK + sparse
MLA attention over a 16 x 128K-context batch (one query per sequence).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload long_decode_16x128k|batched_decode_64x32k|paged_mtp_decode_128seq]

One step = one dsa_forward call over the batch (fused FP8 indexer + exact TopK,
sparse MLA, split combine), inputs resident in HBM.  Every timed step is
bracketed by CUDA events on the launching stream.  No L2 flush runs between
steps: each step streams the whole index-K cache (268 MB at 16 x 128K, more
than twice the 126 MB L2) through L2, which evicts the previous step's data.
(A flush by writing a buffer would leave ~126 MB of dirty lines that the next
step pays to write back.)  The attention-only stage timing, whose inputs are
smaller than L2, evicts L2 before each call by reading a 256 MiB buffer,
outside the timed interval.  With
N > 1 (torchrun) every rank runs its own replica batch (the path has no
exchange step) and the time is the max over ranks.

Printed: one JSON line (rank 0).  `roofline` is for the dominant kernel (the
fused indexer), timed alone over the same workload; `e2e` repeats the step
through the C ABI from pinned host buffers (query-side inputs in, outputs
out; the caches are resident state); `cpu_baseline` is the fp64 oracle timed
on a bounded sample on this host.
"""
from __future__ import annotations

import argparse
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
from long_context_decode_indexer_b200.synth import CONFIGS, make_inputs  # noqa: E402

METRIC = "DSA decode queries/s at 128K ctx (indexer+TopK+sparse MLA); % of HBM/TC roofline"
WORKLOADS = {c["name"]: cid for cid, c in CONFIGS.items() if c["kind"] in ("decode", "paged2")}
DEFAULT_WORKLOAD = CONFIGS[3]["name"]
L2_BYTES = 126 * 1024 * 1024


# DRAM traffic of the fused indexer from one ncu capture (see
# profiles/k1_indexer_long_decode_16x96k.md): read + write bytes per scored
# position, valid only while the kernel sources hash to the captured build.
K1_SOURCES = ("long_context_decode_indexer_b200/csrc/indexer.cu",
              "long_context_decode_indexer_b200/csrc/select.cuh",
              "long_context_decode_indexer_b200/csrc/ptx.cuh",
              "long_context_decode_indexer_b200/csrc/kernels.h")
K1_PROFILED = {"sha256_16": "8a4b7d790e67b55e", "bytes_per_position": 131.10498046875}


def k1_traffic(inp):
    import hashlib
    h = hashlib.sha256()
    for f in K1_SOURCES:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    if h.hexdigest()[:16] != K1_PROFILED["sha256_16"]:
        return None
    n = inp.q_n.astype(np.int64)
    return float(K1_PROFILED["bytes_per_position"] * n[n > inp.topk].sum())


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), "measured"
    except Exception:
        return 6650.0, 1590.0, "fallback"


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


def workload_config(inp, world):
    """The `config` object of the JSON line (the same for both arms)."""
    return {"workload": inp.name, "nq": inp.nq, "context": int(inp.q_n.max()),
            "topk": inp.topk, "h_idx": inp.h_idx, "d_idx": inp.d_idx, "heads": inp.h,
            "d_qk": inp.d_qk, "d_v": inp.d_v, "paged": inp.page_table is not None,
            "parallelism": "replicas" if world > 1 else "single",
            "l2": "inputs larger than L2: each step streams the %.0f MB index-K cache; "
                  "no flush between steps (attention-only stage: L2 evicted by a 256 MiB "
                  "read before each call)" % (algorithmic_bytes(inp)["indexer"] / 1e6)}


def algorithmic_bytes(inp):
    """Bytes the three steps must move at minimum (per batch)."""
    n = inp.q_n.astype(np.int64)
    k = inp.topk
    scored = n > k
    kI = int(n[scored].sum()) * inp.d_idx                        # k^I rows streamed once
    if inp.q_per_seq == 2:                                       # two queries share a stream
        kI = int(np.maximum(n[0::2], n[1::2])[scored[0::2] | scored[1::2]].sum()) * inp.d_idx
    idx_in = inp.nq * (inp.h_idx * inp.d_idx + inp.h_idx * 2)    # q^I + w
    idx_out = inp.nq * k * 4                                     # selected positions
    sel = np.minimum(n, k)
    gather = int(sel.sum()) * inp.d_qk * 2                       # latent rows
    att_io = inp.nq * inp.h * (inp.d_qk * 2 + inp.d_v * 2 + 4) + inp.nq * k * 4
    flops_idx = 2 * int(n[scored].sum()) * inp.h_idx * inp.d_idx
    flops_att = 2 * int(sel.sum()) * inp.h * (inp.d_qk + inp.d_v)
    return dict(indexer=kI + idx_in + idx_out, attention=gather + att_io,
                flops_indexer=flops_idx, flops_attention=flops_att)


# -------------------------------------------------------------- our arm
def run_ours(args, world, rank):
    cid = WORKLOADS[args.workload]
    t_gen = time.time()
    inp = replica_inputs(cid, rank)
    db = upload(inp)
    torch.cuda.synchronize()
    gen_s = time.time() - t_gen
    p = db.params()
    kv = db.kvdesc()
    paged = db.page_table is not None
    st = torch.cuda.current_stream()
    ws = workspace(dsa.workspace_size(p, kv, dsa.OP_FORWARD))
    ws_idx = workspace(dsa.workspace_size(p, kv, dsa.OP_INDEXER_TOPK))
    ws_mla = workspace(dsa.workspace_size(p, kv, dsa.OP_SPARSE_MLA_DECODE))
    out = torch.empty((inp.nq, inp.h, inp.d_v), dtype=torch.int16, device="cuda")
    lse = torch.empty((inp.nq, inp.h), dtype=torch.float32, device="cuda")
    idx = torch.empty((inp.nq, inp.topk), dtype=torch.int32, device="cuda")
    evict_buf = torch.ones(2 * L2_BYTES // 4, dtype=torch.int32, device="cuda")

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

    for _ in range(args.warmup):
        step()
    assert dsa.check_status(ws) == dsa.DSA_OK, dsa.last_error()
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device(), args.clocks_csv) as clk:
        clk.active = True
        t_total = timed(step, args.steps)
        torch.cuda.synchronize()
        barrier(world)
        # stage timings (same workload, same stream) for the roofline
        t_idx = timed(lambda: dsa.indexer_topk(p, kv, db.q_idx, db.w, db.kidx, db.k_scale, idx,
                                               None, ws_idx, stream=st), args.steps)
        t_mla = timed(lambda: dsa.sparse_mla_decode(p, kv, db.q, db.kv, db.kv_row_stride, idx,
                                                    out, lse, ws_mla, stream=st), args.steps,
                      before=evict)
    status = dsa.check_status(ws)
    t_max = max_over_ranks(t_total, world)

    # end to end through the C ABI from pinned host buffers
    h_qidx = torch.from_numpy(inp.q_idx).pin_memory()
    h_w = torch.from_numpy(inp.w.view(np.int16)).pin_memory()
    h_q = torch.from_numpy(inp.q.view(np.int16)).pin_memory()
    h_qn = torch.from_numpy(inp.q_n).pin_memory()
    h_qseq = torch.from_numpy(inp.q_seq).pin_memory()
    h_out = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    h_lse = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()
    h_idx = torch.empty(idx.shape, dtype=idx.dtype).pin_memory()
    d_qidx, d_w, d_q = torch.empty_like(db.q_idx), torch.empty_like(db.w), torch.empty_like(db.q)
    d_qn, d_qseq = torch.empty_like(db.q_n), torch.empty_like(db.q_seq)
    kv_e = dsa.make_kv(q_seq=d_qseq, q_n=d_qn, seq_row0=db.seq_row0, page_table=db.page_table,
                       page_size=inp.page_size, cache_rows=db.kidx.shape[0])
    h2d = sum(t.numel() * t.element_size() for t in (h_qidx, h_w, h_q, h_qn, h_qseq))
    d2h = sum(t.numel() * t.element_size() for t in (h_out, h_lse, h_idx))

    ref_out = out.clone()  # the device-resident path's result, for the check below
    copy_stream = torch.cuda.Stream()

    def e2e_step():
        # The same two stages through the public entry points (dsa_indexer_topk,
        # then dsa_sparse_mla_decode, which is what dsa_forward runs), with the
        # copies overlapped on a second stream: the 2.4 MB attention query goes
        # up while the indexer runs, the indices come down while the attention
        # runs.  `cur` is the capture stream while a graph is recorded.
        cur = torch.cuda.current_stream()
        copy_stream.wait_stream(cur)                 # the previous step is done with d_q
        with torch.cuda.stream(copy_stream):
            d_q.copy_(h_q, non_blocking=True)
        for d, h in ((d_qidx, h_qidx), (d_w, h_w), (d_qn, h_qn), (d_qseq, h_qseq)):
            d.copy_(h, non_blocking=True)
        dsa.indexer_topk(p, kv_e, d_qidx, d_w, db.kidx, db.k_scale, idx, None, ws_idx)
        cur.wait_stream(copy_stream)                 # the query is on the device
        copy_stream.wait_stream(cur)                 # the indices are final
        with torch.cuda.stream(copy_stream):
            h_idx.copy_(idx, non_blocking=True)
        dsa.sparse_mla_decode(p, kv_e, d_q, db.kv, db.kv_row_stride, idx, out, lse, ws_mla)
        h_out.copy_(out, non_blocking=True)
        h_lse.copy_(lse, non_blocking=True)
        cur.wait_stream(copy_stream)                 # join the copy stream

    for _ in range(args.warmup):
        e2e_step()
    torch.cuda.synchronize()
    barrier(world)
    t_e2e_eager = max_over_ranks(timed(e2e_step, args.steps), world)
    # The same step recorded once as a CUDA graph (copies from the pinned
    # buffers, the two stages' launches, copies back, both streams) and
    # replayed: one host launch per step, as a decode loop would run it.
    e2e_launch = "cuda_graph"
    try:
        graph = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream()
        side.wait_stream(st)
        with torch.cuda.stream(side):
            e2e_step()
        st.wait_stream(side)
        torch.cuda.synchronize()
        with torch.cuda.graph(graph):
            e2e_step()
        for _ in range(args.warmup):
            graph.replay()
        torch.cuda.synchronize()
        barrier(world)
        t_e2e = max_over_ranks(timed(graph.replay, args.steps), world)
        del graph
    except RuntimeError as exc:  # capture refused: report the eager loop
        print("e2e graph capture failed (%s); reporting the eager loop" % exc, file=sys.stderr)
        e2e_launch, t_e2e = "eager", t_e2e_eager
    assert dsa.check_status(ws) == dsa.DSA_OK, dsa.last_error()
    assert dsa.check_status(ws_idx) == dsa.DSA_OK, dsa.last_error()
    assert dsa.check_status(ws_mla) == dsa.DSA_OK, dsa.last_error()
    torch.cuda.synchronize()
    e2e_same = bool(torch.equal(h_out, ref_out.cpu()))  # host copy == device-resident result

    alg = algorithmic_bytes(inp)
    hbm, bf16, peak_kind = peaks()
    idx_gbs = alg["indexer"] / (t_idx / args.steps) / 1e9
    mla_gbs = alg["attention"] / (t_mla / args.steps) / 1e9
    mla_tflops = alg["flops_attention"] / (t_mla / args.steps) / 1e12
    step_gbs = (alg["indexer"] + alg["attention"]) / (t_total / args.steps) / 1e9
    total_q = inp.nq * args.steps * world
    qps = job_rate(inp.nq, args.steps, world, t_max)
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
        "config": workload_config(inp, world),
        "roofline": {"bound": "hbm", "achieved": idx_gbs, "peak": hbm, "unit": "GB/s",
                     "frac": idx_gbs / hbm, "traffic": k1_traffic(inp),
                     "kernel": "k1_indexer (fused indexer + TopK)",
                     "peak_source": peak_kind},
        "stages": {
            "indexer_topk_us": t_idx / args.steps * 1e6,
            "indexer_topk_gbs": idx_gbs,
            "indexer_topk_frac_nominal_8tbs": idx_gbs / 8000.0,
            "sparse_mla_us": t_mla / args.steps * 1e6,
            "sparse_mla_gbs": mla_gbs,
            "sparse_mla_tflops": mla_tflops,
            "sparse_mla_frac_hbm": mla_gbs / hbm,
            "sparse_mla_frac_bf16": mla_tflops / bf16,
            "step_gbs": step_gbs,
            "step_frac_hbm": step_gbs / hbm,
            "algorithmic_bytes_per_step": alg["indexer"] + alg["attention"],
        },
        "e2e": {"value": total_q / t_e2e, "unit": "queries/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "launch": e2e_launch,
                "copies": "overlapped with the kernels on a second stream",
                "eager_value": total_q / t_e2e_eager, "matches_device_result": e2e_same},
        "gpu_launches": 3 * args.steps,
        "device_status": status,
        "input_gen_s": gen_s,
        "clocks": clk.summary(),
    }
    return res, inp


# --------------------------------------------------------- oracle timing
def oracle_sample(inp, n_queries, nthreads=0):
    """Time the fp64 oracle (score -> TopK -> attention) on the first
    n_queries queries of the batch; returns (queries/s, cores, seconds)."""
    import oracle
    sel = np.arange(min(n_queries, inp.nq))
    t0 = time.time()
    oracle.forward(inp.q_idx[sel], inp.w[sel], inp.kidx, inp.q[sel], inp.kv, inp.q_seq[sel],
                   inp.q_n[sel], k=inp.topk, scale=inp.scale, seq_row0=inp.seq_row0,
                   page_table=inp.page_table, page_size=inp.page_size, nthreads=nthreads)
    dt = time.time() - t0
    return len(sel) / dt, oracle.max_threads(), dt


def cpu_baseline(inp, target_s=15.0):
    """Bounded sample: one query first, then as many more as ~target_s allows."""
    qps1, cores, dt1 = oracle_sample(inp, 1)
    n = max(1, min(inp.nq, int(target_s / max(dt1, 1e-3))))
    if n > 1:
        qps, cores, dt = oracle_sample(inp, n)
    else:
        qps, dt = qps1, dt1
    return {"value": qps, "unit": "queries/s", "cores": cores, "kind": "oracle",
            "sample": "%d of %d queries of %s (full context), fp64 C oracle, %.1f s"
                      % (n, inp.nq, inp.name, dt),
            "cpu": cpu_model()}


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
    if rank != 0:
        return None
    cid = WORKLOADS[args.workload]
    inp = make_inputs(cid)
    import oracle
    oracle.build()
    # each "step" is a bounded sample: one query of the batch
    for _ in range(min(args.warmup, 1)):
        oracle_sample(inp, 1)
    times = []
    for _ in range(args.steps):
        _, cores, dt = oracle_sample(inp, 1)
        times.append(dt)
    qps = args.steps / sum(times)
    return {
        "metric": METRIC, "value": qps, "unit": "queries/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": sum(times) / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "impl": "reference",
        "config": workload_config(inp, world),
        "cpu_baseline": {"value": qps, "unit": "queries/s", "cores": cores, "kind": "oracle",
                         "sample": "1 query of %s per step (full context), fp64 C oracle"
                                   % inp.name},
        "e2e": {"value": qps, "unit": "queries/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default=DEFAULT_WORKLOAD)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--clocks-csv", default=None,
                    help="also record nvidia-smi clock samples (CSV) during the timed loops")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    world, rank, _ = dist_init() if args.impl == "ours" else (
        int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")), 0)
    if args.impl == "reference":
        res = run_reference(args, world, rank)
        if res is not None:
            print(json.dumps(res))
        return
    res, inp = run_ours(args, world, rank)
    if rank == 0:
        if world == 1 and not args.no_cpu_baseline:
            res["cpu_baseline"] = cpu_baseline(inp)
        print(json.dumps(res))
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
