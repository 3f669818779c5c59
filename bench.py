#!/usr/bin/env python
"""Benchmark of the product-key memory lookup forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload memplus]
                    [--impl ours|reference] [--sharded]

One step = one pkm_forward over a batch of the workload (sub-key norms, the
selection -- query norms, sub-key scoring, per-half top-k, k x k combine,
softmax --, bag gather [+ Memory+ GEMMs]).  The default workload is the
Memory+ forward (16,384 tokens, 16.8 M keys, 32 GiB value table).  For
N > 1 one rank runs per GPU: run directly, ``--gpus N`` starts itself under
torch.distributed.run; under torchrun WORLD_SIZE must equal N.  By default
every rank holds a replica of the tables and processes its own batch (weak
scaling, no data-path collective).  ``--sharded`` instead splits the value
table by rows over the ranks and times the row-sharded step (selection,
all-gather of the selections, each shard's partial bags, reduce-scatter)
over NCCL.  Timings are the maximum over ranks; rank 0 prints one JSON line.

--impl reference times the CPU oracle (plain fp64 C, all host cores) on a
bounded token sample per step, rank 0 only.
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
sys.path.insert(0, ROOT)

import torch  # noqa: E402

METRIC = "memory-layer lookup tokens/sec; bag-gather HBM GB/s vs B200 ~8 TB/s peak"
UNIT = "tokens/s"
L2_FLUSH_BYTES = 256 << 20
PROFILES = os.path.join(ROOT, "profiles")


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=200)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--workload", default="memplus",
                   choices=["pkm", "memplus", "tiny", "decode", "train", "memplus_train",
                            "engram"])
    p.add_argument("--graph", action="store_true",
                   help="capture one step in a CUDA graph and replay it (default for decode)")
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--shards", type=int, default=0,
                   help="pkm workloads: also time the compute of a row-sharded step with this "
                        "many shards held on one GPU (selection + every shard's partial bags)")
    p.add_argument("--engram-rows", type=int, default=0,
                   help="engram workload: rows per head table (0: the workload's own, about "
                        "2^20; smaller tables for profiling captures)")
    p.add_argument("--n-sub", type=int, default=0,
                   help="profiling aid for the product-key workloads: this many sub-keys per "
                        "(head, half) and a value table of n_sub^2 rows instead of the "
                        "workload's own (0), for kernel captures that fit a few GB; its line is "
                        "not the workload's metric and carries no ncu traffic record")
    p.add_argument("--tokens", type=int, default=0,
                   help="profiling aid for the product-key workloads: this many tokens per "
                        "step instead of the workload's own (0); like --n-sub, its line is not "
                        "the workload's metric and carries no ncu traffic record")
    p.add_argument("--select-only", action="store_true",
                   help="profiling aid for the pkm-style workloads: run only the selection "
                        "(no value table on the device) and print its mean time per launch")
    p.add_argument("--cpu-seconds", type=float, default=10.0,
                   help="target CPU time of the oracle baseline sample")
    p.add_argument("--sharded", action="store_true",
                   help="row-shard the value table over the ranks and time the sharded step "
                        "(selection, all-gather, partial bags, reduce-scatter) over NCCL")
    p.add_argument("--launcher-check", action="store_true",
                   help="start the ranks, join their process group and report the world size "
                        "(no GPU work): a check of the multi-process launch")
    return p.parse_args()


def torchrun_command(args_list, gpus: int, port: int):
    """The command that runs this script with the same arguments as one
    process per GPU under torch.distributed.run (rendezvous on 127.0.0.1)."""
    return [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
            f"--nproc-per-node={gpus}", "--master-addr=127.0.0.1", f"--master-port={port}",
            os.path.abspath(__file__)] + list(args_list)


def relaunch(gpus: int) -> int:
    """``--gpus N`` run without torchrun: start the N ranks and return their
    launcher's exit code."""
    import socket

    sk = socket.socket()
    sk.bind(("127.0.0.1", 0))
    port = sk.getsockname()[1]
    sk.close()
    return subprocess.call(torchrun_command(sys.argv[1:], gpus, port))


# ------------------------------------------------------------ plumbing --

def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"bench.py: --gpus {args.gpus} but {world} ranks were started")
    if args.impl == "reference":
        return rank, world, local  # rank 0 alone works; no process group
    if args.launcher_check:
        if world > 1:
            import datetime
            torch.distributed.init_process_group(
                "nccl" if torch.cuda.is_available() else "gloo",
                timeout=datetime.timedelta(seconds=60))
        return rank, world, local
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group(
            "nccl", timeout=datetime.timedelta(seconds=120),
            device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return rank, world, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(x: float, world: int) -> float:
    """Maximum of a per-rank float (timings are max over ranks)."""
    if world == 1:
        return x
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def rank_workload(w, rank: int):
    """Weak scaling: each rank draws its own token batch and holds a replica of
    the tables (same table seed on every rank)."""
    return w.scaled(seed=w.seed + 7919 * rank, table_seed_=w.table_seed)


def whole_job_tokens_per_s(tokens_per_rank: int, world: int, max_ms_per_step: float) -> float:
    """Tokens processed by all ranks per second, timed by the slowest rank."""
    return world * tokens_per_rank / (max_ms_per_step / 1e3)


class Clocks:
    """SM clock and throttle-reason samples of this GPU during the timed region.

    NVML (read-only queries) from a thread every 5 ms, so that even a short
    timed region is covered; the first sample is taken before the region
    starts counting.  Falls back to `nvidia-smi -lms 200` when NVML is not
    importable."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.nvml = None
        self.samples = []  # (sm MHz, max MHz, reason names)
        self.path = os.path.join("/tmp", f"pkm_clocks_{os.getpid()}.csv")

    def _nvml_handle(self):
        import pynvml
        pynvml.nvmlInit()
        try:
            uuid = str(torch.cuda.get_device_properties(self.idx).uuid)
            h = pynvml.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
        except Exception:
            h = pynvml.nvmlDeviceGetHandleByIndex(self.idx)
        return pynvml, h

    def _sample_nvml(self):
        nv, h = self.nvml
        bits = {"hw_slowdown": nv.nvmlClocksEventReasonHwSlowdown,
                "hw_thermal_slowdown": nv.nvmlClocksEventReasonHwThermalSlowdown,
                "sw_thermal_slowdown": nv.nvmlClocksEventReasonSwThermalSlowdown,
                "sw_power_cap": nv.nvmlClocksEventReasonSwPowerCap}
        smax = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
        while True:
            sm = float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
            r = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
            self.samples.append((sm, smax, [n for n, b in bits.items() if r & b]))
            self.started.set()
            if self.stop.wait(0.005):
                return

    def __enter__(self):
        import threading
        try:
            self.nvml = self._nvml_handle()
            self.stop, self.started = threading.Event(), threading.Event()
            self.thread = threading.Thread(target=self._sample_nvml, daemon=True)
            self.thread.start()
            self.started.wait(2.0)
            return self
        except Exception:
            self.nvml = None
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=self.f, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.nvml is not None:
            self.stop.set()
            self.thread.join(timeout=5)
            return
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.f.close()

    def summary(self):
        source = "nvml 5 ms"
        if self.nvml is None:
            source = "nvidia-smi 200 ms"
            if self.proc is None or not os.path.exists(self.path):
                return {"sm_mhz": None, "sm_max_mhz": None,
                        "reasons": ["nvidia-smi unavailable"]}
            for line in open(self.path):
                f = [x.strip() for x in line.split(",")]
                if len(f) < 9:
                    continue
                try:
                    sm_v, smax_v = float(f[1]), float(f[2])
                except ValueError:
                    continue
                self.samples.append((sm_v, smax_v,
                                     [n for n, v in zip(self.NAMES, f[5:9])
                                      if v.lower() == "active"]))
            os.remove(self.path)
        sm = [x[0] for x in self.samples]
        smax = self.samples[-1][1] if self.samples else None
        reasons = sorted({n for x in self.samples for n in x[2]})
        loaded = [v for v in sm if smax and v > 0.5 * smax] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None, "sm_max_mhz": smax,
                "samples": len(sm), "source": source, "reasons": reasons}


def measured_peaks():
    for p in (os.path.join(ROOT, "MEASURED_PEAKS.json"),):
        if os.path.exists(p):
            d = json.load(open(p))
            return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}, "fallback"


def gather_bytes_per_token(w) -> int:
    """Algorithmic bytes of the bag gather per token: every selected value row
    (H*k rows of d_v elements), its row id and weight (8 B), the output row
    and, with Memory+, the gate row read."""
    b = w.elem_bytes
    per = w.H * w.k * (w.d_v * b + 8) + w.d_v * b
    if w.memplus:
        per += w.d_v * b
    return per


def backward_bytes(w, U: int) -> int:
    """Algorithmic bytes of the training backward: the value rows re-gathered
    (R rows), ids and weights (8 B per slot), dy, q and K read, dq and dK
    written (fp32), the sparse value gradient written (U rows of fp32 plus ids)."""
    b = w.elem_bytes
    R = w.T * w.H * w.k
    return (R * (w.d_v * b + 8) + w.T * w.d_v * b + w.T * w.H * 2 * w.d_half * (b + 4)
            + w.H * 2 * w.n_sub * w.d_half * (b + 4) + U * (w.d_v * 4 + 4))


def graph_launches(lib, step) -> int:
    """Kernels one step launches (counted on an eager run)."""
    c0 = lib.pkm_launch_count()
    step()
    torch.cuda.synchronize()
    return lib.pkm_launch_count() - c0


def traffic_record(workload: str):
    """dram bytes per launch of a kernel ("<workload>" the gather,
    "<workload>:select" the selection) from the committed ncu summaries, or
    None when the kernel's source changed since it was captured."""
    rec = traffic_entry(workload)
    return rec["dram_bytes_per_launch"] if rec else None


def traffic_entry(workload: str):
    """The committed ncu record of `workload` in profiles/traffic.json, or None
    when it is missing or any of its kernels' sources changed since."""
    path = os.path.join(PROFILES, "traffic.json")
    if not os.path.exists(path):
        return None
    rec = json.load(open(path)).get(workload)
    if not rec:
        return None
    sources = rec.get("sources") or {rec["source"]: rec["source_sha"]}
    for name, want in sources.items():
        src = os.path.join(ROOT, "sparse_key_value_b200", "csrc", name)
        if hashlib.sha256(open(src, "rb").read()).hexdigest()[:16] != want:
            return None
    return rec


# ------------------------------------------------------------ our arm --

def run_ours(args, rank, world, local):
    import sparse_key_value_b200 as skv
    from sparse_key_value_b200.inputs import WORKLOADS, make_inputs

    skv.load()
    w = WORKLOADS[args.workload]
    if args.workload == "decode":
        w = w.scaled(T=8)
    if args.n_sub > 0:
        w = w.scaled(n_sub=args.n_sub)
    if args.tokens > 0:
        w = w.scaled(T=args.tokens)
    inp = make_inputs(rank_workload(w, rank), "cuda")
    mp = w.memplus
    kw = dict(x=inp["x"], W1=inp["W1"], W2=inp["W2"]) if mp else {}
    T = w.T
    out = torch.empty(T, w.d_out, dtype=w.torch_dtype, device="cuda")
    idx = torch.empty(T, w.H, w.k, dtype=torch.int32, device="cuda")
    wts = torch.empty(T, w.H, w.k, dtype=torch.float32, device="cuda")
    ws = torch.empty(max(16, skv.forward_workspace_size(
        T, w.H, w.d_half, w.n_sub, w.k, w.d_v, 1 if w.dtype == "bf16" else 0, mp, w.d_model)),
        dtype=torch.uint8, device="cuda")
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()
    lib = skv.load()

    train = w.train
    mp_train = train and mp
    if mp_train:
        # Memory+ training: the forward keeps the bag output y; the Memory+
        # backward turns the layer-output gradient into the lookup's dy
        yb = torch.empty(T, w.d_v, dtype=w.torch_dtype, device="cuda")
        dyv = torch.empty(T, w.d_v, dtype=w.torch_dtype, device="cuda")
        mdx = torch.empty(T, w.d_model, dtype=torch.float32, device="cuda")
        mdW1 = torch.empty(w.d_model, w.d_v, dtype=torch.float32, device="cuda")
        mdW2 = torch.empty(w.d_v, w.d_model, dtype=torch.float32, device="cuda")
        margs = skv._lib.MemplusBwdArgs(T, w.d_model, w.d_v, skv._p(inp["x"]), skv._p(inp["W1"]),
                                        skv._p(inp["W2"]), skv._p(yb), skv._p(inp["dy"]),
                                        skv._p(dyv), skv._p(mdx), skv._p(mdW1), skv._p(mdW2),
                                        None, 0)
        mws = torch.empty(max(16, lib.pkm_memplus_backward_workspace_size(
            skv.ctypes.byref(margs))), dtype=torch.uint8, device="cuda")
        margs.workspace, margs.workspace_bytes = skv._p(mws), mws.numel()
        kw["y_out"] = yb
    if train:
        R = T * w.H * w.k
        dq = torch.empty(T, w.H, 2, w.d_half, dtype=torch.float32, device="cuda")
        dK = torch.empty(w.H, 2, w.n_sub, w.d_half, dtype=torch.float32, device="cuda")
        uniq = torch.empty(R, dtype=torch.int32, device="cuda")
        grad = torch.empty(R, w.d_v, dtype=torch.float32, device="cuda")
        n_uniq = torch.zeros(1, dtype=torch.int64, device="cuda")
        bargs = skv._bwd_args(inp["query"], inp["subkeys"], inp["values"], idx, wts,
                              dyv if mp_train else inp["dy"],
                              dquery=skv._p(dq), dsubkeys=skv._p(dK), uniq_rows=skv._p(uniq),
                              grad_rows=skv._p(grad), n_uniq=skv._p(n_uniq), uniq_cap=R)
        bws = torch.empty(max(16, lib.pkm_backward_workspace_size(skv.ctypes.byref(bargs))),
                          dtype=torch.uint8, device="cuda")
        bargs.workspace, bargs.workspace_bytes = skv._p(bws), bws.numel()
        sptr = skv.ctypes.c_void_p(stream.cuda_stream)

    def step(events=None, bev=None):
        skv.pkm_forward(inp["query"], inp["subkeys"], inp["values"], w.k, out=out, idx=idx,
                        weights=wts, workspace=ws, phase_events=events, **kw)
        if train:
            if bev is not None:
                bev[0].record()
            if mp_train:
                skv.check(lib.pkm_memplus_backward(skv.ctypes.byref(margs), sptr),
                          "pkm_memplus_backward")
            if bev is not None:
                bev[2].record()
            skv.check(lib.pkm_backward(skv.ctypes.byref(bargs), sptr), "pkm_backward")
            if bev is not None:
                bev[1].record()

    use_graph = args.graph or args.workload == "decode"
    flush_between = args.workload != "decode"
    for _ in range(args.warmup):
        if flush_between:
            flush.zero_()
        step()
    torch.cuda.synchronize()
    assert skv.device_error() == 0
    graph = None
    if use_graph:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            step()
        graph.replay()
        torch.cuda.synchronize()

    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(7)] for _ in range(K)]
    bev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    for e in sum(ev, []) + sum(bev, []):
        e.record()  # creates the event handles the library records into
    barrier(world)
    torch.cuda.synchronize()
    launches0 = lib.pkm_launch_count()
    with Clocks(local) as clk:
        for i in range(K):
            if flush_between:
                flush.zero_()  # L2 flush between timed steps (outside the events)
            ev[i][0].record()
            if graph is not None:
                graph.replay()
            else:
                step()
            ev[i][6].record()
        torch.cuda.synchronize()
    launches = lib.pkm_launch_count() - launches0
    if graph is not None:  # kernels replayed from the graph: one step's launches x K
        launches = graph_launches(lib, step) * K
    barrier(world)
    step_ms = [e[0].elapsed_time(e[6]) for e in ev]
    total_ms = max_over_ranks(sum(step_ms), world)
    # Phases from separate (untimed) steps with the library's phase events:
    # an event recorded between two kernels serialises them, so the timed
    # steps above run without any (their kernels overlap by programmatic
    # dependent launch) and these give the per-phase split.
    phase_ms = None
    if graph is None:
        P = min(K, 20)
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(7)] for _ in range(P)]
        bev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(P)]
        for e in sum(ev, []) + sum(bev, []):
            e.record()
        torch.cuda.synchronize()
        for i in range(P):
            if flush_between:
                flush.zero_()
            step(ev[i], bev[i] if train else None)
        torch.cuda.synchronize()
        phase_ms = [[e[j].elapsed_time(e[j + 1]) for e in ev] for j in range(6)]
    assert skv.device_error() == 0
    ms_per_step = total_ms / K
    value = whole_job_tokens_per_s(T, world, ms_per_step)

    # roofline of the dominant kernel: the bag gather (phase 4 -> 5)
    peaks, peak_kind = measured_peaks()
    peak = float(peaks["hbm_gbs"])
    bytes_per_launch = gather_bytes_per_token(w) * T
    # the committed records hold the workloads' own sizes
    rec_key = args.workload if args.n_sub <= 0 and args.tokens <= 0 else None
    traffic = traffic_record(rec_key) if rec_key else None
    sel = None
    if phase_ms is not None:
        gather_ms = statistics.mean(phase_ms[4])
        achieved = bytes_per_launch / (gather_ms / 1e3) / 1e9
        roof = {"kernel": "embbag_fwd_kernel (bag gather)", "bound": "hbm",
                "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                "frac": round(achieved / peak, 4), "peak_source": f"{peak_kind} hbm_gbs",
                "algorithmic_bytes_per_launch": bytes_per_launch,
                "traffic": traffic, "gather_us": round(gather_ms * 1e3, 2)}
        phases = dict(zip(["norms", "score_topk", "combine_softmax", "gate_gemm", "gather",
                           "out_gemm"], [round(statistics.mean(p) * 1e3, 2) for p in phase_ms]))
        sel = selection_roofline(w, statistics.mean(phase_ms[1]) + statistics.mean(phase_ms[2]),
                                 peaks, peak_kind,
                                 traffic_record(rec_key + ":select") if rec_key else None)
    else:  # graph replay: only whole steps are timed
        achieved = bytes_per_launch / (ms_per_step / 1e3) / 1e9
        roof = {"kernel": "whole step (graph replay)", "bound": "hbm",
                "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                "frac": round(achieved / peak, 4), "peak_source": f"{peak_kind} hbm_gbs",
                "algorithmic_bytes_per_launch": bytes_per_launch, "traffic": traffic}
        phases = None
    extra = {}
    if sel is not None:
        extra["roofline_select"] = sel
    if args.workload == "decode":
        extra["decode"] = decode_report(skv, w, inp, kw, out, idx, wts, ws, step_ms, K,
                                        bytes_per_launch, peak, peak_kind)
    if args.shards > 1 and not train and not w.memplus and graph is None:
        extra["row_sharded_compute"] = time_sharded_compute(skv, inp, w, args.shards, flush,
                                                            peak, peak_kind)
    if train:
        # the lookup's backward (after the Memory+ part, if any) against HBM
        bwd_ms = statistics.mean([b[2].elapsed_time(b[1]) for b in bev])
        U = int(n_uniq.item())
        bbytes = backward_bytes(w, U)
        extra["backward"] = {"us": round(bwd_ms * 1e3, 1), "distinct_rows": U,
                             "algorithmic_bytes": bbytes,
                             "GBps": round(bbytes / (bwd_ms / 1e3) / 1e9, 1),
                             "frac": round(bbytes / (bwd_ms / 1e3) / 1e9 / peak, 4)}
        # the kernels' own DRAM and L2 bytes (ncu record): repeated (Zipf-hot)
        # rows are L2 hits, so DRAM moves well under the algorithmic bytes; the
        # L2 bytes are reported without a time floor (no library-independent
        # L2 copy reaches the L2 throughput these kernels reach)
        rec = traffic_entry(rec_key + ":backward") if rec_key else None
        if rec:
            db, lb = rec["dram_bytes_per_launch"], rec["l2_bytes_per_launch"]
            extra["backward"].update(
                dram_bytes=db, dram_GBps=round(db / (bwd_ms / 1e3) / 1e9, 1),
                dram_frac=round(db / (bwd_ms / 1e3) / 1e9 / peak, 4),
                hbm_bound_us=round(db / (peak * 1e9) * 1e6, 1),
                l2_bytes=lb, l2_GBps=round(lb / (bwd_ms / 1e3) / 1e9, 1),
                traffic_capture=rec["capture"])
        if mp_train:
            # five GEMMs of 2*T*d_model*d_v FLOPs: a, dz, dx, dW1, dW2
            mp_ms = statistics.mean([b[0].elapsed_time(b[2]) for b in bev])
            flops = 5 * 2 * T * w.d_model * w.d_v
            tf = flops / (mp_ms / 1e3) / 1e12
            pk = float(peaks["bf16_tflops"])
            extra["memplus_backward"] = {"us": round(mp_ms * 1e3, 1), "flops": flops,
                                         "TFLOPs": round(tf, 1), "peak": pk,
                                         "frac": round(tf / pk, 4),
                                         "peak_source": f"{peak_kind} bf16_tflops"}

    if train:
        # the step's dominant work is the lookup backward, so the roofline
        # reports it; the gather's figure over-counts there, since Zipf-skewed
        # rows repeat and the repeats hit L2
        b = extra["backward"]
        extra["gather"] = dict(roof, note="Zipf-skewed rows repeat across tokens; repeated "
                                          "rows are L2 hits, so algorithmic bytes over-count DRAM")
        roof = {"kernel": "pkm_backward (sort, segmented value-gradient sum, dw/dS, dq, dK)",
                "bound": "hbm", "achieved": b["GBps"], "peak": peak, "unit": "GB/s",
                "frac": b["frac"], "peak_source": f"{peak_kind} hbm_gbs",
                "algorithmic_bytes_per_launch": b["algorithmic_bytes"],
                "traffic": b.get("dram_bytes"), "backward_us": b["us"]}

    if train:
        # optimiser step on the touched rows (not part of the timed training
        # step): touched-rows Adam with fp32 moments on the backward's sparse
        # gradient, applied to the table in place after everything else
        moments = 2 * w.N * w.d_v * 4
        if moments <= 40 * 2 ** 30:
            extra["optimizer"] = time_sparse_adam(skv, inp["values"], uniq, grad, n_uniq, U, w,
                                                  peak, peak_kind)
        else:
            extra["optimizer"] = {"skipped": f"Adam moments would take {moments / 2**30:.0f} GiB"}

    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, w, inp, kw, out, idx, wts, ws, flush, world, use_graph=use_graph,
                      backward=(lambda: (
                          skv.check(lib.pkm_memplus_backward(skv.ctypes.byref(margs), sptr),
                                    "pkm_memplus_backward") if mp_train else None,
                          skv.check(lib.pkm_backward(skv.ctypes.byref(bargs), sptr),
                                    "pkm_backward"))) if train else None)

    clocks = clk.summary()
    l2 = "256 MiB L2 flush write before every timed step" if flush_between else \
        "decode steps back to back: the value table (32 GiB) exceeds L2, the sub-keys stay " \
        "L2-resident as in a decode loop"
    res = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world,
        "steps": K, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": w.dtype, "data": "synthetic (seeded generators; no dataset)",
        "config": dict(w.describe(), l2=l2, graph=bool(graph is not None),
                       step="forward + backward" if train else "forward",
                       parallelism=f"replicas x{world}: one token batch per GPU, tables "
                                   f"replicated, no data-path collective"),
        "roofline": roof, "phases_us": phases,
        "gather_GBps": round(achieved, 1), "clocks": clocks,
        "gpu_launches": int(launches), "e2e": e2e, **extra,
    }
    return res, w, inp


def selection_flops(w) -> int:
    """Sub-key scoring FLOPs of one forward: every token, head and half
    against its n_sub sub-keys, 2 d_half FLOPs each (the tensor-core work)."""
    return 2 * w.T * w.H * 2 * w.n_sub * w.d_half


def selection_roofline(w, sel_ms: float, peaks, peak_kind, traffic=None):
    """The selection (sub-key norms and the selection kernel(s)) against the
    measured bf16 tensor peak: the scoring GEMM is its dense contraction.
    `traffic`: the selection kernel's DRAM bytes per launch from the committed
    ncu summary (None when its source changed since the capture)."""
    flops = selection_flops(w)
    tf = flops / (sel_ms / 1e3) / 1e12
    pk = float(peaks["bf16_tflops"])
    return {"kernel": "select_tc_kernel (query norms, scoring, per-half top-k, k x k combine, "
                      "softmax) after the sub-key norms", "bound": "tensor",
            "achieved": round(tf, 1), "peak": pk, "unit": "TFLOP/s", "frac": round(tf / pk, 4),
            "peak_source": f"{peak_kind} bf16_tflops", "flops_per_launch": flops,
            "traffic": traffic, "select_us": round(sel_ms * 1e3, 2)}


def dist_stats(ms):
    """mean / p50 / p99 of per-step times (ms) in microseconds."""
    us = sorted(x * 1e3 for x in ms)
    pick = lambda q: us[min(len(us) - 1, int(round(q * (len(us) - 1))))]  # noqa: E731
    return {"mean": round(statistics.mean(us), 2), "p50": round(pick(0.5), 2),
            "p99": round(pick(0.99), 2), "steps": len(us)}


def decode_report(skv, w, inp, kw, out, idx, wts, ws, graph_step_ms, K, gather_bytes, peak,
                  peak_kind):
    """Decode steps: the per-step time distribution with the CUDA graph (the
    timed steps, back to back) and without it (eager launches), and the bag
    gather's own time and GB/s in both.  In the graph the library's phase
    events are recorded as event nodes, read after each replay."""

    def phase_events():
        ev = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(7)]
        for e in ev:
            e.record()
        torch.cuda.synchronize()
        return ev

    def fwd(ev):
        skv.pkm_forward(inp["query"], inp["subkeys"], inp["values"], w.k, out=out, idx=idx,
                        weights=wts, workspace=ws, phase_events=ev, **kw)

    eager_ms, eager_gather = [], []
    eager_phases = [[] for _ in range(6)]
    ev = phase_events()
    for i in range(K + 3):
        fwd(ev)
        torch.cuda.synchronize()
        if i >= 3:
            eager_ms.append(ev[0].elapsed_time(ev[6]))
            eager_gather.append(ev[4].elapsed_time(ev[5]))
            for j in range(6):
                eager_phases[j].append(ev[j].elapsed_time(ev[j + 1]))
    gev = phase_events()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fwd(gev)
    graph_gather = []
    for i in range(K + 3):
        g.replay()
        torch.cuda.synchronize()
        if i >= 3:
            graph_gather.append(gev[4].elapsed_time(gev[5]))
    del g
    assert skv.device_error() == 0
    ge, gg = statistics.mean(eager_gather), statistics.mean(graph_gather)
    names = ["norms", "score_topk", "combine_softmax", "gate_gemm", "gather", "out_gemm"]
    return {"step_us_graph": dist_stats(graph_step_ms), "step_us_eager": dist_stats(eager_ms),
            "phases_us_eager": {nm: round(statistics.mean(v) * 1e3, 2)
                                for nm, v in zip(names, eager_phases)},
            "gather_bytes_per_step": gather_bytes,
            "gather_us_graph": round(gg * 1e3, 2),
            "gather_GBps_graph": round(gather_bytes / (gg / 1e3) / 1e9, 1),
            "gather_us_eager": round(ge * 1e3, 2),
            "gather_GBps_eager": round(gather_bytes / (ge / 1e3) / 1e9, 1),
            "peak": peak, "peak_source": f"{peak_kind} hbm_gbs",
            "note": "graph steps timed back to back (events outside the graph); the gather's "
                    "time in the graph from the library's phase events, recorded as graph "
                    "event nodes, one replay at a time"}


def time_sharded_compute(skv, inp, w, S, flush, peak, peak_kind, reps=20):
    """The compute of one row-sharded step with all S shards on this GPU:
    the selection (pkm_select) and each shard's fp32 partial bags over all
    tokens (embbag_forward_range); the all-gather and reduce-scatter between
    them are not timed (they need S GPUs).  Bytes: every selected row read
    once (by its owner), ids and weights read by every shard, the S fp32
    partial outputs written."""
    from sparse_key_value_b200.sharded import shard_rows

    T, B = w.T, w.H * w.k
    N = inp["values"].shape[0]
    idx = torch.empty(T, w.H, w.k, dtype=torch.int32, device="cuda")
    wts = torch.empty(T, w.H, w.k, dtype=torch.float32, device="cuda")
    parts = torch.empty(S, T, w.d_v, dtype=torch.float32, device="cuda")
    shares = [shard_rows(N, S, r) for r in range(S)]
    sel, gat = [], []
    for i in range(reps + 3):
        flush.zero_()
        e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        e[0].record()
        skv.pkm_select(inp["query"], inp["subkeys"], w.k, d_v=w.d_v, idx=idx, weights=wts)
        e[1].record()
        for r, (lo, n) in enumerate(shares):
            skv.embbag_forward_range(inp["values"][lo:lo + n], lo, idx.view(T, B),
                                     wts.view(T, B), out=parts[r])
        e[2].record()
        torch.cuda.synchronize()
        if i >= 3:
            sel.append(e[0].elapsed_time(e[1]))
            gat.append(e[1].elapsed_time(e[2]))
    assert skv.device_error() == 0
    g_ms = statistics.mean(gat)
    nbytes = T * B * w.d_v * w.elem_bytes + S * T * B * 8 + S * T * w.d_v * 4
    return {"shards": S, "select_us": round(statistics.mean(sel) * 1e3, 1),
            "partial_gathers_us": round(g_ms * 1e3, 1), "algorithmic_bytes": nbytes,
            "GBps": round(nbytes / (g_ms / 1e3) / 1e9, 1),
            "frac": round(nbytes / (g_ms / 1e3) / 1e9 / peak, 4),
            "peak_source": f"{peak_kind} hbm_gbs",
            "note": "all shards on one GPU; the exchange between the steps is not timed"}


def run_sharded(args, rank, world, local, select=None, gather=None, device="cuda"):
    """The row-sharded step (sparse_key_value_b200.sharded): every rank holds
    ceil(N / world) rows of the value table and the replicated sub-keys,
    selects the rows of its own T tokens, and the ranks all-gather the
    selections, sum the partial bags of the rows they hold for every rank's
    tokens and reduce-scatter them (NCCL).  Weak scaling: T tokens per rank.
    The Memory+ GEMMs are not part of this step.  ``select`` / ``gather`` /
    ``device`` are for host tests of the step order (gloo ranks, injected
    reference steps); the benchmark uses the CUDA library."""
    from sparse_key_value_b200.inputs import WORKLOADS, make_inputs, value_shard
    from sparse_key_value_b200.sharded import (LocalComm, TorchComm, exchange_bytes, shard_rows,
                                               sharded_lookup)

    w = args.workload_obj if hasattr(args, "workload_obj") else WORKLOADS[args.workload]
    w = rank_workload(w, rank)
    if device == "cuda":
        import sparse_key_value_b200 as skv
        skv.load()
    inp = make_inputs(w, device, with_values=False)
    lo, n_local = shard_rows(w.N, world, rank)
    shard = value_shard(w, n_local, rank, device)
    comm = TorchComm() if world > 1 else LocalComm()
    cuda = device == "cuda"
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device) if cuda else None

    def step():
        return sharded_lookup(inp["query"], inp["subkeys"], shard, w.k, lo, comm, select, gather)

    for _ in range(args.warmup):
        if cuda:
            flush.zero_()
        step()
    if cuda:
        torch.cuda.synchronize()
    barrier(world)
    K = args.steps
    ms = []
    clk = Clocks(local) if cuda else None
    if clk is not None:
        clk.__enter__()
    for _ in range(K):
        if cuda:
            flush.zero_()  # L2 flush between timed steps (outside the events)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            y, _, _ = step()
            e1.record()
            e1.synchronize()
            ms.append(e0.elapsed_time(e1))
        else:
            t0 = time.perf_counter()
            y, _, _ = step()
            ms.append((time.perf_counter() - t0) * 1e3)
    if clk is not None:
        clk.__exit__(None, None, None)
    barrier(world)
    total = max_over_ranks(sum(ms), world)
    ms_per_step = total / K
    value = whole_job_tokens_per_s(w.T, world, ms_per_step)
    B = w.H * w.k
    # per rank: its shard's rows of every rank's bags (world*T*B rows spread over world
    # shards: T*B in expectation), every rank's ids and weights, the fp32 partials written
    hbm = w.T * B * w.d_v * w.elem_bytes + world * w.T * B * 8 + world * w.T * w.d_v * 4
    return {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world,
        "steps": K, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": w.dtype,
        "data": "synthetic (seeded generators; no dataset)",
        "config": dict(w.describe(), step="row-sharded lookup (selection, all-gather, partial "
                                          "bags, reduce-scatter); no Memory+ GEMMs",
                       rows_per_rank=n_local, l2="256 MiB L2 flush write before every step",
                       parallelism=f"value table row-sharded x{world}, sub-keys replicated, "
                                   f"{w.T} tokens per rank"),
        "exchange_bytes_per_rank": exchange_bytes(w.T, w.H, w.k, w.d_v, world),
        "hbm_bytes_per_rank": hbm, "y_shape": list(y.shape),
        "clocks": clk.summary() if clk is not None else None,
        "cpu_baseline": None, "e2e": None,
    }


def launcher_check(rank, world):
    """Every rank joined the process group: the sum of the ranks over it."""
    total = 0.0
    if world > 1:
        dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
        if dev == "cuda":
            torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
        t = torch.tensor([float(rank)], device=dev)
        torch.distributed.all_reduce(t)
        total = float(t.item())
    return {"launcher_check": True, "n_gpus": world, "rank_sum": total}


def time_sparse_adam(skv, table, rows, grads, count, U, w, peak, peak_kind, reps=10):
    """CUDA-event time of pkm_sparse_optimizer_step (Adam) on U touched rows.
    Algorithmic bytes per row: gradient read (4 d), parameter read and write
    (2 b d), both moments read and written (16 d)."""
    m = torch.zeros(table.shape[0], table.shape[1], dtype=torch.float32, device="cuda")
    v = torch.zeros_like(m)
    e = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    skv.sparse_optimizer_step(table, rows, grads, count, lr=1e-3, kind="adam", m=m, v=v, step=1)
    torch.cuda.synchronize()
    e[0].record()
    for i in range(reps):
        skv.sparse_optimizer_step(table, rows, grads, count, lr=1e-3, kind="adam", m=m, v=v,
                                  step=i + 2)
    e[1].record()
    torch.cuda.synchronize()
    us = e[0].elapsed_time(e[1]) * 1e3 / reps
    nbytes = U * w.d_v * (4 + 2 * w.elem_bytes + 16)
    gbps = nbytes / (us / 1e6) / 1e9
    del m, v
    return {"kind": "adam (touched rows)", "us": round(us, 1), "rows": U, "bytes": nbytes,
            "GBps": round(gbps, 1), "frac": round(gbps / peak, 4),
            "peak_source": f"{peak_kind} hbm_gbs"}


def run_e2e(args, w, inp, kw, out, idx, wts, ws, flush, world, backward=None, use_graph=False):
    """Same metric through the public API with host buffers: every step
    copies the step's query (and x, and for training dy) from pinned host
    memory, runs the step and copies the output back.  The copies run on
    their own streams with two device buffers, so the host-to-device copy of
    step i+1 and the device-to-host copy of step i-1 overlap the compute of
    step i (each step still moves all its bytes inside the timed region).
    With `use_graph` (decode) the step's forward on each buffer is a CUDA
    graph captured once from the same calls and replayed every step."""
    import sparse_key_value_b200 as skv

    hq = inp["query"].cpu().pin_memory()
    hx = inp["x"].cpu().pin_memory() if w.memplus else None
    hdy = inp["dy"].cpu().pin_memory() if backward is not None else None
    hout = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
    dq = [torch.empty_like(inp["query"]) for _ in range(2)]
    dx = [torch.empty_like(inp["x"]) for _ in range(2)] if w.memplus else None
    ddy = [torch.empty_like(inp["dy"]) for _ in range(2)] if hdy is not None else None
    dout = [out, torch.empty_like(out)]
    comp = torch.cuda.current_stream()
    h2d, d2h = torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()  # noqa: E731
    loaded = [ev(), ev()]  # inputs of buffer b on the device
    used = [ev(), ev()]    # the compute that read buffer b's inputs has run
    done = [ev(), ev()]    # output b computed
    drained = [ev(), ev()]  # output b copied to the host
    for e in used + drained:
        e.record(comp)

    def forward(b):
        kw2 = dict(kw)
        if dx is not None:
            kw2["x"] = dx[b]
        skv.pkm_forward(dq[b], inp["subkeys"], inp["values"], w.k, out=dout[b], idx=idx,
                        weights=wts, workspace=ws, **kw2)

    graphs = None
    if use_graph and backward is None:
        for b in range(2):  # eager calls first (workspace lookups happen outside capture)
            forward(b)
        torch.cuda.synchronize()
        graphs = []
        for b in range(2):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                forward(b)
            graphs.append(g)
        torch.cuda.synchronize()

    def step(i):
        b = i % 2
        h2d.wait_event(used[b])
        with torch.cuda.stream(h2d):
            dq[b].copy_(hq, non_blocking=True)
            if dx is not None:
                dx[b].copy_(hx, non_blocking=True)
            if ddy is not None:
                ddy[b].copy_(hdy, non_blocking=True)
        loaded[b].record(h2d)
        comp.wait_event(loaded[b])
        comp.wait_event(drained[b])
        if ddy is not None:
            inp["dy"].copy_(ddy[b])  # the backward reads dy from its fixed buffer
        if graphs is not None:
            graphs[b].replay()
        else:
            forward(b)
        used[b].record(comp)
        if backward is not None:
            backward()
        done[b].record(comp)
        d2h.wait_event(done[b])
        with torch.cuda.stream(d2h):
            hout[b].copy_(dout[b], non_blocking=True)
        drained[b].record(d2h)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    K = args.steps
    barrier(world)
    flush.zero_()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(h2d)
    for i in range(K):
        step(i)
    comp.wait_stream(d2h)
    e1.record(comp)
    e1.synchronize()
    tot = max_over_ranks(e0.elapsed_time(e1), world)
    ms = tot / K
    nbytes = lambda t: t.numel() * t.element_size()  # noqa: E731
    h2d_b = sum(nbytes(t) for t in (hq, hx, hdy) if t is not None)
    d2h_b = nbytes(hout[0])
    res = {"value": round(world * w.T / (ms / 1e3), 1), "unit": UNIT,
           "h2d_bytes_per_step": h2d_b, "d2h_bytes_per_step": d2h_b, "ms_per_step": round(ms, 4),
           "pipeline": "host-to-device copies, compute and device-to-host copies on three "
                       "streams with two device buffers; one timed region over all steps"
                       + ("; the forward replayed from a CUDA graph per buffer"
                          if graphs is not None else "")}
    del graphs
    return res


# ---------------------------------------------------------- Engram lookup --

def engram_bytes_per_token(w) -> int:
    """Algorithmic bytes of the Engram lookup per token: one row per head,
    the hidden-state row, the output row, the gate value and the token id."""
    b = w.elem_bytes
    return w.heads * w.d * b + 2 * w.d * b + 4 + 4


def run_engram(args, rank, world, local):
    """The Engram lookup (hash, gather of one row per head, context gate) on
    the engram workload: one kernel per step, timed with CUDA events."""
    import sparse_key_value_b200 as skv
    from sparse_key_value_b200.inputs import ENGRAM, make_engram_inputs

    lib = skv.load()
    w = ENGRAM.scaled(seed=ENGRAM.seed + 7919 * rank)  # own tokens per rank, same tables
    if args.engram_rows > 0:
        w = w.scaled(rows_per_head=(args.engram_rows,) * w.heads)
    inp = make_engram_inputs(w, "cuda")
    T, d = w.T, w.d
    v = torch.empty(T, d, dtype=w.torch_dtype, device="cuda")
    alpha = torch.empty(T, dtype=torch.float32, device="cuda")
    od = (skv.ctypes.c_int32 * len(w.orders))(*w.orders)
    sd = (skv.ctypes.c_uint64 * w.heads)(*w.seeds)
    md = (skv.ctypes.c_int64 * w.heads)(*w.rows_per_head)
    cp = lambda a: skv.ctypes.cast(a, skv.ctypes.c_void_p)  # noqa: E731
    eargs = skv._lib.EngramArgs(w.n_seq, w.L, len(w.orders), w.K, cp(od), cp(sd), cp(md), d,
                                1 if w.dtype == "bf16" else 0, skv._p(inp["tokens"]),
                                skv._p(inp["table"]), skv._p(inp["h"]), skv._p(v),
                                skv._p(alpha), None, None)
    stream = torch.cuda.current_stream()
    sptr = skv.ctypes.c_void_p(stream.cuda_stream)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")

    def step():
        skv.check(lib.pkm_engram_forward(skv.ctypes.byref(eargs), sptr), "pkm_engram_forward")

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    assert skv.device_error() == 0
    K = args.steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(K)]
    barrier(world)
    torch.cuda.synchronize()
    launches0 = lib.pkm_launch_count()
    with Clocks(local) as clk:
        for e0, e1 in ev:
            flush.zero_()  # L2 flush between timed steps (outside the events)
            e0.record()
            step()
            e1.record()
        torch.cuda.synchronize()
    launches = lib.pkm_launch_count() - launches0
    barrier(world)
    ms = [e0.elapsed_time(e1) for e0, e1 in ev]
    total_ms = max_over_ranks(sum(ms), world)
    ms_per_step = total_ms / K
    value = whole_job_tokens_per_s(T, world, ms_per_step)
    peaks, peak_kind = measured_peaks()
    peak = float(peaks["hbm_gbs"])
    per_launch = engram_bytes_per_token(w) * T
    kern_ms = statistics.mean(ms)  # one launch per step: the step is the kernel
    achieved = per_launch / (kern_ms / 1e3) / 1e9
    roof = {"kernel": "engram_kernel (hash + gather + context gate)", "bound": "hbm",
            "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
            "frac": round(achieved / peak, 4), "peak_source": f"{peak_kind} hbm_gbs",
            "algorithmic_bytes_per_launch": per_launch, "traffic": None,
            "kernel_us": round(kern_ms * 1e3, 2)}

    e2e = None
    if not args.no_e2e:
        htok = inp["tokens"].cpu().pin_memory()
        hh = inp["h"].cpu().pin_memory()
        hv = torch.empty(v.shape, dtype=v.dtype).pin_memory()
        ha = torch.empty(alpha.shape, dtype=alpha.dtype).pin_memory()
        tok_d, h_d = torch.empty_like(inp["tokens"]), torch.empty_like(inp["h"])

        def e2e_step():
            tok_d.copy_(htok, non_blocking=True)
            h_d.copy_(hh, non_blocking=True)
            r = skv.engram_forward(tok_d, inp["table"], h_d, w.orders, w.K, w.seeds,
                                   w.rows_per_head, out=v)
            hv.copy_(r["v"], non_blocking=True)
            ha.copy_(r["alpha"], non_blocking=True)

        for _ in range(args.warmup):
            e2e_step()
        torch.cuda.synchronize()
        tot = 0.0
        barrier(world)
        for _ in range(K):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            e2e_step()
            e1.record()
            e1.synchronize()
            tot += e0.elapsed_time(e1)
        tot = max_over_ranks(tot, world)
        e2e = {"value": round(world * T / (tot / K / 1e3), 1), "unit": UNIT,
               "h2d_bytes_per_step": htok.numel() * 4 + hh.numel() * hh.element_size(),
               "d2h_bytes_per_step": hv.numel() * hv.element_size() + ha.numel() * 4,
               "ms_per_step": round(tot / K, 4)}
    assert skv.device_error() == 0
    res = {
        "metric": "engram lookup tokens/s", "value": round(value, 1), "unit": UNIT,
        "n_gpus": world, "steps": K, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": w.dtype,
        "data": "synthetic (seeded generators; no dataset)",
        "config": dict(w.describe(), l2="256 MiB L2 flush write before every timed step",
                       step="forward", parallelism=f"replicas x{world}: one token batch per "
                                                   f"GPU, tables replicated"),
        "roofline": roof, "clocks": clk.summary(), "gpu_launches": int(launches), "e2e": e2e,
    }
    return res, w, inp


def engram_oracle_seconds(w, inp, tokens, min_seconds: float = 0.0):
    """Seconds of oracle work per pass over ``tokens`` for the Engram
    lookup: the hashed rows of the whole batch (scaled to the sample) plus
    the gate of the sampled tokens, repeated until ``min_seconds`` of work
    have been timed.  Table rows are fetched from the device once, before
    the timing.  Returns (seconds per pass, threads)."""
    import numpy as np

    import oracle

    tok = inp["tokens"].cpu().numpy()
    rows = oracle.engram_rows(tok, w.orders, w.K, w.seeds, w.rows_per_head)
    sel = rows[np.asarray(tokens)]
    uniq, inv = np.unique(sel, return_inverse=True)
    E = inp["table"][torch.from_numpy(uniq).to(inp["table"].device)].cpu()
    h = inp["h"][torch.as_tensor(tokens).to(inp["h"].device)].cpu()
    inv = inv.reshape(sel.shape)
    passes, secs = 0, 0.0
    while passes == 0 or secs < min_seconds:
        t0 = time.perf_counter()
        oracle.engram_rows(tok, w.orders, w.K, w.seeds, w.rows_per_head)
        t_rows = (time.perf_counter() - t0) * len(tokens) / w.T
        t0 = time.perf_counter()
        oracle.engram_gate(inv, E, h)
        secs += t_rows + time.perf_counter() - t0
        passes += 1
    return secs / passes, oracle.num_threads()


def engram_cpu_baseline(args, w, inp):
    import oracle

    oracle.build()
    tokens = list(range(w.T))
    target = args.cpu_seconds / 2
    per_pass, cores = engram_oracle_seconds(w, inp, tokens, min_seconds=target)
    return {"value": round(w.T / per_pass, 2), "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"all {w.T} tokens of the engram workload, passes repeated for about "
                      f"{target:.0f} s; fp64 hash + gather + gate ({per_pass:.3f} s per pass)"}


# --------------------------------------------------------- oracle timing --

def oracle_tokens_per_s(w, inp, tokens, values_dev):
    """Run the CPU oracle (selection, bag, Memory+) on ``tokens``; returns
    (seconds of oracle work, threads).  Value rows are fetched from the
    device table between the oracle's steps (not timed)."""
    import numpy as np

    import oracle

    q = inp["query"][tokens].cpu()
    K = inp["subkeys"].cpu()
    t0 = time.perf_counter()
    idx, S, wt, _ = oracle.pkm_select(q, K, w.k)
    t_sel = time.perf_counter() - t0
    rows = np.unique(idx)
    dev = values_dev.device
    table = values_dev[torch.from_numpy(rows).to(dev)].cpu()
    pos = np.searchsorted(rows, idx).reshape(len(tokens), -1)
    t0 = time.perf_counter()
    y = oracle.bag(pos, wt.reshape(len(tokens), -1), table)
    if w.memplus:
        oracle.memplus(y, inp["x"][tokens].cpu(), inp["W1"].cpu(), inp["W2"].cpu())
    t_rest = time.perf_counter() - t0
    return t_sel + t_rest, oracle.num_threads()


def cpu_baseline(args, w, inp):
    """The oracle as it stands, on a bounded token sample (about
    --cpu-seconds of CPU work)."""
    import oracle

    oracle.build()
    T = w.T
    m, secs = 4, 0.0
    while True:
        tokens = torch.arange(m) * (T // m)
        secs, cores = oracle_tokens_per_s(w, inp, tokens, inp["values"])
        if secs >= args.cpu_seconds / 4 or m >= T:
            break
        m = min(T, m * max(2, int(args.cpu_seconds / 4 / max(secs, 1e-3))))
    return {"value": round(m / secs, 2), "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{m} of {T} tokens (evenly spaced) of the {w.name} workload; "
                      f"fp64 selection + bag{' + Memory+' if w.memplus else ''}; "
                      f"{secs:.2f} s"}


# ---------------------------------------------------------- reference arm --

def run_reference(args, rank, world):
    """The oracle on the host cores as the reference arm (rank 0 only)."""
    if rank != 0:
        return None
    import oracle
    from sparse_key_value_b200.inputs import WORKLOADS, make_inputs

    oracle.build()
    if args.workload == "engram":
        return engram_reference(args, world)
    w = WORKLOADS[args.workload]
    if args.workload == "decode":
        w = w.scaled(T=8)
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    inp = make_inputs(w, dev)
    per_step = min(w.T, 64)  # tokens per step: the per-call set-up is amortised
    spacing = max(1, w.T // (per_step * max(1, args.steps + args.warmup)))
    times, cores = [], 1
    for i in range(args.warmup + args.steps):
        tokens = (torch.arange(per_step) * spacing * (args.steps + args.warmup) + i * spacing) % w.T
        s, cores = oracle_tokens_per_s(w, inp, tokens, inp["values"])
        if i >= args.warmup:
            times.append(s)
    sec = sum(times) / len(times)
    value = per_step / sec
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 2), "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(sec * 1e3, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded generators; no dataset)",
        "config": dict(w.describe(), parallelism="host cores of rank 0"),
        "cpu_baseline": {"value": round(value, 2), "unit": UNIT, "cores": cores,
                         "kind": "oracle",
                         "sample": f"{per_step} tokens per step of the {w.name} workload"},
        "e2e": {"value": round(value, 2), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def engram_reference(args, world):
    """The Engram oracle on the host cores, 256 tokens per step."""
    from sparse_key_value_b200.inputs import ENGRAM, make_engram_inputs

    w = ENGRAM
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    inp = make_engram_inputs(w, dev)
    per_step = 256
    times, cores = [], 1
    n = args.warmup + args.steps
    for i in range(n):
        tokens = [(j * n + i) * (w.T // (per_step * n)) % w.T for j in range(per_step)]
        s, cores = engram_oracle_seconds(w, inp, tokens)
        if i >= args.warmup:
            times.append(s)
    sec = sum(times) / len(times)
    value = per_step / sec
    return {
        "impl": "reference", "metric": "engram lookup tokens/s", "value": round(value, 2),
        "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(sec * 1e3, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded generators; no dataset)",
        "config": dict(w.describe(), parallelism="host cores of rank 0"),
        "cpu_baseline": {"value": round(value, 2), "unit": UNIT, "cores": cores,
                         "kind": "oracle", "sample": f"{per_step} tokens per step of the "
                                                      f"engram workload"},
        "e2e": {"value": round(value, 2), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def run_select_only(args):
    """The selection alone on the workload's queries and sub-keys (no value
    table is allocated): a small-footprint command for kernel captures.  Its
    line reports the selection's time per launch, not the lookup metric."""
    import sparse_key_value_b200 as skv
    from sparse_key_value_b200.inputs import WORKLOADS, make_inputs

    skv.load()
    w = WORKLOADS[args.workload]
    if args.n_sub > 0:
        w = w.scaled(n_sub=args.n_sub)
    if args.tokens > 0:
        w = w.scaled(T=args.tokens)
    inp = make_inputs(w, "cuda", with_values=False)
    idx = torch.empty(w.T, w.H, w.k, dtype=torch.int32, device="cuda")
    wts = torch.empty(w.T, w.H, w.k, dtype=torch.float32, device="cuda")

    def once():
        skv.pkm_select(inp["query"], inp["subkeys"], w.k, d_v=w.d_v, idx=idx, weights=wts)

    for _ in range(args.warmup):
        once()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        once()
    e1.record()
    torch.cuda.synchronize()
    err = skv.device_error()
    if err:
        raise SystemExit(f"bench.py --select-only: device status {err}")
    return {"metric": "selection time per launch (profiling aid)",
            "value": round(e0.elapsed_time(e1) * 1e3 / max(1, args.steps), 2), "unit": "us",
            "higher_is_better": False, "steps": args.steps, "warmup": args.warmup,
            "config": {"workload": args.workload, "select_only": True, **w.describe()}}


def main():
    args = parse()
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        sys.exit(relaunch(args.gpus))
    rank, world, local = dist_setup(args)
    try:
        if args.launcher_check:
            res = launcher_check(rank, world)
        elif args.impl == "reference":
            res = run_reference(args, rank, world)
        elif args.sharded:
            res = run_sharded(args, rank, world, local)
        elif args.select_only:
            if args.workload in ("engram", "tiny") or world > 1:
                raise SystemExit("bench.py: --select-only is for one GPU and the product-key "
                                 "workloads with bf16 tensor-core selection")
            res = run_select_only(args)
        elif args.workload == "engram":
            res, w, inp = run_engram(args, rank, world, local)
            res["cpu_baseline"] = engram_cpu_baseline(args, w, inp) \
                if rank == 0 and world == 1 and not args.no_cpu_baseline else None
        else:
            res, w, inp = run_ours(args, rank, world, local)
            if rank == 0 and world == 1 and not args.no_cpu_baseline:
                res["cpu_baseline"] = cpu_baseline(args, w, inp)
            else:
                res["cpu_baseline"] = None
        if rank == 0 and res is not None:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1 and torch.distributed.is_initialized():
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
