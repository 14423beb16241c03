"""Benchmark: one decode step = one pa_kv_append_decode launch (append + decode) over one batch.

Default workload: the Qwen3-8B-shaped heavy mixed batch (B=256, Hq=32, Hkv=8,
D=128, block_size=16, log-normal context lengths with median 1024 clipped to
[16, 16384], the first full blocks of every 8 requests shared, bf16): the
largest of the decode batches.  Metric: paged-decode attention HBM GB/s
(algorithmic bytes of the decode / device time of the step) and us per
decode step.  The algorithmic bytes count every K/V block once (a prefix
block several tables name is read once), plus q, out, block-table entries
and lengths; the append's bytes are reported beside them, not in them.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--config 1..5] [--impl reference]

Timing: inputs resident in HBM; R copies of the whole step's inputs are used
in rotation so that the working set of consecutive steps exceeds the L2
cache; the K timed steps are bracketed by a barrier and a device synchronise
and measured with CUDA events on the launching stream (max over ranks).  The
K-step region is timed several times, so that the timed kernels span at
least --min-timed-ms in total and the clock samples see them; the median
region is reported.  The decode kernel's own duration comes from
back-to-back launches timed the same way.  The other decode batches
(Qwen3-0.6B, Llama-3.2-1B, long-context MQA) are timed in regions of their
own and reported under "workloads".  A further leg times the step behind a
~100 MB copy kernel on the same stream (the decode's predecessor is then not
another decode).  Under torchrun each rank runs its own batch (weak scaling,
no collective on the data path).  The end-to-end leg stages each step's
inputs in one pinned host buffer (one copy in) and reads the output back
(one copy out) around the same C call.

  python bench.py --prefill 1|2 [--steps K] [--warmup W]

times the chunked prefill step instead (pa_kv_append of the new tokens, then
pa_prefill): value = algorithmic causal TFLOP/s, roofline against the
measured bf16 tensor peak, end-to-end leg with the step's inputs copied from
pinned host memory and the output copied back every step.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

FALLBACK_HBM_GBS = 6650.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=4000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--config", type=int, default=5)
    ap.add_argument("--partition", type=int, default=-1, help="-1: the workload's own (0 = balanced)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--e2e-steps", type=int, default=200)
    ap.add_argument("--min-timed-ms", type=float, default=250.0,
                    help="repeat the K-step region until the timed kernels span this long in total")
    ap.add_argument("--extra", default="2,3,4,4:0",
                    help="other decode workloads timed in regions of their own (comma list of C or C:P, "
                         "P = partition tokens, 0 = balanced split; '' = none)")
    ap.add_argument("--copies", type=int, default=0,
                    help="rotating input copies of a decode workload (0: enough to exceed L2 three times; "
                         "1 only for profiler captures, whose passes flush the caches themselves)")
    ap.add_argument("--prefill", type=int, default=0,
                    help="time the chunked prefill step of prefill workload N (1, 2) instead of the decode step")
    ap.add_argument("--dynamic-share", type=int, default=-1,
                    help="balanced split: share of each request's tiles handed out at run time, in 1/256 "
                         "(-1: the planner's choice)")
    return ap.parse_args()


def csrc_hash() -> str:
    h = hashlib.sha256()
    d = os.path.join(ROOT, "paged_kv_cache_472_b200", "csrc")
    for fn in sorted(os.listdir(d)):
        h.update(fn.encode())
        h.update(open(os.path.join(d, fn), "rb").read())
    return h.hexdigest()[:16]


def measured_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


FALLBACK_BF16_TFLOPS = 1590.0


def measured_tensor_peak():
    """Dense bf16 TFLOP/s (cuBLAS, burst: the kernel is timed on its own)."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    except Exception:
        return FALLBACK_BF16_TFLOPS, "fallback"


def profiled_traffic(workload: str):
    """DRAM bytes per launch of the workload's kernel from the committed ncu
    summary, if it was taken on the current kernel sources."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
        ent = rec.get(workload)
        if ent and ent.get("csrc_hash") == csrc_hash():
            return float(ent["dram_bytes_per_launch"])
    except Exception:
        pass
    return None


class ClockSampler:
    """SM clock and throttle reasons sampled with NVML while the timed region runs."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
               0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, index: int, period_s: float = 0.01):
        self.samples, self.reasons, self.ok = [], 0, False
        self.period, self.stop_ev = period_s, threading.Event()
        self.max_mhz = None
        if index < 0:   # sampling off
            return
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.max_mhz = None

    def _run(self):
        nv = self.nv
        while not self.stop_ev.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                self.reasons |= nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self.stop_ev.set()
            self.t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"]}
        names = [n for bit, n in self.REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz, "reasons": names,
                "samples": len(self.samples)}


# ---------------------------------------------------------------------------
# multi-rank host logic (replicas: each rank decodes its own batch, no exchange)
def rank_seed(cid: int, rank: int):
    """Seed of rank `rank`'s batch: rank 0 runs the workload's own seed."""
    return None if rank == 0 else 1000 + cid + 7919 * rank


def max_over_ranks(value: float, world: int, device) -> float:
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput_gbs(step_bytes: int, world: int, ms_step: float) -> float:
    """Whole-job GB/s: every rank moved step_bytes per step."""
    return world * step_bytes / (ms_step * 1e-3) / 1e9


# ---------------------------------------------------------------------------
def cpu_baseline(case, seconds: float):
    """The float64 oracle as it stands (append + decode), on the host cores.

    All cores: whole steps of the batch, repeated for about `seconds`; the
    median of three such runs is the value.  One core: the same oracle with
    one thread on a sample of the batch (every eighth request; the others
    get length 0 and cost nothing), median of three runs.  GB/s counts the
    same algorithmic bytes as the GPU line (for the sample: its own)."""
    import oracle
    from synth import algorithmic_bytes
    orc = oracle.default()
    nbytes = algorithmic_bytes(case)["decode_unique"]
    runs, steps_all = [], 0
    for _ in range(3):
        steps, t0 = 0, time.perf_counter()
        while True:
            kc, vc = orc.kv_append(case)
            orc.decode(case, kc, vc)
            steps += 1
            el = time.perf_counter() - t0
            if el >= seconds / 3:
                break
        runs.append(el / steps)
        steps_all += steps
    sec_all = statistics.median(runs)
    # one core, every eighth request
    lens = case.context_lens.copy()
    keep = np.zeros(case.B, dtype=bool)
    keep[::8] = True
    lens[~keep] = 0
    e = case.elem_bytes
    s_bytes = (int(lens.astype(np.int64).sum()) * case.Hkv * case.D * e * 2 + 2 * int(keep.sum()) * case.Hq * case.D * e)
    kc, vc = orc.kv_append(case)
    one = []
    for _ in range(3):
        t0 = time.perf_counter()
        orc.decode(case, kc, vc, context_lens=lens, nthreads=1)
        one.append(time.perf_counter() - t0)
    sec_one = statistics.median(one)
    return {"value": nbytes / sec_all / 1e9, "unit": "GB/s", "cores": orc.max_threads(), "kind": "oracle",
            "sample": f"median of 3 runs of {steps_all // 3}-{steps_all - steps_all // 3 * 2} full steps (append + "
                      f"decode of all {case.B} requests) of {case.name}, {sec_all * 1e3:.1f} ms per step",
            "ms_per_step": sec_all * 1e3,
            "cores_1": {"value": s_bytes / sec_one / 1e9, "unit": "GB/s", "cores": 1,
                        "sample": f"median of 3 single-thread runs over {int(keep.sum())} of {case.B} requests "
                                  f"(every eighth), {sec_one:.2f} s each"}}


def run_reference(args):
    import synth
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    case = synth.make_config(args.config)
    from synth import algorithmic_bytes
    base = cpu_baseline(case, max(args.cpu_seconds, 1.0) if args.steps else args.cpu_seconds)
    ab = algorithmic_bytes(case)
    line = {"impl": "reference", "metric": "paged-decode attention HBM GB/s (% of B200 peak); us/decode step",
            "value": base["value"], "unit": "GB/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": base["ms_per_step"], "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": case.name, "B": case.B, "Hq": case.Hq, "Hkv": case.Hkv, "D": case.D,
                       "block_size": case.block_size, "bytes_per_step": ab["decode_unique"]},
            "cpu_baseline": {k: base[k] for k in ("kind", "cores", "sample", "value", "unit", "cores_1")},
            "e2e": {"value": base["value"], "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "gpu_launches": 0}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
def run_prefill(args):
    """The chunked prefill step of a prefill workload: pa_kv_append of every
    new token, then pa_prefill.  value = algorithmic causal FLOPs per second."""
    import torch
    import synth
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "_pagedattn_build", os.path.join(ROOT, "paged_kv_cache_472_b200", "build.py"))
    libbuild = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(libbuild)
    libbuild.build()
    import ctypes
    import paged_kv_cache_472_b200 as pa
    from synth.device import to_device

    torch.cuda.set_device(0)
    pc = synth.make_prefill_config(args.prefill)
    alg = synth.prefill_algorithmic(pc)
    dt = {"bf16": pa.DTYPE_BF16, "f16": pa.DTYPE_F16}[pc.dtype]
    shape = pa.Shape(pc.B, pc.Hq, pc.Hkv, pc.D, pc.block_size, pc.num_blocks, pc.max_blocks_per_seq, dt)
    ashape = pa.Shape(pc.T, pc.Hq, pc.Hkv, pc.D, pc.block_size, pc.num_blocks, pc.max_blocks_per_seq, dt)
    plan = pa.pa_prefill_plan(shape, int(pc.new_tokens().max()))
    R = 3
    v = lambda a: to_device(a, pc.dtype, "cuda")
    i32 = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()
    copies = []
    for _ in range(R):
        q = v(pc.q)
        copies.append(dict(q=q, kn=v(pc.k_new), vn=v(pc.v_new), kc=v(pc.k_cache), vc=v(pc.v_cache),
                           bt=i32(pc.block_tables), cl=i32(pc.context_lens), qs=i32(pc.query_start),
                           sm=i32(pc.slot_mapping), out=torch.empty_like(q)))
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    lib, byref = pa.lib, ctypes.byref
    stream = torch.cuda.current_stream()
    sp = stream.cuda_stream

    def step(i, append=True):
        c = copies[i % R]
        if append:
            lib.pa_kv_append(c["kn"].data_ptr(), c["vn"].data_ptr(), c["sm"].data_ptr(), c["kc"].data_ptr(),
                             c["vc"].data_ptr(), byref(ashape), err.data_ptr(), sp)
        return lib.pa_prefill(c["q"].data_ptr(), c["kc"].data_ptr(), c["vc"].data_ptr(), c["bt"].data_ptr(),
                              c["cl"].data_ptr(), c["qs"].data_ptr(), ctypes.c_float(pc.scale), c["out"].data_ptr(),
                              byref(shape), byref(plan), err.data_ptr(), sp)

    for i in range(max(args.warmup, 3)):
        if step(i):
            raise RuntimeError(pa.pa_last_error_message())
    torch.cuda.synchronize()
    K = args.steps
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(0) as clk:
        torch.cuda._sleep(20_000_000)
        e0.record(stream)
        for i in range(K):
            step(i)
        e1.record(stream)
        torch.cuda.synchronize()
    ms_step = e0.elapsed_time(e1) / K
    # the prefill kernel alone, back to back
    torch.cuda._sleep(20_000_000)
    e0.record(stream)
    for i in range(K):
        step(i, append=False)
    e1.record(stream)
    torch.cuda.synchronize()
    ms_kernel = e0.elapsed_time(e1) / K
    # end to end: every step copies its inputs (q, the new tokens' K/V and
    # slots, tables, lengths, row offsets) from pinned host memory and the
    # output back; the KV pool is resident state
    host = {k: copies[0][k].cpu().pin_memory() for k in ("q", "kn", "vn", "sm", "bt", "cl", "qs")}
    host_out = torch.empty(copies[0]["out"].shape, dtype=copies[0]["out"].dtype).pin_memory()

    def e2e_step(i):
        c = copies[i % R]
        for k, t in host.items():
            c[k].copy_(t, non_blocking=True)
        rc = step(i)
        host_out.copy_(c["out"], non_blocking=True)
        return rc

    for i in range(3):
        if e2e_step(i):
            raise RuntimeError(pa.pa_last_error_message())
    torch.cuda.synchronize()
    KE = max(1, min(K, args.e2e_steps))
    torch.cuda._sleep(20_000_000)
    e0.record(stream)
    for i in range(KE):
        e2e_step(i)
    e1.record(stream)
    torch.cuda.synchronize()
    ms_e2e_serial = e0.elapsed_time(e1) / KE

    # the same steps double-buffered over the R device copies: step i+1's
    # inputs go up on one copy stream and step i-1's output comes down on
    # another while step i computes
    up_s, dn_s = torch.cuda.Stream(), torch.cuda.Stream()
    ev_up, ev_k, ev_dn = ([torch.cuda.Event() for _ in range(R)] for _ in range(3))
    host_outs = [host_out] + [torch.empty_like(host_out).pin_memory() for _ in range(R - 1)]

    def e2e_pipelined(i):
        r = i % R
        c = copies[r]
        if i == 0:
            up_s.wait_stream(stream)     # nothing is copied before the start event
        up_s.wait_event(ev_k[r])         # the step that last used copy r is done with it
        with torch.cuda.stream(up_s):
            for k, t in host.items():
                c[k].copy_(t, non_blocking=True)
        ev_up[r].record(up_s)
        stream.wait_event(ev_up[r])
        stream.wait_event(ev_dn[r])      # its previous output has been read back
        rc = step(i)
        ev_k[r].record(stream)
        dn_s.wait_event(ev_k[r])
        with torch.cuda.stream(dn_s):
            host_outs[r].copy_(c["out"], non_blocking=True)
        ev_dn[r].record(dn_s)
        return rc

    torch.cuda._sleep(20_000_000)
    e0.record(stream)
    for i in range(KE):
        e2e_pipelined(i)
    for r in range(R):
        stream.wait_event(ev_dn[r])      # the region ends after the last output is home
    e1.record(stream)
    torch.cuda.synchronize()
    ms_e2e = e0.elapsed_time(e1) / KE
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = host_out.numel() * host_out.element_size()
    if int(err.item()):
        raise RuntimeError(f"device error word {int(err.item()):#x}")
    peak, kind = measured_tensor_peak()
    tflops = alg["flops"] / (ms_step * 1e-3) / 1e12
    k_tflops = alg["flops"] / (ms_kernel * 1e-3) / 1e12
    line = {"metric": "paged chunked-prefill attention TFLOP/s (causal, algorithmic)", "value": round(tflops, 2),
            "unit": "TFLOP/s", "n_gpus": 1, "steps": K, "warmup": args.warmup, "ms_per_step": round(ms_step, 6),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": pc.dtype, "data": "synthetic",
            "config": {"workload": pc.name, "B": pc.B, "new_tokens": pc.T, "Hq": pc.Hq, "Hkv": pc.Hkv, "D": pc.D,
                       "block_size": pc.block_size, "context_tokens": int(pc.context_lens.sum()),
                       "flops_per_step": alg["flops"], "min_bytes_per_step": alg["bytes"],
                       "l2": f"{R} rotating input copies"},
            "roofline": {"bound": "tensor", "achieved": round(k_tflops, 2), "peak": peak, "unit": "TFLOP/s",
                         "frac": round(k_tflops / peak, 4), "traffic": profiled_traffic(pc.name),
                         "kernel": "paged_prefill_kernel",
                         "peak_kind": kind, "kernel_us": round(ms_kernel * 1e3, 3),
                         "engine": "tcgen05.mma, S and O in tensor memory, P split into two 16-bit parts"},
            "e2e": {"value": round(alg["flops"] / (ms_e2e * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "us_per_step": round(ms_e2e * 1e3, 3),
                    "mode": "double-buffered: each step's upload and read-back overlap its neighbours' steps",
                    "serial": {"value": round(alg["flops"] / (ms_e2e_serial * 1e-3) / 1e12, 2),
                               "us_per_step": round(ms_e2e_serial * 1e3, 3),
                               "mode": "upload, step, read-back in order on one stream"}},
            "gpu_launches": 2 * K, "clocks": clk.summary()}
    if not args.no_cpu_baseline:
        import oracle
        orc = oracle.default()
        rng = np.random.default_rng(0)
        rows = np.sort(rng.choice(pc.T, size=min(pc.T, 64), replace=False))
        kc, vc = orc.prefill_append(pc)
        t0 = time.perf_counter()
        orc.prefill_rows(pc, rows, kc, vc)
        el = time.perf_counter() - t0
        pos = pc.positions()
        flops = 4 * int((pos[rows] + 1).sum()) * pc.Hq * pc.D
        line["cpu_baseline"] = {"value": flops / el / 1e12, "unit": "TFLOP/s", "cores": orc.max_threads(),
                                "kind": "oracle", "sample": f"{len(rows)} of {pc.T} new tokens, all heads, {el:.1f} s"}
    print(json.dumps(line), flush=True)


def timed_regions(fn, K: int, stream, min_ms: float, world: int, est_ms_step: float, max_regions: int = 200):
    """Time `fn(i)` for i in 0..K-1 as one region (barrier + synchronise on
    both sides, CUDA events on `stream`), repeated until the regions span
    `min_ms` in total; returns (median region ms, regions, all region ms)."""
    import torch
    import torch.distributed as dist
    n = max(1, min(max_regions, math.ceil(min_ms / max(K * est_ms_step, 1e-3))))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    times = []
    base = 0
    for _ in range(n):
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        torch.cuda._sleep(int(min(50e6, 2e6 + K * 40_000)))   # keep the host ahead of the GPU (not timed)
        e0.record(stream)
        for i in range(K):
            fn(base + i)
        e1.record(stream)
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1))
        base += K
    return statistics.median(times), n, times


def decode_workload(cid, args, world, rank, local, stream, lib, pa, extra=False, partition=None):
    """Upload workload `cid` (rank-seeded) in rotating copies and time its
    step (fused append + decode), the decode kernel alone and (main
    workload) the step behind a copy kernel and the end-to-end step."""
    import ctypes
    import torch
    import synth
    from synth import algorithmic_bytes
    from synth.device import shape_fields, upload
    from paged_kv_cache_472_b200.session import PagedDecoder, StepStaging

    case = synth.make_config(cid, seed=rank_seed(cid, rank))
    part = args.partition if partition is None else partition
    pt = case.partition_tokens if part < 0 else part
    ab = algorithmic_bytes(case)
    l2 = torch.cuda.get_device_properties(local).L2_cache_size
    R = max(3, math.ceil(3 * l2 / max(ab["step_total"], 1))) if args.copies <= 0 else args.copies
    copies = [upload(case) for _ in range(R)]
    dec = PagedDecoder(pa.Shape(*shape_fields(case)), int(case.max_blocks_per_seq * case.block_size), pt)
    if args.dynamic_share >= 0 and not extra:
        dec.plan.dynamic_share = args.dynamic_share
    byref = ctypes.byref
    shp, pln = byref(dec.shape), byref(dec.plan)
    ws, wsb = dec.workspace.data_ptr(), dec.workspace.numel()
    ptrs = [(c.k_new.data_ptr(), c.v_new.data_ptr(), c.slot_mapping.data_ptr(), c.k_cache.data_ptr(),
             c.v_cache.data_ptr(), c.q.data_ptr(), c.block_tables.data_ptr(), c.context_lens.data_ptr(),
             c.out.data_ptr()) for c in copies]
    scale = float(case.scale)
    sp = stream.cuda_stream

    def step(i):
        # one decode step through the public C entry point: append + decode in one launch
        kn, vn, sm, kc, vc, q, bt, cl, out = ptrs[i % R]
        return lib.pa_kv_append_decode(kn, vn, sm, q, kc, vc, bt, cl, scale, out, shp, pln, ws, wsb, sp)

    def decode_only(i):
        kn, vn, sm, kc, vc, q, bt, cl, out = ptrs[i % R]
        return lib.pa_decode(q, kc, vc, bt, cl, scale, out, shp, pln, ws, wsb, sp)

    for i in range(max(args.warmup, 3)):
        if step(i):
            raise RuntimeError(pa.pa_last_error_message())
    torch.cuda.synchronize()
    # a first estimate of the step time sizes the number of regions
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(8):
        step(i)
    e1.record(stream)
    torch.cuda.synchronize()
    est = max_over_ranks(e0.elapsed_time(e1) / 8, world, "cuda")   # the same region count on every rank
    K = args.steps
    res = {"case": case, "ab": ab, "R": R, "pt": pt, "dec": dec, "l2": l2}
    KD = max(min(K, 2000), 1)
    # clocks are sampled while the main workload's timed regions run
    with ClockSampler(local if not extra else -1) as clk:
        ms_region, nreg, _ = timed_regions(step, K, stream, args.min_timed_ms, world, est)
        # the decode kernel alone, back to back (events around each region, not between launches)
        ms_dec, nreg_d, _ = timed_regions(decode_only, KD, stream, args.min_timed_ms, world, est)
    res["clocks"] = clk.summary()
    res["ms_step"] = max_over_ranks(ms_region / K, world, "cuda")
    res["regions"] = nreg
    res["ms_decode"] = max_over_ranks(ms_dec / KD, world, "cuda")
    res["decode_regions"], res["decode_launches"] = nreg_d, KD
    err = dec.device_error()
    if err:
        raise RuntimeError(f"{case.name}: device error word {err:#x}")
    if extra:
        return res

    # ---- the step behind another kernel: a ~100 MB copy (50 MB read, 50 MB
    # written) on the same stream before every step, as the projection GEMM
    # before attention would be in an engine ----
    src = torch.empty(25 << 20, dtype=torch.int16, device="cuda")
    dst = torch.empty_like(src)
    KO = max(1, min(K, 500))
    ms_copy, _, _ = timed_regions(lambda i: dst.copy_(src), KO, stream, args.min_timed_ms / 4, world, 0.02)

    def copy_then_step(i):
        dst.copy_(src)
        step(i)

    ms_both, _, _ = timed_regions(copy_then_step, KO, stream, args.min_timed_ms / 2, world, est + 0.02)
    res["us_after_copy"] = max_over_ranks((ms_both - ms_copy) / KO * 1e3, world, "cuda")
    res["copy_us"] = ms_copy / KO * 1e3
    del src, dst

    # ---- end to end: host buffers through the same C call ----
    # the step's inputs staged in one pinned host buffer, uploaded with one
    # copy; the result read back with one copy; the KV pool is resident state
    E = max(1, args.e2e_steps)
    c0 = copies[0]
    names = StepStaging.ORDER
    stg = StepStaging({n: (tuple(getattr(c0, n).shape), getattr(c0, n).dtype) for n in names},
                      tuple(c0.out.shape), c0.out.dtype)
    for n in names:
        stg.host[n].copy_(getattr(c0, n).cpu())
    res["h2d"] = stg.upload_bytes
    res["d2h"] = stg.out.numel() * stg.out.element_size()
    sq, skn, svn, ssm, scl, sbt = (stg.dev[n].data_ptr() for n in names)
    kc, vc, out = c0.k_cache.data_ptr(), c0.v_cache.data_ptr(), c0.out.data_ptr()

    def e2e_step(i):
        stg.upload(stream)
        lib.pa_kv_append_decode(skn, svn, ssm, sq, kc, vc, sbt, scl, scale, out, shp, pln, ws, wsb, sp)
        stg.download(c0.out, stream)

    ms_serial, _, _ = timed_regions(e2e_step, E, stream, args.min_timed_ms / 2, world, est * 2)
    res["ms_e2e_serial"] = max_over_ranks(ms_serial / E, world, "cuda")

    # the same steps double-buffered, as a serving loop runs them: step i+1's
    # inputs go up on one copy stream and step i-1's result comes down on
    # another while step i computes; every step still copies its own inputs
    # in and its own result out inside the timed region
    stg2 = [stg, StepStaging({n: (tuple(getattr(c0, n).shape), getattr(c0, n).dtype) for n in names},
                             tuple(c0.out.shape), c0.out.dtype)]
    for n in names:
        stg2[1].host[n].copy_(stg.host[n])
    outs = [c0.out, torch.empty_like(c0.out)]
    up_s, dn_s = torch.cuda.Stream(), torch.cuda.Stream()
    ev_up = [torch.cuda.Event() for _ in range(2)]
    ev_k = [torch.cuda.Event() for _ in range(2)]
    ev_dn = [torch.cuda.Event() for _ in range(2)]
    dptr = [[st.dev[n].data_ptr() for n in names] for st in stg2]

    def e2e_pipelined(i):
        k = i % 2
        if i % E == 0:
            up_s.wait_stream(stream)     # nothing of a region is copied before its start event
        up_s.wait_event(ev_k[k])         # step i-2 has read this staging slot
        stg2[k].upload(up_s)
        ev_up[k].record(up_s)
        stream.wait_event(ev_up[k])
        stream.wait_event(ev_dn[k])      # step i-2's result has left this output buffer
        q_, kn_, vn_, sm_, cl_, bt_ = dptr[k]
        lib.pa_kv_append_decode(kn_, vn_, sm_, q_, kc, vc, bt_, cl_, scale, outs[k].data_ptr(), shp, pln, ws, wsb,
                                sp)
        ev_k[k].record(stream)
        dn_s.wait_event(ev_k[k])
        stg2[k].download(outs[k], dn_s)
        ev_dn[k].record(dn_s)
        if i % E == E - 1:
            stream.wait_event(ev_dn[k])  # the region ends after its last result is home
            stream.wait_event(ev_dn[1 - k])

    ms_e2e, _, _ = timed_regions(e2e_pipelined, E, stream, args.min_timed_ms / 2, world, est * 2)
    res["ms_e2e"] = max_over_ranks(ms_e2e / E, world, "cuda")
    err = dec.device_error()
    if err:
        raise RuntimeError(f"{case.name}: device error word {err:#x}")
    return res


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    if args.prefill:
        return run_prefill(args)

    import torch
    import torch.distributed as dist
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "_pagedattn_build", os.path.join(ROOT, "paged_kv_cache_472_b200", "build.py"))
    libbuild = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(libbuild)
    libbuild.build()   # before the package import loads the library
    import paged_kv_cache_472_b200 as pa

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    stream = torch.cuda.current_stream()
    peak, peak_kind = measured_peak()
    # extra workloads: "C" (its own partition size) or "C:P" (partition size P, 0 = balanced split)
    extras = []
    for x in args.extra.split(","):
        if not x.strip():
            continue
        cid, _, part = x.partition(":")
        if int(cid) == args.config and not part:
            continue
        extras.append((int(cid), int(part) if part else None))

    m = decode_workload(args.config, args, world, rank, local, stream, pa.lib, pa)
    others = {}
    for cid, part in extras:
        r = decode_workload(cid, args, world, rank, local, stream, pa.lib, pa, extra=True, partition=part)
        ab = r["ab"]
        key = r["case"].name + ("" if part is None else ("-balanced" if part == 0 else f"-partition{part}"))
        others[key] = {
            "step_us": round(r["ms_step"] * 1e3, 3), "decode_us": round(r["ms_decode"] * 1e3, 3),
            "decode_gbs": round(ab["decode_unique"] / (r["ms_decode"] * 1e-3) / 1e9, 1),
            "frac": round(ab["decode_unique"] / (r["ms_decode"] * 1e-3) / 1e9 / peak, 4),
            "step_gbs": round(ab["decode_unique"] / (r["ms_step"] * 1e-3) / 1e9, 1),
            "bytes": ab["decode_unique"], "regions": r["regions"], "partition_tokens": r["pt"]}
        del r
        torch.cuda.empty_cache()

    if rank == 0:
        case, ab = m["case"], m["ab"]
        ms_step = m["ms_step"]
        dbytes = ab["decode_unique"]
        achieved = dbytes / (m["ms_decode"] * 1e-3) / 1e9
        value = job_throughput_gbs(dbytes, world, ms_step)
        line = {
            "metric": "paged-decode attention HBM GB/s (% of B200 peak); us/decode step",
            "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms_step, 6), "us_per_step": round(ms_step * 1e3, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": case.dtype,
            "data": "synthetic",
            "config": {"workload": case.name, "B": case.B, "Hq": case.Hq, "Hkv": case.Hkv, "D": case.D,
                       "block_size": case.block_size, "context_tokens": int(case.context_lens.sum()),
                       "partition_tokens": m["pt"], "dynamic_share": int(m["dec"].plan.dynamic_share),
                       "bytes_per_step": dbytes, "bytes_kind": "algorithmic: K/V of every block once + q + out "
                                                                 "+ tables + lengths",
                       "logical_bytes_per_step": ab["decode_total"], "append_bytes_per_step": ab["append"],
                       "logical_gbs": round(world * ab["decode_total"] / (ms_step * 1e-3) / 1e9, 2),
                       "l2": f"{m['R']} rotating input copies, {m['R'] * ab['step_total'] / 1e6:.0f} MB > L2 "
                             f"{m['l2'] / 1e6:.0f} MB",
                       "timed_regions": m["regions"], "region_stat": "median",
                       "parallelism": f"replicas x{world}" if world > 1 else "1 GPU",
                       "tokens_per_s": round(world * case.B / (ms_step * 1e-3), 1),
                       "pct_of_peak": round(100 * value / world / peak, 2),
                       "step_us_after_copy": round(m["us_after_copy"], 3),
                       "copy_us": round(m["copy_us"], 3)},
            "roofline": {"bound": "hbm", "achieved": round(achieved, 2), "peak": peak, "unit": "GB/s",
                         "frac": round(achieved / peak, 4), "traffic": profiled_traffic(case.name),
                         "kernel": "paged_decode_kernel", "peak_kind": peak_kind,
                         "decode_us": round(m["ms_decode"] * 1e3, 3), "decode_launches_timed": m["decode_launches"],
                         "decode_regions": m["decode_regions"],
                         "algorithmic_bytes_per_launch": dbytes,
                         "engine": "tensor-core mma" if case.dtype != "f32" else "cuda-core fp32"},
            "e2e": {"value": round(job_throughput_gbs(dbytes, world, m["ms_e2e"]), 2), "unit": "GB/s",
                    "h2d_bytes_per_step": m["h2d"], "d2h_bytes_per_step": m["d2h"],
                    "us_per_step": round(m["ms_e2e"] * 1e3, 3),
                    "mode": "double-buffered: each step's upload and read-back overlap its neighbours' steps",
                    "serial": {"value": round(job_throughput_gbs(dbytes, world, m["ms_e2e_serial"]), 2),
                               "us_per_step": round(m["ms_e2e_serial"] * 1e3, 3),
                               "mode": "upload, step, read-back in order on one stream"}},
            "workloads": others,
            "gpu_launches": args.steps,   # one fused append + decode launch per step of the reported region
            "clocks": m["clocks"],
        }
        if not args.no_cpu_baseline:
            cb = cpu_baseline(case, args.cpu_seconds)
            line["cpu_baseline"] = {k: cb[k] for k in ("value", "unit", "cores", "kind", "sample", "cores_1")}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
