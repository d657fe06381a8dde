"""Benchmark: tenant-mixed BitDelta delta-apply throughput on B200 (+ compress GB/s).

Workload (one "step"): one decode step of a 32-layer Llama-3-8B-shaped projection stack
(q, k, v, o 4096-wide; gate/up 14336 x 4096; down 4096 x 14336) with a bf16 base
(~14 GB) and 100 resident tenants (random sign words + fp16 group-128 scales, ~0.98 GB
each, stored in the tiled serving layout of bd_prepare_tenant) for a batch of 512
tokens whose tenant ids are drawn Zipf(1.1); x ~ N(0, 1) bf16, fresh per step.
Each layer is applied as 4 bd_apply_multi calls on the fused matrices a serving engine
keeps (qkv 6144 x 4096, o, gate_up 28672 x 4096, down): 128 calls per step. All inputs
are resident in HBM and together far larger than L2.

Also measured in the same run (reported under "compress"): bd_compress of the 32-layer
stack in bf16 (group 128), W_base ~ N(0, 0.02), delta ~ N(0, 0.001) with 0.05% x30
outliers, with and without the 3-sigma clip.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
For N > 1 launch under torch.distributed.run: each rank runs an independent replica
of the workload on its own GPU (no collective on the data path); value = tokens of all
ranks / the slowest rank's time.
"""

from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from workloads import LLAMA3_8B_FUSED, LLAMA3_8B_PROJECTIONS  # noqa: E402

METRIC = "tenant-mixed delta-apply tokens/s + HBM GB/s vs peak; compress GB/s"
N_LAYERS = 32
N_TENANTS = 100
BATCH = 512
GROUP = 128
ZIPF_S = 1.1
COMPRESS_STREAMS = 4  # compress calls of the stack are spread over this many streams


def tc_min_tokens() -> int:
    """The library's many-token threshold (tensor-core delta from this token count on),
    read from the built library so that the byte accounting follows the build."""
    import tenant_serving_b200 as bd
    return bd.bd_tc_min_tokens()


# DRAM traffic per launch (dram__bytes_read.sum + dram__bytes_write.sum) of a kernel from
# an ncu capture summarised under profiles/, keyed by the hash of the sources the kernel
# was built from: once they change, the number no longer describes the kernel and the
# roofline reports traffic = null.
NCU_TRAFFIC = {
    # ncu capture of the serving workload's 1-layer stack: mean over the qkv, o, gate_up and
    # down calls (each a quarter of a step's launches) of dram__bytes_read.sum +
    # dram__bytes_write.sum
    "delta_lut": {"sources": ["bd_delta_lut.cu", "bd_internal.cuh", "bd_tc.cuh"],
                  "sha256_16": "706ffd8085fd8fc3", "bytes_per_launch": 586094528.0},
}


def ncu_traffic(kernel: str):
    import hashlib
    rec = NCU_TRAFFIC.get(kernel)
    if rec is None:
        return None
    h = hashlib.sha256()
    for f in rec["sources"]:
        with open(os.path.join(ROOT, "tenant_serving_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return rec["bytes_per_launch"] if h.hexdigest()[:16] == rec["sha256_16"] else None


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--layers", type=int, default=N_LAYERS)
    p.add_argument("--tenants", type=int, default=N_TENANTS)
    p.add_argument("--batch", type=int, default=BATCH)
    p.add_argument("--compress-layers", type=int, default=N_LAYERS)
    p.add_argument("--no-compress", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-extra", action="store_true", help="skip the decode, mixed and cold-start workloads")
    p.add_argument("--extra", default="decode,decode_fp8,mixed,cold_start",
                   help="comma-separated extra workloads to run after the serving step (N = 1)")
    p.add_argument("--cpu-seconds", type=float, default=15.0)
    return p.parse_args()


def load_peaks():
    """(HBM GB/s, (bf16 TFLOP/s burst, sustained), source)."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return (d.get("hbm_gbs", 6650.0),
                (d.get("bf16_tflops", 1590.0), d.get("bf16_tflops_sustained", 1400.0)), "measured")
    return 6650.0, (1590.0, 1400.0), "fallback"


# ------------------------------------------------------------------------------------
# clocks sampled during the timed region
# ------------------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        os.unlink(self.path)
        loaded = [s for s in sm if s > 500] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(mx) if mx else None, "samples": len(sm),
                "reasons": sorted(reasons)}


# ------------------------------------------------------------------------------------
# our arm
# ------------------------------------------------------------------------------------
def setup_dist(args):
    """One process per GPU under torch.distributed.run (RANK / WORLD_SIZE / LOCAL_RANK /
    MASTER_* from the environment). NCCL on GPUs; gloo where there is no GPU (the rank
    logic's CPU tests). The group's short timeout turns a missing rank into an error."""
    import datetime
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    on_gpu = torch.cuda.is_available()
    if on_gpu:
        torch.cuda.set_device(local)
    pg = None
    if world > 1:
        import torch.distributed as dist
        kw = {"device_id": torch.device("cuda", local)} if on_gpu else {}
        dist.init_process_group("nccl" if on_gpu else "gloo",
                                timeout=datetime.timedelta(seconds=120), **kw)
        pg = dist
    return world, rank, local, pg


def barrier(pg):
    if pg is not None:
        pg.barrier()


def _reduce(pg, v: float, op) -> float:
    import torch
    dev = "cuda" if pg.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    pg.all_reduce(t, op=op)
    return float(t.item())


def max_over_ranks(pg, v: float) -> float:
    return v if pg is None else _reduce(pg, v, pg.ReduceOp.MAX)


def sum_over_ranks(pg, v: float) -> float:
    return v if pg is None else _reduce(pg, v, pg.ReduceOp.SUM)


def whole_job_rate(pg, units: float, ms: float):
    """Units of all ranks / the slowest rank's time: (units_all, ms_max, units per s)."""
    units_all = sum_over_ranks(pg, units)
    ms_max = max_over_ranks(pg, ms)
    return units_all, ms_max, units_all / (ms_max / 1e3)


def serving_config(args, world: int) -> dict:
    return {"workload": f"serving: {args.layers}-layer Llama-3-8B-shaped projection stack "
                        f"(q, k, v, o, gate, up, down; applied as fused qkv / o / gate_up / down, "
                        f"{4 * args.layers} calls), bf16 base + {args.tenants} resident tenants (sign words + "
                        f"fp16 group-128 scales), batch {args.batch}, Zipf(1.1) tenant ids, one decode step "
                        f"per step",
            "layers": args.layers, "tenants": args.tenants, "batch": args.batch,
            "group_size": GROUP,
            "l2": f"inputs larger than L2 (~{3.5 * args.layers * args.tenants / 100:.0f} GB resident)",
            "parallelism": f"replicas x{world}"}


def zipf_ids_host(rng, batch, n, s):
    k = np.arange(1, n + 1, dtype=np.float64)
    p = k ** (-s)
    p /= p.sum()
    return rng.choice(n, size=batch, p=p).astype(np.int32)


def build_serving(args, seed_base, log):
    """Device-resident serving stack: per layer and projection a bf16 base and a tenant
    table of `tenants` records (random sign words + fp16 group scales)."""
    import torch
    import tenant_serving_b200 as bd
    g = torch.Generator(device="cuda")
    t0 = time.time()
    layers = []
    for layer in range(args.layers):
        projs = []
        for pi, (name, d_out, d_in) in enumerate(LLAMA3_8B_FUSED):
            g.manual_seed(seed_base + 1000 * layer + pi)
            wb = (torch.randn((d_out, d_in), generator=g, device="cuda", dtype=torch.float32)
                  * 0.02).to(torch.bfloat16)
            recs = []
            for u in range(args.tenants):
                words = torch.randint(-(2 ** 31), 2 ** 31 - 1, (d_out, d_in // 32), generator=g,
                                      device="cuda", dtype=torch.int32)
                z = torch.randn((d_out, d_in // GROUP), generator=g, device="cuda")
                s = (0.001 * math.sqrt(2.0 / math.pi) * torch.exp(0.1 * z)).to(torch.float16)
                # serving layout (tiles of 512 rows x 256 columns), written once at load
                tw, ts = bd.bd_prepare_tenant(words, s, bd.BD_SCALE_GROUP, GROUP, d_out, d_in)
                del words, s
                recs.append((tw, ts, bd.BD_SCALE_GROUP, GROUP, bd.BD_LAYOUT_TILED))
            projs.append((name, d_out, d_in, wb, bd.TenantTable(recs, "cuda")))
        layers.append(projs)
        if layer == 0:
            torch.cuda.synchronize()
            log(f"serving: layer 0 generated in {time.time() - t0:.1f}s")
    torch.cuda.synchronize()
    log(f"serving: stack generated in {time.time() - t0:.1f}s, "
        f"{torch.cuda.memory_allocated() / 1e9:.1f} GB allocated")
    return layers


def bench_serving(args, rank, pg, log, peaks):
    import ctypes
    import torch
    import tenant_serving_b200 as bd
    L = bd.lib()
    layers = build_serving(args, 7000 + 1000003 * rank, log)
    steps_total = args.warmup + args.steps
    rng = np.random.default_rng(3000 + rank)
    B = args.batch
    ids_host = [zipf_ids_host(rng, B, args.tenants, ZIPF_S) for _ in range(steps_total)]
    g = torch.Generator(device="cuda")
    xa, xb = [], []
    for st in range(steps_total):
        g.manual_seed(3000 + st + 100000 * rank)
        xa.append(torch.randn((B, 4096), generator=g, device="cuda").to(torch.bfloat16))
        xb.append(torch.randn((B, 14336), generator=g, device="cuda").to(torch.bfloat16))
    ids_dev = [torch.from_numpy(i).cuda() for i in ids_host]
    ys = {name: torch.empty((B, d_out), dtype=torch.bfloat16, device="cuda")
          for name, d_out, d_in in LLAMA3_8B_FUSED}
    wss = {name: torch.empty(bd.bd_apply_workspace_size(d_out, d_in, B, args.tenants),
                             dtype=torch.uint8, device="cuda")
           for name, d_out, d_in in LLAMA3_8B_FUSED}
    stream = torch.cuda.current_stream()
    sp = ctypes.c_void_p(stream.cuda_stream)

    def calls_for(xa_t, xb_t, ids_t):
        out = []
        for projs in layers:
            for name, d_out, d_in, wb, table in projs:
                x = xb_t if d_in == 14336 else xa_t
                y, ws = ys[name], wss[name]
                out.append((ctypes.c_void_p(wb.data_ptr()), bd.BD_BF16, d_out, d_in, table.ptr(),
                            table.n, bd.BD_F16, ctypes.c_void_p(ids_t.data_ptr()),
                            ctypes.c_void_p(x.data_ptr()), B, ctypes.c_void_p(y.data_ptr()),
                            bd.BD_BF16, ctypes.c_void_p(ws.data_ptr()), ws.numel(), sp))
        return out

    step_calls = [calls_for(xa[s], xb[s], ids_dev[s]) for s in range(steps_total)]
    apply = L.bd_apply_multi

    def run_step(s):
        for c in step_calls[s]:
            rc = apply(*c)
            if rc != 0:
                raise bd.BitDeltaError(rc, "bd_apply_multi")

    # warm-up
    for s in range(args.warmup):
        run_step(s)
    torch.cuda.synchronize()
    barrier(pg)
    torch.cuda.synchronize()
    # timed region (device events on the launching stream), clocks sampled meanwhile
    clocks = ClockSampler(torch.cuda.current_device())
    clocks.start()
    time.sleep(0.3)
    n0 = bd.bd_launch_count()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for s in range(args.warmup, steps_total):
        run_step(s)
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    launches = bd.bd_launch_count() - n0
    clk = clocks.stop()
    barrier(pg)
    ms_max = max_over_ranks(pg, ms)

    # the same steps again with the library's per-kernel events on (kernel breakdown and
    # the roofline's per-kernel durations; the events add a little time)
    torch.cuda.synchronize()
    barrier(pg)
    torch.cuda.synchronize()
    bd.bd_profile_enable(True, capacity=args.steps * len(step_calls[0]) * 8 + 16)
    f0 = torch.cuda.Event(enable_timing=True)
    f1 = torch.cuda.Event(enable_timing=True)
    f0.record(stream)
    for s in range(args.warmup, steps_total):
        run_step(s)
    f1.record(stream)
    torch.cuda.synchronize()
    prof = bd.bd_profile_collect()
    bd.bd_profile_enable(False)
    ms_prof = max_over_ranks(pg, f0.elapsed_time(f1))

    # algorithmic bytes of the timed steps. The planner sends a tenant with at least
    # tc_min tokens in the batch (all tenants here are tiled, fp16, group 128) to the
    # tensor-core delta kernel and the others to the lookup-table kernel; each delta kernel
    # is charged the sign words + scales of its tenants and the y rows of its tokens.
    tc_min = tc_min_tokens()
    base_bytes = sum(d_out * d_in * 2 for _, d_out, d_in in LLAMA3_8B_FUSED) * args.layers
    base_flops_per_token = sum(2 * d_out * d_in for _, d_out, d_in in LLAMA3_8B_FUSED) * args.layers
    delta_bytes_per_tenant = sum(d_out * d_in // 8 + d_out * (d_in // GROUP) * 2
                                 for _, d_out, d_in in LLAMA3_8B_FUSED) * args.layers
    y_bytes_per_token = sum(d_out * 2 for _, d_out, _ in LLAMA3_8B_FUSED) * args.layers
    x_bytes_per_token = sum(d_in * 2 for _, _, d_in in LLAMA3_8B_FUSED) * args.layers
    io_bytes = B * (x_bytes_per_token + y_bytes_per_token)
    step_bytes, lut_bytes, tc_bytes = [], 0.0, 0.0
    for s in range(args.warmup, steps_total):
        cnt = np.bincount(ids_host[s], minlength=args.tenants)
        d = int((cnt > 0).sum())
        big = cnt >= tc_min
        step_bytes.append(base_bytes + d * delta_bytes_per_tenant + io_bytes)
        tc_bytes += int(big.sum()) * delta_bytes_per_tenant + int(cnt[big].sum()) * y_bytes_per_token
        small = (cnt > 0) & ~big
        lut_bytes += int(small.sum()) * delta_bytes_per_tenant + int(cnt[small].sum()) * y_bytes_per_token
    distinct = [len(np.unique(ids_host[s])) for s in range(args.warmup, steps_total)]
    total_bytes = float(sum(step_bytes))
    kernel_work = {  # kernel -> (amount over the timed steps, unit, bound)
        "delta_lut": (lut_bytes, "GB/s", "hbm"),
        "delta_tc": (tc_bytes, "GB/s", "hbm"),
        "base_tc": (float(base_flops_per_token) * B * args.steps, "TFLOP/s", "tensor"),
    }

    # e2e through the public API: H2D of this step's inputs (pinned), the 128 calls,
    # D2H of the last projection's output
    pin_xa = [xa[s].cpu().pin_memory() for s in range(steps_total)]
    pin_xb = [xb[s].cpu().pin_memory() for s in range(steps_total)]
    pin_ids = [torch.from_numpy(ids_host[s]).pin_memory() for s in range(steps_total)]
    y_host = torch.empty((B, 4096), dtype=torch.bfloat16).pin_memory()
    last = ys["down"]
    torch.cuda.synchronize()
    barrier(pg)
    g0 = torch.cuda.Event(enable_timing=True)
    g1 = torch.cuda.Event(enable_timing=True)
    g0.record(stream)
    for s in range(args.warmup, steps_total):
        xa[s].copy_(pin_xa[s], non_blocking=True)
        xb[s].copy_(pin_xb[s], non_blocking=True)
        ids_dev[s].copy_(pin_ids[s], non_blocking=True)
        run_step(s)
        y_host.copy_(last, non_blocking=True)
    g1.record(stream)
    torch.cuda.synchronize()
    ms_e2e = max_over_ranks(pg, g0.elapsed_time(g1))
    h2d = B * 4096 * 2 + B * 14336 * 2 + B * 4
    d2h = B * 4096 * 2

    tokens_all, _, value = whole_job_rate(pg, float(B * args.steps), ms)
    e2e_value = tokens_all / (ms_e2e / 1e3)
    hbm_gbs = total_bytes / (ms_max / 1e3) / 1e9

    # dominant kernel by total device time
    dom = max(prof.items(), key=lambda kv: kv[1][1]) if prof else ("delta_lut", (0, 0.0))
    dname, (dl, dms) = dom
    hbm_peak, tensor_peaks, peak_src = peaks
    work, unit, bound = kernel_work.get(dname, (None, "GB/s", "hbm"))
    achieved = None
    if work and dms > 0:
        achieved = work / (dms / 1e3) / (1e12 if unit == "TFLOP/s" else 1e9)
    # a kernel timed inside a long step: the sustained tensor peak
    peak = tensor_peaks[1] if unit == "TFLOP/s" else hbm_peak
    res = {
        "value": value, "ms_per_step": ms_max / args.steps, "ms_per_step_profiled": ms_prof / args.steps,
        "hbm_gbs": hbm_gbs, "hbm_frac": hbm_gbs / hbm_peak, "gpu_launches": launches,
        "clocks": clk, "distinct_tenants_mean": float(np.mean(distinct)),
        "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "kernels": {k: {"launches": v[0], "total_ms": v[1], "share": v[1] / sum(x[1] for x in prof.values())}
                    for k, v in prof.items()},
        "roofline": {"kernel": dname, "bound": bound, "achieved": achieved, "peak": peak,
                     "unit": unit, "frac": (achieved / peak) if achieved else None,
                     "traffic": ncu_traffic(dname),
                     "algorithmic_per_launch": (work / dl) if (work and dl) else None,
                     "peak_source": (f"measured (MEASURED_PEAKS.json "
                                     f"{'bf16_tflops_sustained' if unit == 'TFLOP/s' else 'hbm_gbs'})"
                                     if peak_src == "measured" else
                                     "fallback: the pool's earlier measurement (no MEASURED_PEAKS.json)"),
                     "avg_launch_us": dms / dl * 1e3 if dl else None},
        "kernel_rates": {k: {"achieved": kernel_work[k][0] / (prof[k][1] / 1e3) /
                                         (1e12 if kernel_work[k][1] == "TFLOP/s" else 1e9),
                             "unit": kernel_work[k][1]}
                         for k in kernel_work if k in prof and prof[k][1] > 0},
        "step_bytes_mean": float(np.mean(step_bytes)),
    }
    del layers
    return res


def bench_compress(args, log, peaks):
    """bd_compress over the 32-layer stack: group-128 scales without and with the 3-sigma
    clip, row, column and 128 x 128 block scales; each with the 224 independent calls spread over
    COMPRESS_STREAMS CUDA streams and on a single stream (one call after another)."""
    import torch
    import tenant_serving_b200 as bd
    from workloads import device_weight_pair
    g = torch.Generator(device="cuda")
    t0 = time.time()
    mats = []
    for layer in range(args.compress_layers):
        for pi, (name, d_out, d_in) in enumerate(LLAMA3_8B_PROJECTIONS):
            g.manual_seed(1000 * layer + pi)
            wb, wf = device_weight_pair(g, d_out, d_in, 0.02, 0.001, 0.0005, 30.0)
            mats.append((d_out, d_in, wb, wf))
    torch.cuda.synchronize()
    log(f"compress: {len(mats)} matrices generated in {time.time() - t0:.1f}s")
    params = sum(d_out * d_in for d_out, d_in, _, _ in mats)
    out = {}
    main_s = torch.cuda.current_stream()
    variants = (("group128", bd.BD_SCALE_GROUP, False), ("group128_clip3", bd.BD_SCALE_GROUP, True),
                ("row", bd.BD_SCALE_ROW, False), ("col", bd.BD_SCALE_COL, False),
                ("block128", bd.BD_SCALE_BLOCK, False))
    for label, mode, clip in variants:
        cfg = bd.compress_cfg(mode=mode, group_size=GROUP, clip=clip, clip_k=3.0)
        bufs = []
        for d_out, d_in, wb, wf in mats:
            signs = torch.empty((d_out, d_in // 32), dtype=torch.int32, device="cuda")
            scales = torch.empty(bd.scales_shape(mode, d_out, d_in, GROUP), dtype=torch.float32,
                                 device="cuda")
            ws = torch.empty(max(bd.bd_compress_workspace_size(d_out, d_in, cfg), 16),
                             dtype=torch.uint8, device="cuda")
            bufs.append((signs, scales, ws))
        # algorithmic bytes: bf16 W_base + W_fine read once, sign bits and fp32 scales written
        # (the clip's statistics pass is a second read, not counted)
        scale_bytes = sum(math.prod(bd.scales_shape(mode, d_out, d_in, GROUP)) * 4 for d_out, d_in, _, _ in mats)
        alg = params * (4 + 1 / 8) + scale_bytes
        res = {}
        for nstreams in (COMPRESS_STREAMS, 1):
            streams = [torch.cuda.Stream() for _ in range(nstreams)]

            def one_pass():
                start = torch.cuda.Event()
                start.record(main_s)
                for st in streams:
                    st.wait_event(start)
                for i, ((d_out, d_in, wb, wf), (signs, scales, ws)) in enumerate(zip(mats, bufs)):
                    bd.bd_compress(wb, wf, cfg, signs=signs, scales=scales, workspace=ws,
                                   stream=streams[i % nstreams])
                for st in streams:
                    done = torch.cuda.Event()
                    done.record(st)
                    main_s.wait_event(done)

            for _ in range(2):
                one_pass()
            torch.cuda.synchronize()
            reps = 3
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(main_s)
            for _ in range(reps):
                one_pass()
            e1.record(main_s)
            torch.cuda.synchronize()
            ms = e0.elapsed_time(e1) / reps
            key = "streams4" if nstreams > 1 else "stream1"
            res[key] = {"ms_per_stack": ms, "gbs": alg / (ms / 1e3) / 1e9,
                        "frac": alg / (ms / 1e3) / 1e9 / peaks[0], "streams": nstreams}
            if nstreams == 1:
                # per-kernel device time of a further single-stream pass (kernels do not
                # overlap); the events around each launch are not in the timing above
                bd.bd_profile_enable(True, capacity=len(mats) * 4 + 16)
                one_pass()
                torch.cuda.synchronize()
                prof = bd.bd_profile_collect()
                bd.bd_profile_enable(False)
                res[key]["kernels"] = {k: {"launches": v[0], "ms_per_stack": v[1]} for k, v in prof.items()}
        out[label] = {"params": params, "bytes_per_stack": alg,
                      "tparams_per_s": params / (res["streams4"]["ms_per_stack"] / 1e3) / 1e12, **res}
        if label == "group128":
            out["reconstruct_merged"] = _bench_reconstruct(
                bd, mats, bufs, [torch.cuda.Stream() for _ in range(COMPRESS_STREAMS)], main_s, params,
                peaks)
        del bufs
    del mats
    torch.cuda.empty_cache()
    return out


def _bench_reconstruct(bd, mats, bufs, streams, main_s, params, peaks):
    """The merged weight W_u = W_base + Delta_hat of every matrix of the stack, in bf16,
    from the signs and scales compress just wrote (bd_reconstruct with w_base). Same
    stream arrangement as compress; one reused output buffer per stream."""
    import torch
    biggest = max(d_out * d_in for d_out, d_in, _, _ in mats)
    outs = [torch.empty(biggest, dtype=torch.bfloat16, device="cuda") for _ in streams]

    def one_pass():
        start = torch.cuda.Event()
        start.record(main_s)
        for st in streams:
            st.wait_event(start)
        for i, ((d_out, d_in, wb, wf), (signs, scales, ws)) in enumerate(zip(mats, bufs)):
            k = i % len(streams)
            bd.bd_reconstruct(signs, scales, bd.BD_SCALE_GROUP, GROUP, d_out, d_in, w_base=wb,
                              out=outs[k][: d_out * d_in].view(d_out, d_in), stream=streams[k])
        for st in streams:
            done = torch.cuda.Event()
            done.record(st)
            main_s.wait_event(done)

    for _ in range(2):
        one_pass()
    torch.cuda.synchronize()
    reps = 3
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(main_s)
    for _ in range(reps):
        one_pass()
    e1.record(main_s)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / reps
    # sign bits + fp32 group scales + bf16 W_base read, bf16 W_u written
    alg = params * (1 / 8 + 4 / GROUP + 2 + 2)
    gbs = alg / (ms / 1e3) / 1e9
    return {"ms_per_stack": ms, "gbs": gbs, "frac": gbs / peaks[0], "streams": len(streams)}


def bench_cold_start(args, log, peaks):
    """Cold start of one tenant, as the per-axis delta page measures it: all 224 modules of
    the 32-layer Llama-3-8B stack (group-128 fp16 scales, 981 MB of packed records in
    pinned host memory) loaded by the tenant cache with one transfer per module, against
    loading the dense bf16 merged weights of the same stack (13.96 GB: 32 transfers of one
    layer's 436 MB from pinned host memory). Device time on the copy stream."""
    import torch
    import tenant_serving_b200 as bd
    mods = [(d_out, d_in, GROUP) for _ in range(N_LAYERS) for _, d_out, d_in in LLAMA3_8B_PROJECTIONS]
    rng = np.random.default_rng(4000)
    t0 = time.time()
    records = []
    for d_out, d_in, g in mods:
        words = rng.integers(0, 2 ** 32, size=(d_out, d_in // 32), dtype=np.uint32)
        sc = (0.001 * math.sqrt(2.0 / math.pi) * np.exp(0.1 * rng.standard_normal((d_out, d_in // g)))
              ).astype(np.float16)
        records.append(bd.bd_prepare_record_host(words, sc, bd.BD_SCALE_GROUP, g, d_out, d_in, pin=True))
    log(f"cold start: {len(records)} records packed in {time.time() - t0:.1f}s")
    rec_bytes = sum(r.numel() for r in records)
    # two host tenants with the same records and one slot: every prefetch is a full load
    cache = bd.TenantCache(mods, n_host_tenants=2, n_slots=1)
    for u in range(2):
        for m, r in enumerate(records):
            cache.register(u, m, r, bd.BD_SCALE_GROUP, GROUP)
    cs = torch.cuda.Stream()
    times = []
    for k in range(6):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(cs)
        _, n, ticket = cache.prefetch(np.array([k % 2], dtype=np.int32), stream=cs)
        e1.record(cs)
        cache.acquire(ticket, stream=cs)
        cache.release(ticket, stream=cs)
        torch.cuda.synchronize()
        if k >= 2:
            times.append(e0.elapsed_time(e1))
        assert n == 1
    delta_ms = statistics.median(times)
    stats = cache.resident()[1]
    cache.close()
    del records
    # dense merged weights: one layer's bf16 weights, pinned, moved 32 times
    layer_elems = sum(d_out * d_in for _, d_out, d_in in LLAMA3_8B_PROJECTIONS)
    host_layer = torch.empty(layer_elems, dtype=torch.bfloat16).pin_memory()
    host_layer.view(torch.int16).copy_(torch.from_numpy(
        rng.integers(-2 ** 15, 2 ** 15, size=layer_elems, dtype=np.int16)))
    dev_layer = torch.empty(layer_elems, dtype=torch.bfloat16, device="cuda")
    dtimes = []
    for k in range(3):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(cs)
        with torch.cuda.stream(cs):
            for _ in range(N_LAYERS):
                dev_layer.copy_(host_layer, non_blocking=True)
        e1.record(cs)
        torch.cuda.synchronize()
        if k >= 1:
            dtimes.append(e0.elapsed_time(e1))
    dense_ms = statistics.median(dtimes)
    dense_bytes = layer_elems * 2 * N_LAYERS
    del host_layer, dev_layer
    torch.cuda.empty_cache()
    return {"workload": "one tenant of the 32-layer Llama-3-8B stack, group-128 fp16 scales, pinned host "
                        "memory -> HBM",
            "delta_ms": delta_ms, "delta_bytes": rec_bytes, "delta_gbs": rec_bytes / (delta_ms / 1e3) / 1e9,
            "delta_transfers": len(mods) + 1, "dense_bf16_ms": dense_ms, "dense_bytes": dense_bytes,
            "dense_gbs": dense_bytes / (dense_ms / 1e3) / 1e9, "speedup": dense_ms / delta_ms,
            "cache_stats": stats}


def _time_calls(run, iters, warmup, stream):
    """Device time of `iters` runs of run() after `warmup` runs, plus the library's
    per-kernel times of a second timed pass (ms)."""
    import torch
    import tenant_serving_b200 as bd
    for _ in range(warmup):
        run()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(iters):
        run()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / iters
    bd.bd_profile_enable(True, capacity=iters * 64 + 16)
    for _ in range(iters):
        run()
    torch.cuda.synchronize()
    prof = bd.bd_profile_collect()
    bd.bd_profile_enable(False)
    return ms, {k: {"launches": v[0] // iters, "us_per_run": v[1] / iters * 1e3} for k, v in prof.items()}


def bench_decode(args, log, peaks, fp8=False):
    """Decode GEMV: the up_proj shape 14336 x 4096 with a bf16 base (or, with fp8, the same
    base quantized to e4m3 with per-row scales), 64 resident tenants (sign words + fp16
    group-128 scales, tiled serving layout), 64 tokens, one per tenant (a seeded
    permutation), x ~ N(0, 1) bf16. The ~646 MB (fp8: ~587 MB) read per call is far larger
    than L2, so no flush is needed between calls."""
    import torch
    import tenant_serving_b200 as bd
    d_out, d_in, T, B = 14336, 4096, 64, 64
    g = torch.Generator(device="cuda")
    g.manual_seed(2000)
    wb = (torch.randn((d_out, d_in), generator=g, device="cuda") * 0.02).to(torch.bfloat16)
    recs = []
    for u in range(T):
        words = torch.randint(-(2 ** 31), 2 ** 31 - 1, (d_out, d_in // 32), generator=g, device="cuda",
                              dtype=torch.int32)
        sc = (0.001 * math.sqrt(2.0 / math.pi) *
              torch.exp(0.1 * torch.randn((d_out, d_in // GROUP), generator=g, device="cuda"))).to(torch.float16)
        tw, ts = bd.bd_prepare_tenant(words, sc, bd.BD_SCALE_GROUP, GROUP, d_out, d_in)
        recs.append((tw, ts, bd.BD_SCALE_GROUP, GROUP, bd.BD_LAYOUT_TILED))
    table = bd.TenantTable(recs, "cuda")
    ids = torch.from_numpy(np.random.default_rng(2000).permutation(T).astype(np.int32)).cuda()
    x = (torch.randn((B, d_in), generator=g, device="cuda")).to(torch.bfloat16)
    y = torch.empty((B, d_out), dtype=torch.bfloat16, device="cuda")
    stream = torch.cuda.current_stream()
    if fp8:
        codes, wsc = bd.bd_quantize_base_fp8(wb)
        del wb
        ws = torch.empty(bd.bd_apply_fp8_workspace_size(d_out, d_in, B, T), dtype=torch.uint8, device="cuda")
        run = lambda: bd.bd_apply_multi_fp8(codes, wsc, table, ids, x, y=y, workspace=ws)  # noqa: E731
        base_bytes = d_out * d_in + d_out * 4
    else:
        ws = torch.empty(bd.bd_apply_workspace_size(d_out, d_in, B, T), dtype=torch.uint8, device="cuda")
        run = lambda: bd.bd_apply_multi(wb, table, ids, x, y=y, workspace=ws)  # noqa: E731
        base_bytes = d_out * d_in * 2
    ms, kern = _time_calls(run, 20, 3, stream)
    alg = base_bytes + T * (d_out * d_in // 8 + d_out * (d_in // GROUP) * 2) + B * (d_in + d_out) * 2
    del recs, table
    torch.cuda.empty_cache()
    base_k = "base_fp8" if fp8 else "base_tc"
    out = {"workload": "decode: up_proj 14336x4096 %s base, 64 tenants (group-128 fp16 scales), "
                       "64 tokens one per tenant" % ("e4m3 (per-row fp32 scales)" if fp8 else "bf16"),
           "us_per_call": ms * 1e3, "tokens_per_s": B / (ms / 1e3), "bytes_per_call": alg,
           "gbs": alg / (ms / 1e3) / 1e9, "frac": alg / (ms / 1e3) / 1e9 / peaks[0], "kernels": kern}
    if base_k in kern and kern[base_k]["us_per_run"] > 0:
        out["base_gbs"] = base_bytes / (kern[base_k]["us_per_run"] / 1e6) / 1e9
    return out


def bench_mixed(args, log, peaks):
    """Mixed batch: one Llama-3-8B-shaped layer applied as its 7 projections, 32 resident
    tenants with per-axis fp16 scale vectors (row or column per (tenant, projection),
    Bernoulli(1/2) from the seed), 256 tokens with Zipf(1.1) ids over the 32 tenants,
    bf16 base product on the tensor cores. One run = the 7 calls (~1.25 GB read, far
    larger than L2)."""
    import torch
    import tenant_serving_b200 as bd
    B, T = 256, 32
    rng = np.random.default_rng(3000)
    g = torch.Generator(device="cuda")
    g.manual_seed(3000)
    ids_host = zipf_ids_host(rng, B, T, ZIPF_S)
    ids = torch.from_numpy(ids_host).cuda()
    distinct = np.unique(ids_host)
    calls, alg = [], 0
    for name, d_out, d_in in LLAMA3_8B_PROJECTIONS:
        wb = (torch.randn((d_out, d_in), generator=g, device="cuda") * 0.02).to(torch.bfloat16)
        recs, scale_bytes = [], []
        for u in range(T):
            mode = bd.BD_SCALE_ROW if rng.random() < 0.5 else bd.BD_SCALE_COL
            words = torch.randint(-(2 ** 31), 2 ** 31 - 1, (d_out, d_in // 32), generator=g, device="cuda",
                                  dtype=torch.int32)
            n = d_out if mode == bd.BD_SCALE_ROW else d_in
            sc = (0.001 * math.sqrt(2.0 / math.pi) *
                  torch.exp(0.1 * torch.randn((n,), generator=g, device="cuda"))).to(torch.float16)
            tw, ts = bd.bd_prepare_tenant(words, sc, mode, GROUP, d_out, d_in)
            recs.append((tw, ts, mode, GROUP, bd.BD_LAYOUT_TILED))
            scale_bytes.append(n * 2)
        table = bd.TenantTable(recs, "cuda")
        x = torch.randn((B, d_in), generator=g, device="cuda").to(torch.bfloat16)
        y = torch.empty((B, d_out), dtype=torch.bfloat16, device="cuda")
        ws = torch.empty(bd.bd_apply_workspace_size(d_out, d_in, B, T), dtype=torch.uint8, device="cuda")
        calls.append((wb, table, x, y, ws, recs))
        alg += d_out * d_in * 2 + sum(d_out * d_in // 8 + scale_bytes[u] for u in distinct) + B * (d_in + d_out) * 2
    stream = torch.cuda.current_stream()

    def run():
        for wb, table, x, y, ws, _ in calls:
            bd.bd_apply_multi(wb, table, ids, x, y=y, workspace=ws)

    ms, kern = _time_calls(run, 20, 3, stream)
    del calls
    torch.cuda.empty_cache()
    return {"workload": "mixed: one Llama-3-8B-shaped layer (7 projections), 32 tenants with per-axis "
                        "fp16 scales (row or column per tenant and projection), 256 tokens, Zipf(1.1) ids",
            "us_per_layer": ms * 1e3, "tokens_per_s": B / (ms / 1e3), "bytes_per_layer": alg,
            "distinct_tenants": int(len(distinct)), "gbs": alg / (ms / 1e3) / 1e9,
            "frac": alg / (ms / 1e3) / 1e9 / peaks[0], "kernels": kern}


# ------------------------------------------------------------------------------------
# oracle on host cores (cpu_baseline and the reference arm)
# ------------------------------------------------------------------------------------
def oracle_sample(seconds: float):
    """Run the fp64 oracle's apply on a bounded sample of the serving step: layer-0-shaped
    projections (same shapes, same tenant count and batch, Zipf ids) restricted to a few
    output rows each; returns (tokens/s extrapolated to the full 32-layer step, cores,
    description)."""
    import oracle as O
    from workloads import activations, bf16_bits, random_tenant
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        threads = 1
    rng = np.random.default_rng(11)
    B = BATCH
    ids = zipf_ids_host(rng, B, N_TENANTS, ZIPF_S)
    rows_per = 16
    t_total, frac_total = 0.0, 0.0
    it = 0
    while t_total < seconds and it < 64:
        name, d_out, d_in = LLAMA3_8B_PROJECTIONS[it % 7]
        it += 1
        rows = rows_per
        wb = bf16_bits(rng.normal(0, 0.02, size=(rows, d_in)))
        tenants = [random_tenant(rng, rows, d_in, 0, GROUP) for _ in range(N_TENANTS)]
        x = activations(rng, B, d_in)
        t0 = time.perf_counter()
        O.apply_multi(wb, "bf16", tenants, ids, x, "bf16")
        t_total += time.perf_counter() - t0
        frac_total += rows / (sum(o for _, o, _ in LLAMA3_8B_PROJECTIONS) * N_LAYERS)
    step_seconds = t_total / frac_total
    desc = (f"oracle apply_multi (numpy fp64) on {it} projections of Llama-3-8B shape, "
            f"{rows_per} output rows each, batch {B}, {N_TENANTS} tenants, Zipf(1.1) ids; "
            f"time scaled by output rows to the 32-layer step")
    return B / step_seconds, threads, desc


def cpu_baseline(seconds: float) -> dict:
    """The oracle's serving sample on the host: with the BLAS pool as configured (the
    reported value) and with one thread. cores = the host's logical CPUs; blas_threads =
    the threads the multi-threaded run could use."""
    value, threads, desc = oracle_sample(seconds)
    one = None
    try:
        from threadpoolctl import threadpool_limits
        with threadpool_limits(limits=1):
            one, _, _ = oracle_sample(max(2.0, seconds / 3))
    except Exception:
        pass
    return {"value": value, "unit": "tokens/s", "cores": threads, "host_cpus": os.cpu_count(),
            "blas_threads": threads, "single_thread_value": one, "kind": "oracle", "sample": desc}


def reference_arm(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if world > 1 and rank != 0:
        return 0
    per_step_budget = max(2.0, 60.0 / max(1, args.steps + args.warmup))
    vals = []
    cores = 1
    desc = ""
    for i in range(args.warmup + args.steps):
        v, cores, desc = oracle_sample(per_step_budget)
        if i >= args.warmup:
            vals.append(v)
    value = float(np.mean(vals))
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * BATCH / value, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": serving_config(args, world),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line))
    return 0


# ------------------------------------------------------------------------------------
def main():
    args = parse()
    if args.impl == "reference":
        return reference_arm(args)
    import torch
    world, rank, local, pg = setup_dist(args)

    def log(msg):
        if rank == 0:
            print(f"[bench] {msg}", file=sys.stderr, flush=True)

    from tenant_serving_b200 import build
    if rank == 0:
        build.build()
    barrier(pg)
    import tenant_serving_b200 as bd
    bd.lib()
    peaks = load_peaks()
    comp = None
    if not args.no_compress:
        comp = bench_compress(args, log, peaks)
        barrier(pg)
    res = bench_serving(args, rank, pg, log, peaks)
    cpu = None
    dec = dec8 = mix = None
    cold = None
    if rank == 0 and world == 1 and not args.no_extra:
        extra = set(e for e in args.extra.split(",") if e)
        dec = bench_decode(args, log, peaks) if "decode" in extra else None
        dec8 = bench_decode(args, log, peaks, fp8=True) if "decode_fp8" in extra else None
        mix = bench_mixed(args, log, peaks) if "mixed" in extra else None
        cold = bench_cold_start(args, log, peaks) if "cold_start" in extra else None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(args.cpu_seconds)
    if rank == 0:
        line = {
            "metric": METRIC, "value": res["value"], "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": res["ms_per_step"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": serving_config(args, world),
            "hbm_gbs": res["hbm_gbs"], "hbm_frac_of_measured_peak": res["hbm_frac"],
            "roofline": res["roofline"], "cpu_baseline": cpu, "e2e": res["e2e"],
            "gpu_launches": res["gpu_launches"], "clocks": res["clocks"],
            "ms_per_step_profiled": res["ms_per_step_profiled"],
            "distinct_tenants_mean": res["distinct_tenants_mean"],
            "kernels": res["kernels"], "kernel_rates": res["kernel_rates"], "compress": comp,
            "decode": dec, "decode_fp8_base": dec8, "mixed": mix, "cold_start": cold,
        }
        print(json.dumps(line))
    if pg is not None:
        pg.barrier()
        pg.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
