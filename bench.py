#!/usr/bin/env python3
"""Benchmark: one 8B-shaped body pass (252 direct-packed matrices, batch 1) per step.

Default run (one GPU):  python bench.py
Replicas on N GPUs:     python -m torch.distributed.run --nproc-per-node N ... bench.py --gpus N
Oracle (CPU) arm:       python bench.py --impl reference
Second workload:        python bench.py --workload pq2_body8b   (the same 252 shapes as
                        plain-ternary PQ2_0 blocks, 34 bytes per 128 weights)

Prints ONE JSON line (rank 0).  The metric is microseconds per body pass at
batch 1 (lower is better) together with the weight stream in GB/s against the
measured HBM copy bandwidth.
"""
import argparse
import json
import math
import os
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

METRIC = "µs per 8B body pass (batch 1) + weight GB/s as % of B200 HBM roofline"
UNIT = "us/pass"
WORKLOAD = "body8b"
FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0  # B200 HBM3e, DGX figure


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None,
                    help="timed steps (default: 200 body passes on the GPU, 20 oracle samples on the CPU)")
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["wal", "reference"], default="wal")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-sample-matrices", type=int, default=4)
    ap.add_argument("--workload", choices=["body8b", "pq2_body8b"], default="body8b")
    a = ap.parse_args()
    if a.steps is None:
        a.steps = 20 if a.impl == "reference" else 200
    global WORKLOAD
    WORKLOAD = a.workload
    return a


def is_pq2():
    return WORKLOAD == "pq2_body8b"


def workload_text():
    if is_pq2():
        return ("8B-shaped body pass in PQ2_0: 36 layers x 7 plain-ternary matrices (q,k,v,o 4096-wide; gate/up "
                "4096->12288; down 12288->4096), 34-byte blocks (FP16 scale + 32 code bytes) per 128 weights, "
                "batch 1, one CUDA graph holding one persistent cooperative launch, 144 dependency stages "
                "separated by grid barriers")
    return ("8B-shaped body pass: 36 layers x 7 matrices (q,k,v,o 4096-wide; gate/up 4096->12288; "
            "down 12288->4096), k=8 sites per 128-group, 213 of 252 with WALB2 r=8, batch 1, "
            "one CUDA graph holding one persistent cooperative launch, 144 dependency stages "
            "separated by grid barriers")


def seed_id():
    from wal_synth import workload_id
    return workload_id(WORKLOAD)


def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("LOCAL_RANK", 0)), int(os.environ.get("WORLD_SIZE", 1))


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as fh:
            d = json.load(fh)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    """SM clock and clock-event reasons sampled every few milliseconds in a
    thread through NVML (read-only queries; the library nvidia-smi reads),
    each sample stamped with time.monotonic(), so that the summary keeps only
    the samples taken inside the timed window.  Falls back to an
    `nvidia-smi -lms` child when the NVML binding is missing."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, device_index, period_s=0.002):
        self.dev = device_index
        self.period = period_s
        self.rows = []  # (t, sm_mhz, sm_max_mhz, [reason names])
        self.proc = None
        self.thread = None
        self.halt = threading.Event()
        self.source = "none"

    def _nvml_handle(self):
        import pynvml
        import torch
        pynvml.nvmlInit()
        uuid = getattr(torch.cuda.get_device_properties(self.dev), "uuid", None)
        if uuid is not None:
            try:
                return pynvml, pynvml.nvmlDeviceGetHandleByUUID("GPU-" + str(uuid))
            except Exception:
                pass
        return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.dev)

    def start(self):
        try:
            nv, h = self._nvml_handle()
        except Exception:
            return self._start_smi()
        bits = {"hw_slowdown": nv.nvmlClocksEventReasonHwSlowdown,
                "hw_thermal_slowdown": nv.nvmlClocksEventReasonHwThermalSlowdown,
                "sw_thermal_slowdown": nv.nvmlClocksEventReasonSwThermalSlowdown,
                "sw_power_cap": nv.nvmlClocksEventReasonSwPowerCap}
        smax = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
        self.source = "nvml"

        def loop():
            while not self.halt.is_set():
                t = time.monotonic()
                try:
                    sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                    mask = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                except Exception:
                    break
                self.rows.append((t, float(sm), float(smax), [n for n, b in bits.items() if mask & b]))
                time.sleep(self.period)
        self.thread = threading.Thread(target=loop, daemon=True)
        self.thread.start()

    def _start_smi(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.source = "nvidia-smi"

        def read():
            for line in self.proc.stdout:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9 and parts[1].replace(".", "").isdigit():
                    self.rows.append((time.monotonic(), float(parts[1]), float(parts[2]) if parts[2].replace(
                        ".", "").isdigit() else float("nan"),
                        [n for n, v in zip(self.NAMES, parts[5:9]) if v.lower() == "active"]))
        self.thread = threading.Thread(target=read, daemon=True)
        self.thread.start()

    def stop(self):
        self.halt.set()
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        if self.source == "nvml" and not (self.thread and self.thread.is_alive()):
            try:
                import pynvml
                pynvml.nvmlShutdown()
            except Exception:
                pass

    def summary(self, t0=None, t1=None):
        """Samples with t0 <= t <= t1 (all of them without a window)."""
        rows = [r for r in self.rows if (t0 is None or r[0] >= t0) and (t1 is None or r[0] <= t1)]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0,
                    "source": self.source}
        sm = [r[1] for r in rows]
        smax = [r[2] for r in rows if r[2] == r[2]]
        return {"sm_mhz": float(np.median(sm)), "sm_min_mhz": float(min(sm)),
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted({n for r in rows for n in r[3]}), "samples": len(rows), "source": self.source,
                "window_ms": round(1e3 * (rows[-1][0] - rows[0][0]), 1)}


# ---------------------------------------------------------------------------
# workload
# ---------------------------------------------------------------------------
def weight_bytes(s):
    """Algorithmic (payload) bytes of one matrix, before the 16-byte padding.
    Layout v1: codes N K / 4, sites N G k, scales N G (4 | 2), U N ceil(r/32) 4,
    V r K / 8, per-rank scales 2 r.  PQ2_0: 34 bytes per 128 weights."""
    G = s.K // 128
    if is_pq2():
        return s.N * G * 34
    return (s.N * s.K // 4 + s.N * G * s.k + s.N * G * (4 if s.k else 2) + s.N * ((s.r + 31) // 32) * 4
            + s.r * s.K // 8 + 2 * s.r)


def algorithmic_bytes(specs):
    wbytes = sum(weight_bytes(s) for s in specs)
    io = sum(2 * s.K + 4 * s.N for s in specs)
    return wbytes, io


def build_workload(device):
    import torch
    import ternary_sparse_binary_b200 as wal
    from wal_synth import config_plan, gen_matrix, gen_pq2, gen_x
    specs = config_plan(WORKLOAD)
    mats = []
    t0 = time.time()
    for s in specs:
        if is_pq2():
            T, d = gen_pq2(s.N, s.K, seed_id(), s.index)
            mats.append(wal.Pq2Matrix(wal.pack_pq2_host(T, d, s.N, s.K), s.N, s.K, device=device))
            del T, d
        else:
            c = gen_matrix(WORKLOAD, s)
            mats.append(wal.PackedMatrix(wal.pack_host(c), s.N, s.K, s.k, s.r, device=device))
            del c
    setup_s = time.time() - t0
    xoff, yoff = [0], [0]
    for s in specs:
        xoff.append(xoff[-1] + s.K)
        yoff.append(yoff[-1] + s.N)
    x_host = np.concatenate([gen_x(s.K, 1, seed_id(), s.index)[0] for s in specs]).view(np.int16)
    x_pinned = torch.from_numpy(x_host).pin_memory()
    x_dev = x_pinned.to(device)
    y_dev = torch.empty(yoff[-1], dtype=torch.float32, device=device)
    y_pinned = torch.empty(yoff[-1], dtype=torch.float32).pin_memory()
    xs = [x_dev[xoff[i]:xoff[i + 1]] for i in range(len(specs))]
    ys = [y_dev[yoff[i]:yoff[i + 1]] for i in range(len(specs))]
    bp = wal.BodyPass(mats, [s.stage for s in specs], xs, ys, M=1, device=device)
    return dict(specs=specs, mats=mats, bp=bp, x_dev=x_dev, y_dev=y_dev, x_pinned=x_pinned,
                y_pinned=y_pinned, setup_s=setup_s)


def count_launches(specs, M=1):
    """Kernel launches of one body pass: the graph holds a header clear and one
    persistent launch of the decode-GEMV kernel that runs every stage."""
    return 1


def time_gate_product(w, device, reps=20):
    """Per-launch timing of one product (wal_gemv = one decode-GEMV launch) on
    the first gate matrix, L2 flushed between launches."""
    import torch
    import ternary_sparse_binary_b200 as wal
    idx = next(i for i, s in enumerate(w["specs"]) if s.name.endswith("gate"))
    s, pm = w["specs"][idx], w["mats"][idx]
    pq2 = is_pq2()
    x = w["x_dev"][: s.K]
    y = torch.empty(s.N, dtype=torch.float32, device=device)
    nb = pm.workspace_bytes(1)
    ws = torch.empty(nb, dtype=torch.uint8, device=device)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream()
    durs = []
    for i in range(reps + 3):
        flush.zero_()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        if pq2:
            wal.wal_pq2_gemm(pm.desc, x.data_ptr(), 1, s.K, y.data_ptr(), s.N, ws.data_ptr(), nb, stream.cuda_stream)
        else:
            wal.wal_gemv(pm.desc, x.data_ptr(), y.data_ptr(), ws.data_ptr(), nb, stream.cuda_stream)
        e1.record(stream)
        e1.synchronize()
        if i >= 3:
            durs.append(e0.elapsed_time(e1) * 1e-3)
    wbytes = weight_bytes(s) + 2 * s.K + 4 * s.N
    dur = float(np.mean(durs))
    what = f"{s.name} {s.K}->{s.N} PQ2_0" if pq2 else f"{s.name} {s.K}->{s.N} k={s.k} r={s.r}"
    return {"matrix": what, "bytes_per_launch": wbytes,
            "us_per_launch": dur * 1e6, "gbs": wbytes / dur / 1e9}


def load_traffic(kernel="stream_kernel"):
    """Traffic per launch from the committed ncu summary, if it was taken on
    the current kernel source (and the workload's format)."""
    if is_pq2():
        kernel = "stream_kernel_pq2"
    import hashlib
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(p) as fh:
            d = json.load(fh)
        src = os.path.join(ROOT, "ternary_sparse_binary_b200", "csrc", "wal_stream.cu")
        h = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
        if d.get("source_sha256_16") != h:
            return None
        return d.get(kernel)
    except Exception:
        return None


def cpu_baseline(specs, n_sample):
    """The FP64 oracle as it stands on a bounded sample of the body pass:
    n_sample matrices (one of each role, cycling), scaled to a full pass by
    weight count."""
    import oracle
    from oracle import pq2_oracle
    from wal_synth import gen_matrix, gen_pq2, gen_x
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        cores = os.cpu_count() or 1
    roles_seen, sample = set(), []
    for s in specs:
        role = s.name.split(".")[1]
        if role not in roles_seen:
            roles_seen.add(role)
            sample.append(s)
        if len(sample) >= n_sample:
            break
    t_total, w_sample = 0.0, 0
    for s in sample:
        x = gen_x(s.K, 1, seed_id(), s.index)[0]
        if is_pq2():
            T, d = gen_pq2(s.N, s.K, seed_id(), s.index)
            buf = pq2_oracle.pack(pq2_oracle.Pq2(s.N, s.K, T, d))
            t0 = time.perf_counter()
            pq2_oracle.matmul(pq2_oracle.unpack(buf, s.N, s.K), x.reshape(1, -1))
        else:
            c = gen_matrix(WORKLOAD, s)
            t0 = time.perf_counter()
            oracle.matvec(c, x)
        t_total += time.perf_counter() - t0
        w_sample += s.N * s.K
    w_all = sum(s.N * s.K for s in specs)
    us_per_pass = t_total * (w_all / w_sample) * 1e6
    return {"value": us_per_pass, "unit": UNIT, "cores": int(cores), "kind": "oracle",
            "sample": f"{len(sample)} of 252 matrices ({', '.join(x.name for x in sample)}), "
                      f"{t_total:.1f} s, scaled to a pass by weight count"}


# ---------------------------------------------------------------------------
# job timing over replicas
# ---------------------------------------------------------------------------
def max_over_ranks(ms, world, device=None):
    """The largest of the ranks' times (every rank takes part; world 1: itself)."""
    if world <= 1:
        return float(ms)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_rate(max_ms, steps, world):
    """Microseconds per body pass for the whole job: every rank ran `steps`
    independent passes (replicas), all inside the slowest rank's time."""
    return max_ms * 1e3 / (steps * world)


# ---------------------------------------------------------------------------
# arms
# ---------------------------------------------------------------------------
def run_reference(args):
    rank, _, world = dist_env()
    if rank != 0:
        return 0
    from wal_synth import config_plan
    specs = config_plan(WORKLOAD)
    n = max(1, args.cpu_sample_matrices // 2)
    vals = []
    for i in range(args.warmup + args.steps):
        cb = cpu_baseline(specs, n)
        if i >= args.warmup:
            vals.append(cb["value"])
    v = float(np.mean(vals))
    cb["value"] = v
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": v / 1e3, "higher_is_better": False,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": workload_text()},
            "cpu_baseline": cb,
            "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def run_wal(args):
    import torch
    import torch.distributed as dist
    rank, local_rank, world = dist_env()
    if world > 1:
        torch.cuda.set_device(local_rank)
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=torch.device("cuda", local_rank))
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)

    w = build_workload(device)
    specs, bp = w["specs"], w["bp"]
    stream = torch.cuda.current_stream()
    wbytes, iobytes = algorithmic_bytes(specs)
    launches_per_step = count_launches(specs)

    for _ in range(max(3, args.warmup)):
        bp.run()
    torch.cuda.synchronize()

    clocks = ClockSampler(local_rank)
    clocks.start()
    time.sleep(0.05)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    h_start = time.monotonic()
    t_start.record(stream)
    for i in range(args.steps):
        ev[i][0].record(stream)
        bp.run()
        ev[i][1].record(stream)
    t_end.record(stream)
    torch.cuda.synchronize()
    h_end = time.monotonic()
    if world > 1:
        dist.barrier()
    clocks.stop()
    total_ms = t_start.elapsed_time(t_end)
    per_step = np.array([a.elapsed_time(b) for a, b in ev]) * 1e3  # us
    total_ms = max_over_ranks(total_ms, world, device)
    ms_per_step = total_ms / args.steps
    us_per_pass_job = job_rate(total_ms, args.steps, world)
    gbs = (wbytes + iobytes) / (ms_per_step * 1e-3) / 1e9

    # end to end: pinned host x -> device, body pass, device y -> host, every step
    h2d = w["x_pinned"].numel() * 2
    d2h = w["y_pinned"].numel() * 4
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        w["x_dev"].copy_(w["x_pinned"], non_blocking=True)
        bp.run()
        w["y_pinned"].copy_(w["y_dev"], non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, device)
    e2e_us = job_rate(e2e_ms, args.steps, world)

    kernel = time_gate_product(w, device) if rank == 0 else None
    peak, peak_kind = measured_peaks()

    cb = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cb = cpu_baseline(specs, args.cpu_sample_matrices)

    if rank == 0:
        traffic = load_traffic()
        line = {
            "metric": METRIC, "value": us_per_pass_job, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": False, "scaling": "weak",
            "vs_baseline": None, "dtype": "int32+f32 (dp4a on a 24-bit fixed-point x image, FP32 scales and accumulation)",
            "data": "synthetic",
            "config": {"workload": workload_text(),
                       "weights_bytes": wbytes, "io_bytes": iobytes,
                       "l2": f"inputs larger than L2 ({wbytes / 1e9:.2f} GB of packed weights per pass vs 126 MB L2)",
                       "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                       "step_us_p10_p50_p90": [float(np.percentile(per_step, q)) for q in (10, 50, 90)],
                       "weight_gbs": gbs, "setup_s": round(w["setup_s"], 1)},
            # dominant kernel: stream_kernel, timed per launch on the largest matrix of the pass
            "roofline": {"bound": "hbm", "achieved": kernel["gbs"], "peak": peak, "unit": "GB/s",
                         "frac": kernel["gbs"] / peak, "traffic": traffic,
                         "peak_kind": f"{peak_kind} copy bandwidth (MEASURED_PEAKS hbm_gbs)",
                         "kernel": "stream_kernel", "launch": kernel["matrix"],
                         "bytes_per_launch": kernel["bytes_per_launch"], "us_per_launch": kernel["us_per_launch"],
                         "timing": "CUDA events around each launch on its stream, L2 flushed between launches"},
            "pass_roofline": {"achieved": gbs, "unit": "GB/s", "frac": gbs / peak,
                              "frac_of_nominal_8tbs": gbs / NOMINAL_HBM_GBS,
                              "scope": "whole body pass (graph): packed weights + x + y per pass / ms per pass"},
            "e2e": {"value": e2e_us, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            "gpu_launches": launches_per_step * args.steps,
            "clocks": clocks.summary(h_start, h_end),
        }
        if cb:
            line["cpu_baseline"] = cb
        print(json.dumps(line), flush=True)
    bp.close()
    if world > 1:
        dist.destroy_process_group()
    return 0


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    return run_wal(args)


if __name__ == "__main__":
    sys.exit(main())
