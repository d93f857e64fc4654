"""Batch sweep of one product: gate 4096->12288 and down 12288->4096 (k=8,
r=16), M in {1, 4, 8, 16, 64, 256, 1024}; one JSON line per case.

    python -m ternary_sparse_binary_b200.sweep [--reps 20] [--M 64,256]

Each call of the public entry point (wal_gemv for M = 1, wal_gemm_small_m
otherwise) is timed with CUDA events on its stream, L2 flushed (a 256 MiB
write) before every call.  Reported per case:
  us        mean time per call
  gbs       algorithmic bytes / time: packed weights + 2 M K (x) + 4 M N (y)
  tflops    algorithmic FLOPs / time: 2 M N K (ternary) + 2 M N G k (sites)
            + 2 M r (N + K) (WALB2)
  issued_tflops  what the tensor cores execute for M >= 8: two K-passes over
            the FP16 planes (ternary and residual) + the WALB2 MMA with K = 64
  frac_hbm, frac_tensor  against MEASURED_PEAKS.json (copy GB/s, bf16 burst
            TFLOP/s; FP16 runs at the bf16 rate)
"""
import argparse
import json
import os
import sys

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import ternary_sparse_binary_b200 as wal  # noqa: E402
from wal_synth import config_plan, gen_matrix, gen_x  # noqa: E402


def payload_bytes(N, K, k, r):
    G = K // 128
    return N * K // 4 + N * G * k + N * G * (4 if k else 2) + N * 4 * ((r + 31) // 32) + r * K // 8 + 2 * r


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as fh:
            d = json.load(fh)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), "measured"
    except Exception:
        return 6650.0, 1590.0, "fallback"


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--reps", type=int, default=20)
    ap.add_argument("--M", default="1,4,8,16,64,256,1024")
    a = ap.parse_args()
    Ms = [int(v) for v in a.M.split(",")]
    dev = torch.device("cuda", 0)
    stream = torch.cuda.current_stream()
    hbm, tfl, kind = peaks()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    for spec in config_plan("sweep"):
        c = gen_matrix("sweep", spec)
        pm = wal.PackedMatrix(wal.pack_host(c), spec.N, spec.K, spec.k, spec.r, device=dev)
        N, K, k, r = spec.N, spec.K, spec.k, spec.r
        G = K // 128
        for M in Ms:
            X = torch.from_numpy(gen_x(K, M, 4, 100 + spec.index).view(np.int16)).to(dev)
            Y = torch.empty((M, N), dtype=torch.float32, device=dev)
            nb = pm.workspace_bytes(M)
            ws = torch.empty(nb, dtype=torch.uint8, device=dev)
            durs = []
            for i in range(a.reps + 3):
                flush.zero_()
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                if M == 1:
                    wal.wal_gemv(pm.desc, X.data_ptr(), Y.data_ptr(), ws.data_ptr(), nb, stream.cuda_stream)
                else:
                    wal.wal_gemm_small_m(pm.desc, X.data_ptr(), M, K, Y.data_ptr(), N, ws.data_ptr(), nb,
                                         stream.cuda_stream)
                e1.record(stream)
                e1.synchronize()
                if i >= 3:
                    durs.append(e0.elapsed_time(e1) * 1e-3)
            wal.wal_device_status(ws.data_ptr(), stream.cuda_stream)
            t = float(np.mean(durs))
            nbytes = payload_bytes(N, K, k, r) + 2 * M * K + 4 * M * N
            flops = 2 * M * N * K + 2 * M * N * G * k + 2 * M * r * (N + K)
            issued = (2 * (2 if k else 1) * M * N * K + 2 * M * N * 64) if M >= 8 else 0
            print(json.dumps({
                "matrix": f"{spec.name} {K}->{N} k={k} r={r}", "M": M, "us": round(t * 1e6, 2),
                "gbs": round(nbytes / t / 1e9, 1), "frac_hbm": round(nbytes / t / 1e9 / hbm, 4),
                "tflops": round(flops / t / 1e12, 2), "issued_tflops": round(issued / t / 1e12, 2),
                "frac_tensor": round(issued / t / 1e12 / tfl, 4) if issued else None,
                "path": "tcgen05" if M >= 8 else "cuda-core", "peaks": kind}), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
