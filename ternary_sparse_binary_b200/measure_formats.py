"""Timing of the format kernels on one GPU: one JSON line per case.

    python -m ternary_sparse_binary_b200.measure_formats [--reps 20]

Cases:
  base3   the base-3 -> layout-v1 conversion (wal_base3_convert) of a
          32768 x 16384 matrix: bytes read (base-3 codes + BF16 scales) and
          written (2-bit code plane + FP16 scales) per call.  The call
          synchronises its stream (it returns the format check), so the
          event-timed interval includes a 4-byte read-back.
  pq2     one PQ2_0 product (wal_pq2_gemm, M = 1) for the 8B gate and down
          shapes and a 27B MLP shape: packed blocks + x + y per launch.
  int4    the INT4/g128 LM head of an 8B model (151936 x 4096, M = 1):
          nibble plane + FP16 scales + x + logits per launch.
  rc1     one prepared RC1 product (wal_rc1_gemm, M = 1) of the 8B gate
          shape, k = 8, two paths of rank 4: code plane + sites + FP32 scales
          + low-rank planes + x + y per launch.
Every call is timed with CUDA events on its stream after 3 warm-up calls,
with a 256 MiB buffer written between calls to flush L2.
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
from wal_synth import gen_base3, gen_int4, gen_pq2, gen_rc1, gen_x  # noqa: E402


def peak_gbs():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as fh:
            return float(json.load(fh)["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def timed(fn, reps):
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    s = torch.cuda.current_stream()
    out = []
    for i in range(reps + 3):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s)
        fn()
        e1.record(s)
        e1.synchronize()
        if i >= 3:
            out.append(e0.elapsed_time(e1) * 1e-3)
    return float(np.mean(out)), float(np.min(out))


def case_base3(reps):
    N, K = 32768, 16384
    T, s = gen_base3(N, K, 6, 1)
    raw = np.empty(wal.wal_base3_bytes(N, K), np.uint8)
    wal.wal_base3_pack(T.ctypes.data, N, K, raw.ctypes.data)
    del T
    sizes = wal.wal_packed_sizes(N, K, 0, 0)
    b3d = torch.from_numpy(raw).cuda()
    sd = torch.from_numpy(s.view(np.int16).reshape(-1)).cuda()
    codes = torch.empty(sizes[0], dtype=torch.uint8, device="cuda")
    alpha = torch.empty(sizes[2], dtype=torch.uint8, device="cuda")
    ws = torch.empty(512, dtype=torch.uint8, device="cuda")
    st = torch.cuda.current_stream().cuda_stream

    def call():
        wal.wal_base3_convert(b3d.data_ptr(), sd.data_ptr(), N, K, codes.data_ptr(), alpha.data_ptr(),
                              ws.data_ptr(), 512, st)
    mean, best = timed(call, reps)
    G = K // 128
    bytes_moved = N * ((K + 4) // 5) + 2 * N * G + N * K // 4 + 2 * N * G
    pk, kind = peak_gbs()
    return {"case": "base3_convert", "shape": [N, K], "bytes_per_call": bytes_moved, "us_per_call": mean * 1e6,
            "us_best": best * 1e6, "gbs": bytes_moved / mean / 1e9, "frac": bytes_moved / mean / 1e9 / pk,
            "peak": pk, "peak_kind": kind}


def case_pq2(N, K, reps, name):
    T, d = gen_pq2(N, K, 6, N + K)
    pm = wal.Pq2Matrix(wal.pack_pq2_host(T, d, N, K), N, K)
    x = torch.from_numpy(gen_x(K, 1, 6, 1).view(np.int16)).cuda()
    y = torch.empty(N, dtype=torch.float32, device="cuda")
    nb = pm.workspace_bytes(1)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    st = torch.cuda.current_stream().cuda_stream

    def call():
        wal.wal_pq2_gemm(pm.desc, x.data_ptr(), 1, K, y.data_ptr(), N, ws.data_ptr(), nb, st)
    mean, best = timed(call, reps)
    bytes_moved = N * (K // 128) * 34 + 2 * K + 4 * N
    pk, kind = peak_gbs()
    return {"case": f"pq2_gemm {name}", "shape": [N, K], "bytes_per_call": bytes_moved, "us_per_call": mean * 1e6,
            "us_best": best * 1e6, "gbs": bytes_moved / mean / 1e9, "frac": bytes_moved / mean / 1e9 / pk,
            "peak": pk, "peak_kind": kind}


def case_int4(reps):
    N, K = 151936, 4096
    q, d = gen_int4(N, K, 6, 2)
    sc, ss = wal.wal_int4_sizes(N, K)
    c, s = np.empty(sc, np.uint8), np.empty(ss, np.uint8)
    wal.wal_int4_pack(q.ctypes.data, d.ctypes.data, N, K, c.ctypes.data, s.ctypes.data)
    del q
    cd, sd = torch.from_numpy(c).cuda(), torch.from_numpy(s).cuda()
    m = wal.wal_int4_matrix(N, K, cd.data_ptr(), sd.data_ptr())
    x = torch.from_numpy(gen_x(K, 1, 6, 3).view(np.int16)).cuda()
    y = torch.empty(N, dtype=torch.float32, device="cuda")
    nb = wal.wal_int4_workspace_bytes(m, 1)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    st = torch.cuda.current_stream().cuda_stream

    def call():
        wal.wal_int4_gemm(m, x.data_ptr(), 1, K, y.data_ptr(), N, ws.data_ptr(), nb, st)
    mean, best = timed(call, reps)
    bytes_moved = N * K // 2 + N * (K // 128) * 2 + 2 * K + 4 * N
    pk, kind = peak_gbs()
    return {"case": "int4_gemm LM head 4096->151936", "shape": [N, K], "bytes_per_call": bytes_moved,
            "us_per_call": mean * 1e6, "us_best": best * 1e6, "gbs": bytes_moved / mean / 1e9,
            "frac": bytes_moved / mean / 1e9 / pk, "peak": pk, "peak_kind": kind}


def case_rc1(reps):
    N, K, k, r1, r2 = 12288, 4096, 8, 4, 4
    dd = gen_rc1(N, K, k, r1, r2, 6, 4)
    G = K // 128
    from wal_synth import Components
    base = wal.pack_host(Components(N, K, k, 0, dd["T"], dd["site_pos"], dd["site_sign"], np.zeros((N, G), np.uint16),
                                    np.zeros((N, G), np.uint16), np.zeros((N, 0), np.int8), np.zeros((K, 0), np.int8),
                                    np.zeros(0, np.uint16)))
    pad = lambda a: np.concatenate([np.ascontiguousarray(a).reshape(-1).view(np.uint8),
                                    np.zeros((-a.nbytes) % 16, np.uint8)])
    paths = []
    for U, V, s in ((dd["U1"], dd["V1"], dd["s1"]), (dd["U2"], dd["V2"], dd["s2"])):
        pb = wal.pack_host(Components(N, K, 0, U.shape[1], np.zeros((N, K), np.int8), np.zeros((N, G, 0), np.uint8),
                                      np.zeros((N, G, 0), np.int8), np.zeros((N, G), np.uint16),
                                      np.zeros((N, G), np.uint16), U, V, np.zeros(U.shape[1], np.uint16)))
        paths.append((U.shape[1], pb[3], pb[4], pad(s)))
    m = wal.Rc1Matrix.prepare(base[0], base[1], pad(np.concatenate([dd["alpha24"], dd["beta24"]], axis=2)),
                              paths[0], paths[1], N, K, k)
    x = torch.from_numpy(gen_x(K, 1, 6, 5).view(np.int16)).cuda()
    y = torch.empty(N, dtype=torch.float32, device="cuda")
    nb = m.workspace_bytes(1)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    st = torch.cuda.current_stream().cuda_stream

    def call():
        wal.wal_rc1_gemm(m.desc, x.data_ptr(), 1, K, y.data_ptr(), N, ws.data_ptr(), nb, st)
    mean, best = timed(call, reps)
    r = r1 + r2
    bytes_moved = N * K // 4 + N * G * k + N * G * 8 + N * 4 + r * K // 8 + 4 * r + 2 * K + 4 * N
    pk, kind = peak_gbs()
    return {"case": "rc1_gemm 8B gate 4096->12288 k=8 r=4+4", "shape": [N, K], "bytes_per_call": bytes_moved,
            "us_per_call": mean * 1e6, "us_best": best * 1e6, "gbs": bytes_moved / mean / 1e9,
            "frac": bytes_moved / mean / 1e9 / pk, "peak": pk, "peak_kind": kind}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--reps", type=int, default=20)
    ap.add_argument("--only", default="")
    a = ap.parse_args()
    cases = {
        "base3": lambda: case_base3(a.reps),
        "pq2_gate": lambda: case_pq2(12288, 4096, a.reps, "8B gate 4096->12288"),
        "pq2_down": lambda: case_pq2(4096, 12288, a.reps, "8B down 12288->4096"),
        "pq2_27b_up": lambda: case_pq2(17408, 5120, a.reps, "27B up 5120->17408"),
        "int4": lambda: case_int4(a.reps),
        "rc1": lambda: case_rc1(a.reps),
    }
    for name, fn in cases.items():
        if a.only and name not in a.only.split(","):
            continue
        print(json.dumps(fn()), flush=True)


if __name__ == "__main__":
    main()
