"""Run one seeded product (or a small body pass) repeatedly: a fixed case for ncu.

    python -m ternary_sparse_binary_b200.profile_case --N 12288 --K 4096 --k 8 --r 8 --reps 4
    python -m ternary_sparse_binary_b200.profile_case --body layer8b --reps 3
"""
import argparse
import os
import sys

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import ternary_sparse_binary_b200 as wal  # noqa: E402
from wal_synth import gen_components, gen_x, config_plan, gen_matrix  # noqa: E402


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--N", type=int, default=12288)
    ap.add_argument("--K", type=int, default=4096)
    ap.add_argument("--k", type=int, default=8)
    ap.add_argument("--r", type=int, default=8)
    ap.add_argument("--M", type=int, default=1)
    ap.add_argument("--reps", type=int, default=4)
    ap.add_argument("--body", default=None, help="run a named workload as a body pass instead")
    a = ap.parse_args()
    dev = torch.device("cuda", 0)
    s = torch.cuda.current_stream()
    if a.body:
        specs = config_plan(a.body)
        mats, xs, ys = [], [], []
        for sp in specs:
            c = gen_matrix(a.body, sp)
            mats.append(wal.PackedMatrix(wal.pack_host(c), sp.N, sp.K, sp.k, sp.r, device=dev))
            xs.append(torch.from_numpy(gen_x(sp.K, a.M, 5, sp.index).view(np.int16)).to(dev))
            ys.append(torch.empty((a.M, sp.N), dtype=torch.float32, device=dev))
        bp = wal.BodyPass(mats, [sp.stage for sp in specs], xs, ys, M=a.M, device=dev)
        for _ in range(a.reps):
            bp.run()
        torch.cuda.synchronize()
        bp.close()
        print(f"body {a.body}: {len(specs)} matrices x {a.reps} passes done")
        return 0
    c = gen_components(a.N, a.K, a.k, a.r, config_id=5, matrix_index=1)
    pm = wal.PackedMatrix(wal.pack_host(c), a.N, a.K, a.k, a.r, device=dev)
    X = torch.from_numpy(gen_x(a.K, a.M, 5, 1).view(np.int16)).to(dev)
    Y = torch.empty((a.M, a.N), dtype=torch.float32, device=dev)
    nb = pm.workspace_bytes(a.M)
    ws = torch.empty(nb, dtype=torch.uint8, device=dev)
    for _ in range(a.reps):
        if a.M == 1:
            wal.wal_gemv(pm.desc, X.data_ptr(), Y.data_ptr(), ws.data_ptr(), nb, s.cuda_stream)
        else:
            wal.wal_gemm_small_m(pm.desc, X.data_ptr(), a.M, a.K, Y.data_ptr(), a.N, ws.data_ptr(), nb,
                                 s.cuda_stream)
    torch.cuda.synchronize()
    print(f"product {a.N}x{a.K} k={a.k} r={a.r} M={a.M}: {a.reps} launches done")
    return 0


if __name__ == "__main__":
    sys.exit(main())
