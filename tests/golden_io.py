"""Reader for the hand-derived fixtures in tests/golden/."""
import os

import numpy as np

from wal_synth import Components

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def fixture_names():
    return sorted(f[:-4] for f in os.listdir(GOLDEN) if f.endswith(".txt") and f != "README.txt")


def load(name):
    N = K = k = r = None
    lines = []
    with open(os.path.join(GOLDEN, name + ".txt")) as fh:
        for raw in fh:
            line = raw.split("#", 1)[0].strip()
            if not line:
                continue
            key, val = line.split(":", 1)
            lines.append((key.strip(), val.split()))
    for key, v in lines:
        if key == "shape":
            N, K, k, r = map(int, v)
    G = K // 128
    T = np.zeros((N, K), np.int8)
    alpha = np.zeros((N, G), np.uint16)
    beta = np.zeros((N, G), np.uint16)
    U = np.ones((N, r), np.int8)
    V = np.ones((K, r), np.int8)
    s = np.zeros(r, np.uint16)
    x = np.zeros(K, np.uint16)
    sites = {}
    y = np.zeros(N, np.float64)
    codes_hex = None
    for key, v in lines:
        if key == "alpha":
            alpha[int(v[0]), int(v[1])] = int(v[2], 16)
        elif key == "beta":
            beta[int(v[0]), int(v[1])] = int(v[2], 16)
        elif key == "trit":
            T[int(v[0]), int(v[1])] = int(v[2])
        elif key == "site":
            sites.setdefault((int(v[0]), int(v[1])), []).append((int(v[2]), int(v[3])))
        elif key == "u":
            U[int(v[0]), int(v[1])] = int(v[2])
        elif key == "vneg":
            V[int(v[0]), int(v[1])] = -1
        elif key == "s":
            s[int(v[0])] = int(v[1], 16)
        elif key == "x":
            x[int(v[0])] = int(v[1], 16)
        elif key == "x_all":
            x[:] = int(v[0], 16)
        elif key == "y":
            y[int(v[0])] = float(v[1])
        elif key == "codes_hex":
            codes_hex = bytes.fromhex("".join(v))
    pos = np.zeros((N, G, k), np.uint8)
    sgn = np.ones((N, G, k), np.int8)
    if k:
        for n in range(N):
            for g in range(G):
                lst = sorted(sites[(n, g)])
                assert len(lst) == k, f"{name}: need exactly {k} sites in ({n},{g})"
                for i, (p, sg) in enumerate(lst):
                    pos[n, g, i] = p
                    sgn[n, g, i] = sg
    c = Components(N, K, k, r, T, pos, sgn, alpha, beta, U, V, s)
    return c, x, y, codes_hex
