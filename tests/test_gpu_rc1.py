"""RC1 storage on the GPU: the prepare step bit for bit, and the FP32-scale
products vs the FP64 oracle (needs a B200).

Tolerance (applied by oracle.check_tolerance, the decoded alpha in the role
of max|alpha|): rel-L2 <= 1e-5 over the output, and per activation row m
max |y_m - y*_m| <= 1e-3 * ||x_m||_2 * max|alpha|.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import rc1_oracle as rc
from wal_synth import Components, gen_components, gen_rc1, gen_x, body_plan, LAYER_27B, ROLE_K_27B

from gpu_util import needs_gpu, wal, device_bf16, stream, assert_parity, device_matrix, run_gemm

pytestmark = [pytest.mark.gpu, needs_gpu]


def _pad16(a):
    b = np.ascontiguousarray(a).reshape(-1).view(np.uint8)
    out = np.zeros((b.size + 15) // 16 * 16, np.uint8)
    out[: b.size] = b
    return out


def _v1_planes(N, K, k, T, pos, sgn, U, V):
    """Layout-v1 planes from the library's host packer (codes, sites, u_bits, v_bits)."""
    G = K // 128
    r = U.shape[1]
    c = Components(N, K, k, r, T, pos, sgn, np.zeros((N, G), np.uint16), np.zeros((N, G), np.uint16), U, V,
                   np.zeros(r, np.uint16))
    return wal().pack_host(c)


def device_rc1(d):
    N, K, k = d["N"], d["K"], d["k"]
    base = _v1_planes(N, K, k, d["T"], d["site_pos"], d["site_sign"], np.zeros((N, 0), np.int8),
                      np.zeros((K, 0), np.int8))
    s24 = np.concatenate([d["alpha24"], d["beta24"]], axis=2) if k else d["alpha24"]
    paths = []
    for U, V, s in ((d["U1"], d["V1"], d["s1"]), (d["U2"], d["V2"], d["s2"])):
        r = U.shape[1]
        if r:
            pb = _v1_planes(N, K, 0, np.zeros((N, K), np.int8), np.zeros((N, K // 128, 0), np.uint8),
                            np.zeros((N, K // 128, 0), np.int8), U, V)
            paths.append((r, pb[3], pb[4], _pad16(s)))
        else:
            paths.append((0, None, None, None))
    return wal().Rc1Matrix.prepare(base[0], base[1] if k else None, _pad16(s24), paths[0], paths[1], N, K, k)


def _rc1(d):
    return rc.Rc1(d["N"], d["K"], d["k"], d["T"], d["site_pos"], d["site_sign"], d["alpha24"], d["beta24"],
                  d["U1"], d["V1"], d["s1"], d["U2"], d["V2"], d["s2"])


def _gemm(m, X):
    w = wal()
    M = X.shape[0]
    Y = torch.full((M, m.N), float("nan"), dtype=torch.float32, device="cuda")
    nb = m.workspace_bytes(M)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    w.wal_rc1_gemm(m.desc, device_bf16(X).data_ptr(), M, m.K, Y.data_ptr(), m.N, ws.data_ptr(), nb, stream())
    torch.cuda.synchronize()
    w.wal_device_status(ws.data_ptr(), stream())
    return Y.cpu().numpy().astype(np.float64)


def _alpha_f32(d):
    return rc.f24_to_f64(d["alpha24"])


def _check(Y, ref, X, d, what):
    # check_tolerance takes alpha as fp16 bits; pass max|alpha| through an equivalent fp16 value bound
    ok, rel, worst = oracle.check_tolerance(Y, ref, X, np.array([0], np.uint16))
    amax = float(np.abs(_alpha_f32(d)).max())
    Xf = oracle.widen_bf16(X).reshape(X.shape[0], -1)
    diff = np.abs(Y.reshape(X.shape[0], -1) - ref.reshape(X.shape[0], -1))
    bound = 1e-3 * np.linalg.norm(Xf, axis=1) * amax
    assert rel <= 1e-5, f"{what}: rel-L2 {rel:.3e}"
    assert np.all(diff.max(axis=1) <= bound), f"{what}: max-abs {diff.max():.3e} above {bound.min():.3e}"


SHAPES = [  # N, K, k, r1, r2
    (512, 1024, 8, 4, 4),
    (37, 384, 2, 1, 0),
    (1000, 2176, 4, 0, 3),
    (64, 128, 0, 0, 0),
    (300, 5120, 4, 8, 8),
    (9, 17408, 8, 16, 16),
    (2051, 4224, 2, 5, 2),
]


@pytest.mark.parametrize("N,K,k,r1,r2", SHAPES)
def test_rc1_prepare_bit_exact(N, K, k, r1, r2):
    d = gen_rc1(N, K, k, r1, r2, 65, N + K)
    m = device_rc1(d)
    want = rc.prepared(_rc1(d))
    for got, ref, name in zip(m.bufs[2:], want, ("scales32", "u_bits", "v_bits", "lr32")):
        if got is None:
            assert not np.any(ref), name
            continue
        assert np.array_equal(got.cpu().numpy(), ref), name


@pytest.mark.parametrize("N,K,k,r1,r2", SHAPES)
@pytest.mark.parametrize("M", [1, 4])
def test_rc1_product_parity(N, K, k, r1, r2, M):
    d = gen_rc1(N, K, k, r1, r2, 66, N + K + M)
    X = gen_x(K, M, 66, N + K)
    Y = _gemm(device_rc1(d), X)
    _check(Y, rc.matmul(_rc1(d), X), X, d, f"RC1 {N}x{K} k={k} r={r1}+{r2} M={M}")


def test_rc1_equals_layout_v1_bitwise_with_fp16_scales():
    """Every scale an FP16 value: the FP32-scale kernel and the layout-v1
    kernel do the same arithmetic, so their outputs are equal bit for bit."""
    from wal_synth import f24_bytes_from_f32
    c = gen_components(2000, 4096, 8, 8, config_id=67, matrix_index=1)
    f24 = lambda b: f24_bytes_from_f32(np.asarray(b, np.uint16).view(np.float16).astype(np.float32))
    d = dict(N=c.N, K=c.K, k=c.k, T=c.T, site_pos=c.site_pos, site_sign=c.site_sign, alpha24=f24(c.alpha),
             beta24=f24(c.beta), U1=c.U[:, :3], V1=c.V[:, :3], s1=f24(c.lr_scale[:3]), U2=c.U[:, 3:],
             V2=c.V[:, 3:], s2=f24(c.lr_scale[3:]))
    X = gen_x(4096, 3, 67, 2)
    y_rc1 = _gemm(device_rc1(d), X)
    y_v1 = run_gemm(device_matrix(c), device_bf16(X), 3)
    assert np.array_equal(y_rc1, y_v1)


def test_rc1_body_two_layers_27b_shapes():
    """Two 27B-shaped layers in RC1 storage (k by role, two WALB2 paths of
    rank 4 on every matrix), run as one body pass; every output checked."""
    w = wal()
    specs = body_plan(2, LAYER_27B, ROLE_K_27B, 8, 7)
    mats, xs, ys, refs = [], [], [], []
    for s in specs:
        d = gen_rc1(s.N, s.K, s.k, 4, 4, 7, 700 + s.index)
        X = gen_x(s.K, 1, 7, 700 + s.index)
        refs.append((s, d, X, rc.matmul(_rc1(d), X)))
        mats.append(device_rc1(d))
        xs.append(device_bf16(X))
        ys.append(torch.full((s.N,), float("nan"), dtype=torch.float32, device="cuda"))
    bp = w.BodyPass(mats, [s.stage for s in specs], xs, ys, M=1)
    for _ in range(2):
        bp.run()
        torch.cuda.synchronize()
        w.wal_device_status(bp.ws.data_ptr(), stream())
    for (s, d, X, ref), y in zip(refs, ys):
        _check(y.cpu().numpy().astype(np.float64).reshape(1, -1), ref, X, d, s.name)
    bp.close()
