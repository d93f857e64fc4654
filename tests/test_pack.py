"""Host converter (wal_pack_matrix) against the oracle's own packer, CPU only."""
import numpy as np
import pytest

import oracle
import ternary_sparse_binary_b200 as wal
from wal_synth import Components, gen_components

from golden_io import fixture_names, load


SHAPES = [(512, 1024, 8, 4), (3, 128, 2, 1), (7, 256, 0, 0), (5, 384, 4, 32), (33, 2176, 8, 8),
          (1, 128, 8, 0), (17, 640, 2, 31), (4, 4096, 0, 3)]


@pytest.mark.parametrize("N,K,k,r", SHAPES)
def test_pack_matches_oracle_bytes(N, K, k, r):
    c = gen_components(N, K, k, r, config_id=81, matrix_index=N + K + k + r)
    mine = wal.pack_host(c)
    ref = oracle.pack(c)
    assert [m.size for m in mine] == oracle.packed_sizes(N, K, k, r)
    for i, (a, b) in enumerate(zip(mine, ref)):
        assert np.array_equal(a, b), f"buffer {i} differs"


@pytest.mark.parametrize("name", fixture_names())
def test_pack_golden(name):
    c, _, _, codes_hex = load(name)
    mine = wal.pack_host(c)
    assert all(np.array_equal(a, b) for a, b in zip(mine, oracle.pack(c)))
    if codes_hex is not None:
        assert mine[0][: len(codes_hex)].tobytes() == codes_hex


def test_pack_roundtrip_through_oracle_decoder():
    c = gen_components(64, 1024, 8, 16, config_id=82)
    u = oracle.unpack(wal.pack_host(c), 64, 1024, 8, 16)
    for f in ("T", "site_pos", "site_sign", "alpha", "beta", "U", "V", "lr_scale"):
        assert np.array_equal(getattr(u, f), getattr(c, f)), f


@pytest.mark.parametrize("shape", [(2, 100, 0, 0), (2, 128, 3, 0), (2, 128, 0, 33), (0, 128, 0, 0), (2, 0, 0, 0)])
def test_sizes_reject_bad_shapes(shape):
    with pytest.raises(wal.WalError) as e:
        wal.wal_packed_sizes(*shape)
    assert e.value.status == wal.WAL_ERR_SHAPE


def _bad(mut):
    c = gen_components(4, 256, 4, 2, config_id=83)
    mut(c)
    with pytest.raises(wal.WalError) as e:
        wal.pack_host(c)
    return e.value.status


def test_pack_rejects_trit_out_of_range():
    def m(c): c.T[1, 7] = 2
    assert _bad(m) == wal.WAL_ERR_FORMAT


def test_pack_rejects_duplicate_site():
    def m(c): c.site_pos[2, 1, 1] = c.site_pos[2, 1, 0]
    assert _bad(m) == wal.WAL_ERR_FORMAT


def test_pack_rejects_unsorted_sites():
    def m(c): c.site_pos[0, 0, :] = c.site_pos[0, 0, ::-1].copy()
    assert _bad(m) == wal.WAL_ERR_FORMAT


def test_pack_rejects_position_128():
    def m(c): c.site_pos[0, 1, 3] = 128
    assert _bad(m) == wal.WAL_ERR_FORMAT


def test_pack_rejects_bad_sign_and_lowrank():
    def m(c): c.site_sign[3, 0, 0] = 0
    assert _bad(m) == wal.WAL_ERR_FORMAT

    def m2(c): c.V[5, 1] = 0
    assert _bad(m2) == wal.WAL_ERR_FORMAT


def test_pack_rejects_null_buffers():
    c = gen_components(4, 256, 4, 2, config_id=83)
    with pytest.raises(wal.WalError) as e:
        wal.wal_pack_matrix(c.T.ctypes.data, None, None, c.alpha.ctypes.data, None, None, None, None,
                            4, 256, 4, 2, [None] * 6)
    assert e.value.status == wal.WAL_ERR_ARG


# ---------------------------------------------------------------------------
# PQ2_0 block format
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("N,K", [(1, 128), (3, 256), (64, 4096), (5, 12288), (7, 1152), (33, 5120)])
def test_pq2_pack_matches_oracle_bytes(N, K):
    from oracle import pq2_oracle as pq
    from wal_synth import gen_pq2
    T, d = gen_pq2(N, K, 83, N + K)
    mine = wal.pack_pq2_host(T, d, N, K)
    assert mine.size == pq.packed_bytes(N, K) == wal.wal_pq2_bytes(N, K)
    assert np.array_equal(mine, pq.pack(pq.Pq2(N, K, T, d)))


def test_pq2_pack_rejects_bad_trit():
    T = np.zeros((1, 128), np.int8)
    T[0, 7] = 2
    with pytest.raises(wal.WalError) as e:
        wal.pack_pq2_host(T, np.zeros((1, 1), np.uint16), 1, 128)
    assert e.value.status == wal.WAL_ERR_FORMAT


def test_pq2_sizes_reject_bad_shape():
    assert wal.wal_pq2_bytes(4, 100) == 0
    assert wal.wal_pq2_bytes(0, 128) == 0
    assert wal.wal_pq2_bytes(2, 128) == 80


# ---------------------------------------------------------------------------
# base-3 container
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("N,K", [(1, 128), (2, 256), (3, 384), (4, 512), (5, 640), (2, 4096), (1, 17408)])
def test_base3_pack_matches_oracle_bytes(N, K):
    from oracle import base3_oracle as b3
    from wal_synth import gen_base3
    T, _ = gen_base3(N, K, 84, N + K)
    out = np.empty(wal.wal_base3_bytes(N, K), np.uint8)
    wal.wal_base3_pack(T.ctypes.data, N, K, out.ctypes.data)
    assert out.size == b3.packed_bytes(N, K)
    assert np.array_equal(out, b3.pack(T))


def test_base3_sizes():
    assert wal.wal_base3_bytes(1, 128) == 32  # 26 bytes, padded
    assert wal.wal_base3_bytes(2, 5120) == 2048
    assert wal.wal_base3_bytes(1, 100) == 0


# ---------------------------------------------------------------------------
# INT4 LM head and INT3 embedding planes
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("N,K", [(1, 128), (3, 256), (7, 4096), (2, 12288)])
def test_int4_int3_pack_match_oracle(N, K):
    from oracle import head_oracle as ho
    from wal_synth import gen_int3, gen_int4
    for gen, sizes, pack, ref in ((gen_int4, wal.wal_int4_sizes, wal.wal_int4_pack, ho.int4_pack),
                                  (gen_int3, wal.wal_int3_sizes, wal.wal_int3_pack, ho.int3_pack)):
        q, d = gen(N, K, 85, N + K)
        sc, ss = sizes(N, K)
        c, s = np.empty(sc, np.uint8), np.empty(ss, np.uint8)
        pack(q.ctypes.data, d.ctypes.data, N, K, c.ctypes.data, s.ctypes.data)
        rc, rs = ref(q, d)
        assert np.array_equal(c, rc) and np.array_equal(s, rs)


def test_int_pack_rejects_range():
    c, s = np.empty(64, np.uint8), np.empty(16, np.uint8)
    q = np.zeros((1, 128), np.int8)
    q[0, 9] = 8
    with pytest.raises(wal.WalError):
        wal.wal_int4_pack(q.ctypes.data, np.zeros(1, np.uint16).ctypes.data, 1, 128, c.ctypes.data, s.ctypes.data)
    q[0, 9] = -5
    c3 = np.empty(48, np.uint8)
    with pytest.raises(wal.WalError):
        wal.wal_int3_pack(q.ctypes.data, np.zeros(1, np.uint16).ctypes.data, 1, 128, c3.ctypes.data, s.ctypes.data)


@pytest.mark.parametrize("N,K,k,r1,r2", [(512, 1024, 8, 4, 4), (37, 384, 0, 1, 0), (9, 17408, 2, 16, 16),
                                         (64, 128, 4, 0, 3)])
def test_rc1_sizes_match_oracle_planes(N, K, k, r1, r2):
    """The library's RC1 plane sizes equal the byte counts of the oracle's own
    canonical and prepared planes (each zero-padded to 16 bytes)."""
    from oracle import rc1_oracle as rc
    from wal_synth import gen_rc1
    d = gen_rc1(N, K, k, r1, r2, 68, N + K)
    c = rc.Rc1(N, K, k, d["T"], d["site_pos"], d["site_sign"], d["alpha24"], d["beta24"],
               d["U1"], d["V1"], d["s1"], d["U2"], d["V2"], d["s2"])
    can, prep = wal.wal_rc1_sizes(N, K, k, r1, r2)
    assert can[0] == rc.scales24_plane(c).size
    for (U, V, s), idx in (((d["U1"], d["V1"], d["s1"]), (1, 2, 3)), ((d["U2"], d["V2"], d["s2"]), (4, 5, 6))):
        assert [can[i] for i in idx] == [p.size for p in rc.path_planes(U, V, s)]
    assert list(prep) == [p.size for p in rc.prepared(c)]


@pytest.mark.parametrize("args", [(4, 128, 0, 20, 20), (4, 128, 0, -1, 0), (4, 100, 0, 1, 1), (4, 128, 3, 1, 1)])
def test_rc1_sizes_reject(args):
    with pytest.raises(wal.WalError) as e:
        wal.wal_rc1_sizes(*args)
    assert e.value.status == wal.WAL_ERR_SHAPE


def test_last_error_names_the_reason():
    """A failing call leaves its reason in the thread's error text, which the
    binding's exception carries."""
    with pytest.raises(wal.WalError) as e:
        wal.wal_rc1_sizes(4, 128, 0, 20, 20)
    assert "r1 + r2" in wal.wal_last_error()
    assert "r1 + r2" in str(e.value) and "WAL_ERR_SHAPE" in str(e.value)
