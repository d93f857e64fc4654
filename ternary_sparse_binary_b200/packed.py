"""Device-resident packed matrices and the body-pass helper (argument marshalling only)."""
import ctypes

import numpy as np
import torch

from . import _abi
from ._abi import wal_matrix, wal_pq2_matrix, wal_rc1_matrix


def _ptr(a):
    if a is None:
        return None
    if isinstance(a, torch.Tensor):
        return a.data_ptr()
    return a.ctypes.data


def pack_host(c):
    """Pack dense components (attributes N, K, k, r, T, site_pos, site_sign, alpha,
    beta, U, V, lr_scale as numpy arrays) with the library's host converter.
    Returns the six layout-v1 buffers as numpy uint8 arrays."""
    sizes = _abi.wal_packed_sizes(c.N, c.K, c.k, c.r)
    out = [np.empty(s, dtype=np.uint8) for s in sizes]
    arrs = [np.ascontiguousarray(c.T, np.int8),
            np.ascontiguousarray(c.site_pos, np.uint8) if c.k else None,
            np.ascontiguousarray(c.site_sign, np.int8) if c.k else None,
            np.ascontiguousarray(c.alpha, np.uint16),
            np.ascontiguousarray(c.beta, np.uint16) if c.k else None,
            np.ascontiguousarray(c.U, np.int8) if c.r else None,
            np.ascontiguousarray(c.V, np.int8) if c.r else None,
            np.ascontiguousarray(c.lr_scale, np.uint16) if c.r else None]
    _abi.wal_pack_matrix(*[_ptr(a) for a in arrs], c.N, c.K, c.k, c.r,
                         [_ptr(o) if o.size else None for o in out])
    return out


class PackedMatrix:
    """Six layout-v1 buffers on a CUDA device plus their wal_matrix descriptor."""

    def __init__(self, bufs, N, K, k, r, device="cuda"):
        self.N, self.K, self.k, self.r = N, K, k, r
        self.bufs = [torch.from_numpy(np.ascontiguousarray(b).view(np.uint8).reshape(-1)).to(device)
                     if np.size(b) else None for b in bufs]
        self.desc = wal_matrix(N, K, k, r, *[_ptr(b) if b is not None else None for b in self.bufs])

    @property
    def nbytes(self):
        return sum(b.numel() for b in self.bufs if b is not None)

    def workspace_bytes(self, M=1):
        return _abi.wal_workspace_bytes(self.desc, M)


def pack_pq2_host(T, d, N, K):
    """Pack T (int8 [N, K]) and d (fp16 bits [N, K/128]) into a PQ2_0 buffer
    with the library's host packer; returns a numpy uint8 array."""
    out = np.empty(_abi.wal_pq2_bytes(N, K), dtype=np.uint8)
    T = np.ascontiguousarray(T, np.int8)
    d = np.ascontiguousarray(d, np.uint16)
    _abi.wal_pq2_pack(_ptr(T), _ptr(d), N, K, _ptr(out))
    return out


class Pq2Matrix:
    """A PQ2_0 block buffer on a CUDA device plus its wal_pq2_matrix descriptor."""

    def __init__(self, buf, N, K, device="cuda"):
        self.N, self.K = N, K
        self.buf = torch.from_numpy(np.ascontiguousarray(buf).view(np.uint8).reshape(-1)).to(device)
        self.desc = wal_pq2_matrix(N, K, self.buf.data_ptr())

    @property
    def nbytes(self):
        return self.buf.numel()

    def workspace_bytes(self, M=1):
        return _abi.wal_pq2_workspace_bytes(self.desc, M)


def _dev(a, device):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.uint8).reshape(-1)).to(device)


class Rc1Matrix:
    """A prepared RC1 matrix on a CUDA device: the layout-v1 code plane and
    site bytes, FP32 scales and one WALB2 rank block, with its
    wal_rc1_matrix descriptor.  Built by prepare() from the canonical planes
    (24-bit scales, two paths) with the library's GPU prepare step."""

    def __init__(self, N, K, k, r, codes, sites, scales32, u_bits, v_bits, lr32):
        self.N, self.K, self.k, self.r = N, K, k, r
        self.bufs = [codes, sites, scales32, u_bits, v_bits, lr32]
        ptr = lambda t: t.data_ptr() if t is not None and t.numel() else None
        self.desc = wal_rc1_matrix(N, K, k, r, *[ptr(b) for b in self.bufs])

    @classmethod
    def prepare(cls, codes, sites, scales24, path1, path2, N, K, k, device="cuda", stream=None):
        """codes, sites: layout-v1 host planes; scales24: host bytes of the
        24-bit scale plane; path1, path2: (r_p, u_bits, v_bits, s24) host
        planes (r_p may be 0 with None buffers)."""
        (r1, u1, v1, s1), (r2, u2, v2, s2) = path1, path2
        _, prep = _abi.wal_rc1_sizes(N, K, k, r1, r2)
        d = lambda a: _dev(a, device) if a is not None and np.size(a) else None
        c, st, s24 = d(codes), d(sites), d(scales24)
        ins = [d(u1), d(v1), d(s1), d(u2), d(v2), d(s2)]
        out = [torch.zeros(n, dtype=torch.uint8, device=device) if n else None for n in prep]
        ptr = lambda t: t.data_ptr() if t is not None else None
        _abi.wal_rc1_prepare(N, K, k, ptr(s24), r1, ptr(ins[0]), ptr(ins[1]), ptr(ins[2]), r2, ptr(ins[3]),
                             ptr(ins[4]), ptr(ins[5]), *[ptr(o) for o in out], _stream_handle(stream))
        torch.cuda.current_stream(device).synchronize() if stream is None else stream.synchronize()
        return cls(N, K, k, r1 + r2, c, st, *out)

    @property
    def nbytes(self):
        return sum(b.numel() for b in self.bufs if b is not None)

    def workspace_bytes(self, M=1):
        return _abi.wal_rc1_workspace_bytes(self.desc, M)


def to_device(bufs, N, K, k, r, device="cuda"):
    return PackedMatrix(bufs, N, K, k, r, device)


def _stream_handle(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


class BodyPass:
    """Owns a wal_body_plan handle and its workspace; run() replays the graph.
    The matrices are all PackedMatrix (layout v1), all Pq2Matrix (PQ2_0) or
    all Rc1Matrix (prepared RC1)."""

    def __init__(self, mats, stage_of, xs, ys, M=1, device="cuda"):
        self.mats = list(mats)
        self.descs = [m.desc for m in self.mats]
        kind = type(self.mats[0])
        if any(type(m) is not kind for m in self.mats):
            raise ValueError("a body pass takes matrices of one format")
        self._ws_fn, self._pass_fn = {
            PackedMatrix: (_abi.wal_body_workspace_bytes, _abi.wal_body_pass),
            Pq2Matrix: (_abi.wal_pq2_body_workspace_bytes, _abi.wal_pq2_body_pass),
            Rc1Matrix: (_abi.wal_rc1_body_workspace_bytes, _abi.wal_rc1_body_pass),
        }[kind]
        self.stage_of = [int(s) for s in stage_of]
        self.xs, self.ys, self.M = list(xs), list(ys), M
        nb = self._ws_fn(self.descs, M)
        if nb == 0:
            raise _abi.WalError(_abi.WAL_ERR_ARG, "wal_body_workspace_bytes")
        self.ws = torch.empty(nb, dtype=torch.uint8, device=device)
        self.plan = ctypes.c_void_p(None)

    def run(self, stream=None):
        self._pass_fn(self.plan, self.descs, self.stage_of, [x.data_ptr() for x in self.xs],
                           [y.data_ptr() for y in self.ys], self.M, self.ws.data_ptr(), self.ws.numel(),
                           _stream_handle(stream))

    def close(self):
        if self.plan.value:
            _abi.wal_body_plan_destroy(self.plan)
            self.plan = ctypes.c_void_p(None)

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
