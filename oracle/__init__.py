"""Python front of the CPU oracle (``bev_oracle.c``).

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the bench's
CPU-baseline leg are the only callers.  The product path (the CUDA library and
its binding) never imports this package.

The oracle is the plain definition of the exact dense Sampling-VT written as a
loop nest (FlashBEV reading notes, "Method" items 1 and 4): per height bin the
mean over valid cameras of the bilinear samples, summed over height.  See the
header comment of ``bev_oracle.c`` for every reading it takes.

Also the multi-scale form (``ms_forward`` / ``ms_backward``: several
feature-pyramid levels sampled through one geometry and summed inside the
valid mean; pins in ``tests/test_oracle_multiscale.py``), the lift-splat BEV pooling of the LSS tutorial ("Lift", "Splat"):
``lss_forward`` / ``lss_backward`` (pins in ``tests/test_oracle_lss.py``), and
the deformable aggregation of the SparseDriveV2 notes ("Deformable
Aggregation", steps 1-3): ``deform_forward`` / ``deform_backward`` (pins in
``tests/test_oracle_deform.py``).

Pins (in ``tests/test_oracle.py``): a materialised tensorized evaluation with
``torch.nn.functional.grid_sample`` on tiny grids, a hand-derived worked example
(``tests/golden/``), affine and constant feature closed forms, camera
permutation, duplicate-camera and per-bin decompositions, linearity, the
adjoint identity and finite differences for the backward.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "bev_oracle.c")
_LIB = os.path.join(_HERE, "libbevoracle.so")
_lib = None

CFLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
          "-fno-fast-math", "-msse2", "-mfpmath=sse", "-Wall"]


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (fp contraction off, SSE float math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.run(["gcc", *CFLAGS, _SRC, "-o", tmp, "-lm"], check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        I = ctypes.c_int
        F = ctypes.c_float
        lib.oracle_grid_spec.argtypes = [P, P, P, P]
        lib.oracle_grid_spec.restype = I
        lib.oracle_project.argtypes = [P, P, F, F, F, I, I, I, I, P, P, P, P]
        lib.oracle_project.restype = I
        lib.oracle_forward.argtypes = [P, I, I, I, I, I, P, P, I, I, I, I, I, P, P, P, P, P, I]
        lib.oracle_forward.restype = None
        lib.oracle_backward.argtypes = [P, I, I, I, I, I, P, P, I, I, I, I, I, P, P, P, P, I]
        lib.oracle_backward.restype = None
        lib.oracle_ms_forward.argtypes = [P, I, P, P, I, I, I, P, P, I, I, I, I, I, P, P, P, P, P, I]
        lib.oracle_ms_forward.restype = None
        lib.oracle_ms_backward.argtypes = [P, I, P, P, I, I, I, P, P, I, I, I, I, I, P, P, P, P, I]
        lib.oracle_ms_backward.restype = None
        lib.oracle_deform_forward.argtypes = [P, I, I, I, I, I, P, P, I, I, P, P, P, I, I, P, P, I]
        lib.oracle_deform_forward.restype = None
        lib.oracle_deform_backward.argtypes = [P, P, I, I, I, I, I, P, P, I, I, P, P, P, I, I,
                                               P, P, P, P, P, P, I]
        lib.oracle_deform_backward.restype = None
        lib.oracle_lss_cell.argtypes = [P, P, I, I, I, I, I, I, I, F, F, I, I, P, F, P, P]
        lib.oracle_lss_cell.restype = I
        lib.oracle_lss_forward.argtypes = [P, P, I, I, I, I, I, I, P, P, I, I, F, F, I, I, P, F, P, P, P, P]
        lib.oracle_lss_forward.restype = None
        lib.oracle_lss_backward.argtypes = [P, P, P, I, I, I, I, I, I, P, P, I, I, F, F, I, I, P, F, P,
                                            P, P, P, P]
        lib.oracle_lss_backward.restype = None
        _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _np(x, dtype):
    """Contiguous numpy copy; torch tensors (any dtype, incl. bf16) widen exactly."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().cpu()
            if dtype == np.float64:
                x = x.double()
            elif dtype == np.float32:
                x = x.float()
            x = x.numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x, dtype=dtype))


class Grid:
    """Counts and fp32 cell sizes from ranges and resolutions (oracle's own)."""

    def __init__(self, ranges, res):
        r = np.asarray(ranges, dtype=np.float32)
        s = np.asarray(res, dtype=np.float32)
        counts = np.zeros(3, dtype=np.int32)
        cell = np.zeros(3, dtype=np.float32)
        if _load().oracle_grid_spec(_ptr(r), _ptr(s), _ptr(counts), _ptr(cell)) != 0:
            raise ValueError(f"grid ranges {ranges} / resolution {res} do not give integral counts")
        self.X, self.Y, self.Z = (int(v) for v in counts)
        self.lo = np.array([r[0], r[2], r[4]], dtype=np.float32)
        self.cell = cell

    def centres(self, axis: int) -> np.ndarray:
        n = (self.X, self.Y, self.Z)[axis]
        return (self.lo[axis] + ((np.arange(n, dtype=np.float32) + np.float32(0.5))
                                 * self.cell[axis]).astype(np.float32)).astype(np.float32)


def project(K, E, p, img_h, img_w, Hf, Wf):
    """Single point through single camera: (valid, u, v, fx, fy)."""
    K = _np(K, np.float32).reshape(9)
    E = _np(E, np.float32).reshape(16)
    u, v, fx, fy = (np.zeros(1, dtype=np.float32) for _ in range(4))
    ok = _load().oracle_project(_ptr(K), _ptr(E), float(np.float32(p[0])), float(np.float32(p[1])),
                                float(np.float32(p[2])), img_h, img_w, Hf, Wf,
                                _ptr(u), _ptr(v), _ptr(fx), _ptr(fy))
    out = [u[0], v[0], fx[0], fy[0]]
    return bool(ok), float(out[0]), float(out[1]), float(out[2]), float(out[3])


def forward(features, K, E, img_h, img_w, grid: Grid, threads: int = 0):
    """Returns (out [B,C,X,Y] f64, bound [B,C,X,Y] f64, count [B,X,Y,Z] int32).

    ``features`` is [B,N,C,Hf,Wf] (fp32 or bf16; widened exactly to fp64).
    ``threads`` = OpenMP threads (0: the runtime default).
    """
    F = _np(features, np.float64)
    B, N, C, Hf, Wf = F.shape
    Kc = _np(K, np.float32).reshape(B, N, 3, 3)
    Ec = _np(E, np.float32).reshape(B, N, 4, 4)
    out = np.zeros((B, C, grid.X, grid.Y), dtype=np.float64)
    bound = np.zeros_like(out)
    count = np.zeros((B, grid.X, grid.Y, grid.Z), dtype=np.int32)
    _load().oracle_forward(_ptr(F), B, N, C, Hf, Wf, _ptr(Kc), _ptr(Ec), img_h, img_w,
                           grid.X, grid.Y, grid.Z, _ptr(grid.lo), _ptr(grid.cell),
                           _ptr(out), _ptr(bound), _ptr(count), threads)
    return out, bound, count


def backward(dout, N, Hf, Wf, K, E, img_h, img_w, grid: Grid, threads: int = 0):
    """Returns (dF [B,N,C,Hf,Wf] f64, bound [B,N,C,Hf,Wf] f64) for dout [B,C,X,Y]."""
    G = _np(dout, np.float64)
    B, C, X, Y = G.shape
    assert (X, Y) == (grid.X, grid.Y)
    Kc = _np(K, np.float32).reshape(B, N, 3, 3)
    Ec = _np(E, np.float32).reshape(B, N, 4, 4)
    dF = np.zeros((B, N, C, Hf, Wf), dtype=np.float64)
    dB = np.zeros_like(dF)
    _load().oracle_backward(_ptr(G), B, N, C, Hf, Wf, _ptr(Kc), _ptr(Ec), img_h, img_w,
                            grid.X, grid.Y, grid.Z, _ptr(grid.lo), _ptr(grid.cell),
                            _ptr(dF), _ptr(dB), threads)
    return dF, dB


def _ptr_array(arrays):
    return (ctypes.c_void_p * len(arrays))(*[a.ctypes.data for a in arrays])


def ms_forward(levels, K, E, img_h, img_w, grid: Grid, threads: int = 0):
    """Multi-scale forward: ``levels`` = list of [B,N,C,H_l,W_l] feature maps
    (fp32 or bf16, widened exactly).  Returns (out, bound, count) as
    ``forward`` does; the levels' samples are summed inside the valid mean."""
    Fs = [_np(f, np.float64) for f in levels]
    B, N, C = Fs[0].shape[:3]
    assert all(f.shape[:3] == (B, N, C) for f in Fs)
    H = np.array([f.shape[3] for f in Fs], dtype=np.int32)
    W = np.array([f.shape[4] for f in Fs], dtype=np.int32)
    Kc = _np(K, np.float32).reshape(B, N, 3, 3)
    Ec = _np(E, np.float32).reshape(B, N, 4, 4)
    out = np.zeros((B, C, grid.X, grid.Y), dtype=np.float64)
    bound = np.zeros_like(out)
    count = np.zeros((B, grid.X, grid.Y, grid.Z), dtype=np.int32)
    _load().oracle_ms_forward(_ptr_array(Fs), len(Fs), _ptr(H), _ptr(W), B, N, C, _ptr(Kc), _ptr(Ec),
                              img_h, img_w, grid.X, grid.Y, grid.Z, _ptr(grid.lo), _ptr(grid.cell),
                              _ptr(out), _ptr(bound), _ptr(count), threads)
    return out, bound, count


def ms_backward(dout, N, sizes, K, E, img_h, img_w, grid: Grid, threads: int = 0):
    """Multi-scale backward: ``sizes`` = [(H_l, W_l), ...].  Returns
    (list of dF_l [B,N,C,H_l,W_l] f64, list of bounds)."""
    G = _np(dout, np.float64)
    B, C, X, Y = G.shape
    assert (X, Y) == (grid.X, grid.Y)
    H = np.array([h for h, _ in sizes], dtype=np.int32)
    W = np.array([w for _, w in sizes], dtype=np.int32)
    Kc = _np(K, np.float32).reshape(B, N, 3, 3)
    Ec = _np(E, np.float32).reshape(B, N, 4, 4)
    dF = [np.zeros((B, N, C, h, w), dtype=np.float64) for h, w in sizes]
    dB = [np.zeros_like(d) for d in dF]
    _load().oracle_ms_backward(_ptr(G), len(sizes), _ptr(H), _ptr(W), B, N, C, _ptr(Kc), _ptr(Ec),
                               img_h, img_w, grid.X, grid.Y, grid.Z, _ptr(grid.lo), _ptr(grid.cell),
                               _ptr_array(dF), _ptr_array(dB), threads)
    return dF, dB


def deform_forward(features, K, E, img_h, img_w, anchors, offsets, weights, threads: int = 0):
    """Deformable aggregation (SparseDriveV2 notes, "Deformable Aggregation"
    steps 1-3).  features [B,N,C,Hf,Wf]; anchors [B,Q,3]; offsets [B,Q,Kp,3];
    weights [B,Q,N,Kp].  Returns (out [B,Q,C] f64, bound [B,Q,C] f64)."""
    F = _np(features, np.float64)
    B, N, C, Hf, Wf = F.shape
    A = _np(anchors, np.float32)
    D = _np(offsets, np.float32)
    W = _np(weights, np.float32)
    Q, Kp = D.shape[1], D.shape[2]
    assert A.shape == (B, Q, 3) and D.shape == (B, Q, Kp, 3) and W.shape == (B, Q, N, Kp)
    Kc = _np(K, np.float32).reshape(B, N, 3, 3)
    Ec = _np(E, np.float32).reshape(B, N, 4, 4)
    out = np.zeros((B, Q, C), dtype=np.float64)
    bound = np.zeros_like(out)
    _load().oracle_deform_forward(_ptr(F), B, N, C, Hf, Wf, _ptr(Kc), _ptr(Ec), img_h, img_w,
                                  _ptr(A), _ptr(D), _ptr(W), Q, Kp, _ptr(out), _ptr(bound), threads)
    return out, bound


def deform_backward(features, dout, K, E, img_h, img_w, anchors, offsets, weights, threads: int = 0):
    """Gradients of the deformable aggregation for dout [B,Q,C]: returns a dict
    with dF [B,N,C,Hf,Wf], dW [B,Q,N,Kp], dOff [B,Q,Kp,3] (f64) and their
    bounds dF_bound, dW_bound, dOff_bound."""
    F = _np(features, np.float64)
    B, N, C, Hf, Wf = F.shape
    G = _np(dout, np.float64)
    A = _np(anchors, np.float32)
    D = _np(offsets, np.float32)
    W = _np(weights, np.float32)
    Q, Kp = D.shape[1], D.shape[2]
    assert G.shape == (B, Q, C) and W.shape == (B, Q, N, Kp)
    Kc = _np(K, np.float32).reshape(B, N, 3, 3)
    Ec = _np(E, np.float32).reshape(B, N, 4, 4)
    r = {k: np.zeros(s, dtype=np.float64) for k, s in
         [("dF", F.shape), ("dF_bound", F.shape), ("dW", W.shape), ("dW_bound", W.shape),
          ("dOff", D.shape), ("dOff_bound", D.shape)]}
    _load().oracle_deform_backward(_ptr(F), _ptr(G), B, N, C, Hf, Wf, _ptr(Kc), _ptr(Ec), img_h, img_w,
                                   _ptr(A), _ptr(D), _ptr(W), Q, Kp,
                                   _ptr(r["dF"]), _ptr(r["dF_bound"]), _ptr(r["dW"]), _ptr(r["dW_bound"]),
                                   _ptr(r["dOff"]), _ptr(r["dOff_bound"]), threads)
    return r


class LssGrid:
    """BEV pillars of the lift-splat pooling: counts X, Y from x/y ranges and
    cell sizes (oracle's own), one z slab [zmin, zmax), depth bins."""

    def __init__(self, ranges, res_xy, dbound):
        g = Grid((ranges[0], ranges[1], ranges[2], ranges[3], ranges[4], ranges[5]),
                 (res_xy[0], res_xy[1], ranges[5] - ranges[4]))
        self.X, self.Y = g.X, g.Y
        self.lo = g.lo
        self.zmax = np.float32(ranges[5])
        self.cell = np.ascontiguousarray(g.cell[:2])
        self.dmin, self.dmax, self.dstep = (np.float32(v) for v in dbound)
        self.D = int(round((float(dbound[1]) - float(dbound[0])) / float(dbound[2])))


def lss_cell(K, E, h, w, k, img_h, img_w, Hf, Wf, grid: LssGrid):
    """(cell index i*Y + j or -1, ego point) of one frustum point."""
    K = _np(K, np.float32).reshape(9)
    E = _np(E, np.float32).reshape(16)
    p = np.zeros(3, dtype=np.float32)
    c = _load().oracle_lss_cell(_ptr(K), _ptr(E), h, w, k, img_h, img_w, Hf, Wf, float(grid.dmin), float(grid.dstep),
                                grid.X, grid.Y, _ptr(grid.lo), float(grid.zmax), _ptr(grid.cell), _ptr(p))
    return int(c), p


def lss_forward(depth, feat, K, E, img_h, img_w, grid: LssGrid):
    """Lift-splat pooling.  depth [B,N,D,Hf,Wf], feat [B,N,C,Hf,Wf].  Returns
    (out [B,C,X,Y] f64, bound [B,C,X,Y] f64, count [B,X,Y] int32)."""
    A = _np(depth, np.float64)
    Fe = _np(feat, np.float64)
    B, N, D, Hf, Wf = A.shape
    C = Fe.shape[2]
    assert Fe.shape == (B, N, C, Hf, Wf) and D == grid.D
    Kc = _np(K, np.float32).reshape(B, N, 3, 3)
    Ec = _np(E, np.float32).reshape(B, N, 4, 4)
    out = np.zeros((B, C, grid.X, grid.Y), dtype=np.float64)
    bound = np.zeros_like(out)
    count = np.zeros((B, grid.X, grid.Y), dtype=np.int32)
    _load().oracle_lss_forward(_ptr(A), _ptr(Fe), B, N, D, C, Hf, Wf, _ptr(Kc), _ptr(Ec), img_h, img_w,
                               float(grid.dmin), float(grid.dstep), grid.X, grid.Y, _ptr(grid.lo), float(grid.zmax),
                               _ptr(grid.cell), _ptr(out), _ptr(bound), _ptr(count))
    return out, bound, count


def lss_backward(depth, feat, dout, K, E, img_h, img_w, grid: LssGrid):
    """Returns dict ddepth, ddepth_bound [B,N,D,Hf,Wf], dfeat, dfeat_bound [B,N,C,Hf,Wf] (f64)."""
    A = _np(depth, np.float64)
    Fe = _np(feat, np.float64)
    G = _np(dout, np.float64)
    B, N, D, Hf, Wf = A.shape
    C = Fe.shape[2]
    Kc = _np(K, np.float32).reshape(B, N, 3, 3)
    Ec = _np(E, np.float32).reshape(B, N, 4, 4)
    r = {k: np.zeros(s, dtype=np.float64) for k, s in
         [("ddepth", A.shape), ("ddepth_bound", A.shape), ("dfeat", Fe.shape), ("dfeat_bound", Fe.shape)]}
    _load().oracle_lss_backward(_ptr(A), _ptr(Fe), _ptr(G), B, N, D, C, Hf, Wf, _ptr(Kc), _ptr(Ec), img_h, img_w,
                                float(grid.dmin), float(grid.dstep), grid.X, grid.Y, _ptr(grid.lo), float(grid.zmax),
                                _ptr(grid.cell), _ptr(r["ddepth"]), _ptr(r["ddepth_bound"]), _ptr(r["dfeat"]),
                                _ptr(r["dfeat_bound"]))
    return r
