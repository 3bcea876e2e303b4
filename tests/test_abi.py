"""The C ABI without a GPU: the library loads, exports every function the
header declares, and rejects bad arguments before touching CUDA."""
import ctypes
import os
import re

import pytest
import torch

from camera_bev_view_b200 import build as B
from camera_bev_view_b200 import ops

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "bevsample.h")
FAKE = 0x10000  # non-NULL, never dereferenced by the paths tested here


@pytest.fixture(scope="module")
def L():
    B.build()
    return ops.lib()


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^[A-Za-z_][\w\s\*]*?\b(bev_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ["bev_grid_spec", "bev_workspace_size", "bev_sample_forward", "bev_sample_backward",
              "bev_status_string"]:
        assert n in names


def test_library_exports_every_declared_symbol(L):
    for name in declared_functions():
        assert hasattr(L, name), name


def test_status_strings(L):
    assert ops.bev_status_string(0) == "ok"
    for s in (-1, -2, -3, -4, -5):
        assert ops.bev_status_string(s) not in ("ok", "unknown status")
    assert ops.bev_status_string(42) == "unknown status"
    # a device-side check failure of the bounds-checked build is reported as
    # BEV_ERR_INTERNAL, with its own text and name in the binding's error
    assert ops.bev_status_string(-5) == "internal consistency check failed"
    e = ops.BevError(-5, "bev_sample_forward")
    assert e.status == -5 and "BEV_ERR_INTERNAL" in str(e) and "internal consistency" in str(e)


def test_bounds_checked_library_exports_the_same_boundary(L):
    """The normal library says it is not bounds-checked; its checked twin
    exports every declared function and says it is."""
    assert L.bev_bounds_checked() == 0
    C = ctypes.CDLL(B.LIB_CHECKED)
    for name in declared_functions():
        assert hasattr(C, name), name
    C.bev_bounds_checked.restype = ctypes.c_int
    assert C.bev_bounds_checked() == 1


def test_noalloc_size_constant_matches_the_header():
    m = re.search(r"#define BEV_NOALLOC_SCRATCH_BYTES \((\d+)u << (\d+)\)", open(HEADER).read())
    assert m and int(m.group(1)) << int(m.group(2)) == ops.BEV_NOALLOC_SCRATCH_BYTES


def test_grid_spec(L):
    g = ops.bev_grid_spec((-50, 50, -50, 50, -5, 3), (0.5, 0.5, 1.0))
    assert (g.X, g.Y, g.Z) == (200, 200, 8)
    assert (g.dx, g.dy, g.dz) == (0.5, 0.5, 1.0)
    g = ops.bev_grid_spec((-50, 50, -50, 50, -5, 3), (0.25, 0.25, 0.5))
    assert (g.X, g.Y, g.Z) == (400, 400, 16)
    g = ops.bev_grid_spec((-25, 25, -25, 25, -5, 3), (1.0, 1.0, 2.0))
    assert (g.X, g.Y, g.Z, g.xmin, g.zmax) == (50, 50, 4, -25.0, 3.0)
    bad = [((-50, 50, -50, 50, -5, 3), (0.3, 0.5, 1.0)),       # non-integral
           ((50, -50, -50, 50, -5, 3), (0.5, 0.5, 1.0)),       # max < min
           ((-50, 50, -50, 50, -5, 3), (0.0, 0.5, 1.0)),       # zero res
           ((-50, 50, -50, 50, -5, float("nan")), (0.5, 0.5, 1.0)),
           ((-50, 50, -50, 50, -5, 3), (1e-4, 0.5, 1.0)),      # count above the limit
           ((-50, 50, -50, 50, -5, 3), (0.5, 0.5, 1e-3))]      # Z above the limit
    for r, s in bad:
        with pytest.raises(ops.BevError) as e:
            ops.bev_grid_spec(r, s)
        assert e.value.status == -1
    assert L.bev_grid_spec(None, None, None) == -1


def test_workspace_sizes(L):
    # NCHW fp32: channels-last copy, C padded to 4, 256-byte aligned
    assert ops.bev_workspace_size(0, 0, 1, 6, 64, 16, 44, 0) == 6 * 16 * 44 * 64 * 4
    assert ops.bev_workspace_size(1, 0, 4, 6, 128, 32, 88, 0) == 4 * 6 * 32 * 88 * 128 * 2
    assert ops.bev_workspace_size(0, 0, 1, 1, 3, 2, 2, 0) == 256          # 16 floats -> 256
    # NHWC with aligned channel count: used in place
    assert ops.bev_workspace_size(0, 1, 1, 6, 64, 16, 44, 0) == 0
    assert ops.bev_workspace_size(1, 1, 1, 6, 120, 16, 44, 0) == 0
    # NHWC with C not a multiple of the 16-byte chunk: repacked
    assert ops.bev_workspace_size(1, 1, 1, 6, 12, 16, 44, 0) == 6 * 16 * 44 * 16 * 2
    # backward: fp32 channels-last gradient
    assert ops.bev_workspace_size(0, 0, 2, 6, 64, 16, 44, 1) == 2 * 6 * 16 * 44 * 64 * 4
    for args in [(0, 0, 0, 6, 64, 16, 44, 0), (0, 0, 1, 33, 64, 16, 44, 0), (2, 0, 1, 6, 64, 16, 44, 0),
                 (0, 2, 1, 6, 64, 16, 44, 0), (0, 0, 1, 6, 64, 0, 44, 1)]:
        with pytest.raises(ops.BevError):
            ops.bev_workspace_size(*args)


def _fwd(L, **kw):
    g = ops.bev_grid_spec((-50, 50, -50, 50, -5, 3), (0.5, 0.5, 1.0))
    a = dict(features=FAKE, dtype=0, layout=0, B=1, N=6, C=64, Hf=16, Wf=44, K=FAKE, E=FAKE,
             img_h=256, img_w=704, grid=ctypes.byref(g), out=FAKE, count=None, ws=FAKE,
             ws_bytes=1 << 30, stream=None)
    a.update(kw)
    return L.bev_sample_forward(a["features"], a["dtype"], a["layout"], a["B"], a["N"], a["C"], a["Hf"],
                                a["Wf"], a["K"], a["E"], a["img_h"], a["img_w"], a["grid"], a["out"],
                                a["count"], a["ws"], a["ws_bytes"], a["stream"])


def _bwd(L, **kw):
    g = ops.bev_grid_spec((-50, 50, -50, 50, -5, 3), (0.5, 0.5, 1.0))
    a = dict(dout=FAKE, B=2, N=6, C=64, Hf=16, Wf=44, K=FAKE, E=FAKE, img_h=256, img_w=704,
             grid=ctypes.byref(g), dF=FAKE, ws=FAKE, ws_bytes=1 << 30, stream=None)
    a.update(kw)
    return L.bev_sample_backward(a["dout"], a["B"], a["N"], a["C"], a["Hf"], a["Wf"], a["K"], a["E"],
                                 a["img_h"], a["img_w"], a["grid"], a["dF"], a["ws"], a["ws_bytes"],
                                 a["stream"])


def test_forward_argument_errors(L):
    bad_grid = ops.BevGrid(0, 10, 10, 0, 1, 0, 1, 0, 1, 0.1, 0.1, 0.1)
    nan_grid = ops.BevGrid(10, 10, 10, float("nan"), 1, 0, 1, 0, 1, 0.1, 0.1, 0.1)
    cases = [
        (dict(features=None), -1), (dict(K=None), -1), (dict(E=None), -1), (dict(out=None), -1),
        (dict(grid=None), -1), (dict(B=0), -1), (dict(N=0), -1), (dict(N=33), -1), (dict(C=0), -1),
        (dict(Hf=0), -1), (dict(Wf=-3), -1), (dict(img_h=0), -1), (dict(img_w=0), -1),
        (dict(grid=ctypes.byref(bad_grid)), -1), (dict(grid=ctypes.byref(nan_grid)), -1),
        (dict(B=20000), -1),                         # B * N beyond the launch limits
        (dict(dtype=2), -2), (dict(layout=5), -2),
        (dict(ws=None), -3), (dict(ws_bytes=100), -3), (dict(ws=FAKE + 8), -3),
        (dict(layout=1, features=FAKE + 4, ws=None, ws_bytes=0), -1),   # NHWC in place must be 16B aligned
    ]
    for kw, want in cases:
        assert _fwd(L, **kw) == want, kw


def test_backward_argument_errors(L):
    cases = [(dict(dout=None), -1), (dict(dF=None), -1), (dict(K=None), -1), (dict(N=40), -1),
             (dict(C=0), -1), (dict(grid=None), -1), (dict(img_w=-1), -1),
             (dict(ws=None), -3), (dict(ws_bytes=1024), -3), (dict(ws=FAKE + 16), -3)]
    for kw, want in cases:
        assert _bwd(L, **kw) == want, kw


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device path")
def test_valid_host_checks_then_cuda_error_without_device(L):
    # every host-side check passes; the first CUDA call reports that no device is usable
    assert _fwd(L) == -4
    assert _bwd(L) == -4


# --------------------------------------------------------------------------
# deformable aggregation
# --------------------------------------------------------------------------

def test_header_declares_the_deformable_calls():
    names = declared_functions()
    for n in ["bev_deform_workspace_size", "bev_deform_forward", "bev_deform_backward"]:
        assert n in names


def test_deform_workspace_sizes(L):
    # fp32 NCHW: repack (B N Hf Wf C 4) for the forward; + gradient buffer for the backward
    fwd = L.bev_deform_workspace_size(0, 0, 1, 6, 256, 64, 176, 0)
    assert fwd == 6 * 64 * 176 * 256 * 4
    bwd = L.bev_deform_workspace_size(0, 0, 1, 6, 256, 64, 176, 1)
    assert bwd == fwd + 6 * 64 * 176 * 256 * 4
    # NHWC with whole chunks is used in place: no repack
    assert L.bev_deform_workspace_size(0, 1, 1, 6, 256, 64, 176, 0) == 0
    # bf16: chunks of 8 channels, fp32 gradient buffer padded to them
    assert L.bev_deform_workspace_size(1, 1, 2, 6, 12, 8, 22, 1) == ((2 * 6 * 8 * 22 * 16 * 2 + 255) // 256 * 256
                                                                      + (2 * 6 * 8 * 22 * 16 * 4 + 255) // 256 * 256)
    assert L.bev_deform_workspace_size(0, 0, 0, 6, 16, 8, 22, 0) == ctypes.c_size_t(-1).value
    assert L.bev_deform_workspace_size(3, 0, 1, 6, 16, 8, 22, 0) == ctypes.c_size_t(-1).value


def _dfwd(L, **kw):
    a = dict(features=FAKE, dtype=0, layout=0, B=1, N=6, C=256, Hf=64, Wf=176, K=FAKE, E=FAKE, img_h=512,
             img_w=1408, A=FAKE, D=FAKE, W=FAKE, Q=900, Kp=13, out=FAKE, ws=FAKE, ws_bytes=1 << 30, stream=None)
    a.update(kw)
    return L.bev_deform_forward(a["features"], a["dtype"], a["layout"], a["B"], a["N"], a["C"], a["Hf"], a["Wf"],
                                a["K"], a["E"], a["img_h"], a["img_w"], a["A"], a["D"], a["W"], a["Q"], a["Kp"],
                                a["out"], a["ws"], a["ws_bytes"], a["stream"])


def _dbwd(L, **kw):
    a = dict(features=FAKE, dtype=0, layout=0, B=1, N=6, C=256, Hf=64, Wf=176, K=FAKE, E=FAKE, img_h=512,
             img_w=1408, A=FAKE, D=FAKE, W=FAKE, Q=900, Kp=13, dout=FAKE, dF=FAKE, dW=FAKE, dO=FAKE,
             ws=FAKE, ws_bytes=1 << 30, stream=None)
    a.update(kw)
    return L.bev_deform_backward(a["features"], a["dtype"], a["layout"], a["B"], a["N"], a["C"], a["Hf"],
                                 a["Wf"], a["K"], a["E"], a["img_h"], a["img_w"], a["A"], a["D"], a["W"], a["Q"],
                                 a["Kp"], a["dout"], a["dF"], a["dW"], a["dO"], a["ws"], a["ws_bytes"],
                                 a["stream"])


def test_deform_argument_errors(L):
    common = [(dict(features=None), -1), (dict(K=None), -1), (dict(A=None), -1), (dict(D=None), -1),
              (dict(W=None), -1), (dict(Q=0), -1), (dict(Kp=0), -1), (dict(Kp=65), -1), (dict(N=33), -1),
              (dict(img_h=0), -1), (dict(dtype=2), -2), (dict(layout=7), -2),
              (dict(C=513), -2),                                  # beyond 4 chunks per lane (fp32)
              (dict(ws=None), -3), (dict(ws_bytes=64), -3), (dict(ws=FAKE + 8), -3)]
    for kw, want in common + [(dict(out=None), -1)]:
        assert _dfwd(L, **kw) == want, kw
    for kw, want in common + [(dict(dout=None), -1), (dict(dF=None), -1), (dict(dW=None), -1),
                              (dict(dO=None), -1)]:
        assert _dbwd(L, **kw) == want, kw
    # bf16 takes up to 1024 channels
    assert _dfwd(L, dtype=1, C=1024) != -2 and _dfwd(L, dtype=1, C=1032) == -2


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device path")
def test_deform_valid_host_checks_then_cuda_error_without_device(L):
    assert _dfwd(L) == -4
    assert _dbwd(L) == -4


# --------------------------------------------------------------------------
# lift-splat pooling
# --------------------------------------------------------------------------

def test_header_declares_the_lss_calls():
    names = declared_functions()
    for n in ["bev_lss_workspace_size", "bev_lss_forward", "bev_lss_backward"]:
        assert n in names


def test_lss_workspace_sizes(L):
    assert L.bev_lss_workspace_size(1, 6, 64, 41, 8, 22, 200, 200, 0) == 256 + 200 * 200 * 64 * 8
    assert L.bev_lss_workspace_size(1, 6, 64, 41, 8, 22, 200, 200, 1) == 200 * 200 * 64 * 4
    assert L.bev_lss_workspace_size(1, 6, 64, 0, 8, 22, 200, 200, 0) == ctypes.c_size_t(-1).value
    assert L.bev_lss_workspace_size(1, 6, 64, 41, 8, 22, 0, 200, 0) == ctypes.c_size_t(-1).value


def _lfwd(L, **kw):
    g = ops.bev_grid_spec((-50, 50, -50, 50, -10, 10), (0.5, 0.5, 20.0))
    a = dict(depth=FAKE, feat=FAKE, B=1, N=6, D=41, C=64, Hf=8, Wf=22, K=FAKE, E=FAKE, img_h=128, img_w=352,
             dmin=4.0, dstep=1.0, grid=ctypes.byref(g), out=FAKE, ws=FAKE, ws_bytes=1 << 30, stream=None)
    a.update(kw)
    return L.bev_lss_forward(a["depth"], a["feat"], a["B"], a["N"], a["D"], a["C"], a["Hf"], a["Wf"], a["K"],
                             a["E"], a["img_h"], a["img_w"], a["dmin"], a["dstep"], a["grid"], a["out"], a["ws"],
                             a["ws_bytes"], a["stream"])


def _lbwd(L, **kw):
    g = ops.bev_grid_spec((-50, 50, -50, 50, -10, 10), (0.5, 0.5, 20.0))
    a = dict(depth=FAKE, feat=FAKE, dout=FAKE, B=1, N=6, D=41, C=64, Hf=8, Wf=22, K=FAKE, E=FAKE, img_h=128,
             img_w=352, dmin=4.0, dstep=1.0, grid=ctypes.byref(g), dd=FAKE, df=FAKE, ws=FAKE, ws_bytes=1 << 30,
             stream=None)
    a.update(kw)
    return L.bev_lss_backward(a["depth"], a["feat"], a["dout"], a["B"], a["N"], a["D"], a["C"], a["Hf"], a["Wf"],
                              a["K"], a["E"], a["img_h"], a["img_w"], a["dmin"], a["dstep"], a["grid"], a["dd"],
                              a["df"], a["ws"], a["ws_bytes"], a["stream"])


def test_lss_argument_errors(L):
    common = [(dict(depth=None), -1), (dict(feat=None), -1), (dict(K=None), -1), (dict(grid=None), -1),
              (dict(D=0), -1), (dict(N=40), -1), (dict(img_w=0), -1), (dict(dstep=0.0), -1),
              (dict(dstep=float("nan")), -1), (dict(dmin=float("inf")), -1), (dict(C=257), -2),
              (dict(ws=None), -3), (dict(ws_bytes=64), -3), (dict(ws=FAKE + 8), -3)]
    for kw, want in common + [(dict(out=None), -1)]:
        assert _lfwd(L, **kw) == want, kw
    for kw, want in common + [(dict(dout=None), -1), (dict(dd=None), -1), (dict(df=None), -1)]:
        assert _lbwd(L, **kw) == want, kw


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device path")
def test_lss_valid_host_checks_then_cuda_error_without_device(L):
    assert _lfwd(L) == -4
    assert _lbwd(L) == -4


# --------------------------------------------------------------------------
# multi-scale dense Sampling-VT
# --------------------------------------------------------------------------

def test_header_declares_the_multiscale_calls():
    names = declared_functions()
    for n in ["bev_multiscale_workspace_size", "bev_sample_forward_multiscale", "bev_sample_backward_multiscale"]:
        assert n in names
    assert re.search(r"#define BEV_MAX_LEVELS 4\b", open(HEADER).read())


P2_P5 = [(64, 176), (32, 88), (16, 44), (8, 22)]


def test_multiscale_workspace_sizes(L):
    per = [ops.bev_workspace_size(0, 0, 1, 6, 64, h, w, 0) for h, w in P2_P5]
    assert ops.bev_multiscale_workspace_size(0, 0, 1, 6, 64, P2_P5, 0) == sum(per)
    assert ops.bev_multiscale_workspace_size(0, 1, 1, 6, 64, P2_P5, 0) == 0          # NHWC in place
    # per-level regions are 256-byte aligned: 1x1x3 channels of 2x2 texels -> 256 bytes each
    assert ops.bev_multiscale_workspace_size(0, 0, 1, 1, 3, [(2, 2), (1, 1), (1, 2)], 0) == 3 * 256
    bw = [ops.bev_workspace_size(0, 0, 2, 6, 64, h, w, 1) for h, w in P2_P5]
    assert ops.bev_multiscale_workspace_size(0, 0, 2, 6, 64, P2_P5, 1) == sum(bw)
    assert ops.bev_multiscale_workspace_size(0, 0, 1, 6, 64, P2_P5[:1], 0) == per[0]
    for args in [(0, 0, 1, 6, 64, [], 0), (0, 0, 1, 6, 64, P2_P5 + [(4, 11)], 0),
                 (0, 0, 1, 6, 64, [(16, 44), (0, 22)], 0), (2, 0, 1, 6, 64, P2_P5, 0), (0, 0, 1, 33, 64, P2_P5, 1)]:
        with pytest.raises(ops.BevError):
            ops.bev_multiscale_workspace_size(*args)


def _ms_fwd(L, levels=P2_P5, feats=None, **kw):
    g = ops.bev_grid_spec((-50, 50, -50, 50, -5, 3), (0.5, 0.5, 1.0))
    n = len(levels)
    fp = feats if feats is not None else (ctypes.c_void_p * max(n, 1))(*([FAKE] * max(n, 1)))
    a = dict(features=fp, n=n, H=ops._int_array([h for h, _ in levels] or [0]),
             W=ops._int_array([w for _, w in levels] or [0]), dtype=0, layout=0, B=1, N=6, C=64, K=FAKE, E=FAKE,
             img_h=256, img_w=704, grid=ctypes.byref(g), out=FAKE, count=None, ws=FAKE, ws_bytes=1 << 30,
             stream=None)
    a.update(kw)
    return L.bev_sample_forward_multiscale(a["features"], a["n"], a["H"], a["W"], a["dtype"], a["layout"], a["B"],
                                           a["N"], a["C"], a["K"], a["E"], a["img_h"], a["img_w"], a["grid"],
                                           a["out"], a["count"], a["ws"], a["ws_bytes"], a["stream"])


def _ms_bwd(L, levels=P2_P5, grads=None, **kw):
    g = ops.bev_grid_spec((-50, 50, -50, 50, -5, 3), (0.5, 0.5, 1.0))
    n = len(levels)
    gp = grads if grads is not None else (ctypes.c_void_p * max(n, 1))(*([FAKE] * max(n, 1)))
    a = dict(dout=FAKE, n=n, H=ops._int_array([h for h, _ in levels] or [0]),
             W=ops._int_array([w for _, w in levels] or [0]), B=2, N=6, C=64, K=FAKE, E=FAKE, img_h=256,
             img_w=704, grid=ctypes.byref(g), dF=gp, ws=FAKE, ws_bytes=1 << 30, stream=None)
    a.update(kw)
    return L.bev_sample_backward_multiscale(a["dout"], a["n"], a["H"], a["W"], a["B"], a["N"], a["C"], a["K"],
                                            a["E"], a["img_h"], a["img_w"], a["grid"], a["dF"], a["ws"],
                                            a["ws_bytes"], a["stream"])


def test_multiscale_argument_errors(L):
    one_null = (ctypes.c_void_p * 4)(FAKE, FAKE, None, FAKE)
    cases = [
        (dict(features=None), -1), (dict(n=0), -1), (dict(n=5), -1), (dict(H=None), -1), (dict(W=None), -1),
        (dict(K=None), -1), (dict(out=None), -1), (dict(grid=None), -1), (dict(N=33), -1), (dict(C=0), -1),
        (dict(img_w=0), -1), (dict(feats=one_null), -1),
        (dict(dtype=2), -2), (dict(layout=3), -2),
        (dict(ws=None), -3), (dict(ws_bytes=1000), -3), (dict(ws=FAKE + 8), -3),
    ]
    for kw, want in cases:
        feats = kw.pop("feats", None)
        assert _ms_fwd(L, feats=feats, **kw) == want, kw
    assert _ms_fwd(L, levels=[(16, 44), (0, 22)]) == -1
    unaligned = (ctypes.c_void_p * 4)(FAKE, FAKE + 4, FAKE, FAKE)
    assert _ms_fwd(L, feats=unaligned, layout=1, ws=None, ws_bytes=0) == -1   # NHWC in place must be 16B aligned
    bwd = [(dict(dout=None), -1), (dict(dF=None), -1), (dict(n=0), -1), (dict(n=5), -1), (dict(N=40), -1),
           (dict(grads=one_null), -1), (dict(ws=None), -3), (dict(ws_bytes=4096), -3), (dict(ws=FAKE + 16), -3)]
    for kw, want in bwd:
        grads = kw.pop("grads", None)
        assert _ms_bwd(L, grads=grads, **kw) == want, kw


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device path")
def test_multiscale_valid_host_checks_then_cuda_error_without_device(L):
    assert _ms_fwd(L) == -4
    assert _ms_bwd(L) == -4
