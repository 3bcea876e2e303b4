"""ctypes binding of ``libbevsample.so`` (C ABI in ``include/bevsample.h``).

Argument marshalling only: every step of the view transform runs in the CUDA
library.  PyTorch supplies device memory and the current stream.  If the
library has not been built this module raises on first use -- there is no
CPU fallback.

The functions keep the C names:

    bev_grid_spec(range6, res3)                      -> BevGrid
    bev_workspace_size(dtype, layout, B, N, C, Hf, Wf, for_backward) -> int
    bev_sample_forward(features, K, E, img_h, img_w, grid, ...) -> (out, count)
    bev_sample_backward(dout, K, E, img_h, img_w, grid, N, Hf, Wf, ...) -> dfeatures
    bev_sample_backward_noalloc(dout, K, E, img_h, img_w, grid, N, Hf, Wf, out) -> dfeatures
    bev_features_to_channels_last(features, out=None) -> [B,N,Hf,Wf,C] copy
    bev_deform_workspace_size(dtype, layout, B, N, C, Hf, Wf, for_backward) -> int
    bev_deform_forward(features, K, E, img_h, img_w, anchors, offsets, weights, ...) -> [B,Q,C]
    bev_deform_backward(features, K, E, img_h, img_w, anchors, offsets, weights, dout, ...)
                                                     -> (dfeatures, dweights, doffsets)
    bev_lss_workspace_size(B, N, C, D, Hf, Wf, X, Y, for_backward) -> int
    bev_lss_forward(depth, feat, K, E, img_h, img_w, dmin, dstep, grid, ...) -> [B,C,X,Y]
    bev_lss_backward(depth, feat, dout, K, E, img_h, img_w, dmin, dstep, grid, ...) -> (ddepth, dfeat)
    bev_status_string(status)                        -> str
"""
from __future__ import annotations

import ctypes
import os

import torch

from . import build as _build

F32, BF16 = 0, 1
NCHW, NHWC = 0, 1
BEV_NOALLOC_SCRATCH_BYTES = 16 << 20  # include/bevsample.h: size of the built-in array of the no-alloc backward
STATUS = {0: "BEV_OK", -1: "BEV_ERR_INVALID_ARG", -2: "BEV_ERR_UNSUPPORTED",
          -3: "BEV_ERR_WORKSPACE", -4: "BEV_ERR_CUDA", -5: "BEV_ERR_INTERNAL"}


class BevError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)} ({bev_status_string(status)})")


class BevGrid(ctypes.Structure):
    _fields_ = [("X", ctypes.c_int), ("Y", ctypes.c_int), ("Z", ctypes.c_int),
                ("xmin", ctypes.c_float), ("xmax", ctypes.c_float),
                ("ymin", ctypes.c_float), ("ymax", ctypes.c_float),
                ("zmin", ctypes.c_float), ("zmax", ctypes.c_float),
                ("dx", ctypes.c_float), ("dy", ctypes.c_float), ("dz", ctypes.c_float)]

    def __repr__(self):
        return (f"BevGrid(X={self.X}, Y={self.Y}, Z={self.Z}, x=[{self.xmin},{self.xmax}], "
                f"y=[{self.ymin},{self.ymax}], z=[{self.zmin},{self.zmax}], "
                f"d=({self.dx},{self.dy},{self.dz}))")


_lib = None


def library_path() -> str:
    return _build.LIB


def lib():
    """Load the library (never builds it implicitly on a GPU run)."""
    global _lib
    if _lib is None:
        path = _build.LIB
        if not os.path.exists(path):
            raise RuntimeError(f"{path} is missing: build it with `python -m camera_bev_view_b200.build` "
                               "(nvcc, sm_100a); this package has no CPU fallback")
        L = ctypes.CDLL(path)
        P, I, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        L.bev_bounds_checked.argtypes = []
        L.bev_bounds_checked.restype = I
        L.bev_grid_spec.argtypes = [P, P, ctypes.POINTER(BevGrid)]
        L.bev_grid_spec.restype = I
        L.bev_workspace_size.argtypes = [I, I, I, I, I, I, I, I]
        L.bev_workspace_size.restype = S
        L.bev_sample_forward.argtypes = [P, I, I, I, I, I, I, I, P, P, I, I, ctypes.POINTER(BevGrid),
                                         P, P, P, S, P]
        L.bev_sample_forward.restype = I
        L.bev_sample_backward.argtypes = [P, I, I, I, I, I, P, P, I, I, ctypes.POINTER(BevGrid),
                                          P, P, S, P]
        L.bev_sample_backward.restype = I
        L.bev_sample_backward_noalloc.argtypes = [P, I, I, I, I, I, P, P, I, I, ctypes.POINTER(BevGrid),
                                                  P, P]
        L.bev_sample_backward_noalloc.restype = I
        L.bev_features_to_channels_last.argtypes = [P, I, I, I, I, I, I, P, P]
        L.bev_features_to_channels_last.restype = I
        L.bev_deform_workspace_size.argtypes = [I, I, I, I, I, I, I, I]
        L.bev_deform_workspace_size.restype = S
        L.bev_deform_forward.argtypes = [P, I, I, I, I, I, I, I, P, P, I, I, P, P, P, I, I, P, P, S, P]
        L.bev_deform_forward.restype = I
        L.bev_deform_backward.argtypes = [P, I, I, I, I, I, I, I, P, P, I, I, P, P, P, I, I, P, P, P, P, P, S, P]
        L.bev_deform_backward.restype = I
        Fl = ctypes.c_float
        L.bev_lss_workspace_size.argtypes = [I, I, I, I, I, I, I, I, I]
        L.bev_lss_workspace_size.restype = S
        L.bev_lss_forward.argtypes = [P, P, I, I, I, I, I, I, P, P, I, I, Fl, Fl, ctypes.POINTER(BevGrid), P, P, S, P]
        L.bev_lss_forward.restype = I
        L.bev_lss_backward.argtypes = [P, P, P, I, I, I, I, I, I, P, P, I, I, Fl, Fl, ctypes.POINTER(BevGrid),
                                       P, P, P, S, P]
        L.bev_lss_backward.restype = I
        L.bev_multiscale_workspace_size.argtypes = [I, I, I, I, I, I, P, P, I]
        L.bev_multiscale_workspace_size.restype = S
        L.bev_sample_forward_multiscale.argtypes = [P, I, P, P, I, I, I, I, I, P, P, I, I,
                                                    ctypes.POINTER(BevGrid), P, P, P, S, P]
        L.bev_sample_forward_multiscale.restype = I
        L.bev_sample_backward_multiscale.argtypes = [P, I, P, P, I, I, I, P, P, I, I, ctypes.POINTER(BevGrid),
                                                     P, P, S, P]
        L.bev_sample_backward_multiscale.restype = I
        L.bev_status_string.argtypes = [I]
        L.bev_status_string.restype = ctypes.c_char_p
        _lib = L
    return _lib


def bev_bounds_checked() -> bool:
    """True when the loaded library is the bounds-checked build."""
    return bool(lib().bev_bounds_checked())


def bev_status_string(status: int) -> str:
    return lib().bev_status_string(int(status)).decode()


def bev_grid_spec(range6, res3) -> BevGrid:
    r = (ctypes.c_float * 6)(*[float(v) for v in range6])
    s = (ctypes.c_float * 3)(*[float(v) for v in res3])
    g = BevGrid()
    st = lib().bev_grid_spec(r, s, ctypes.byref(g))
    if st != 0:
        raise BevError(st, "bev_grid_spec")
    return g


def bev_workspace_size(dtype: int, layout: int, B: int, N: int, C: int, Hf: int, Wf: int,
                       for_backward: int) -> int:
    v = lib().bev_workspace_size(dtype, layout, B, N, C, Hf, Wf, for_backward)
    if v == ctypes.c_size_t(-1).value:
        raise BevError(-1, "bev_workspace_size")
    return int(v)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return F32
    if t.dtype == torch.bfloat16:
        return BF16
    raise TypeError(f"features must be float32 or bfloat16, got {t.dtype}")


def _stream_ptr(stream) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return int(s.cuda_stream)


def _workspace(nbytes: int, device, workspace):
    if nbytes == 0:
        return None, 0
    if workspace is not None:
        return workspace, workspace.numel() * workspace.element_size()
    return torch.empty(nbytes, dtype=torch.uint8, device=device), nbytes


def bev_sample_forward(features: torch.Tensor, K: torch.Tensor, E: torch.Tensor, img_h: int, img_w: int,
                       grid: BevGrid, layout: int = NCHW, out: torch.Tensor | None = None,
                       count: torch.Tensor | bool | None = None, workspace: torch.Tensor | None = None,
                       stream=None):
    """Forward on device tensors.  ``features`` is [B,N,C,Hf,Wf] (NCHW) or
    [B,N,Hf,Wf,C] (NHWC).  Returns (out [B,C,X,Y] fp32, count [B,X,Y,Z] uint8 or None)."""
    if layout == NCHW:
        B, N, C, Hf, Wf = features.shape
    else:
        B, N, Hf, Wf, C = features.shape
    dev = features.device
    dtype = _dtype_code(features)
    if out is None:
        out = torch.empty((B, C, grid.X, grid.Y), dtype=torch.float32, device=dev)
    if count is True:
        count = torch.empty((B, grid.X, grid.Y, grid.Z), dtype=torch.uint8, device=dev)
    elif count is False:
        count = None
    ws, ws_bytes = _workspace(bev_workspace_size(dtype, layout, B, N, C, Hf, Wf, 0), dev, workspace)
    st = lib().bev_sample_forward(
        features.data_ptr(), dtype, layout, B, N, C, Hf, Wf, K.data_ptr(), E.data_ptr(), int(img_h),
        int(img_w), ctypes.byref(grid), out.data_ptr(), count.data_ptr() if count is not None else None,
        ws.data_ptr() if ws is not None else None, ws_bytes, _stream_ptr(stream))
    if st != 0:
        raise BevError(st, "bev_sample_forward")
    return out, count


def bev_sample_backward(dout: torch.Tensor, K: torch.Tensor, E: torch.Tensor, img_h: int, img_w: int,
                        grid: BevGrid, N: int, Hf: int, Wf: int, out: torch.Tensor | None = None,
                        workspace: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """dL/dfeatures [B,N,C,Hf,Wf] fp32 for dout [B,C,X,Y] fp32."""
    B, C = dout.shape[:2]
    dev = dout.device
    if out is None:
        out = torch.empty((B, N, C, Hf, Wf), dtype=torch.float32, device=dev)
    ws, ws_bytes = _workspace(bev_workspace_size(F32, NCHW, B, N, C, Hf, Wf, 1), dev, workspace)
    st = lib().bev_sample_backward(
        dout.data_ptr(), B, N, C, Hf, Wf, K.data_ptr(), E.data_ptr(), int(img_h), int(img_w),
        ctypes.byref(grid), out.data_ptr(), ws.data_ptr() if ws is not None else None, ws_bytes,
        _stream_ptr(stream))
    if st != 0:
        raise BevError(st, "bev_sample_backward")
    return out


def _int_array(vals):
    return (ctypes.c_int * len(vals))(*[int(v) for v in vals])


def _ptr_array(tensors):
    return (ctypes.c_void_p * len(tensors))(*[t.data_ptr() for t in tensors])


def bev_multiscale_workspace_size(dtype: int, layout: int, B: int, N: int, C: int, sizes,
                                  for_backward: int) -> int:
    """``sizes`` = [(H_l, W_l), ...]."""
    v = lib().bev_multiscale_workspace_size(dtype, layout, B, N, C, len(sizes), _int_array([h for h, _ in sizes]),
                                            _int_array([w for _, w in sizes]), for_backward)
    if v == ctypes.c_size_t(-1).value:
        raise BevError(-1, "bev_multiscale_workspace_size")
    return int(v)


def bev_sample_forward_multiscale(levels, K: torch.Tensor, E: torch.Tensor, img_h: int, img_w: int,
                                  grid: BevGrid, layout: int = NCHW, out: torch.Tensor | None = None,
                                  count: torch.Tensor | bool | None = None, workspace: torch.Tensor | None = None,
                                  stream=None):
    """Multi-scale forward.  ``levels`` = list of device tensors, level l
    [B,N,C,H_l,W_l] (NCHW) or [B,N,H_l,W_l,C] (NHWC), one dtype.  Returns
    (out [B,C,X,Y] fp32, count [B,X,Y,Z] uint8 or None)."""
    levels = list(levels)
    if layout == NCHW:
        B, N, C = levels[0].shape[:3]
        sizes = [tuple(f.shape[3:5]) for f in levels]
    else:
        B, N = levels[0].shape[:2]
        C = levels[0].shape[4]
        sizes = [tuple(f.shape[2:4]) for f in levels]
    dev = levels[0].device
    dtype = _dtype_code(levels[0])
    if out is None:
        out = torch.empty((B, C, grid.X, grid.Y), dtype=torch.float32, device=dev)
    if count is True:
        count = torch.empty((B, grid.X, grid.Y, grid.Z), dtype=torch.uint8, device=dev)
    elif count is False:
        count = None
    ws, ws_bytes = _workspace(bev_multiscale_workspace_size(dtype, layout, B, N, C, sizes, 0), dev, workspace)
    st = lib().bev_sample_forward_multiscale(
        _ptr_array(levels), len(levels), _int_array([h for h, _ in sizes]), _int_array([w for _, w in sizes]),
        dtype, layout, B, N, C, K.data_ptr(), E.data_ptr(), int(img_h), int(img_w), ctypes.byref(grid),
        out.data_ptr(), count.data_ptr() if count is not None else None,
        ws.data_ptr() if ws is not None else None, ws_bytes, _stream_ptr(stream))
    if st != 0:
        raise BevError(st, "bev_sample_forward_multiscale")
    return out, count


def bev_sample_backward_multiscale(dout: torch.Tensor, K: torch.Tensor, E: torch.Tensor, img_h: int, img_w: int,
                                   grid: BevGrid, N: int, sizes, out=None, workspace: torch.Tensor | None = None,
                                   stream=None):
    """dL/dF_l for every level: list of [B,N,C,H_l,W_l] fp32 for dout [B,C,X,Y]."""
    B, C = dout.shape[:2]
    dev = dout.device
    sizes = [tuple(s) for s in sizes]
    if out is None:
        out = [torch.empty((B, N, C, h, w), dtype=torch.float32, device=dev) for h, w in sizes]
    ws, ws_bytes = _workspace(bev_multiscale_workspace_size(F32, NCHW, B, N, C, sizes, 1), dev, workspace)
    st = lib().bev_sample_backward_multiscale(
        dout.data_ptr(), len(sizes), _int_array([h for h, _ in sizes]), _int_array([w for _, w in sizes]),
        B, N, C, K.data_ptr(), E.data_ptr(), int(img_h), int(img_w), ctypes.byref(grid),
        _ptr_array(out), ws.data_ptr() if ws is not None else None, ws_bytes, _stream_ptr(stream))
    if st != 0:
        raise BevError(st, "bev_sample_backward_multiscale")
    return out


def bev_features_to_channels_last(features: torch.Tensor, out: torch.Tensor | None = None, stream=None):
    """[B,N,C,Hf,Wf] -> [B,N,Hf,Wf,C] (same dtype) on the device."""
    B, N, C, Hf, Wf = features.shape
    if out is None:
        out = torch.empty((B, N, Hf, Wf, C), dtype=features.dtype, device=features.device)
    st = lib().bev_features_to_channels_last(features.data_ptr(), _dtype_code(features), B, N, C, Hf, Wf,
                                             out.data_ptr(), _stream_ptr(stream))
    if st != 0:
        raise BevError(st, "bev_features_to_channels_last")
    return out


def bev_sample_backward_noalloc(dout: torch.Tensor, K: torch.Tensor, E: torch.Tensor, img_h: int, img_w: int,
                                grid: BevGrid, N: int, Hf: int, Wf: int, out: torch.Tensor,
                                stream=None) -> torch.Tensor:
    """Feature gradient without a workspace, for callers that cannot allocate:
    the library accumulates in its own fixed 16 MiB device array.  ``out``
    ([B,N,C,Hf,Wf] fp32) must be supplied; this wrapper allocates nothing."""
    if dout.dim() != 4 or dout.dtype != torch.float32 or not dout.is_contiguous():
        raise ValueError("dout must be a contiguous fp32 [B,C,X,Y] tensor")
    B, C = dout.shape[:2]
    if (tuple(out.shape) != (B, N, C, Hf, Wf) or out.dtype != torch.float32 or not out.is_contiguous()
            or out.device != dout.device):
        raise ValueError(f"out must be a contiguous fp32 tensor of shape {(B, N, C, Hf, Wf)} on {dout.device}")
    st = lib().bev_sample_backward_noalloc(
        dout.data_ptr(), B, N, C, Hf, Wf, K.data_ptr(), E.data_ptr(), int(img_h), int(img_w),
        ctypes.byref(grid), out.data_ptr(), _stream_ptr(stream))
    if st != 0:
        raise BevError(st, "bev_sample_backward_noalloc")
    return out


def bev_deform_workspace_size(dtype: int, layout: int, B: int, N: int, C: int, Hf: int, Wf: int,
                              for_backward: int) -> int:
    v = lib().bev_deform_workspace_size(dtype, layout, B, N, C, Hf, Wf, for_backward)
    if v == ctypes.c_size_t(-1).value:
        raise BevError(-1, "bev_deform_workspace_size")
    return int(v)


def _feature_dims(features: torch.Tensor, layout: int):
    if layout == NCHW:
        B, N, C, Hf, Wf = features.shape
    else:
        B, N, Hf, Wf, C = features.shape
    return B, N, C, Hf, Wf


def bev_deform_forward(features: torch.Tensor, K: torch.Tensor, E: torch.Tensor, img_h: int, img_w: int,
                       anchors: torch.Tensor, offsets: torch.Tensor, weights: torch.Tensor, layout: int = NCHW,
                       out: torch.Tensor | None = None, workspace: torch.Tensor | None = None, stream=None):
    """Deformable aggregation on device tensors: anchors [B,Q,3], offsets
    [B,Q,Kp,3], weights [B,Q,N,Kp] (fp32).  Returns out [B,Q,C] fp32."""
    B, N, C, Hf, Wf = _feature_dims(features, layout)
    Q, Kp = offsets.shape[1], offsets.shape[2]
    dev = features.device
    dtype = _dtype_code(features)
    if out is None:
        out = torch.empty((B, Q, C), dtype=torch.float32, device=dev)
    ws, ws_bytes = _workspace(bev_deform_workspace_size(dtype, layout, B, N, C, Hf, Wf, 0), dev, workspace)
    st = lib().bev_deform_forward(
        features.data_ptr(), dtype, layout, B, N, C, Hf, Wf, K.data_ptr(), E.data_ptr(), int(img_h), int(img_w),
        anchors.data_ptr(), offsets.data_ptr(), weights.data_ptr(), Q, Kp, out.data_ptr(),
        ws.data_ptr() if ws is not None else None, ws_bytes, _stream_ptr(stream))
    if st != 0:
        raise BevError(st, "bev_deform_forward")
    return out


def bev_deform_backward(features: torch.Tensor, K: torch.Tensor, E: torch.Tensor, img_h: int, img_w: int,
                        anchors: torch.Tensor, offsets: torch.Tensor, weights: torch.Tensor, dout: torch.Tensor,
                        layout: int = NCHW, out: tuple | None = None, workspace: torch.Tensor | None = None,
                        stream=None):
    """Gradients for dout [B,Q,C]: returns (dfeatures [B,N,C,Hf,Wf], dweights
    [B,Q,N,Kp], doffsets [B,Q,Kp,3]), all fp32."""
    B, N, C, Hf, Wf = _feature_dims(features, layout)
    Q, Kp = offsets.shape[1], offsets.shape[2]
    dev = features.device
    dtype = _dtype_code(features)
    if out is None:
        out = (torch.empty((B, N, C, Hf, Wf), dtype=torch.float32, device=dev),
               torch.empty((B, Q, N, Kp), dtype=torch.float32, device=dev),
               torch.empty((B, Q, Kp, 3), dtype=torch.float32, device=dev))
    dF, dW, dO = out
    ws, ws_bytes = _workspace(bev_deform_workspace_size(dtype, layout, B, N, C, Hf, Wf, 1), dev, workspace)
    st = lib().bev_deform_backward(
        features.data_ptr(), dtype, layout, B, N, C, Hf, Wf, K.data_ptr(), E.data_ptr(), int(img_h), int(img_w),
        anchors.data_ptr(), offsets.data_ptr(), weights.data_ptr(), Q, Kp, dout.data_ptr(), dF.data_ptr(),
        dW.data_ptr(), dO.data_ptr(), ws.data_ptr() if ws is not None else None, ws_bytes, _stream_ptr(stream))
    if st != 0:
        raise BevError(st, "bev_deform_backward")
    return dF, dW, dO


def bev_lss_workspace_size(B: int, N: int, C: int, D: int, Hf: int, Wf: int, X: int, Y: int,
                           for_backward: int) -> int:
    v = lib().bev_lss_workspace_size(B, N, C, D, Hf, Wf, X, Y, for_backward)
    if v == ctypes.c_size_t(-1).value:
        raise BevError(-1, "bev_lss_workspace_size")
    return int(v)


def bev_lss_forward(depth: torch.Tensor, feat: torch.Tensor, K: torch.Tensor, E: torch.Tensor, img_h: int,
                    img_w: int, dmin: float, dstep: float, grid: BevGrid, out: torch.Tensor | None = None,
                    workspace: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Lift-splat pooling: depth [B,N,D,Hf,Wf], feat [B,N,C,Hf,Wf] fp32 ->
    out [B,C,X,Y] fp32."""
    B, N, D, Hf, Wf = depth.shape
    C = feat.shape[2]
    dev = depth.device
    if out is None:
        out = torch.empty((B, C, grid.X, grid.Y), dtype=torch.float32, device=dev)
    ws, ws_bytes = _workspace(bev_lss_workspace_size(B, N, C, D, Hf, Wf, grid.X, grid.Y, 0), dev, workspace)
    st = lib().bev_lss_forward(depth.data_ptr(), feat.data_ptr(), B, N, D, C, Hf, Wf, K.data_ptr(), E.data_ptr(),
                               int(img_h), int(img_w), float(dmin), float(dstep), ctypes.byref(grid), out.data_ptr(),
                               ws.data_ptr() if ws is not None else None, ws_bytes, _stream_ptr(stream))
    if st != 0:
        raise BevError(st, "bev_lss_forward")
    return out


def bev_lss_backward(depth: torch.Tensor, feat: torch.Tensor, dout: torch.Tensor, K: torch.Tensor, E: torch.Tensor,
                     img_h: int, img_w: int, dmin: float, dstep: float, grid: BevGrid, out: tuple | None = None,
                     workspace: torch.Tensor | None = None, stream=None):
    """Gradients for dout [B,C,X,Y]: (ddepth [B,N,D,Hf,Wf], dfeat [B,N,C,Hf,Wf])."""
    B, N, D, Hf, Wf = depth.shape
    C = feat.shape[2]
    dev = depth.device
    if out is None:
        out = (torch.empty_like(depth, dtype=torch.float32), torch.empty_like(feat, dtype=torch.float32))
    dd, df = out
    ws, ws_bytes = _workspace(bev_lss_workspace_size(B, N, C, D, Hf, Wf, grid.X, grid.Y, 1), dev, workspace)
    st = lib().bev_lss_backward(depth.data_ptr(), feat.data_ptr(), dout.data_ptr(), B, N, D, C, Hf, Wf,
                                K.data_ptr(), E.data_ptr(), int(img_h), int(img_w), float(dmin), float(dstep),
                                ctypes.byref(grid), dd.data_ptr(), df.data_ptr(),
                                ws.data_ptr() if ws is not None else None, ws_bytes, _stream_ptr(stream))
    if st != 0:
        raise BevError(st, "bev_lss_backward")
    return dd, df
