"""GPU parity of the deformable aggregation (SparseDriveV2 notes, "Deformable
Aggregation" steps 1-3) against the CPU oracle, through the C ABI.

Error metric as for the dense path: max |gpu - oracle| / bound, where bound
is the oracle's sum of absolute terms of the same output; where the bound is
0 the GPU value must be exactly 0.  Gate 1e-5: fp32 (and bf16 features,
which widen exactly to fp32) with fp32 accumulation of at most a few hundred
terms per output.
"""
import numpy as np
import pytest
import torch

import oracle
from camera_bev_view_b200 import inputs as I
from camera_bev_view_b200 import ops

pytestmark = pytest.mark.gpu

TOL = 1e-5


def _err(gpu, ref, bound):
    gpu = gpu.detach().double().cpu().numpy()
    diff = np.abs(gpu - ref)
    zero = bound == 0
    assert np.all(gpu[zero] == 0.0), "nonzero output where the oracle has no term"
    return float((diff[~zero] / bound[~zero]).max()) if (~zero).any() else 0.0


def _inputs(w, dev="cuda"):
    F = I.make_features(w)
    K, E = I.make_rigs(w)
    A, D, W = I.make_queries(w)
    g = I.make_query_dout(w)
    return F, K, E, A, D, W, g


def _to(dev, *ts):
    return [t.to(dev) for t in ts]


def _check(w, F, K, E, A, D, W, g, layout=ops.NCHW, backward=True, nonzero=True):
    Fd, Kd, Ed, Ad, Dd, Wd, gd = _to("cuda", F, K, E, A, D, W, g)
    if layout == ops.NHWC:
        Fd = Fd.permute(0, 1, 3, 4, 2).contiguous()
    out = ops.bev_deform_forward(Fd, Kd, Ed, w.img_h, w.img_w, Ad, Dd, Wd, layout=layout)
    torch.cuda.synchronize()
    ref, bound = oracle.deform_forward(F, K, E, w.img_h, w.img_w, A, D, W)
    assert (np.abs(ref).max() > 0) == nonzero
    e = _err(out, ref, bound)
    assert e <= TOL, ("forward", e)
    if not backward:
        return out
    dF, dW, dO = ops.bev_deform_backward(Fd, Kd, Ed, w.img_h, w.img_w, Ad, Dd, Wd, gd, layout=layout)
    torch.cuda.synchronize()
    r = oracle.deform_backward(F, g, K, E, w.img_h, w.img_w, A, D, W)
    for name, got in (("dF", dF), ("dW", dW), ("dOff", dO)):
        e = _err(got, r[name], r[name + "_bound"])
        assert e <= TOL, (name, e)
    return out


def test_deform_tiny_forward_backward():
    w = I.DEFORM_WORKLOADS["deform_tiny"]
    _check(w, *_inputs(w))


def test_deform_full_size_forward_backward():
    """900 queries x 13 keypoints, 6 cameras, C = 256, 64 x 176 maps."""
    w = I.DEFORM_WORKLOADS["deform"]
    _check(w, *_inputs(w))


def test_deform_bf16_batched_forward_backward():
    w = I.DEFORM_WORKLOADS["deform_bf16"]
    _check(w, *_inputs(w))


def test_deform_nhwc_input_is_bitwise_the_same():
    w = I.DEFORM_WORKLOADS["deform_tiny"].scaled(C=32)
    F, K, E, A, D, W, g = _inputs(w)
    o1 = _check(w, F, K, E, A, D, W, g, layout=ops.NCHW, backward=False)
    o2 = _check(w, F, K, E, A, D, W, g, layout=ops.NHWC, backward=False)
    assert torch.equal(o1, o2)


@pytest.mark.parametrize("C,dtype", [(13, "f32"), (3, "f32"), (20, "bf16"), (500, "f32"), (1000, "bf16")])
def test_deform_ragged_and_wide_channels(C, dtype):
    w = I.DEFORM_WORKLOADS["deform_tiny"].scaled(C=C, dtype=dtype, Q=24)
    _check(w, *_inputs(w))


def test_deform_max_keypoints_single_camera_single_query():
    w = I.DEFORM_WORKLOADS["deform_tiny"].scaled(N=1, Q=1, Kp=64)
    F, K, E, A, D, W, g = _inputs(w)
    A[0, 0] = torch.tensor([10.0, 0.0, 0.0])    # 9 m ahead of camera 0: its keypoints are in view
    _check(w, F, K, E, A, D, W, g)
    w = I.DEFORM_WORKLOADS["deform_tiny"].scaled(N=32, Q=5, Kp=3)
    _check(w, *_inputs(w))


def test_deform_invalid_keypoints_and_zero_weights():
    """Keypoints far below the ground plane and behind every camera's field of
    view (200 m below): all samples invalid, so out, dW and dOff are 0 and dF
    is 0.  Then zero weights on valid keypoints: out and dOff are 0 but dW is
    the samples."""
    w = I.DEFORM_WORKLOADS["deform_tiny"]
    F, K, E, A, D, W, g = _inputs(w)
    A2 = A.clone()
    A2[..., 2] = -200.0
    Fd, Kd, Ed, Ad, Dd, Wd, gd = _to("cuda", F, K, E, A2, D, W, g)
    out = ops.bev_deform_forward(Fd, Kd, Ed, w.img_h, w.img_w, Ad, Dd, Wd)
    dF, dW, dO = ops.bev_deform_backward(Fd, Kd, Ed, w.img_h, w.img_w, Ad, Dd, Wd, gd)
    torch.cuda.synchronize()
    for t in (out, dF, dW, dO):
        assert torch.count_nonzero(t) == 0
    _check(w, F, K, E, A, D, torch.zeros_like(W), g, nonzero=False)


def test_deform_unaligned_output_uses_scalar_stores():
    w = I.DEFORM_WORKLOADS["deform_tiny"]
    F, K, E, A, D, W, g = _inputs(w)
    Fd, Kd, Ed, Ad, Dd, Wd = _to("cuda", F, K, E, A, D, W)
    buf = torch.zeros(w.B * w.Q * w.C + 1, device="cuda")
    out = buf[1:].view(w.B, w.Q, w.C)       # 4-byte, not 16-byte, aligned
    ops.bev_deform_forward(Fd, Kd, Ed, w.img_h, w.img_w, Ad, Dd, Wd, out=out)
    torch.cuda.synchronize()
    ref, bound = oracle.deform_forward(F, K, E, w.img_h, w.img_w, A, D, W)
    assert _err(out, ref, bound) <= TOL
    assert buf[0].item() == 0.0


def test_deform_forward_and_weight_offset_gradients_are_deterministic():
    w = I.DEFORM_WORKLOADS["deform"]
    F, K, E, A, D, W, g = _to("cuda", *_inputs(w))
    o1 = ops.bev_deform_forward(F, K, E, w.img_h, w.img_w, A, D, W)
    o2 = ops.bev_deform_forward(F, K, E, w.img_h, w.img_w, A, D, W)
    _, w1, d1 = ops.bev_deform_backward(F, K, E, w.img_h, w.img_w, A, D, W, g)
    _, w2, d2 = ops.bev_deform_backward(F, K, E, w.img_h, w.img_w, A, D, W, g)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(w1, w2) and torch.equal(d1, d2)


def test_deform_rejects_host_pointers():
    w = I.DEFORM_WORKLOADS["deform_tiny"]
    F, K, E, A, D, W, g = _inputs(w)
    Fd, Kd, Ed, Dd, Wd = _to("cuda", F, K, E, D, W)
    with pytest.raises(ops.BevError) as ei:
        ops.bev_deform_forward(Fd, Kd, Ed, w.img_h, w.img_w, A, Dd, Wd)   # anchors on the host
    assert ei.value.status == -1
