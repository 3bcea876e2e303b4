"""GPU parity of the lift-splat BEV pooling (LSS tutorial, "Lift" and
"Splat") against the CPU oracle, through the C ABI.  Metric as for the other
paths: max |gpu - oracle| / bound (the oracle's sum of |terms|), exact 0
where the bound is 0; gate 1e-5 (fp32 inputs; the forward's pillar sums
are exact fixed-point sums, the backward accumulates in fp32)."""
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
    zero = bound == 0
    assert np.all(gpu[zero] == 0.0), "nonzero output where the oracle has no term"
    return float((np.abs(gpu - ref)[~zero] / bound[~zero]).max()) if (~zero).any() else 0.0


def _run(w, depth=None, feat=None, K=None, E=None, dout=None, backward=True):
    if depth is None:
        depth, feat = I.make_lss_inputs(w)
    if K is None:
        K, E = I.make_rigs(w)
    if dout is None:
        dout = I.make_lss_dout(w)
    g = ops.bev_grid_spec(w.ranges, w.res_xy + (w.zr[1] - w.zr[0],))
    og = oracle.LssGrid(w.ranges, w.res_xy, w.dbound)
    dd, fd, Kd, Ed, gd = (t.cuda() for t in (depth, feat, K, E, dout))
    dmin, _, dstep = w.dbound
    out = ops.bev_lss_forward(dd, fd, Kd, Ed, w.img_h, w.img_w, dmin, dstep, g)
    torch.cuda.synchronize()
    ref, bound, count = oracle.lss_forward(depth, feat, K, E, w.img_h, w.img_w, og)
    e = _err(out, ref, bound)
    assert e <= TOL, ("forward", e)
    res = {"out": out, "count": count}
    if backward:
        ddep, dfe = ops.bev_lss_backward(dd, fd, gd, Kd, Ed, w.img_h, w.img_w, dmin, dstep, g)
        torch.cuda.synchronize()
        r = oracle.lss_backward(depth, feat, dout, K, E, w.img_h, w.img_w, og)
        for name, got in (("ddepth", ddep), ("dfeat", dfe)):
            e = _err(got, r[name], r[name + "_bound"])
            assert e <= TOL, (name, e)
        res.update(ddepth=ddep, dfeat=dfe)
    return res


@pytest.mark.parametrize("name", ["lss_tiny", "lss", "lss_b4"])
def test_lss_workloads_forward_backward(name):
    r = _run(I.LSS_WORKLOADS[name])
    assert r["count"].sum() > 0


@pytest.mark.parametrize("C,D", [(1, 41), (256, 8), (33, 1), (100, 17)])
def test_lss_channel_and_bin_counts(C, D):
    w = I.LSS_WORKLOADS["lss_tiny"].scaled(C=C, D=D, dbound=(4.0, 4.0 + D, 1.0))
    _run(w)


def test_lss_random_rig_and_partial_grid():
    """Pitch and roll, off-centre principal points, and a grid that covers only
    part of the frustum (points outside are dropped)."""
    w = I.LSS_WORKLOADS["lss_tiny"].scaled(xr=(-5.0, 15.0), yr=(-12.0, 4.0), X=40, Y=32, zr=(-1.0, 2.5))
    K, E = I.random_rig(77, w.N, w.img_h, w.img_w)
    _run(w, K=torch.from_numpy(K)[None], E=torch.from_numpy(E)[None])


def test_lss_zero_depth_gives_zero_output_and_feat_gradient():
    w = I.LSS_WORKLOADS["lss_tiny"]
    depth, feat = I.make_lss_inputs(w)
    r = _run(w, depth=torch.zeros_like(depth), feat=feat)
    assert torch.count_nonzero(r["out"]) == 0 and torch.count_nonzero(r["dfeat"]) == 0


def test_lss_results_are_reproducible_bit_for_bit():
    w = I.LSS_WORKLOADS["lss_b4"]
    depth, feat = I.make_lss_inputs(w)
    K, E = I.make_rigs(w)
    dout = I.make_lss_dout(w)
    g = ops.bev_grid_spec(w.ranges, w.res_xy + (w.zr[1] - w.zr[0],))
    dd, fd, Kd, Ed, gd = (t.cuda() for t in (depth, feat, K, E, dout))
    outs = [ops.bev_lss_forward(dd, fd, Kd, Ed, w.img_h, w.img_w, 4.0, 1.0, g) for _ in range(2)]
    grads = [ops.bev_lss_backward(dd, fd, gd, Kd, Ed, w.img_h, w.img_w, 4.0, 1.0, g) for _ in range(2)]
    torch.cuda.synchronize()
    assert torch.equal(outs[0], outs[1])
    assert torch.equal(grads[0][0], grads[1][0]) and torch.equal(grads[0][1], grads[1][1])


def test_lss_rejects_host_pointers():
    w = I.LSS_WORKLOADS["lss_tiny"]
    depth, feat = I.make_lss_inputs(w)
    K, E = I.make_rigs(w)
    g = ops.bev_grid_spec(w.ranges, w.res_xy + (w.zr[1] - w.zr[0],))
    with pytest.raises(ops.BevError) as ei:
        ops.bev_lss_forward(depth.cuda(), feat, K.cuda(), E.cuda(), w.img_h, w.img_w, 4.0, 1.0, g)
    assert ei.value.status == -1
