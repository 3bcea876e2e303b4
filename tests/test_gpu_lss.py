"""GPU parity of the lift-splat BEV pooling (LSS tutorial, "Lift" and
"Splat") against the CPU oracle, through the C ABI.  Metric as for the other
paths: max |gpu - oracle| / bound (the oracle's sum of |terms|), exact 0
where the bound is 0; gate 1e-5 (fp32 inputs; the backward accumulates in
fp32).  The forward's pillar sums are exact sums of fixed-point terms; its
stated error (bev_lss_forward in include/bevsample.h) is at most (the
pillar's points) * 2^-(s+1) absolute plus the final fp32 rounding, so that
absolute allowance is taken off before the relative gate.  It matters only
for pillars whose few terms are within a few fixed-point quanta of zero."""
import math

import numpy as np
import pytest
import torch

import oracle
from camera_bev_view_b200 import inputs as I
from camera_bev_view_b200 import ops

pytestmark = pytest.mark.gpu

TOL = 1e-5


def _err(gpu, ref, bound, allow=0.0):
    gpu = gpu.detach().double().cpu().numpy()
    zero = bound == 0
    assert np.all(gpu[zero] == 0.0), "nonzero output where the oracle has no term"
    excess = np.maximum(np.abs(gpu - ref) - allow, 0.0)
    return float((excess[~zero] / bound[~zero]).max()) if (~zero).any() else 0.0


def _half_quantum(depth, feat):
    """2^-(s+1) of the forward's fixed point, s = 62 - e(max|depth| max|feat|)
    - e(N D Hf Wf) clamped to [-126, 127], e(v) the smallest e with v < 2^e
    (the product of the two maxima rounded to fp32)."""
    B, N, D, Hf, Wf = depth.shape
    m = float(np.float32(np.abs(depth.numpy()).max()) * np.float32(np.abs(feat.numpy()).max()))
    if not m > 0.0:
        return 0.0
    s = max(-126, min(127, 62 - math.frexp(m)[1] - math.frexp(N * D * Hf * Wf)[1]))
    return 2.0 ** -(s + 1)


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
    e = _err(out, ref, bound, np.asarray(count, dtype=np.float64)[:, None] * _half_quantum(depth, feat))
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


@pytest.mark.parametrize("C,D,rig", [(100, 17, "config"), (33, 41, "tilted"), (256, 5, "tilted")])
def test_lss_column_block_backward(C, D, rig):
    """Maps large enough for the backward's column blocks (at least one CTA
    per SM): ragged channel chunks (33, 100, 256 channels), an odd bin count,
    a height that is not a multiple of the 16-row block and a width that is
    not a multiple of the 4-column block; on the tilted rig the rows of a
    column fall in different pillars, so runs break inside a column."""
    w = I.LSS_WORKLOADS["lss_b4"].scaled(C=C, D=D, dbound=(4.0, 4.0 + D, 1.0), Hf=21, Wf=42)
    if rig == "config":
        _run(w)
    else:
        Ks, Es = zip(*(I.random_rig(91 + b, w.N, w.img_h, w.img_w) for b in range(w.B)))
        _run(w, K=torch.from_numpy(np.stack(Ks)), E=torch.from_numpy(np.stack(Es)))


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
