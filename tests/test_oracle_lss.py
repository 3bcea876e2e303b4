"""Pins of the oracle's lift-splat BEV pooling (LSS tutorial, "Lift" and
"Splat") against things other than itself: a hand-computed frustum point,
the materialised float64 form (inverse matrices, explicit outer product,
index_add), the count closed form, linearity, the adjoints and camera
permutation.
"""
import numpy as np
import pytest
import torch

import oracle
from camera_bev_view_b200 import inputs as I
from tensorized_vt import tensorized_lss


def _grid(w):
    return oracle.LssGrid(w.ranges, w.res_xy, w.dbound)


def test_lss_principal_ray_lands_straight_ahead():
    """Jitter-free rig; camera 0 (yaw 0, at (1, 0, 1.5)) with its principal
    point moved to the centre of feature texel (3, 10) (u = 10.5 * 16 = 168,
    v = 3.5 * 16 = 56): bin k lies straight ahead at depth 4 + k, i.e. at ego
    (5 + k, 0, 1.5), in pillar (floor((5 + k + 20) / 1), floor(20 / 1))."""
    w = I.LSS_WORKLOADS["lss_tiny"]
    K, E = I.make_rig(0, 6, 128, 352, jitter=False)
    K[0, 0, 2], K[0, 1, 2] = 168.0, 56.0
    g = _grid(w)
    for k in range(8):
        cell, p = oracle.lss_cell(K[0], E[0], 3, 10, k, 128, 352, 8, 22, g)
        np.testing.assert_allclose(p, [5.0 + k, 0.0, 1.5], atol=2e-5)
        assert cell == (5 + k + 20) * 40 + 20
    # a point behind the 12 m depth range would be bin 8: not part of the frustum;
    # points below the slab are dropped
    g2 = oracle.LssGrid((-20, 20, -20, 20, 2.0, 10.0), (1.0, 1.0), (4.0, 12.0, 1.0))
    assert oracle.lss_cell(K[0], E[0], 3, 10, 0, 128, 352, 8, 22, g2)[0] == -1


CASES = [
    # workload, rig kind, seed
    ("lss_tiny", "config", 31),
    ("lss_tiny", "random", 32),
    ("lss", "config", 33),
]


def _inputs(name, kind, seed):
    w = I.LSS_WORKLOADS[name]
    depth, feat = I.make_lss_inputs(w)
    if kind == "config":
        K, E = I.make_rigs(w)
    else:
        K, E = I.random_rig(seed, w.N, w.img_h, w.img_w)
        K, E = torch.from_numpy(K)[None], torch.from_numpy(E)[None]
    return w, depth, feat, K, E


@pytest.mark.parametrize("case", CASES, ids=[f"{c[0]}-{c[1]}" for c in CASES])
def test_lss_oracle_matches_tensorized(case):
    w, depth, feat, K, E = _inputs(*case)
    _, _, amb = tensorized_lss(depth, feat, K, E, w.img_h, w.img_w, w.ranges, (w.X, w.Y), w.dbound)
    depth = depth * (~amb).to(depth.dtype)           # points on a cell edge carry no weight
    g = _grid(w)
    out, bound, count = oracle.lss_forward(depth, feat, K, E, w.img_h, w.img_w, g)
    ref, ref_count, _ = tensorized_lss(depth, feat, K, E, w.img_h, w.img_w, w.ranges, (w.X, w.Y), w.dbound)
    assert count.sum() > 0
    err = np.abs(out - ref.numpy()) / np.maximum(bound, 1e-30)
    err = np.where(bound > 0, err, np.abs(out - ref.numpy()))
    assert err.max() < 1e-9
    # every point in a cell (ambiguous ones included) is counted the same way
    amb_any = amb.any()
    if not amb_any:
        np.testing.assert_array_equal(count, ref_count.numpy().astype(np.int32))


def test_lss_unit_inputs_give_the_point_count():
    """feat = 1 and depth = 1 everywhere: each pillar sums to the number of
    frustum points it holds."""
    w = I.LSS_WORKLOADS["lss_tiny"]
    K, E = I.make_rigs(w)
    g = _grid(w)
    depth = torch.ones((1, 6, w.D, w.Hf, w.Wf))
    feat = torch.ones((1, 6, 3, w.Hf, w.Wf))
    out, _, count = oracle.lss_forward(depth, feat, K, E, w.img_h, w.img_w, g)
    for c in range(3):
        np.testing.assert_array_equal(out[0, c], count[0].astype(np.float64))
    assert count.sum() > 0.5 * 6 * w.D * w.Hf * w.Wf


def test_lss_linearity_permutation_and_adjoints():
    w = I.LSS_WORKLOADS["lss_tiny"]
    depth, feat = I.make_lss_inputs(w)
    K, E = I.make_rigs(w)
    g = _grid(w)
    out, _, _ = oracle.lss_forward(depth, feat, K, E, w.img_h, w.img_w, g)
    o2, _, _ = oracle.lss_forward(depth, 3.0 * feat.double(), K, E, w.img_h, w.img_w, g)
    np.testing.assert_allclose(o2, 3.0 * out, rtol=1e-13, atol=1e-13)
    o3, _, _ = oracle.lss_forward(0.5 * depth.double(), feat, K, E, w.img_h, w.img_w, g)
    np.testing.assert_allclose(o3, 0.5 * out, rtol=1e-13, atol=1e-13)
    perm = torch.tensor([2, 5, 0, 1, 4, 3])
    op, _, _ = oracle.lss_forward(depth[:, perm], feat[:, perm], K[:, perm], E[:, perm], w.img_h, w.img_w, g)
    np.testing.assert_allclose(op, out, rtol=1e-12, atol=1e-12)
    dout = I.make_lss_dout(w).double()
    r = oracle.lss_backward(depth, feat, dout, K, E, w.img_h, w.img_w, g)
    lhs = float((out * dout.numpy()).sum())
    for name, x in (("ddepth", depth), ("dfeat", feat)):
        rhs = float((x.double().numpy() * r[name]).sum())
        assert abs(lhs - rhs) <= 1e-12 * (abs(lhs) + abs(rhs)) + 1e-12, name


def test_lss_backward_matches_autograd_of_tensorized():
    w, depth, feat, K, E = _inputs("lss_tiny", "random", 34)
    _, _, amb = tensorized_lss(depth, feat, K, E, w.img_h, w.img_w, w.ranges, (w.X, w.Y), w.dbound)
    keep = (~amb).to(torch.float64)
    g = _grid(w)
    dout = I.make_lss_dout(w).double()
    A = (depth.double() * keep).requires_grad_()
    Fe = feat.double().requires_grad_()
    ref, _, _ = tensorized_lss(A, Fe, K, E, w.img_h, w.img_w, w.ranges, (w.X, w.Y), w.dbound)
    (ref * dout).sum().backward()
    r = oracle.lss_backward(A.detach(), feat, dout, K, E, w.img_h, w.img_w, g)
    ref_dd = A.grad.numpy() * keep.numpy()
    got_dd = r["ddepth"] * keep.numpy()
    for name, got, ref_, bnd in (("ddepth", got_dd, ref_dd, r["ddepth_bound"]),
                                 ("dfeat", r["dfeat"], Fe.grad.numpy(), r["dfeat_bound"])):
        assert np.abs(got).max() > 0, name
        err = np.abs(got - ref_) / np.maximum(bnd, 1e-30)
        err = np.where(bnd > 0, err, np.abs(got - ref_))
        assert err.max() < 1e-9, (name, err.max())
