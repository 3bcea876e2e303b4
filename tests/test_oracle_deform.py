"""Pins of the oracle's deformable aggregation (SparseDriveV2 notes,
"Deformable Aggregation" steps 1-3) against things other than itself: a
hand-derived example, one-hot weights against a bilinear read written out
here, the materialised float64 form with grid_sample and its autograd
gradients, linearity, the adjoint identity and camera permutation.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from camera_bev_view_b200 import inputs as I
from tensorized_vt import tensorized_deform


def _case(seed, B, N, C, Hf, Wf, ih, iw, Q, Kp, kind="config", spread=2.0):
    if kind == "config":
        rigs = [I.make_rig(seed + b, N, ih, iw) for b in range(B)]
    else:
        rigs = [I.random_rig(seed + b, N, ih, iw) for b in range(B)]
    K = torch.from_numpy(np.stack([r[0] for r in rigs]))
    E = torch.from_numpy(np.stack([r[1] for r in rigs]))
    g = torch.Generator().manual_seed(seed)
    F = torch.randn((B, N, C, Hf, Wf), generator=g, dtype=torch.float32)
    rng = np.random.default_rng(seed)
    A = np.stack([rng.uniform(-12, 12, (B, Q)), rng.uniform(-12, 12, (B, Q)), rng.uniform(-1, 2, (B, Q))], -1)
    D = rng.uniform(-spread, spread, (B, Q, Kp, 3))
    W = rng.uniform(-1.0, 1.0, (B, Q, N, Kp))
    return (F, K, E, torch.from_numpy(A.astype(np.float32)), torch.from_numpy(D.astype(np.float32)),
            torch.from_numpy(W.astype(np.float32)))


CASES = [
    # seed, B, N, C, Hf, Wf, img_h, img_w, Q, Kp, rig
    (21, 1, 6, 5, 8, 22, 128, 352, 40, 5, "config"),
    (22, 2, 6, 3, 16, 44, 256, 704, 24, 7, "config"),
    (23, 1, 3, 4, 6, 10, 48, 80, 30, 3, "random"),
    (24, 2, 4, 2, 9, 5, 72, 40, 16, 6, "random"),
    (25, 1, 4, 3, 8, 11, 64, 176, 20, 4, "random"),     # strides differ: 8 rows, 16 columns
]


def _unambiguous_weights(W, amb):
    """Zero the weights of (n, k) keypoints whose validity sits on an edge."""
    keep = (~amb).permute(0, 2, 1, 3).to(W.dtype)       # [B,Q,N,Kp]
    return W * keep


def test_deform_worked_example_exact():
    """Jitter-free rig, 128x352 images, 8x22 features: the keypoint
    (10, 0, 1.5) is 9 m straight ahead of camera 0 and (-10, 0, 1.5) 9 m ahead
    of camera 3 (yaw 180 deg), both at the principal point, i.e. feature
    position (10.5, 3.5): each sample is the mean of texels (3..4, 10..11).
    No other camera sees either point (65 deg off their axes, beyond the
    35.6 deg half field of view).  So out = 0.25 (w[0,0] S_0 + w[3,1] S_3)
    with S_n the sum of those four texels of camera n."""
    K, E = I.make_rig(0, 6, 128, 352, jitter=False)
    K, E = torch.from_numpy(K)[None], torch.from_numpy(E)[None]
    F = torch.randn((1, 6, 3, 8, 22), generator=torch.Generator().manual_seed(5), dtype=torch.float32)
    A = torch.tensor([[[0.0, 0.0, 1.5]]])
    D = torch.tensor([[[[10.0, 0.0, 0.0], [-10.0, 0.0, 0.0]]]])
    W = torch.arange(1, 13, dtype=torch.float32).reshape(1, 1, 6, 2) / 8.0
    out, bound = oracle.deform_forward(F, K, E, 128, 352, A, D, W)
    S = lambda n: F[0, n, :, 3:5, 10:12].double().sum(dim=(1, 2)).numpy()
    expect = 0.25 * (W[0, 0, 0, 0].item() * S(0) + W[0, 0, 3, 1].item() * S(3))
    np.testing.assert_allclose(out[0, 0], expect, rtol=1e-14, atol=1e-14)
    assert np.all(bound >= np.abs(out))


def _bilinear(Fn, fx, fy):
    """Zero-padded bilinear read of Fn [C,H,W] at feature position (fx, fy)."""
    C, H, W = Fn.shape
    x0, y0 = math.floor(fx), math.floor(fy)
    ax, ay = fx - x0, fy - y0
    acc = np.zeros(C)
    for yy, xx, wt in ((y0, x0, (1 - ay) * (1 - ax)), (y0, x0 + 1, (1 - ay) * ax),
                       (y0 + 1, x0, ay * (1 - ax)), (y0 + 1, x0 + 1, ay * ax)):
        if 0 <= yy < H and 0 <= xx < W:
            acc += wt * Fn[:, yy, xx]
    return acc


def test_deform_one_hot_weights_read_one_keypoint_in_one_camera():
    """A single nonzero weight w[q, n, k] = 1 must give query q exactly the
    bilinear read of camera n at keypoint k (zero when that keypoint is not
    valid in camera n) and every other query zero: pins the (q, n, k)
    indexing of weights, offsets and cameras."""
    F, K, E, A, D, W = _case(31, 1, 6, 4, 8, 22, 128, 352, 12, 3)
    Fd = F.double().numpy()
    valid, invalid = [], []
    for q in range(12):
        for n in range(6):
            for k in range(3):
                p = (A[0, q] + D[0, q, k]).numpy()
                ok, u, v, fx, fy = oracle.project(K[0, n], E[0, n], p, 128, 352, 8, 22)
                (valid if ok else invalid).append((q, n, k, fx, fy))
    assert len(valid) >= 6 and len(invalid) >= 2
    picks = valid[:: max(1, len(valid) // 6)][:6] + invalid[:2]
    assert len({(q, n) for q, n, k, _, _ in picks[:6]}) >= 3
    for (q, n, k, fx, fy) in picks:
        Wh = torch.zeros_like(W)
        Wh[0, q, n, k] = 1.0
        out, _ = oracle.deform_forward(F, K, E, 128, 352, A, D, Wh)
        ok = (q, n, k, fx, fy) in valid
        expect = _bilinear(Fd[0, n], fx, fy) if ok else np.zeros(4)
        # the oracle rounds each corner weight to fp32 (pinned geometry); here
        # they are fp64, so agreement is to fp32 rounding of the weights
        np.testing.assert_allclose(out[0, q], expect, rtol=1e-6, atol=1e-6)
        assert np.all(np.delete(out[0], q, axis=0) == 0.0)


@pytest.mark.parametrize("case", CASES, ids=[f"s{c[0]}" for c in CASES])
def test_deform_oracle_matches_tensorized_forward(case):
    seed, B, N, C, Hf, Wf, ih, iw, Q, Kp, kind = case
    F, K, E, A, D, W = _case(seed, B, N, C, Hf, Wf, ih, iw, Q, Kp, kind)
    _, mask, amb, _, _ = tensorized_deform(F, K, E, ih, iw, A, D, W)
    W = _unambiguous_weights(W, amb)
    out, bound = oracle.deform_forward(F, K, E, ih, iw, A, D, W)
    ref, _, _, _, _ = tensorized_deform(F, K, E, ih, iw, A, D, W)
    assert mask.sum() > 0.1 * mask.numel() / N
    err = np.abs(out - ref.numpy()) / np.maximum(bound, 1e-30)
    err = np.where(bound > 0, err, np.abs(out - ref.numpy()))
    assert err.max() < 2e-3


BWD_CASES = CASES[:3] + CASES[4:]


@pytest.mark.parametrize("case", BWD_CASES, ids=[f"s{c[0]}" for c in BWD_CASES])
def test_deform_backward_matches_autograd_of_tensorized(case):
    """dF, dW and dOff against autograd of the float64 materialised form.
    Keypoints within 1e-3 texel of a cell edge (where the bilinear derivative
    jumps, so fp32 and fp64 positions may pick different sides) or on a
    validity edge carry zero weight in both."""
    seed, B, N, C, Hf, Wf, ih, iw, Q, Kp, kind = case
    F, K, E, A, D, W = _case(seed, B, N, C, Hf, Wf, ih, iw, Q, Kp, kind)
    _, mask, amb, fx, fy = tensorized_deform(F, K, E, ih, iw, A, D, W)
    near = lambda f: ((f - torch.floor(f)) < 1e-3) | ((f - torch.floor(f)) > 1 - 1e-3)
    amb = amb | (mask & (near(fx) | near(fy)))
    W = _unambiguous_weights(W, amb)
    g = torch.randn((B, Q, C), generator=torch.Generator().manual_seed(seed + 7), dtype=torch.float64)
    r = oracle.deform_backward(F, g, K, E, ih, iw, A, D, W)
    Fv = F.double().requires_grad_()
    Wv = W.double().requires_grad_()
    Dv = D.double().requires_grad_()
    out, _, _, _, _ = tensorized_deform(Fv, K, E, ih, iw, A, D, Wv, offsets64=Dv)
    (out * g).sum().backward()
    for name, ref in (("dF", Fv.grad), ("dW", Wv.grad), ("dOff", Dv.grad)):
        got, bnd = r[name], r[name + "_bound"]
        ref = ref.numpy()
        if name == "dW":   # weights of invalid keypoints get no gradient in the oracle
            ref = ref * mask.permute(0, 2, 1, 3).numpy()
        assert np.abs(got).max() > 0, name
        err = np.abs(got - ref) / np.maximum(bnd, 1e-30)
        err = np.where(bnd > 0, err, np.abs(got - ref))
        assert err.max() < 2e-3, (name, err.max())


def test_deform_adjoint_and_linearity():
    F, K, E, A, D, W = _case(41, 2, 6, 3, 8, 22, 128, 352, 20, 4)
    g = torch.randn((2, 20, 3), generator=torch.Generator().manual_seed(3), dtype=torch.float64)
    out, _ = oracle.deform_forward(F, K, E, 128, 352, A, D, W)
    r = oracle.deform_backward(F, g, K, E, 128, 352, A, D, W)
    lhs = float((out * g.numpy()).sum())
    rhs = float((F.double().numpy() * r["dF"]).sum())
    assert abs(lhs - rhs) <= 1e-12 * (abs(lhs) + abs(rhs)) + 1e-12
    rhs_w = float((W.double().numpy() * r["dW"]).sum())        # out is linear in W too
    assert abs(lhs - rhs_w) <= 1e-12 * (abs(lhs) + abs(rhs_w)) + 1e-12
    o2, _ = oracle.deform_forward(F, K, E, 128, 352, A, D, 2.0 * W)
    np.testing.assert_allclose(o2, 2.0 * out, rtol=1e-13, atol=1e-13)
    # float64 features reach the oracle unrounded, so 3 F - 1 is exact
    o3, _ = oracle.deform_forward(3.0 * F.double() - 1.0, K, E, 128, 352, A, D, W)
    o1, _ = oracle.deform_forward(torch.ones_like(F), K, E, 128, 352, A, D, W)
    np.testing.assert_allclose(o3, 3.0 * out - o1, rtol=1e-10, atol=1e-10)


def test_deform_camera_permutation_invariance():
    F, K, E, A, D, W = _case(51, 1, 6, 3, 8, 22, 128, 352, 16, 4)
    perm = torch.tensor([3, 0, 5, 1, 4, 2])
    out, _ = oracle.deform_forward(F, K, E, 128, 352, A, D, W)
    outp, _ = oracle.deform_forward(F[:, perm], K[:, perm], E[:, perm], 128, 352, A, D, W[:, :, perm])
    np.testing.assert_allclose(outp, out, rtol=1e-12, atol=1e-12)


def test_deform_offsets_finite_differences():
    """Central differences of the oracle's own forward in one offset
    coordinate at a time (h = 2 mm), on keypoints well inside their cells and
    the image: they must match dOff to the differencing error."""
    F, K, E, A, D, W = _case(61, 1, 6, 3, 16, 44, 256, 704, 10, 3, spread=1.0)
    g = torch.randn((1, 10, 3), generator=torch.Generator().manual_seed(9), dtype=torch.float64)
    r = oracle.deform_backward(F, g, K, E, 256, 704, A, D, W)
    _, mask, amb, fx, fy = tensorized_deform(F, K, E, 256, 704, A, D, W)
    frac = lambda f: f - torch.floor(f)
    checked = 0
    for q in range(10):
        for k in range(3):
            sel = mask[0, :, q, k]
            if not sel.any() or amb[0, :, q, k].any():
                continue
            fxs, fys = fx[0, :, q, k][sel], fy[0, :, q, k][sel]
            if ((frac(fxs) < 0.05) | (frac(fxs) > 0.95) | (frac(fys) < 0.05) | (frac(fys) > 0.95)).any():
                continue
            for d in range(3):
                h = 2e-3
                Dp, Dm = D.clone(), D.clone()
                Dp[0, q, k, d] += h
                Dm[0, q, k, d] -= h
                hp = float(Dp[0, q, k, d] - D[0, q, k, d])
                hm = float(D[0, q, k, d] - Dm[0, q, k, d])
                op, _ = oracle.deform_forward(F, K, E, 256, 704, A, Dp, W)
                om, _ = oracle.deform_forward(F, K, E, 256, 704, A, Dm, W)
                fd = float(((op - om) * g.numpy()).sum()) / (hp + hm)
                an = r["dOff"][0, q, k, d]
                assert abs(fd - an) <= 2e-2 * r["dOff_bound"][0, q, k, d] + 1e-6, (q, k, d, fd, an)
                checked += 1
    assert checked >= 6
