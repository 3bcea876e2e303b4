"""Pins of the CPU oracle against things other than itself (no GPU needed).

Each test fixes one part of the definition (FlashBEV reading notes, "Method"
item 1 and "Key Insight"; SparseDriveV2 notes, "Deformable Aggregation" step 2
and pitfalls) so that a dropped term, a wrong sign, index or operand order
in the oracle fails at least one of them.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from camera_bev_view_b200 import inputs as I
from tensorized_vt import project_all, tensorized_backward, tensorized_forward

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _grid(ranges, counts):
    X, Y, Z = counts
    r = ranges
    return oracle.Grid(r, ((r[1] - r[0]) / X, (r[3] - r[2]) / Y, (r[5] - r[4]) / Z))


def _rig(kind, seed, N, img_h, img_w):
    if kind == "config":
        return I.make_rig(seed, N, img_h, img_w)
    return I.random_rig(seed, N, img_h, img_w)


# --------------------------------------------------------------------------
# hand-derived worked example (tests/golden/worked_example.json)
# --------------------------------------------------------------------------

def test_worked_example_forward_exact():
    g = json.load(open(os.path.join(GOLDEN, "worked_example.json")))
    grid = oracle.Grid(g["range"], g["res"])
    assert (grid.X, grid.Y, grid.Z) == (1, 1, 4)
    F = np.array(g["features"], dtype=np.float32)
    out, bound, count = oracle.forward(F, np.array(g["K"], np.float32), np.array(g["E"], np.float32),
                                       g["img_h"], g["img_w"], grid)
    np.testing.assert_array_equal(count, np.array(g["expected_count"]))
    np.testing.assert_array_equal(out, np.array(g["expected_out"]))
    assert np.all(bound >= np.abs(out))


def test_worked_example_backward_exact():
    g = json.load(open(os.path.join(GOLDEN, "worked_example.json")))
    grid = oracle.Grid(g["range"], g["res"])
    dF, _ = oracle.backward(np.array(g["dout"]), 3, g["Hf"], g["Wf"], np.array(g["K"], np.float32),
                            np.array(g["E"], np.float32), g["img_h"], g["img_w"], grid)
    np.testing.assert_array_equal(dF, np.array(g["expected_dF"]))


# --------------------------------------------------------------------------
# geometry: hand-computed single points and the validity edges
# --------------------------------------------------------------------------

def test_principal_point_of_level_camera():
    """Jitter-free rig, yaw-0 camera at (1, 0, 1.5): ego (10, 0, 1.5) is 9 m
    straight ahead, so it lands on the principal point (cx, cy) = (176, 64);
    at stride 16 that is feature position (176/16 - 0.5, 64/16 - 0.5)."""
    K, E = I.make_rig(0, 6, 128, 352, jitter=False)
    ok, u, v, fx, fy = oracle.project(K[0], E[0], (10.0, 0.0, 1.5), 128, 352, 8, 22)
    assert ok and (u, v, fx, fy) == (176.0, 64.0, 10.5, 3.5)
    # every nominal camera sees a point 9 m along its own axis at mount height
    for n in range(6):
        yaw = math.radians(60 * n)
        p = (math.cos(yaw) * 10, math.sin(yaw) * 10, 1.5)
        ok, u, v, fx, fy = oracle.project(K[n], E[n], p, 128, 352, 8, 22)
        assert ok and abs(u - 176) < 1e-3 and abs(v - 64) < 1e-3


def test_validity_edges_closed_image_strict_depth():
    K = np.array([[2, 0, 2], [0, 2, 2], [0, 0, 1]], np.float32)
    E = np.array([[0, -1, 0, 0], [0, 0, -1, 0], [1, 0, 0, 0], [0, 0, 0, 1]], np.float32)
    # u == W_img exactly: inside (closed interval); fx = 4 * 0.5 - 0.5 = 1.5
    assert oracle.project(K, E, (8.0, -8.0, 0.0), 4, 4, 2, 2)[0]
    assert oracle.project(K, E, (8.0, -8.0, 0.0), 4, 4, 2, 2)[3] == 1.5
    # u == 0 exactly: inside
    assert oracle.project(K, E, (8.0, 8.0, 0.0), 4, 4, 2, 2)[0]
    # just beyond either edge: outside
    assert not oracle.project(K, E, (8.0, -8.01, 0.0), 4, 4, 2, 2)[0]
    assert not oracle.project(K, E, (8.0, 8.01, 0.0), 4, 4, 2, 2)[0]
    assert not oracle.project(K, E, (8.0, 0.0, 8.01), 4, 4, 2, 2)[0]
    # depth exactly 0.1 (fp32) is not valid; a little more is
    assert not oracle.project(K, E, (0.1, 0.0, 0.0), 4, 4, 2, 2)[0]
    assert oracle.project(K, E, (0.1001, 0.0, 0.0), 4, 4, 2, 2)[0]
    # behind the camera
    assert not oracle.project(K, E, (-8.0, 0.0, 0.0), 4, 4, 2, 2)[0]


def test_fp32_geometry_agrees_with_fp64_off_edges():
    """Oracle validity (pinned fp32) vs float64 projection on the full
    nuScenes-like grid: any disagreement must sit within 0.05 px of an image
    edge or 1 mm of the depth threshold."""
    w = I.WORKLOADS["nuscenes"]
    K, E = I.make_rigs(w)
    grid = oracle.Grid(w.ranges, w.res)
    _, _, count = oracle.forward(torch.zeros(1, 6, 1, w.Hf, w.Wf), K, E, w.img_h, w.img_w, grid)
    u, v, depth, mask = project_all(K, E, w.ranges, (w.X, w.Y, w.Z), w.img_h, w.img_w)
    from tensorized_vt import ambiguous
    amb = ambiguous(u, v, depth, w.img_h, w.img_w).any(dim=1).numpy()
    c64 = mask.sum(dim=1).numpy()
    diff = c64 != count
    assert not np.any(diff & ~amb)
    assert count.sum() > 0.5 * count.size


# --------------------------------------------------------------------------
# brute force: materialised tensorized form with grid_sample (tiny grids)
# --------------------------------------------------------------------------

CASES = [
    # (rig kind, seed, N, C, Hf, Wf, img_h, img_w, ranges, counts)
    ("config", 11, 6, 4, 8, 22, 128, 352, (-25, 25, -25, 25, -5, 3), (8, 8, 3)),
    ("config", 12, 3, 3, 8, 22, 128, 352, (-6, 6, -6, 6, -3, 3), (7, 6, 3)),
    ("random", 13, 3, 4, 6, 10, 48, 80, (-10, 10, -8, 8, -2, 4), (8, 7, 2)),
    ("random", 14, 2, 2, 5, 7, 40, 56, (-4, 4, -4, 4, -1, 3), (6, 8, 3)),
    ("random", 15, 3, 3, 9, 5, 72, 40, (-20, 20, -20, 20, -4, 4), (5, 5, 3)),
    ("random", 16, 3, 3, 8, 11, 64, 176, (-12, 12, -12, 12, -2, 3), (6, 7, 3)),  # row / column strides differ
]


@pytest.mark.parametrize("case", CASES, ids=[f"{c[0]}{c[1]}" for c in CASES])
def test_oracle_matches_tensorized_forward(case):
    kind, seed, N, C, Hf, Wf, ih, iw, ranges, counts = case
    K, E = _rig(kind, seed, N, ih, iw)
    K, E = K[None], E[None]
    F = torch.randn((1, N, C, Hf, Wf), generator=torch.Generator().manual_seed(seed), dtype=torch.float32)
    grid = _grid(ranges, counts)
    out, bound, count = oracle.forward(F, K, E, ih, iw, grid)
    ref, ref_count, amb = tensorized_forward(F, K, E, ranges, counts, ih, iw)
    amb = amb.numpy()
    assert count.sum() > 0
    np.testing.assert_array_equal(count[~amb], ref_count.numpy()[~amb])
    cell_ok = ~amb.any(axis=-1)                       # [B,X,Y]
    err = np.abs(out - ref.numpy()) / np.maximum(bound, 1e-30)
    err = np.where(bound > 0, err, np.abs(out - ref.numpy()))
    # away from the edge-ambiguous samples the fp64 tensorized form and the
    # pinned-fp32 oracle differ by the geometry's rounding only (measured
    # <= 5.3e-6 of the bound on these cases)
    assert err.transpose(0, 2, 3, 1)[cell_ok].max() < 1e-5


@pytest.mark.parametrize("case", CASES[:3] + CASES[5:], ids=[f"{c[0]}{c[1]}" for c in CASES[:3] + CASES[5:]])
def test_oracle_backward_matches_autograd_of_tensorized(case):
    kind, seed, N, C, Hf, Wf, ih, iw, ranges, counts = case
    K, E = _rig(kind, seed, N, ih, iw)
    K, E = K[None], E[None]
    grid = _grid(ranges, counts)
    g = torch.randn((1, C) + counts[:2], generator=torch.Generator().manual_seed(seed + 1), dtype=torch.float64)
    _, _, amb = tensorized_forward(torch.zeros(1, N, C, Hf, Wf), K, E, ranges, counts, ih, iw)
    g = g * (~amb.any(dim=-1))[:, None].to(torch.float64)   # drop cells with edge-ambiguous samples
    dF, dB = oracle.backward(g, N, Hf, Wf, K, E, ih, iw, grid)
    ref, _ = tensorized_backward(g, N, Hf, Wf, K, E, ranges, counts, ih, iw)
    assert np.abs(dF).max() > 0
    err = np.abs(dF - ref.numpy()) / np.maximum(dB, 1e-30)
    err = np.where(dB > 0, err, np.abs(dF - ref.numpy()))
    # a texel's bound can be dominated by small bilinear weights, which the
    # fp64-vs-pinned-fp32 sample position (~1e-6 px) moves by ~1e-4 of
    # themselves (measured <= 8.1e-5 of the bound on these cases)
    assert err.max() < 2e-4


# --------------------------------------------------------------------------
# closed forms
# --------------------------------------------------------------------------

def test_affine_features_closed_form():
    """One level camera at the origin, mount height h, looking along +x:
    camera coordinates (-y, h - z, x), so u = f(-y)/x + cx, v = f(h - z)/x + cy.
    With F[c, r, s] = a_c s + b_c r + g_c, bilinear sampling reproduces the
    affine function exactly at any interior point (fx, fy):
        out[c, i, j] = sum_{valid k} (a_c fx_k + b_c fy_k + g_c)
    with fx = u Wf / W_img - 0.5, fy = v Hf / H_img - 0.5 (align_corners=False).
    Also pins x -> output row i and y -> output column j."""
    ih, iw, Hf, Wf, C, h, f = 64, 160, 8, 20, 3, 1.5, 80.0
    K = np.array([[[[f, 0, iw / 2], [0, f, ih / 2], [0, 0, 1]]]], np.float32)
    E = np.array([[[[0, -1, 0, 0], [0, 0, -1, h], [1, 0, 0, 0], [0, 0, 0, 1]]]], np.float32)
    a = np.array([0.7, -1.3, 0.0])
    b = np.array([0.25, 0.5, -2.0])
    gam = np.array([1.0, 0.0, 3.5])
    rows, cols = np.meshgrid(np.arange(Hf), np.arange(Wf), indexing="ij")
    F = (a[:, None, None] * cols + b[:, None, None] * rows + gam[:, None, None])[None, None]
    ranges, counts = (4, 28, -9, 9, -1, 3), (6, 9, 4)
    grid = _grid(ranges, counts)
    out, _, count = oracle.forward(F.astype(np.float32), K, E, ih, iw, grid)
    xs = 4 + (np.arange(6) + 0.5) * 4.0
    ys = -9 + (np.arange(9) + 0.5) * 2.0
    zs = -1 + (np.arange(4) + 0.5) * 1.0
    checked = 0
    for i, x in enumerate(xs):
        for j, y in enumerate(ys):
            expect = np.zeros(C)
            interior = True
            for k, z in enumerate(zs):
                u = f * (-y) / x + iw / 2
                v = f * (h - z) / x + ih / 2
                if not (0 <= u <= iw and 0 <= v <= ih):
                    assert count[0, i, j, k] == 0
                    continue
                assert count[0, i, j, k] == 1
                fx, fy = u * Wf / iw - 0.5, v * Hf / ih - 0.5
                interior &= (0.001 < fx < Wf - 1.001) and (0.001 < fy < Hf - 1.001)
                expect += a * fx + b * fy + gam
            if interior:
                checked += 1
                np.testing.assert_allclose(out[0, :, i, j], expect, rtol=0, atol=1e-3)
    assert checked >= 20


def test_constant_features_closed_form():
    """F == k: a valid sample whose four corners lie in the map returns k, so
    a cell all of whose valid samples are interior gives k * #{z: cnt_z >= 1};
    any cell gives at most that (zero padding only removes weight)."""
    w = I.WORKLOADS["tiny"]
    K, E = I.make_rigs(w)
    grid = oracle.Grid(w.ranges, w.res)
    k = 2.5
    F = torch.full((1, 6, 2, w.Hf, w.Wf), k)
    out, _, count = oracle.forward(F, K, E, w.img_h, w.img_w, grid)
    u, v, depth, mask = project_all(K, E, w.ranges, (w.X, w.Y, w.Z), w.img_h, w.img_w)
    fx = u * w.Wf / w.img_w - 0.5
    fy = v * w.Hf / w.img_h - 0.5
    interior = (fx > 1e-3) & (fx < w.Wf - 1 - 1e-3) & (fy > 1e-3) & (fy < w.Hf - 1 - 1e-3)
    all_interior = (~mask | interior).all(dim=1).all(dim=-1).numpy()     # [B,X,Y]
    nz = (count > 0).sum(axis=-1)                                        # [B,X,Y]
    strict = all_interior & (nz > 0)
    assert strict.sum() > 100
    for c in range(2):
        np.testing.assert_allclose(out[:, c][strict], k * nz[strict], rtol=1e-6)
        # corner weights are fp32 products, so they sum to 1 within a few ulp
        assert np.all(out[:, c] <= k * nz * (1 + 1e-6))
        assert np.all(out[:, c] >= 0)
    assert np.any(out[:, 0][~all_interior & (nz > 0)] < k * nz[~all_interior & (nz > 0)] - 1e-3)


# --------------------------------------------------------------------------
# structural invariants
# --------------------------------------------------------------------------

def test_camera_permutation_invariance():
    w = I.WORKLOADS["tiny"]
    F = I.make_features(w)
    K, E = I.make_rigs(w)
    grid = oracle.Grid(w.ranges, w.res)
    out, _, count = oracle.forward(F, K, E, w.img_h, w.img_w, grid)
    perm = [3, 0, 5, 1, 4, 2]
    out_p, _, count_p = oracle.forward(F[:, perm], K[:, perm], E[:, perm], w.img_h, w.img_w, grid)
    np.testing.assert_array_equal(count, count_p)
    np.testing.assert_allclose(out_p, out, rtol=1e-12, atol=1e-12)


def test_duplicate_camera_halves_each_sample():
    """Rig [A, A] with features [F1, F2]: every valid bin has count 2 and the
    valid mean is (sample(F1) + sample(F2)) / 2 -- pins the mean denominator."""
    w = I.WORKLOADS["tiny"]
    K, E = I.make_rigs(w)
    grid = oracle.Grid(w.ranges, w.res)
    gen = torch.Generator().manual_seed(7)
    F1 = torch.randn((1, 1, 4, w.Hf, w.Wf), generator=gen)
    F2 = torch.randn((1, 1, 4, w.Hf, w.Wf), generator=gen)
    KA, EA = K[:, :1], E[:, :1]
    o1, _, c1 = oracle.forward(F1, KA, EA, w.img_h, w.img_w, grid)
    o2, _, _ = oracle.forward(F2, KA, EA, w.img_h, w.img_w, grid)
    o12, _, c12 = oracle.forward(torch.cat([F1, F2], 1), torch.cat([KA, KA], 1), torch.cat([EA, EA], 1),
                                 w.img_h, w.img_w, grid)
    np.testing.assert_array_equal(c12, 2 * c1)
    np.testing.assert_allclose(o12, (o1 + o2) / 2, rtol=1e-12, atol=1e-12)
    assert c1.max() == 1 and c1.sum() > 0


def test_height_sum_decomposes_over_bins():
    """Summing over height: the Z-bin result equals the sum of Z single-bin
    grids with the same centres (z in [-5,3] at 1 m: centres are exact)."""
    w = I.WORKLOADS["tiny"]
    F = I.make_features(w)
    K, E = I.make_rigs(w)
    ranges = (-25, 25, -25, 25, -5, 3)
    full = _grid(ranges, (20, 20, 8))
    out, _, count = oracle.forward(F, K, E, w.img_h, w.img_w, full)
    total = np.zeros_like(out)
    for k in range(8):
        one = _grid((-25, 25, -25, 25, -5 + k, -4 + k), (20, 20, 1))
        o, _, c = oracle.forward(F, K, E, w.img_h, w.img_w, one)
        np.testing.assert_array_equal(c[..., 0], count[..., k])
        total += o
    np.testing.assert_allclose(out, total, rtol=1e-12, atol=1e-12)


def test_linearity_in_features():
    w = I.WORKLOADS["tiny"]
    K, E = I.make_rigs(w)
    grid = oracle.Grid(w.ranges, w.res)
    gen = torch.Generator().manual_seed(8)
    F = torch.randn((1, 6, 3, w.Hf, w.Wf), generator=gen, dtype=torch.float64)
    G = torch.randn((1, 6, 3, w.Hf, w.Wf), generator=gen, dtype=torch.float64)
    oF, _, _ = oracle.forward(F, K, E, w.img_h, w.img_w, grid)
    oG, _, _ = oracle.forward(G, K, E, w.img_h, w.img_w, grid)
    oFG, _, _ = oracle.forward(2.0 * F - 0.75 * G, K, E, w.img_h, w.img_w, grid)
    np.testing.assert_allclose(oFG, 2.0 * oF - 0.75 * oG, rtol=1e-10, atol=1e-10)


def test_adjoint_identity():
    """<A F, g> = <F, A^T g> (fp64) on the tiny workload at full size."""
    w = I.WORKLOADS["tiny"]
    K, E = I.make_rigs(w)
    grid = oracle.Grid(w.ranges, w.res)
    gen = torch.Generator().manual_seed(9)
    F = torch.randn((1, 6, w.C, w.Hf, w.Wf), generator=gen, dtype=torch.float64)
    g = torch.randn((1, w.C, w.X, w.Y), generator=gen, dtype=torch.float64)
    out, _, _ = oracle.forward(F, K, E, w.img_h, w.img_w, grid)
    dF, _ = oracle.backward(g, 6, w.Hf, w.Wf, K, E, w.img_h, w.img_w, grid)
    lhs = float((out * g.numpy()).sum())
    rhs = float((F.numpy() * dF).sum())
    assert abs(lhs - rhs) <= 1e-12 * (abs(lhs) + abs(rhs)) + 1e-12
    assert abs(lhs) > 1.0


def test_backward_finite_differences_6x6x2():
    """Central differences of L(F) = <A F, g> on a 6x6x2 grid over the
    nuScenes-like ranges, backward-workload channel count.  The operator is
    linear in F, so the difference quotient equals dL/dF up to rounding: 256
    touched texels and 64 untouched ones (gradient exactly 0)."""
    w = I.WORKLOADS["backward"]
    K, E = I.make_rigs(w)
    K, E = K[:1], E[:1]
    ranges = w.ranges
    grid = _grid(ranges, (6, 6, 2))
    gen = torch.Generator().manual_seed(10)
    F = torch.randn((1, 6, w.C, w.Hf, w.Wf), generator=gen, dtype=torch.float64)
    g = torch.randn((1, w.C, 6, 6), generator=gen, dtype=torch.float64).numpy()
    dF, _ = oracle.backward(g, 6, w.Hf, w.Wf, K, E, w.img_h, w.img_w, grid)
    touched = np.argwhere(dF != 0)
    untouched = np.argwhere(dF == 0)
    assert len(touched) >= 256 and len(untouched) >= 64
    rng = np.random.default_rng(11)
    picks = [tuple(t) for t in touched[rng.choice(len(touched), 256, replace=False)]]
    picks += [tuple(t) for t in untouched[rng.choice(len(untouched), 64, replace=False)]]
    h = 0.5

    def L(Fx):
        o, _, _ = oracle.forward(Fx, K, E, w.img_h, w.img_w, grid)
        return float((o * g).sum())

    # batch the perturbations: perturb 16 texels of distinct channels at a time is not
    # separable, so evaluate one at a time (the grid is tiny)
    for idx in picks:
        Fp = F.clone()
        Fm = F.clone()
        Fp[idx] += h
        Fm[idx] -= h
        fd = (L(Fp) - L(Fm)) / (2 * h)
        assert abs(fd - dF[idx]) <= 1e-9 * max(1.0, abs(dF[idx])), (idx, fd, dF[idx])


def test_grid_spec_counts_and_rejects_non_integral():
    g = oracle.Grid((-50, 50, -50, 50, -5, 3), (0.5, 0.5, 1.0))
    assert (g.X, g.Y, g.Z) == (200, 200, 8)
    assert g.cell[0] == np.float32(0.5) and g.cell[2] == np.float32(1.0)
    g = oracle.Grid((-50, 50, -50, 50, -5, 3), (0.25, 0.25, 0.5))
    assert (g.X, g.Y, g.Z) == (400, 400, 16)
    with pytest.raises(ValueError):
        oracle.Grid((-50, 50, -50, 50, -5, 3), (0.3, 0.5, 1.0))
    with pytest.raises(ValueError):
        oracle.Grid((50, -50, -50, 50, -5, 3), (0.5, 0.5, 1.0))
