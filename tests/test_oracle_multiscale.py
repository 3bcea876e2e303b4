"""Pins of the oracle's multi-scale form (FlashBEV reading notes, "Takeaway"
4: multi-scale fused view transformation; SparseDriveV2 notes, "Image
Encoder": FPN levels with a common channel count) against things other than
itself.

- brute force: the materialised form with one ``grid_sample`` per level
  (forward, and its autograd for the backward);
- reduction: one level is the single-level operator, bit for bit;
- additivity: with the count shared by all levels, the output is the sum of
  the single-level outputs at each level's own resolution;
- the adjoint identity between the multi-scale forward and backward;
- a level whose map is all zeros changes nothing, but its own gradient is
  the single-level gradient at its size.

A level sampled at another level's scale, a count taken per level, levels
averaged instead of summed or a gradient sent to the wrong level fails at
least one of these.
"""
import numpy as np
import pytest
import torch

import oracle
from camera_bev_view_b200 import inputs as I
from tensorized_vt import tensorized_ms_backward, tensorized_ms_forward


def _grid(ranges, counts):
    X, Y, Z = counts
    r = ranges
    return oracle.Grid(r, ((r[1] - r[0]) / X, (r[3] - r[2]) / Y, (r[5] - r[4]) / Z))


def _levels(seed, B, N, C, sizes, dtype=torch.float32):
    gen = torch.Generator().manual_seed(seed)
    return [torch.randn((B, N, C, h, w), generator=gen, dtype=dtype) for h, w in sizes]


CASES = [
    # (rig kind, seed, N, C, level sizes, img_h, img_w, ranges, counts)
    ("config", 21, 6, 3, [(8, 22), (4, 11), (2, 6)], 128, 352, (-25, 25, -25, 25, -5, 3), (8, 8, 3)),
    ("random", 22, 3, 2, [(6, 10), (3, 5)], 48, 80, (-10, 10, -8, 8, -2, 4), (8, 7, 2)),
    ("random", 23, 3, 3, [(9, 5), (5, 3), (3, 2), (2, 1)], 72, 40, (-20, 20, -20, 20, -4, 4), (5, 5, 3)),
]


def _rig(kind, seed, N, ih, iw):
    K, E = (I.make_rig if kind == "config" else I.random_rig)(seed, N, ih, iw)
    return K[None], E[None]


@pytest.mark.parametrize("case", CASES, ids=[f"{c[0]}{c[1]}" for c in CASES])
def test_ms_matches_tensorized_forward(case):
    kind, seed, N, C, sizes, ih, iw, ranges, counts = case
    K, E = _rig(kind, seed, N, ih, iw)
    Fs = _levels(seed, 1, N, C, sizes)
    out, bound, count = oracle.ms_forward(Fs, K, E, ih, iw, _grid(ranges, counts))
    ref, ref_count, amb = tensorized_ms_forward(Fs, K, E, ranges, counts, ih, iw)
    amb = amb.numpy()
    assert count.sum() > 0
    np.testing.assert_array_equal(count[~amb], ref_count.numpy()[~amb])
    cell_ok = ~amb.any(axis=-1)
    err = np.where(bound > 0, np.abs(out - ref.numpy()) / np.maximum(bound, 1e-30), np.abs(out - ref.numpy()))
    assert err.transpose(0, 2, 3, 1)[cell_ok].max() < 2e-3


@pytest.mark.parametrize("case", CASES, ids=[f"{c[0]}{c[1]}" for c in CASES])
def test_ms_backward_matches_autograd_of_tensorized(case):
    kind, seed, N, C, sizes, ih, iw, ranges, counts = case
    K, E = _rig(kind, seed, N, ih, iw)
    g = torch.randn((1, C) + counts[:2], generator=torch.Generator().manual_seed(seed + 1), dtype=torch.float64)
    _, _, amb = tensorized_ms_forward(_levels(0, 1, N, C, sizes), K, E, ranges, counts, ih, iw)
    g = g * (~amb.any(dim=-1))[:, None].to(torch.float64)
    dF, dB = oracle.ms_backward(g, N, sizes, K, E, ih, iw, _grid(ranges, counts))
    ref, _ = tensorized_ms_backward(g, N, sizes, K, E, ranges, counts, ih, iw)
    for l in range(len(sizes)):
        assert np.abs(dF[l]).max() > 0
        r = ref[l].numpy()
        err = np.where(dB[l] > 0, np.abs(dF[l] - r) / np.maximum(dB[l], 1e-30), np.abs(dF[l] - r))
        assert err.max() < 2e-3, l


def test_ms_one_level_is_the_single_level_operator():
    w = I.WORKLOADS["tiny"]
    K, E = I.make_rigs(w)
    grid = oracle.Grid(w.ranges, w.res)
    F = I.make_features(w)
    o1, b1, c1 = oracle.forward(F, K, E, w.img_h, w.img_w, grid)
    o2, b2, c2 = oracle.ms_forward([F], K, E, w.img_h, w.img_w, grid)
    assert np.array_equal(o1, o2) and np.array_equal(b1, b2) and np.array_equal(c1, c2)
    g = torch.randn((1, w.C, w.X, w.Y), generator=torch.Generator().manual_seed(5), dtype=torch.float64)
    d1, e1 = oracle.backward(g, 6, w.Hf, w.Wf, K, E, w.img_h, w.img_w, grid)
    d2, e2 = oracle.ms_backward(g, 6, [(w.Hf, w.Wf)], K, E, w.img_h, w.img_w, grid)
    assert np.array_equal(d1, d2[0]) and np.array_equal(e1, e2[0])


def test_ms_output_is_the_sum_of_single_level_outputs():
    """The count depends on the image plane only, so the valid mean of the
    summed samples is the sum of the per-level valid means."""
    w = I.WORKLOADS["tiny"]
    K, E = I.make_rigs(w)
    grid = oracle.Grid(w.ranges, w.res)
    sizes = [(8, 22), (4, 11), (3, 7)]   # the last is not a halving: its own scale is 7 / W_img
    Fs = _levels(31, 1, 6, w.C, sizes, torch.float64)
    out, bound, count = oracle.ms_forward(Fs, K, E, w.img_h, w.img_w, grid)
    total = np.zeros_like(out)
    btot = np.zeros_like(out)
    for F in Fs:
        o, b, c = oracle.forward(F, K, E, w.img_h, w.img_w, grid)
        assert np.array_equal(c, count)
        total += o
        btot += b
    np.testing.assert_allclose(out, total, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(bound, btot, rtol=1e-12, atol=1e-12)
    assert np.abs(out).max() > 0.1


def test_ms_adjoint_identity():
    w = I.WORKLOADS["tiny"]
    K, E = I.make_rigs(w)
    grid = oracle.Grid(w.ranges, w.res)
    sizes = [(8, 22), (4, 11), (2, 6)]
    Fs = _levels(41, 1, 6, w.C, sizes, torch.float64)
    g = torch.randn((1, w.C, w.X, w.Y), generator=torch.Generator().manual_seed(42), dtype=torch.float64)
    out, _, _ = oracle.ms_forward(Fs, K, E, w.img_h, w.img_w, grid)
    dF, _ = oracle.ms_backward(g, 6, sizes, K, E, w.img_h, w.img_w, grid)
    lhs = float((out * g.numpy()).sum())
    rhs = sum(float((F.numpy() * d).sum()) for F, d in zip(Fs, dF))
    assert abs(lhs - rhs) <= 1e-12 * (abs(lhs) + abs(rhs)) + 1e-12
    assert abs(lhs) > 1.0


def test_ms_zero_level_adds_nothing_and_gets_its_own_gradient():
    w = I.WORKLOADS["tiny"]
    K, E = I.make_rigs(w)
    grid = oracle.Grid(w.ranges, w.res)
    F = I.make_features(w)
    Z = torch.zeros((1, 6, w.C, 5, 13))
    o1, _, _ = oracle.forward(F, K, E, w.img_h, w.img_w, grid)
    o2, _, _ = oracle.ms_forward([Z, F], K, E, w.img_h, w.img_w, grid)
    np.testing.assert_allclose(o2, o1, rtol=1e-13, atol=1e-13)
    g = torch.randn((1, w.C, w.X, w.Y), generator=torch.Generator().manual_seed(6), dtype=torch.float64)
    dF, _ = oracle.ms_backward(g, 6, [(5, 13), (w.Hf, w.Wf)], K, E, w.img_h, w.img_w, grid)
    d_small, _ = oracle.backward(g, 6, 5, 13, K, E, w.img_h, w.img_w, grid)
    d_full, _ = oracle.backward(g, 6, w.Hf, w.Wf, K, E, w.img_h, w.img_w, grid)
    assert np.array_equal(dF[0], d_small) and np.array_equal(dF[1], d_full)
