"""CUDA path (through the C ABI) against the CPU oracle, element by element.

Gates: valid-camera counts bit-exact; outputs within a condition-aware
relative error err = max |gpu - oracle| / bound, where bound is the oracle's
fp64 sum of |terms| for that element (elements with bound 0 must be exactly
0).  Tolerance 1e-5 for fp32 and bf16 features alike: bf16 features are
inputs, read as the same exact values by both sides (the oracle widens them
to fp64, the kernels to fp32), so the only difference left is the fp32
accumulation order, as for fp32 features.  Every workload runs at its full
size in the launch configuration the bench times.
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle
from camera_bev_view_b200 import inputs as I
from camera_bev_view_b200 import ops

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
TOL = {"f32": 1e-5, "bf16": 1e-5}
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def naive_errors(got, ref):
    """The naive figures reported beside the gate: the largest per-element
    relative error among elements with |o| >= 1e-3 max|o|, and max|delta| /
    max|o| (o = the oracle's output)."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    top = float(np.abs(ref).max()) if ref.size else 0.0
    if top == 0.0:
        return {"rel_on_large": 0.0, "max_abs_over_max": 0.0}
    big = np.abs(ref) >= 1e-3 * top
    return {"rel_on_large": float((np.abs(got - ref)[big] / np.abs(ref[big])).max()),
            "max_abs_over_max": float(np.abs(got - ref).max() / top)}


def report(kind, got, ref, err):
    """Print the gate and the naive figures; append them as a JSON line to
    $BEV_PARITY_REPORT when that names a file."""
    row = {"test": os.environ.get("PYTEST_CURRENT_TEST", "?").split(" ")[0], "kind": kind,
           "err_over_bound": err, **naive_errors(got, ref)}
    print(json.dumps(row))
    path = os.environ.get("BEV_PARITY_REPORT")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps(row) + "\n")


def rel_err(got, ref, bound):
    got = np.asarray(got, dtype=np.float64)
    zero = bound == 0
    assert np.all(got[zero] == 0), "elements with no contribution must be exactly 0"
    if np.all(zero):
        return 0.0
    return float((np.abs(got - ref)[~zero] / bound[~zero]).max())


def gpu_forward(F, K, E, img_h, img_w, ranges, res, layout=ops.NCHW, count=True, stream=None):
    g = ops.bev_grid_spec(ranges, res)
    Fd = F.to(DEV)
    if layout == ops.NHWC:
        Fd = Fd.permute(0, 1, 3, 4, 2).contiguous()
    out, cnt = ops.bev_sample_forward(Fd, K.to(DEV), E.to(DEV), img_h, img_w, g, layout=layout,
                                      count=count, stream=stream)
    torch.cuda.synchronize()
    return out.cpu(), (cnt.cpu() if cnt is not None else None)


def gpu_backward(dout, K, E, img_h, img_w, ranges, res, N, Hf, Wf):
    g = ops.bev_grid_spec(ranges, res)
    dF = ops.bev_sample_backward(dout.to(DEV), K.to(DEV), E.to(DEV), img_h, img_w, g, N, Hf, Wf)
    torch.cuda.synchronize()
    return dF.cpu()


def check_forward(F, K, E, img_h, img_w, ranges, res, tol, layout=ops.NCHW):
    out, cnt = gpu_forward(F, K, E, img_h, img_w, ranges, res, layout=layout)
    ref, bound, ref_cnt = oracle.forward(F, K, E, img_h, img_w, oracle.Grid(ranges, res))
    np.testing.assert_array_equal(cnt.numpy().astype(np.int32), ref_cnt)
    err = rel_err(out.numpy(), ref, bound)
    report("forward", out.numpy(), ref, err)
    assert err <= tol, err
    return out, ref, ref_cnt, err


def check_backward(dout, K, E, img_h, img_w, ranges, res, N, Hf, Wf, tol=1e-5):
    dF = gpu_backward(dout, K, E, img_h, img_w, ranges, res, N, Hf, Wf)
    ref, bound = oracle.backward(dout, N, Hf, Wf, K, E, img_h, img_w, oracle.Grid(ranges, res))
    err = rel_err(dF.numpy(), ref, bound)
    report("backward", dF.numpy(), ref, err)
    assert err <= tol, err
    return dF, ref, err


# --------------------------------------------------------------------------
# the workloads at full size
# --------------------------------------------------------------------------

@pytest.mark.parametrize("name", ["tiny", "nuscenes", "batched_bf16", "large"])
def test_forward_workload_full_size(name):
    w = I.WORKLOADS[name]
    F = I.make_features(w)
    K, E = I.make_rigs(w)
    out, ref, cnt, err = check_forward(F, K, E, w.img_h, w.img_w, w.ranges, w.res, TOL[w.dtype])
    assert err <= 1e-5
    assert cnt.sum() > 0.5 * cnt.size


@pytest.mark.parametrize("name", ["nuscenes", "batched_bf16"])
def test_forward_channels_last_input(name):
    w = I.WORKLOADS[name]
    F = I.make_features(w)
    K, E = I.make_rigs(w)
    out_nhwc, _ = gpu_forward(F, K, E, w.img_h, w.img_w, w.ranges, w.res, layout=ops.NHWC)
    out_nchw, _ = gpu_forward(F, K, E, w.img_h, w.img_w, w.ranges, w.res, layout=ops.NCHW)
    assert torch.equal(out_nhwc, out_nchw)   # same kernel, same order: bitwise equal


def _tilted_rigs(w, seed):
    Ks, Es = zip(*(I.random_rig(seed + b, w.N, w.img_h, w.img_w) for b in range(w.B)))
    return torch.from_numpy(np.stack(Ks)), torch.from_numpy(np.stack(Es))


@pytest.mark.parametrize("name", ["batched_bf16", "large"])
def test_forward_full_size_tilted_rigs(name):
    """The full-size workloads on rigs with random yaw, +-8 degree pitch and
    roll and off-centre principal points: a cell's voxels then project to a
    slanted segment, so merged patches are wider than two columns and the
    unmerged path is taken more often."""
    w = I.WORKLOADS[name]
    K, E = _tilted_rigs(w, 300)
    check_forward(I.make_features(w), K, E, w.img_h, w.img_w, w.ranges, w.res, TOL[w.dtype])


def test_backward_full_size_tilted_rigs():
    """The feature gradient at the batched_bf16 sizes (B4, C128, 200x200x16)
    on the tilted rigs: groups of cells then share slanted boxes."""
    w = I.WORKLOADS["batched_bf16"]
    K, E = _tilted_rigs(w, 300)
    check_backward(I.make_dout(w), K, E, w.img_h, w.img_w, w.ranges, w.res, w.N, w.Hf, w.Wf)


def test_backward_workload_full_size():
    w = I.WORKLOADS["backward"]
    K, E = I.make_rigs(w)
    dout = I.make_dout(w)
    check_backward(dout, K, E, w.img_h, w.img_w, w.ranges, w.res, w.N, w.Hf, w.Wf)


def test_backward_tiny_and_adjoint_on_gpu():
    w = I.WORKLOADS["tiny"]
    K, E = I.make_rigs(w)
    gen = torch.Generator().manual_seed(5)
    F = torch.randn((1, 6, w.C, w.Hf, w.Wf), generator=gen)
    g = torch.randn((1, w.C, w.X, w.Y), generator=gen)
    check_backward(g, K, E, w.img_h, w.img_w, w.ranges, w.res, 6, w.Hf, w.Wf)
    out, _ = gpu_forward(F, K, E, w.img_h, w.img_w, w.ranges, w.res)
    dF = gpu_backward(g, K, E, w.img_h, w.img_w, w.ranges, w.res, 6, w.Hf, w.Wf)
    lhs = float((out.double() * g.double()).sum())
    rhs = float((F.double() * dF.double()).sum())
    assert abs(lhs - rhs) <= 1e-5 * (abs(lhs) + abs(rhs))


def test_worked_example_exact_on_gpu():
    gj = json.load(open(os.path.join(GOLDEN, "worked_example.json")))
    F = torch.tensor(gj["features"], dtype=torch.float32)
    K = torch.tensor(gj["K"], dtype=torch.float32)
    E = torch.tensor(gj["E"], dtype=torch.float32)
    out, cnt = gpu_forward(F, K, E, gj["img_h"], gj["img_w"], gj["range"], gj["res"])
    np.testing.assert_array_equal(cnt.numpy(), np.array(gj["expected_count"]))
    np.testing.assert_array_equal(out.numpy(), np.array(gj["expected_out"], dtype=np.float32))
    dF = gpu_backward(torch.tensor(gj["dout"], dtype=torch.float32), K, E, gj["img_h"], gj["img_w"],
                      gj["range"], gj["res"], 3, gj["Hf"], gj["Wf"])
    np.testing.assert_array_equal(dF.numpy(), np.array(gj["expected_dF"], dtype=np.float32))


# --------------------------------------------------------------------------
# edge cases: ragged tiles, padded and sliced channels, height chunks, many
# cameras, empty views, degenerate grids
# --------------------------------------------------------------------------

def _random_case(seed, B, N, C, Hf, Wf, img_h, img_w, dtype=torch.float32):
    Ks, Es = [], []
    for b in range(B):
        K, E = I.random_rig(seed + b, N, img_h, img_w)
        Ks.append(K)
        Es.append(E)
    F = torch.randn((B, N, C, Hf, Wf), generator=torch.Generator().manual_seed(seed)).to(dtype)
    return F, torch.from_numpy(np.stack(Ks)), torch.from_numpy(np.stack(Es))


EDGE = [
    # id, seed, B, N, C, Hf, Wf, img, ranges, counts, dtype
    ("ragged_c3", 21, 2, 4, 3, 9, 13, (72, 104), (-12, 14, -10, 11, -2, 3), (13, 21, 5), torch.float32),
    ("ragged_bf16_c12", 22, 1, 5, 12, 7, 19, (56, 152), (-9, 9, -8, 9, -2, 2), (11, 17, 3), torch.bfloat16),
    ("slices_c200", 23, 1, 6, 200, 8, 22, (128, 352), (-20, 20, -20, 20, -4, 4), (24, 16, 4), torch.float32),
    ("slices_bf16_c264", 24, 1, 3, 264, 8, 22, (128, 352), (-16, 16, -16, 16, -4, 4), (16, 16, 3), torch.bfloat16),
    ("zchunks_z40", 25, 1, 6, 16, 8, 22, (128, 352), (-10, 10, -10, 10, -6, 4), (16, 16, 40), torch.float32),
    ("c80_lanes", 26, 1, 6, 80, 10, 30, (80, 240), (-15, 15, -15, 15, -3, 3), (20, 20, 6), torch.float32),
    ("c4_one_lane", 27, 1, 6, 4, 10, 30, (80, 240), (-15, 15, -15, 15, -3, 3), (20, 20, 6), torch.float32),
    ("single_cell", 28, 1, 6, 8, 10, 30, (80, 240), (3, 4, -0.5, 0.5, 0, 1), (1, 1, 1), torch.float32),
]


@pytest.mark.parametrize("case", EDGE, ids=[c[0] for c in EDGE])
def test_forward_edge_cases(case):
    _, seed, B, N, C, Hf, Wf, (ih, iw), ranges, counts, dt = case
    F, K, E = _random_case(seed, B, N, C, Hf, Wf, ih, iw, dt)
    res = tuple((ranges[2 * a + 1] - ranges[2 * a]) / counts[a] for a in range(3))
    check_forward(F, K, E, ih, iw, ranges, res, 1e-5)
    for layout in (ops.NHWC,):
        check_forward(F, K, E, ih, iw, ranges, res, 1e-5, layout=layout)


@pytest.mark.parametrize("case", [c for c in EDGE if c[10] == torch.float32], ids=[c[0] for c in EDGE if c[10] == torch.float32])
def test_backward_edge_cases(case):
    _, seed, B, N, C, Hf, Wf, (ih, iw), ranges, counts, _ = case
    _, K, E = _random_case(seed, B, N, 1, Hf, Wf, ih, iw)
    res = tuple((ranges[2 * a + 1] - ranges[2 * a]) / counts[a] for a in range(3))
    dout = torch.randn((B, C, counts[0], counts[1]), generator=torch.Generator().manual_seed(seed + 7))
    check_backward(dout, K, E, ih, iw, ranges, res, N, Hf, Wf)


def test_thirty_two_cameras_force_height_chunks():
    """32 cameras, 16 of them duplicated: many valid cameras per voxel, so a
    tile stages its height bins in several chunks."""
    K1, E1 = I.random_rig(31, 16, 64, 160, spread=0.2)
    K = torch.from_numpy(np.concatenate([K1, K1]))[None]
    E = torch.from_numpy(np.concatenate([E1, E1]))[None]
    F = torch.randn((1, 32, 8, 8, 20), generator=torch.Generator().manual_seed(32))
    ranges, res = (-12, 12, -12, 12, -3, 3), (1.0, 1.0, 0.5)
    out, ref, cnt, _ = check_forward(F, K, E, 64, 160, ranges, res, 1e-5)
    assert cnt.max() >= 4
    dout = torch.randn((1, 8, 24, 24), generator=torch.Generator().manual_seed(33))
    check_backward(dout, K, E, 64, 160, ranges, res, 32, 8, 20)


def test_tall_patches_take_the_unmerged_path():
    """One camera close to a fine column of 32 bins with a tall feature map:
    each cell's bins span the whole map height, so the merged patches of a
    tile exceed shared memory and the kernels fall back to unmerged taps."""
    K = np.array([[[[448.0, 0, 320], [0, 448.0, 128], [0, 0, 1]]]], np.float32)
    E = np.array([[[[0, -1, 0, 0], [0, 0, -1, 0], [1, 0, 0, 0], [0, 0, 0, 1]]]], np.float32)
    K, E = torch.from_numpy(K), torch.from_numpy(E)
    F = torch.randn((1, 1, 8, 64, 160), generator=torch.Generator().manual_seed(41))
    ranges, res = (1.5, 5.5, -1.0, 1.0, -2.0, 2.0), (0.25, 0.25, 0.125)
    out, ref, cnt, _ = check_forward(F, K, E, 256, 640, ranges, res, 1e-5)
    assert cnt.sum() > 1000
    dout = torch.randn((1, 8, 16, 8), generator=torch.Generator().manual_seed(42))
    check_backward(dout, K, E, 256, 640, ranges, res, 1, 64, 160)


def test_empty_view_gives_zeros():
    """Grid entirely behind a single forward-looking camera."""
    K, E = I.make_rig(0, 1, 128, 352, jitter=False)
    K, E = torch.from_numpy(K)[None], torch.from_numpy(E)[None]
    F = torch.randn((1, 1, 16, 8, 22))
    out, cnt = gpu_forward(F, K, E, 128, 352, (-30, -10, -10, 10, -2, 2), (1, 1, 1))
    assert torch.count_nonzero(out) == 0 and torch.count_nonzero(cnt) == 0
    dF = gpu_backward(torch.randn(1, 16, 20, 20), K, E, 128, 352, (-30, -10, -10, 10, -2, 2), (1, 1, 1),
                      1, 8, 22)
    assert torch.count_nonzero(dF) == 0


def test_forward_without_count_and_on_side_stream_is_deterministic():
    w = I.WORKLOADS["nuscenes"]
    F = I.make_features(w)
    K, E = I.make_rigs(w)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        a, c = gpu_forward(F, K, E, w.img_h, w.img_w, w.ranges, w.res, count=False, stream=s)
    b, _ = gpu_forward(F, K, E, w.img_h, w.img_w, w.ranges, w.res)
    assert c is None
    assert torch.equal(a, b)


def test_camera_permutation_on_gpu():
    w = I.WORKLOADS["tiny"]
    F = I.make_features(w)
    K, E = I.make_rigs(w)
    perm = [5, 2, 0, 4, 1, 3]
    a, ca = gpu_forward(F, K, E, w.img_h, w.img_w, w.ranges, w.res)
    b, cb = gpu_forward(F[:, perm], K[:, perm], E[:, perm], w.img_h, w.img_w, w.ranges, w.res)
    assert torch.equal(ca, cb)
    torch.testing.assert_close(a, b, rtol=1e-5, atol=1e-5)


def test_host_pointers_are_rejected_without_launch():
    w = I.WORKLOADS["tiny"]
    F = I.make_features(w).to(DEV)
    K, E = I.make_rigs(w)
    g = ops.bev_grid_spec(w.ranges, w.res)
    with pytest.raises(ops.BevError) as e:
        ops.bev_sample_forward(F, K, E.to(DEV), w.img_h, w.img_w, g)     # K on the host
    assert e.value.status == -1
    with pytest.raises(ops.BevError) as e:
        ops.bev_sample_backward(torch.zeros(1, w.C, w.X, w.Y, device=DEV), K, E.to(DEV), w.img_h,
                                w.img_w, g, 6, w.Hf, w.Wf)                # K on the host
    assert e.value.status == -1
    torch.cuda.synchronize()


# --------------------------------------------------------------------------
# the largest sizes the boundary accepts along each axis (small elsewhere)
# --------------------------------------------------------------------------

def test_maximum_height_bins():
    """Z = 1024 (the limit): 64 height chunks per cell in the forward."""
    K, E = I.make_rig(51, 6, 128, 352)
    K, E = torch.from_numpy(K)[None], torch.from_numpy(E)[None]
    F = torch.randn((1, 6, 8, 8, 22), generator=torch.Generator().manual_seed(51))
    ranges, res = (-8, 8, -8, 8, -5, 3), (2.0, 2.0, 8.0 / 1024)
    out, ref, cnt, _ = check_forward(F, K, E, 128, 352, ranges, res, 1e-5)
    assert cnt.shape[-1] == 1024 and cnt.sum() > 10000
    dout = torch.randn((1, 8, 8, 8), generator=torch.Generator().manual_seed(52))
    check_backward(dout, K, E, 128, 352, ranges, res, 6, 8, 22)


def test_two_thousand_channels_in_sixteen_slices():
    K, E = I.make_rig(53, 6, 128, 352)
    K, E = torch.from_numpy(K)[None], torch.from_numpy(E)[None]
    F = torch.randn((1, 6, 2048, 4, 11), generator=torch.Generator().manual_seed(53))
    ranges, res = (-12, 12, -12, 12, -4, 4), (1.5, 1.5, 2.0)
    check_forward(F, K, E, 128, 352, ranges, res, 1e-5)
    dout = torch.randn((1, 2048, 16, 16), generator=torch.Generator().manual_seed(54))
    check_backward(dout, K, E, 128, 352, ranges, res, 6, 4, 11)


def test_widest_feature_map():
    """Wf = 16384 (the limit) on a 2048 x 16384 image: texel offsets beyond
    2^16 within one row."""
    K = np.array([[[[4000.0, 0, 8192], [0, 4000.0, 1024], [0, 0, 1]]]], np.float32)
    E = np.array([[[[0, -1, 0, 0], [0, 0, -1, 0], [1, 0, 0, 0], [0, 0, 0, 1]]]], np.float32)
    K, E = torch.from_numpy(K), torch.from_numpy(E)
    F = torch.randn((1, 1, 4, 2, 16384), generator=torch.Generator().manual_seed(55))
    ranges, res = (5, 25, -20, 20, -1, 1), (1.0, 0.25, 0.5)
    out, ref, cnt, _ = check_forward(F, K, E, 2048, 16384, ranges, res, 1e-5)
    assert cnt.sum() > 1000
    dout = torch.randn((1, 4, 20, 160), generator=torch.Generator().manual_seed(56))
    check_backward(dout, K, E, 2048, 16384, ranges, res, 1, 2, 16384)
