"""The bounds-checked build (libbevsample_checked.so, -DBEV_BOUNDS_CHECK).

In that build the dense kernels test every geometry-derived address -- each
group's texel box (every gather load and gradient reduction lies in it), each
merge word, group-table slot, output, count and dout index -- before touching
it; a failed test skips the access and the call returns BEV_ERR_INTERNAL.
These tests load that library in place of the normal one and run the tiny
workload, the edge cases, the unmerged fallback and the largest sizes the
boundary accepts, through the C ABI: every call must return BEV_OK (a zero
device error word) and still match the oracle.
"""
import os

import numpy as np
import pytest
import torch

import oracle
from camera_bev_view_b200 import build, inputs as I, ops
from test_gpu_parity import EDGE, _random_case, check_backward, check_forward

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def checked_library():
    if not os.path.exists(build.LIB_CHECKED):
        build.build(checked=True)
    saved_path, saved_lib = build.LIB, ops._lib
    build.LIB, ops._lib = build.LIB_CHECKED, None
    assert ops.bev_bounds_checked()
    yield
    build.LIB, ops._lib = saved_path, saved_lib


def test_tiny_workload_forward_and_backward():
    w = I.WORKLOADS["tiny"]
    F = I.make_features(w)
    K, E = I.make_rigs(w)
    check_forward(F, K, E, w.img_h, w.img_w, w.ranges, w.res, 1e-5)
    check_backward(I.make_dout(w), K, E, w.img_h, w.img_w, w.ranges, w.res, w.N, w.Hf, w.Wf)


@pytest.mark.parametrize("case", EDGE, ids=[c[0] for c in EDGE])
def test_edge_cases(case):
    _, seed, B, N, C, Hf, Wf, (ih, iw), ranges, counts, dt = case
    F, K, E = _random_case(seed, B, N, C, Hf, Wf, ih, iw, dt)
    res = tuple((ranges[2 * a + 1] - ranges[2 * a]) / counts[a] for a in range(3))
    check_forward(F, K, E, ih, iw, ranges, res, 1e-5)
    dout = torch.randn((B, C, counts[0], counts[1]), generator=torch.Generator().manual_seed(seed + 7))
    check_backward(dout, K, E, ih, iw, ranges, res, N, Hf, Wf)


def test_tall_boxes_fall_back_cell_by_cell_and_bin_by_bin():
    K = np.array([[[[448.0, 0, 320], [0, 448.0, 128], [0, 0, 1]]]], np.float32)
    E = np.array([[[[0, -1, 0, 0], [0, 0, -1, 0], [1, 0, 0, 0], [0, 0, 0, 1]]]], np.float32)
    K, E = torch.from_numpy(K), torch.from_numpy(E)
    F = torch.randn((1, 1, 8, 64, 160), generator=torch.Generator().manual_seed(41))
    ranges, res = (1.5, 5.5, -1.0, 1.0, -2.0, 2.0), (0.25, 0.25, 0.125)
    check_forward(F, K, E, 256, 640, ranges, res, 1e-5)
    check_backward(torch.randn((1, 8, 16, 8), generator=torch.Generator().manual_seed(42)), K, E, 256, 640,
                   ranges, res, 1, 64, 160)


def test_largest_sizes():
    # Z = 1024
    K, E = I.make_rig(51, 6, 128, 352)
    K, E = torch.from_numpy(K)[None], torch.from_numpy(E)[None]
    F = torch.randn((1, 6, 8, 8, 22), generator=torch.Generator().manual_seed(51))
    ranges, res = (-8, 8, -8, 8, -5, 3), (2.0, 2.0, 8.0 / 1024)
    check_forward(F, K, E, 128, 352, ranges, res, 1e-5)
    check_backward(torch.randn((1, 8, 8, 8), generator=torch.Generator().manual_seed(52)), K, E, 128, 352,
                   ranges, res, 6, 8, 22)
    # 2048 channels
    F = torch.randn((1, 6, 2048, 4, 11), generator=torch.Generator().manual_seed(53))
    ranges, res = (-12, 12, -12, 12, -4, 4), (1.5, 1.5, 2.0)
    check_forward(F, K, E, 128, 352, ranges, res, 1e-5)
    # Wf = 16384
    K = torch.from_numpy(np.array([[[[4000.0, 0, 8192], [0, 4000.0, 1024], [0, 0, 1]]]], np.float32))
    E = torch.from_numpy(np.array([[[[0, -1, 0, 0], [0, 0, -1, 0], [1, 0, 0, 0], [0, 0, 0, 1]]]], np.float32))
    F = torch.randn((1, 1, 4, 2, 16384), generator=torch.Generator().manual_seed(55))
    ranges, res = (5, 25, -20, 20, -1, 1), (1.0, 0.25, 0.5)
    check_forward(F, K, E, 2048, 16384, ranges, res, 1e-5)
    check_backward(torch.randn((1, 4, 20, 160), generator=torch.Generator().manual_seed(56)), K, E, 2048, 16384,
                   ranges, res, 1, 2, 16384)


def test_thirty_two_cameras():
    K1, E1 = I.random_rig(31, 16, 64, 160, spread=0.2)
    K = torch.from_numpy(np.concatenate([K1, K1]))[None]
    E = torch.from_numpy(np.concatenate([E1, E1]))[None]
    F = torch.randn((1, 32, 8, 8, 20), generator=torch.Generator().manual_seed(32))
    ranges, res = (-12, 12, -12, 12, -3, 3), (1.0, 1.0, 0.5)
    check_forward(F, K, E, 64, 160, ranges, res, 1e-5)
    check_backward(torch.randn((1, 8, 24, 24), generator=torch.Generator().manual_seed(33)), K, E, 64, 160,
                   ranges, res, 32, 8, 20)


def test_multiscale_tiny():
    w = I.MS_WORKLOADS["ms_tiny"]
    Fs = I.make_ms_features(w)
    K, E = I.make_rigs(w)
    g = ops.bev_grid_spec(w.ranges, w.res)
    out, _ = ops.bev_sample_forward_multiscale([f.to("cuda") for f in Fs], K.to("cuda"), E.to("cuda"), w.img_h,
                                               w.img_w, g)
    torch.cuda.synchronize()
    ref, bound, _ = oracle.ms_forward(Fs, K, E, w.img_h, w.img_w, oracle.Grid(w.ranges, w.res))
    got = out.cpu().double().numpy()
    nz = bound > 0
    assert np.all(got[~nz] == 0)
    assert float((np.abs(got - ref)[nz] / bound[nz]).max()) <= 1e-5
