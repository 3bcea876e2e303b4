"""GPU parity of the multi-scale dense Sampling-VT (FlashBEV reading notes,
"Takeaway" 4: multi-scale fused view transformation) against the oracle,
through the C ABI.

Gates as for the single-level path: valid counts bit-exact; outputs within
err = max |gpu - oracle| / bound <= 1e-5, bound = the oracle's fp64 sum of
|terms| (elements with bound 0 must be exactly 0), for fp32 and bf16
features alike (both sides read the same bf16 values).
"""
import numpy as np
import pytest
import torch

import oracle
from camera_bev_view_b200 import inputs as I
from camera_bev_view_b200 import ops

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
TOL = 1e-5


def rel_err(got, ref, bound):
    got = np.asarray(got, dtype=np.float64)
    zero = bound == 0
    assert np.all(got[zero] == 0), "elements with no contribution must be exactly 0"
    if np.all(zero):
        return 0.0
    return float((np.abs(got - ref)[~zero] / bound[~zero]).max())


def _grid(w):
    return ops.bev_grid_spec(w.ranges, w.res)


def run_forward(w, Fs, K, E, layout=ops.NCHW):
    Fd = [f.to(DEV) for f in Fs]
    if layout == ops.NHWC:
        Fd = [f.permute(0, 1, 3, 4, 2).contiguous() for f in Fd]
    out, cnt = ops.bev_sample_forward_multiscale(Fd, K.to(DEV), E.to(DEV), w.img_h, w.img_w, _grid(w),
                                                 layout=layout, count=True)
    torch.cuda.synchronize()
    return out.cpu(), cnt.cpu()


def check(w, Fs=None, K=None, E=None, backward=True):
    Fs = Fs if Fs is not None else I.make_ms_features(w)
    if K is None:
        K, E = I.make_rigs(w)
    out, cnt = run_forward(w, Fs, K, E)
    grid = oracle.Grid(w.ranges, w.res)
    ref, bound, ref_cnt = oracle.ms_forward(Fs, K, E, w.img_h, w.img_w, grid)
    np.testing.assert_array_equal(cnt.numpy().astype(np.int32), ref_cnt)
    e = rel_err(out.numpy(), ref, bound)
    assert e <= TOL, ("forward", e)
    if not backward:
        return out
    g = I.make_dout(w)
    sizes = [tuple(f.shape[3:5]) for f in Fs]
    dF = ops.bev_sample_backward_multiscale(g.to(DEV), K.to(DEV), E.to(DEV), w.img_h, w.img_w, _grid(w), w.N, sizes)
    torch.cuda.synchronize()
    rF, rB = oracle.ms_backward(g, w.N, sizes, K, E, w.img_h, w.img_w, grid)
    for l in range(len(sizes)):
        e = rel_err(dF[l].cpu().numpy(), rF[l], rB[l])
        assert e <= TOL, ("backward level", l, e)
    return out


@pytest.mark.parametrize("name", ["ms_tiny", "ms", "ms_bf16"])
def test_multiscale_workload_full_size(name):
    check(I.MS_WORKLOADS[name])


@pytest.mark.parametrize("name", ["ms", "ms_bf16"])
def test_multiscale_full_size_tilted_rigs(name):
    """The full-size pyramids on rigs with random yaw, +-8 degree pitch and
    roll and off-centre principal points: slanted projections on every
    level, forward and every level's gradient."""
    w = I.MS_WORKLOADS[name]
    Ks, Es = zip(*(I.random_rig(400 + b, w.N, w.img_h, w.img_w) for b in range(w.B)))
    check(w, K=torch.from_numpy(np.stack(Ks)), E=torch.from_numpy(np.stack(Es)))


def test_one_level_is_bitwise_the_single_level_forward():
    w = I.WORKLOADS["nuscenes"]
    F = I.make_features(w)
    K, E = I.make_rigs(w)
    g = _grid(w)
    o1, c1 = ops.bev_sample_forward(F.to(DEV), K.to(DEV), E.to(DEV), w.img_h, w.img_w, g, count=True)
    o2, c2 = ops.bev_sample_forward_multiscale([F.to(DEV)], K.to(DEV), E.to(DEV), w.img_h, w.img_w, g, count=True)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(c1, c2)


def test_channels_last_levels_are_bitwise_the_same():
    w = I.MS_WORKLOADS["ms_tiny"]
    Fs = I.make_ms_features(w)
    K, E = I.make_rigs(w)
    o1, _ = run_forward(w, Fs, K, E, ops.NCHW)
    o2, _ = run_forward(w, Fs, K, E, ops.NHWC)
    assert torch.equal(o1, o2)


@pytest.mark.parametrize("C,dtype", [(13, "f32"), (20, "bf16"), (300, "f32"), (3, "f32")])
def test_ragged_and_wide_channels(C, dtype):
    check(I.MS_WORKLOADS["ms_tiny"].scaled(C=C, dtype=dtype))


def test_levels_that_are_not_halvings_and_a_one_texel_level():
    """Sizes 7x19, 3x5 and 1x1 on a 128x352 image: each level's own scale
    W_l / W_img, and a level whose only texel is every valid sample's corner."""
    check(I.MS_WORKLOADS["ms_tiny"].scaled(levels=((7, 19), (3, 5), (1, 1))))


def test_two_levels_batched_with_a_third_of_the_grid():
    check(I.MS_WORKLOADS["ms"].scaled(B=2, C=8, X=67, Y=41, levels=((16, 44), (8, 22))))


def test_forward_is_deterministic_and_backward_reproducible():
    w = I.MS_WORKLOADS["ms"]
    Fs = [f.to(DEV) for f in I.make_ms_features(w)]
    K, E = (t.to(DEV) for t in I.make_rigs(w))
    g = _grid(w)
    o1, _ = ops.bev_sample_forward_multiscale(Fs, K, E, w.img_h, w.img_w, g)
    o2, _ = ops.bev_sample_forward_multiscale(Fs, K, E, w.img_h, w.img_w, g)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2)


def test_host_pointers_are_rejected():
    w = I.MS_WORKLOADS["ms_tiny"]
    Fs = I.make_ms_features(w)
    K, E = I.make_rigs(w)
    Fd = [f.to(DEV) for f in Fs]
    Fd[2] = Fs[2]                      # one level left on the host
    with pytest.raises(ops.BevError) as ei:
        ops.bev_sample_forward_multiscale(Fd, K.to(DEV), E.to(DEV), w.img_h, w.img_w, _grid(w))
    assert ei.value.status == -1
