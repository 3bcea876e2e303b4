"""The allocation-free feature gradient, bev_sample_backward_noalloc.

It exists for callers that cannot allocate device memory or pass a
workspace (engine plugins with pre-planned memory, deployments that forbid
allocation after start-up, real-time loops that cannot afford cudaMalloc's
stalls).  These tests call it through the C ABI and compare it with
bev_sample_backward, which takes a caller workspace, on two calls in a row
with different upstream gradients: the second call must not see anything the
first left in the shared built-in array.  The file is named to be collected
last, and it passes alone in a fresh process as well as after the other tests.
"""
import numpy as np
import pytest
import torch

import oracle
from camera_bev_view_b200 import inputs as I
from camera_bev_view_b200 import ops

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
TOL = 1e-5   # the fp32 parity tolerance of the other GPU tests, relative to the oracle's bound


def _err(got, ref, bound):
    got = got.cpu().double().numpy()
    ref = ref.cpu().double().numpy()
    zero = bound == 0
    assert np.all(got[zero] == 0) and np.all(ref[zero] == 0)
    return float((np.abs(got - ref)[~zero] / bound[~zero]).max())


def test_noalloc_backward_matches_workspace_backward_on_two_calls():
    w = I.WORKLOADS["backward"]
    K, E = I.make_rigs(w)
    g = ops.bev_grid_spec(w.ranges, w.res)
    og = oracle.Grid(w.ranges, w.res)
    Kd, Ed = K.to(DEV), E.to(DEV)
    douts = [I.make_dout(w), 3.0 * torch.randn(w.B, w.C, w.X, w.Y, generator=torch.Generator().manual_seed(77))]
    out = torch.empty((w.B, w.N, w.C, w.Hf, w.Wf), dtype=torch.float32, device=DEV)
    for dout in douts:
        d = dout.to(DEV)
        ref = ops.bev_sample_backward(d, Kd, Ed, w.img_h, w.img_w, g, w.N, w.Hf, w.Wf)
        got = ops.bev_sample_backward_noalloc(d, Kd, Ed, w.img_h, w.img_w, g, w.N, w.Hf, w.Wf, out=out)
        torch.cuda.synchronize()
        _, bound = oracle.backward(dout, w.N, w.Hf, w.Wf, K, E, w.img_h, w.img_w, og)
        assert _err(got, ref, bound) <= TOL


def test_noalloc_rejects_shapes_beyond_the_builtin_array():
    w = I.WORKLOADS["backward"]
    K, E = I.make_rigs(w)
    g = ops.bev_grid_spec(w.ranges, w.res)
    C = 1024                    # 2*6*16*44*1024*4 bytes = 34.6 MB > 16 MiB
    dout = torch.zeros((w.B, C, w.X, w.Y), device=DEV)
    out = torch.empty((w.B, w.N, C, w.Hf, w.Wf), device=DEV)
    with pytest.raises(ops.BevError) as e:
        ops.bev_sample_backward_noalloc(dout, K.to(DEV), E.to(DEV), w.img_h, w.img_w, g, w.N, w.Hf, w.Wf,
                                        out=out)
    assert e.value.status == -2
