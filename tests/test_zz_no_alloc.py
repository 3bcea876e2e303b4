"""The allocation-free feature gradient, bev_sample_backward_noalloc.

It exists for callers that cannot allocate device memory or pass a
workspace (engine plugins with pre-planned memory, deployments that forbid
allocation after start-up, real-time loops that cannot afford cudaMalloc's
stalls).  These tests call it through the C ABI and compare it with
bev_sample_backward, which takes a caller workspace, and with the CPU oracle,
on calls in a row with different upstream gradients and shapes: a later call
must not see anything an earlier one left in the shared built-in array.  The
file is named to be collected last, and it passes alone in a fresh process as
well as after the other tests.
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


def test_noalloc_backward_matches_workspace_backward_and_oracle_on_two_calls():
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
        oref, bound = oracle.backward(dout, w.N, w.Hf, w.Wf, K, E, w.img_h, w.img_w, og)
        assert _err(got, ref, bound) <= TOL
        assert _err(got, torch.from_numpy(oref), bound) <= TOL


def _one_camera_case(C, Hf, Wf, seed):
    """The tiny workload's grid seen by its first camera only, with C channels
    on an Hf x Wf feature map."""
    w = I.WORKLOADS["tiny"]
    K, E = I.make_rigs(w)
    K, E = K[:, :1].contiguous(), E[:, :1].contiguous()
    dout = torch.randn(1, C, w.X, w.Y, generator=torch.Generator().manual_seed(seed))
    return w, K, E, dout, ops.bev_grid_spec(w.ranges, w.res)


def test_noalloc_at_the_limit_then_a_smaller_ragged_call():
    # B*N*Hf*Wf*round_up(C,4)*4 = 1*1*64*64*1024*4 bytes: exactly the built-in 16 MiB
    assert 64 * 64 * 1024 * 4 == ops.BEV_NOALLOC_SCRATCH_BYTES
    for C, Hf, Wf, seed in ((1024, 64, 64, 5), (3, 16, 44, 6)):   # the second call: C % 4 != 0
        w, K, E, dout, g = _one_camera_case(C, Hf, Wf, seed)
        d, Kd, Ed = dout.to(DEV), K.to(DEV), E.to(DEV)
        out = torch.empty((1, 1, C, Hf, Wf), dtype=torch.float32, device=DEV)
        got = ops.bev_sample_backward_noalloc(d, Kd, Ed, w.img_h, w.img_w, g, 1, Hf, Wf, out=out)
        ref = ops.bev_sample_backward(d, Kd, Ed, w.img_h, w.img_w, g, 1, Hf, Wf)
        torch.cuda.synchronize()
        _, bound = oracle.backward(dout, 1, Hf, Wf, K, E, w.img_h, w.img_w, oracle.Grid(w.ranges, w.res))
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


def test_noalloc_binding_checks_the_output_tensor():
    w = I.WORKLOADS["tiny"]
    K, E = I.make_rigs(w)
    g = ops.bev_grid_spec(w.ranges, w.res)
    dout = torch.zeros((w.B, w.C, w.X, w.Y), device=DEV)
    for bad in (torch.empty((w.B, w.N, w.C, w.Hf, w.Wf + 1), device=DEV),        # shape
                torch.empty((w.B, w.N, w.C, w.Hf, w.Wf), dtype=torch.float64, device=DEV),
                torch.empty((w.B, w.N, w.C, w.Wf, w.Hf), device=DEV).transpose(3, 4)):   # not contiguous
        with pytest.raises(ValueError):
            ops.bev_sample_backward_noalloc(dout, K.to(DEV), E.to(DEV), w.img_h, w.img_w, g, w.N, w.Hf, w.Wf,
                                            out=bad)
