"""Materialised ("tensorized") Sampling-VT in float64 on the CPU, for tiny grids.

This is the form the FlashBEV reading notes describe as the baseline ("Problem
Setting"): build the voxel grid, project every voxel into every camera, build
the validity mask, sample a Features3D volume of shape B x N x C x X x Y x Z with
``torch.nn.functional.grid_sample`` (bilinear, zero padding,
align_corners=False), take the masked mean over cameras and sum over height.
It is written independently of the loop-nest oracle -- whole-tensor einsums,
float64 geometry, and the library sampler for the bilinear step -- and is used
only to pin that oracle.

Because its geometry is float64, a validity decision can differ from the
oracle's fp32 one when a sample sits on an edge of the image or at the depth
threshold.  ``ambiguous`` flags every (b, n, x, y, z) within ``margin`` of such
an edge so that callers can leave those cells out of the comparison.
"""
from __future__ import annotations

import torch
import torch.nn.functional as Fn


def voxel_centres(ranges, counts):
    xmin, xmax, ymin, ymax, zmin, zmax = (float(r) for r in ranges)
    X, Y, Z = counts
    xs = xmin + (torch.arange(X, dtype=torch.float64) + 0.5) * ((xmax - xmin) / X)
    ys = ymin + (torch.arange(Y, dtype=torch.float64) + 0.5) * ((ymax - ymin) / Y)
    zs = zmin + (torch.arange(Z, dtype=torch.float64) + 0.5) * ((zmax - zmin) / Z)
    return xs, ys, zs


def project_all(K, E, ranges, counts, img_h, img_w):
    """uv, depth, mask for every (b, n, x, y, z): float64, shapes [B,N,X,Y,Z]."""
    K = torch.as_tensor(K, dtype=torch.float64)
    E = torch.as_tensor(E, dtype=torch.float64)
    xs, ys, zs = voxel_centres(ranges, counts)
    P = torch.stack(torch.meshgrid(xs, ys, zs, indexing="ij"), dim=-1)        # [X,Y,Z,3]
    Ph = torch.cat([P, torch.ones_like(P[..., :1])], dim=-1)                  # [X,Y,Z,4]
    cam = torch.einsum("bnrk,xyzk->bnxyzr", E[:, :, :3, :], Ph)               # ego -> camera
    pix = torch.einsum("bnrk,bnxyzk->bnxyzr", K, cam)                         # camera -> image
    depth = cam[..., 2]
    safe = torch.where(depth.abs() > 1e-12, depth, torch.ones_like(depth))
    u = pix[..., 0] / safe
    v = pix[..., 1] / safe
    mask = (depth > 0.1) & (u >= 0) & (u <= img_w) & (v >= 0) & (v <= img_h)
    return u, v, depth, mask


def ambiguous(u, v, depth, img_h, img_w, margin_px=0.05, margin_depth=1e-3):
    near_edge = ((u.abs() < margin_px) | ((u - img_w).abs() < margin_px) |
                 (v.abs() < margin_px) | ((v - img_h).abs() < margin_px))
    return ((depth - 0.1).abs() < margin_depth) | ((depth > 0.1) & near_edge)


def tensorized_forward(features, K, E, ranges, counts, img_h, img_w):
    """Returns out [B,C,X,Y], count [B,X,Y,Z], ambiguous [B,X,Y,Z] (any camera)."""
    F = torch.as_tensor(features).to(torch.float64)
    B, N, C, Hf, Wf = F.shape
    X, Y, Z = counts
    u, v, depth, mask = project_all(K, E, ranges, counts, img_h, img_w)
    # normalised grid for align_corners=False: pixel = ((g + 1) * size - 1) / 2
    gx = 2.0 * u / img_w - 1.0
    gy = 2.0 * v / img_h - 1.0
    grid = torch.stack([gx, gy], dim=-1)
    grid = torch.where(mask[..., None], grid, torch.zeros_like(grid))
    grid = grid.reshape(B * N, X * Y * Z, 1, 2)
    feats3d = Fn.grid_sample(F.reshape(B * N, C, Hf, Wf), grid, mode="bilinear",
                             padding_mode="zeros", align_corners=False)      # [BN,C,XYZ,1]
    feats3d = feats3d.reshape(B, N, C, X, Y, Z) * mask[:, :, None].to(torch.float64)
    count = mask.sum(dim=1)                                                   # [B,X,Y,Z]
    mean = feats3d.sum(dim=1) / count.clamp(min=1)[:, None].to(torch.float64)  # [B,C,X,Y,Z]
    out = mean.sum(dim=-1)
    amb = ambiguous(u, v, depth, img_h, img_w).any(dim=1)
    return out, count, amb


def tensorized_backward(dout, N, Hf, Wf, K, E, ranges, counts, img_h, img_w):
    """dL/dF by autograd through the materialised form (float64)."""
    dout = torch.as_tensor(dout, dtype=torch.float64)
    B, C = dout.shape[:2]
    F = torch.zeros((B, N, C, Hf, Wf), dtype=torch.float64, requires_grad=True)
    out, _, amb = tensorized_forward(F, K, E, ranges, counts, img_h, img_w)
    (out * dout).sum().backward()
    return F.grad, amb


# --------------------------------------------------------------------------
# Deformable aggregation (SparseDriveV2 notes, "Deformable Aggregation"
# steps 1-3), materialised: every (b, n, q, k) keypoint projected in float64,
# the validity mask, a grid_sample of every keypoint in every camera, the
# masked weighted sum.  Differentiable in the features, the weights and the
# offsets (autograd through grid_sample's sampling grid).
# --------------------------------------------------------------------------

def deform_keypoints(anchors, offsets, offsets64=None):
    """p = a + d, valued as the float32 sum; when ``offsets64`` (float64,
    requiring grad) is given the result carries its gradient with slope 1."""
    p32 = (torch.as_tensor(anchors, dtype=torch.float32)[:, :, None, :] +
           torch.as_tensor(offsets, dtype=torch.float32)).to(torch.float64)
    if offsets64 is None:
        return p32
    return p32 + (offsets64 - offsets64.detach())


def deform_project(K, E, p, img_h, img_w):
    """uv, depth, mask for every (b, n, q, k): float64, shapes [B,N,Q,Kp]."""
    K = torch.as_tensor(K, dtype=torch.float64)
    E = torch.as_tensor(E, dtype=torch.float64)
    cam = torch.einsum("bnrk,bqtk->bnqtr", E[:, :, :3, :3], p) + E[:, :, None, None, :3, 3]
    pix = torch.einsum("bnrk,bnqtk->bnqtr", K, cam)
    depth = cam[..., 2]
    safe = torch.where(depth.abs() > 1e-12, depth, torch.ones_like(depth))
    u = pix[..., 0] / safe
    v = pix[..., 1] / safe
    mask = (depth > 0.1) & (u >= 0) & (u <= img_w) & (v >= 0) & (v <= img_h)
    return u, v, depth, mask


def tensorized_deform(features, K, E, img_h, img_w, anchors, offsets, weights, offsets64=None):
    """Returns (out [B,Q,C], mask [B,N,Q,Kp], ambiguous [B,N,Q,Kp], fx, fy)."""
    F = torch.as_tensor(features)
    if F.dtype != torch.float64:
        F = F.to(torch.float64)
    B, N, C, Hf, Wf = F.shape
    W = torch.as_tensor(weights)
    if W.dtype != torch.float64:
        W = W.to(torch.float64)
    p = deform_keypoints(anchors, offsets, offsets64)                      # [B,Q,Kp,3]
    Q, Kp = p.shape[1], p.shape[2]
    u, v, depth, mask = deform_project(K, E, p, img_h, img_w)
    gx = 2.0 * u / img_w - 1.0
    gy = 2.0 * v / img_h - 1.0
    grid = torch.stack([gx, gy], dim=-1)
    grid = torch.where(mask[..., None], grid, torch.zeros_like(grid))
    phi = Fn.grid_sample(F.reshape(B * N, C, Hf, Wf), grid.reshape(B * N, Q, Kp, 2), mode="bilinear",
                         padding_mode="zeros", align_corners=False).reshape(B, N, C, Q, Kp)
    wm = W.permute(0, 2, 1, 3) * mask.to(torch.float64)                    # [B,N,Q,Kp]
    out = torch.einsum("bncqk,bnqk->bqc", phi, wm)
    amb = ambiguous(u, v, depth, img_h, img_w)
    fx = u * (Wf / img_w) - 0.5
    fy = v * (Hf / img_h) - 0.5
    return out, mask, amb, fx, fy
