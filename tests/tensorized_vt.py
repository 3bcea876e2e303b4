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


def tensorized_ms_forward(levels, K, E, ranges, counts, img_h, img_w):
    """Multi-scale form: one projection and mask, one grid_sample per level
    (the normalised grid is the same for every level: align_corners=False
    maps it to u * W_l / W_img - 0.5 on a map of width W_l), the levels'
    samples summed before the masked mean over cameras.  Returns out, count,
    ambiguous as ``tensorized_forward`` does."""
    Fs = [torch.as_tensor(f).to(torch.float64) for f in levels]
    B, N, C = Fs[0].shape[:3]
    X, Y, Z = counts
    u, v, depth, mask = project_all(K, E, ranges, counts, img_h, img_w)
    grid = torch.stack([2.0 * u / img_w - 1.0, 2.0 * v / img_h - 1.0], dim=-1)
    grid = torch.where(mask[..., None], grid, torch.zeros_like(grid)).reshape(B * N, X * Y * Z, 1, 2)
    total = torch.zeros((B, N, C, X, Y, Z), dtype=torch.float64)
    for F in Fs:
        Hl, Wl = F.shape[3:]
        s = Fn.grid_sample(F.reshape(B * N, C, Hl, Wl), grid, mode="bilinear", padding_mode="zeros",
                           align_corners=False)
        total = total + s.reshape(B, N, C, X, Y, Z)
    total = total * mask[:, :, None].to(torch.float64)
    count = mask.sum(dim=1)
    out = (total.sum(dim=1) / count.clamp(min=1)[:, None].to(torch.float64)).sum(dim=-1)
    return out, count, ambiguous(u, v, depth, img_h, img_w).any(dim=1)


def tensorized_ms_backward(dout, N, sizes, K, E, ranges, counts, img_h, img_w):
    """dL/dF_l of every level by autograd through the multi-scale form."""
    dout = torch.as_tensor(dout, dtype=torch.float64)
    B, C = dout.shape[:2]
    Fs = [torch.zeros((B, N, C, h, w), dtype=torch.float64, requires_grad=True) for h, w in sizes]
    out, _, amb = tensorized_ms_forward(Fs, K, E, ranges, counts, img_h, img_w)
    (out * dout).sum().backward()
    return [F.grad for F in Fs], amb


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


# --------------------------------------------------------------------------
# Lift-splat BEV pooling (LSS tutorial, "Lift" and "Splat"), materialised:
# every frustum point (b, n, k, h, w) in float64 -- pixel centre, depth of
# bin k, K^-1 by torch.linalg.inv, E^-1 by torch.linalg.inv -- its pillar by
# floor, the outer product depth x feat as an explicit [.., D, C] tensor, and
# a float64 index_add into the BEV grid.
# --------------------------------------------------------------------------

def lss_points(K, E, Hf, Wf, img_h, img_w, dbound):
    """Ego points [B,N,D,Hf,Wf,3] of every frustum point, float64."""
    K = torch.as_tensor(K, dtype=torch.float64)
    E = torch.as_tensor(E, dtype=torch.float64)
    dmin, dmax, dstep = (float(v) for v in dbound)
    D = int(round((dmax - dmin) / dstep))
    ds = dmin + dstep * torch.arange(D, dtype=torch.float64)
    us = (torch.arange(Wf, dtype=torch.float64) + 0.5) * (img_w / Wf)
    vs = (torch.arange(Hf, dtype=torch.float64) + 0.5) * (img_h / Hf)
    v, u = torch.meshgrid(vs, us, indexing="ij")
    pix = torch.stack([u, v, torch.ones_like(u)], dim=-1)                      # [Hf,Wf,3]
    rays = torch.einsum("bnrk,hwk->bnhwr", torch.linalg.inv(K), pix)           # camera frame, depth 1
    pc = ds[None, None, :, None, None, None] * rays[:, :, None]                # [B,N,D,Hf,Wf,3]
    Einv = torch.linalg.inv(E)
    return torch.einsum("bnrk,bndhwk->bndhwr", Einv[:, :, :3, :3], pc) + Einv[:, :, None, None, None, :3, 3]


def tensorized_lss(depth, feat, K, E, img_h, img_w, ranges, counts_xy, dbound, margin=1e-4):
    """Returns (out [B,C,X,Y], count [B,X,Y], ambiguous [B,N,D,Hf,Wf]) in float64;
    ``ambiguous`` marks points within ``margin`` (relative to the cell) of a
    cell edge or of the z slab's bounds."""
    A = torch.as_tensor(depth)
    A = A if A.dtype == torch.float64 else A.to(torch.float64)
    Fe = torch.as_tensor(feat)
    Fe = Fe if Fe.dtype == torch.float64 else Fe.to(torch.float64)
    B, N, D, Hf, Wf = A.shape
    C = Fe.shape[2]
    X, Y = counts_xy
    xmin, xmax, ymin, ymax, zmin, zmax = (float(r) for r in ranges)
    dx, dy = (xmax - xmin) / X, (ymax - ymin) / Y
    P = lss_points(K, E, Hf, Wf, img_h, img_w, dbound)
    fi = (P[..., 0] - xmin) / dx
    fj = (P[..., 1] - ymin) / dy
    i, j = torch.floor(fi), torch.floor(fj)
    inside = (i >= 0) & (i < X) & (j >= 0) & (j < Y) & (P[..., 2] >= zmin) & (P[..., 2] < zmax)
    amb = (((fi - torch.round(fi)).abs() < margin) | ((fj - torch.round(fj)).abs() < margin) |
           ((P[..., 2] - zmin).abs() < margin) | ((P[..., 2] - zmax).abs() < margin))
    pts = A[:, :, :, None] * Fe[:, :, None]                                    # [B,N,D,C,Hf,Wf] outer product
    cellid = torch.where(inside, (i * Y + j).long(), torch.zeros_like(i).long())
    out = torch.zeros((B, C, X * Y), dtype=torch.float64)
    count = torch.zeros((B, X * Y), dtype=torch.float64)
    for b in range(B):
        m = inside[b].reshape(-1)
        idx = cellid[b].reshape(-1)[m]
        vals = pts[b].permute(0, 1, 3, 4, 2).reshape(-1, C)[m]                 # [points, C]
        out[b].index_add_(1, idx, vals.t())
        count[b].index_add_(0, idx, torch.ones_like(idx, dtype=torch.float64))
    return out.reshape(B, C, X, Y), count.reshape(B, X, Y), amb
