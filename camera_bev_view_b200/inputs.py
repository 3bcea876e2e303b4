"""Seeded synthetic inputs shared by the oracle tests, the GPU tests and the bench.

This module draws random numbers and lays out camera rigs. It holds none of
the view transform's arithmetic (no projection, no validity test, no
sampling) and imports nothing else from this package, so that the oracle
and the CUDA path can both consume identical bytes without sharing code.

Workloads (shapes after the LSS tutorial's worked sizes, "Lift" section:
128x352 images at stride 16 give an 8x22 feature map; "Splat" section: a
-50..50 m BEV at 0.5 m per cell gives 200x200):

  tiny        B1 N6 C16  8x22  (img 128x352)   50x50x4   over +-25 m  fp32
  nuscenes    B1 N6 C64  16x44 (img 256x704)   200x200x8 over +-50 m  fp32
  batched     B4 N6 C128 32x88 (img 512x1408)  200x200x16 over +-50 m bf16
  large       B1 N6 C80  32x88 (img 512x1408)  400x400x16 over +-50 m fp32
  backward    nuscenes shapes with B2, upstream gradient N(0,1)

Deformable-aggregation workloads (SparseDriveV2 notes, "Deformable
Aggregation": Nq queries of K keypoints each, with Nq ~ 10^2-10^3 and K in
the tens, over six surround cameras):

  deform_tiny  B1 N6 C16  8x22   (img 128x352)  Q32  K4   fp32
  deform       B1 N6 C256 64x176 (img 512x1408) Q900 K13  fp32
  deform_bf16  B4 N6 C256 64x176 (img 512x1408) Q900 K13  bf16

Lift-splat pooling workloads (LSS tutorial, "Lift" and "Splat": 41 depth
bins over [4, 45) m at 1 m, 64-d context, 8x22 features per camera from
128x352 images, 6 cameras, a 200x200 BEV at 0.5 m; z is one pillar, taken
as [-10, 10] m):

  lss_tiny  B1 N6 C8  D8  8x22  (img 128x352)  40x40 over +-20 m   fp32
  lss       B1 N6 C64 D41 8x22  (img 128x352)  200x200 over +-50 m fp32
  lss_b4    B4 N6 C64 D41 16x44 (img 256x704)  200x200 over +-50 m fp32

Multi-scale workloads (FlashBEV reading notes, "Takeaway" 4: multi-scale
fused view transformation; SparseDriveV2 notes, "Image Encoder": an FPN
gives P2..P5 at strides 4, 8, 16 and 32 with one channel count; 256x704
images as in the nuScenes-like workload):

  ms_tiny   B1 N6 C16  32x88,16x44,8x22,4x11 (img 128x352)  50x50x4   over +-25 m fp32
  ms        B1 N6 C64  64x176,32x88,16x44,8x22 (img 256x704) 200x200x8 over +-50 m fp32
  ms_bf16   B2 N6 C128 64x176,32x88,16x44,8x22 (img 256x704) 200x200x8 over +-50 m bf16

Level l of the features is drawn i.i.d. N(0, 1) from its own seed.

Depth distributions are a softmax over the bins of N(0, 1) * 2 logits;
context features and the upstream gradient are N(0, 1).

Anchors are uniform over x, y in [-50, 50] m and z in [-2, 2] m; keypoint
offsets uniform in [-2, 2] m per axis; weights uniform in [0, 1) / (N K);
the upstream gradient is N(0, 1).

z always spans [-5, 3] m.  Rig: camera n has nominal yaw 60 deg * n, sits at
(cos yaw, sin yaw, 1.5) m plus U(-0.05, 0.05) m jitter per axis, and looks
horizontally along yaw + U(-2, 2) deg with no pitch or roll.  Ego frame:
x forward, y left, z up.  Camera frame: x right, y down, z forward.  The
extrinsic maps ego to camera (SparseDriveV2 notes, "Deformable Aggregation"
pitfalls: the extrinsic takes ego coordinates into the camera frame).
Pinhole intrinsics fx = fy = 0.7 * W_img, cx = W_img / 2, cy = H_img / 2.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    index: int            # seed family
    B: int
    N: int
    C: int
    Hf: int
    Wf: int
    img_h: int
    img_w: int
    X: int
    Y: int
    Z: int
    xr: tuple
    yr: tuple
    zr: tuple
    dtype: str            # "f32" or "bf16" feature storage
    backward: bool = False

    @property
    def ranges(self):
        return (self.xr[0], self.xr[1], self.yr[0], self.yr[1], self.zr[0], self.zr[1])

    @property
    def res(self):
        """Cell sizes that reproduce the stated counts (extent / count)."""
        return ((self.xr[1] - self.xr[0]) / self.X,
                (self.yr[1] - self.yr[0]) / self.Y,
                (self.zr[1] - self.zr[0]) / self.Z)

    @property
    def out_elems(self):
        return self.B * self.C * self.X * self.Y

    def scaled(self, **kw):
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    "tiny": Workload("tiny", 0, 1, 6, 16, 8, 22, 128, 352, 50, 50, 4,
                     (-25.0, 25.0), (-25.0, 25.0), (-5.0, 3.0), "f32"),
    "nuscenes": Workload("nuscenes", 1, 1, 6, 64, 16, 44, 256, 704, 200, 200, 8,
                         (-50.0, 50.0), (-50.0, 50.0), (-5.0, 3.0), "f32"),
    "batched_bf16": Workload("batched_bf16", 2, 4, 6, 128, 32, 88, 512, 1408, 200, 200, 16,
                             (-50.0, 50.0), (-50.0, 50.0), (-5.0, 3.0), "bf16"),
    "large": Workload("large", 3, 1, 6, 80, 32, 88, 512, 1408, 400, 400, 16,
                      (-50.0, 50.0), (-50.0, 50.0), (-5.0, 3.0), "f32"),
    "backward": Workload("backward", 4, 2, 6, 64, 16, 44, 256, 704, 200, 200, 8,
                         (-50.0, 50.0), (-50.0, 50.0), (-5.0, 3.0), "f32", backward=True),
}


@dataclasses.dataclass(frozen=True)
class DeformWorkload:
    name: str
    index: int            # seed family
    B: int
    N: int
    C: int
    Hf: int
    Wf: int
    img_h: int
    img_w: int
    Q: int                # queries per batch item
    Kp: int               # keypoints per query
    dtype: str            # "f32" or "bf16" feature storage

    @property
    def out_elems(self):
        return self.B * self.Q * self.C

    def scaled(self, **kw):
        return dataclasses.replace(self, **kw)


DEFORM_WORKLOADS = {
    "deform_tiny": DeformWorkload("deform_tiny", 10, 1, 6, 16, 8, 22, 128, 352, 32, 4, "f32"),
    "deform": DeformWorkload("deform", 11, 1, 6, 256, 64, 176, 512, 1408, 900, 13, "f32"),
    "deform_bf16": DeformWorkload("deform_bf16", 12, 4, 6, 256, 64, 176, 512, 1408, 900, 13, "bf16"),
}


@dataclasses.dataclass(frozen=True)
class MultiScaleWorkload:
    name: str
    index: int            # seed family
    B: int
    N: int
    C: int
    levels: tuple         # ((H_0, W_0), (H_1, W_1), ...)
    img_h: int
    img_w: int
    X: int
    Y: int
    Z: int
    xr: tuple
    yr: tuple
    zr: tuple
    dtype: str            # "f32" or "bf16" feature storage

    @property
    def ranges(self):
        return (self.xr[0], self.xr[1], self.yr[0], self.yr[1], self.zr[0], self.zr[1])

    @property
    def res(self):
        return ((self.xr[1] - self.xr[0]) / self.X,
                (self.yr[1] - self.yr[0]) / self.Y,
                (self.zr[1] - self.zr[0]) / self.Z)

    @property
    def out_elems(self):
        return self.B * self.C * self.X * self.Y

    def scaled(self, **kw):
        return dataclasses.replace(self, **kw)


_P2_P5_256x704 = ((64, 176), (32, 88), (16, 44), (8, 22))

MS_WORKLOADS = {
    "ms_tiny": MultiScaleWorkload("ms_tiny", 30, 1, 6, 16, ((32, 88), (16, 44), (8, 22), (4, 11)), 128, 352,
                                  50, 50, 4, (-25.0, 25.0), (-25.0, 25.0), (-5.0, 3.0), "f32"),
    "ms": MultiScaleWorkload("ms", 31, 1, 6, 64, _P2_P5_256x704, 256, 704, 200, 200, 8,
                             (-50.0, 50.0), (-50.0, 50.0), (-5.0, 3.0), "f32"),
    "ms_bf16": MultiScaleWorkload("ms_bf16", 32, 2, 6, 128, _P2_P5_256x704, 256, 704, 200, 200, 8,
                                  (-50.0, 50.0), (-50.0, 50.0), (-5.0, 3.0), "bf16"),
}


def make_ms_features(w: MultiScaleWorkload, shard: int = 0, layout: str = "nchw"):
    """One i.i.d. N(0,1) feature map per level, [B,N,C,H_l,W_l] (or
    [B,N,H_l,W_l,C] for ``nhwc``) on CPU; bf16 rounds the float32 draw."""
    out = []
    for l, (h, wl) in enumerate(w.levels):
        g = torch.Generator().manual_seed(5000 + 10 * w.index + l + 100003 * shard)
        f = torch.randn((w.B, w.N, w.C, h, wl), generator=g, dtype=torch.float32)
        if w.dtype == "bf16":
            f = f.to(torch.bfloat16)
        if layout == "nhwc":
            f = f.permute(0, 1, 3, 4, 2).contiguous()
        out.append(f)
    return out


@dataclasses.dataclass(frozen=True)
class LssWorkload:
    name: str
    index: int            # seed family
    B: int
    N: int
    C: int
    D: int                # depth bins
    Hf: int
    Wf: int
    img_h: int
    img_w: int
    X: int
    Y: int
    xr: tuple
    yr: tuple
    zr: tuple
    dbound: tuple         # (dmin, dmax, dstep)
    dtype: str = "f32"

    @property
    def ranges(self):
        return (self.xr[0], self.xr[1], self.yr[0], self.yr[1], self.zr[0], self.zr[1])

    @property
    def res_xy(self):
        return ((self.xr[1] - self.xr[0]) / self.X, (self.yr[1] - self.yr[0]) / self.Y)

    @property
    def out_elems(self):
        return self.B * self.C * self.X * self.Y

    def scaled(self, **kw):
        return dataclasses.replace(self, **kw)


LSS_WORKLOADS = {
    "lss_tiny": LssWorkload("lss_tiny", 20, 1, 6, 8, 8, 8, 22, 128, 352, 40, 40, (-20.0, 20.0), (-20.0, 20.0),
                            (-10.0, 10.0), (4.0, 12.0, 1.0)),
    "lss": LssWorkload("lss", 21, 1, 6, 64, 41, 8, 22, 128, 352, 200, 200, (-50.0, 50.0), (-50.0, 50.0),
                       (-10.0, 10.0), (4.0, 45.0, 1.0)),
    "lss_b4": LssWorkload("lss_b4", 22, 4, 6, 64, 41, 16, 44, 256, 704, 200, 200, (-50.0, 50.0), (-50.0, 50.0),
                          (-10.0, 10.0), (4.0, 45.0, 1.0)),
}


def make_lss_inputs(w: LssWorkload, shard: int = 0):
    """(depth [B,N,D,Hf,Wf], feat [B,N,C,Hf,Wf]) float32 torch (CPU): depth is a
    softmax over the bins of N(0,1) * 2 logits; feat is N(0,1)."""
    g = torch.Generator().manual_seed(7000 + w.index + 100003 * shard)
    logits = 2.0 * torch.randn((w.B, w.N, w.D, w.Hf, w.Wf), generator=g, dtype=torch.float32)
    depth = torch.softmax(logits, dim=2)
    feat = torch.randn((w.B, w.N, w.C, w.Hf, w.Wf), generator=g, dtype=torch.float32)
    return depth.contiguous(), feat


def make_lss_dout(w: LssWorkload, shard: int = 0) -> torch.Tensor:
    """Upstream gradient [B,C,X,Y] float32, i.i.d. N(0,1)."""
    g = torch.Generator().manual_seed(8000 + w.index + 100003 * shard)
    return torch.randn((w.B, w.C, w.X, w.Y), generator=g, dtype=torch.float32)


def make_queries(w: DeformWorkload, shard: int = 0):
    """(anchors [B,Q,3], offsets [B,Q,Kp,3], weights [B,Q,N,Kp]) float32 torch (CPU)."""
    rng = np.random.default_rng(5000 + w.index + 100003 * shard)
    anchors = np.stack([rng.uniform(-50.0, 50.0, size=(w.B, w.Q)), rng.uniform(-50.0, 50.0, size=(w.B, w.Q)),
                        rng.uniform(-2.0, 2.0, size=(w.B, w.Q))], axis=-1)
    offsets = rng.uniform(-2.0, 2.0, size=(w.B, w.Q, w.Kp, 3))
    weights = rng.uniform(0.0, 1.0, size=(w.B, w.Q, w.N, w.Kp)) / (w.N * w.Kp)
    return (torch.from_numpy(anchors.astype(np.float32)), torch.from_numpy(offsets.astype(np.float32)),
            torch.from_numpy(weights.astype(np.float32)))


def make_query_dout(w: DeformWorkload, shard: int = 0) -> torch.Tensor:
    """Upstream gradient [B,Q,C] float32, i.i.d. N(0,1)."""
    g = torch.Generator().manual_seed(6000 + w.index + 100003 * shard)
    return torch.randn((w.B, w.Q, w.C), generator=g, dtype=torch.float32)


def pinhole_intrinsics(img_h: int, img_w: int) -> np.ndarray:
    f = 0.7 * img_w
    return np.array([[f, 0.0, img_w / 2.0], [0.0, f, img_h / 2.0], [0.0, 0.0, 1.0]])


def camera_extrinsic(yaw: float, pos) -> np.ndarray:
    """Ego-to-camera 4x4 for a level camera looking along ``yaw`` from ``pos``.

    Rows of R are the camera axes written in ego coordinates:
    x_c = (sin yaw, -cos yaw, 0), y_c = (0, 0, -1), z_c = (cos yaw, sin yaw, 0);
    E = [R | -R pos; 0 0 0 1].  Built in float64.
    """
    R = np.array([[math.sin(yaw), -math.cos(yaw), 0.0],
                  [0.0, 0.0, -1.0],
                  [math.cos(yaw), math.sin(yaw), 0.0]])
    E = np.eye(4)
    E[:3, :3] = R
    E[:3, 3] = -R @ np.asarray(pos, dtype=np.float64)
    return E


def make_rig(seed: int, N: int, img_h: int, img_w: int, jitter: bool = True):
    """Return (K [N,3,3], E [N,4,4]) as float32 arrays for one batch item.

    Per camera, in order, the generator draws the yaw jitter and then the
    three position jitters.
    """
    rng = np.random.default_rng(seed)
    K = np.empty((N, 3, 3))
    E = np.empty((N, 4, 4))
    for n in range(N):
        yaw0 = math.radians(60.0 * n)
        dyaw = rng.uniform(-2.0, 2.0) if jitter else 0.0
        dpos = rng.uniform(-0.05, 0.05, size=3) if jitter else np.zeros(3)
        pos = np.array([math.cos(yaw0), math.sin(yaw0), 1.5]) + dpos
        K[n] = pinhole_intrinsics(img_h, img_w)
        E[n] = camera_extrinsic(yaw0 + math.radians(dyaw), pos)
    return K.astype(np.float32), E.astype(np.float32)


def rig_seed(w: Workload, b: int, shard: int = 0) -> int:
    return 2000 + 16 * w.index + b + 100003 * shard


def make_rigs(w: Workload, shard: int = 0):
    """Calibrations for every batch item: (K [B,N,3,3], E [B,N,4,4]) float32 torch (CPU)."""
    Ks, Es = [], []
    for b in range(w.B):
        K, E = make_rig(rig_seed(w, b, shard), w.N, w.img_h, w.img_w)
        Ks.append(K)
        Es.append(E)
    return torch.from_numpy(np.stack(Ks)), torch.from_numpy(np.stack(Es))


def make_features(w: Workload, shard: int = 0, layout: str = "nchw") -> torch.Tensor:
    """i.i.d. N(0,1) features [B,N,C,Hf,Wf] (or [B,N,Hf,Wf,C] for ``nhwc``) on CPU.

    bf16 workloads round the float32 draw to nearest-even.
    """
    g = torch.Generator().manual_seed(1000 + w.index + 100003 * shard)
    f = torch.randn((w.B, w.N, w.C, w.Hf, w.Wf), generator=g, dtype=torch.float32)
    if w.dtype == "bf16":
        f = f.to(torch.bfloat16)
    if layout == "nhwc":
        f = f.permute(0, 1, 3, 4, 2).contiguous()
    return f


def make_dout(w: Workload, shard: int = 0) -> torch.Tensor:
    """Upstream gradient [B,C,X,Y] float32, i.i.d. N(0,1)."""
    g = torch.Generator().manual_seed(3000 + w.index + 100003 * shard)
    return torch.randn((w.B, w.C, w.X, w.Y), generator=g, dtype=torch.float32)


def random_rig(seed: int, N: int, img_h: int, img_w: int, height=(0.5, 2.5), spread=1.0):
    """A looser rig for property tests: random yaw, small pitch and roll, random mount.

    Cameras get yaw U(0, 360) deg, pitch and roll U(-8, 8) deg, position within
    ``spread`` m of the origin at a random height, and intrinsics with unequal
    focal lengths, skew 0 and a principal point off centre.  Float32 output.
    """
    rng = np.random.default_rng(seed)
    K = np.empty((N, 3, 3))
    E = np.empty((N, 4, 4))
    for n in range(N):
        yaw = rng.uniform(0, 2 * math.pi)
        pitch = math.radians(rng.uniform(-8, 8))
        roll = math.radians(rng.uniform(-8, 8))
        pos = np.array([rng.uniform(-spread, spread), rng.uniform(-spread, spread),
                        rng.uniform(*height)])
        base = camera_extrinsic(yaw, np.zeros(3))[:3, :3]
        cp, sp, cr, sr = math.cos(pitch), math.sin(pitch), math.cos(roll), math.sin(roll)
        Rx = np.array([[1, 0, 0], [0, cp, -sp], [0, sp, cp]])
        Rz = np.array([[cr, -sr, 0], [sr, cr, 0], [0, 0, 1]])
        R = Rz @ Rx @ base
        E[n] = np.eye(4)
        E[n, :3, :3] = R
        E[n, :3, 3] = -R @ pos
        fx = rng.uniform(0.5, 0.9) * img_w
        fy = fx * rng.uniform(0.9, 1.1)
        K[n] = np.array([[fx, 0.0, img_w * rng.uniform(0.4, 0.6)],
                         [0.0, fy, img_h * rng.uniform(0.4, 0.6)],
                         [0.0, 0.0, 1.0]])
    return K.astype(np.float32), E.astype(np.float32)
