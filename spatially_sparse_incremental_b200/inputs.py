"""Seeded synthetic inputs for the SIGE sparse-conv workloads.

This module only draws random numbers and places synthetic edits; it holds none
of the method's arithmetic (no difference mask, no tile reduction, no conv).
Both the CPU oracle tests and the CUDA path take their inputs from here, so the
two sides see the same bytes.

The pages evaluate on edited LSUN-Church / Cityscapes images, which are not
available here.  The generators below stand in for them with edits of the
size the pages quote ("about 1.2% of the area", mer.dev notes on SIGE,
Abstract; SIGE project page, "Performance"): seeded rectangles, discs and
ellipses whose union covers a requested fraction of the image.

Everything returns CPU torch tensors.  Activations are NHWC (N=1) unless a
function says otherwise; conv weights are [C_out][k][k][C_in] (KRSC); biases
and GroupNorm affine parameters are float32.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

__all__ = [
    "rect_mask", "blob_mask", "pool_any", "kaiming_uniform", "bias_uniform",
    "ConvLayer", "make_cfg1", "make_cfg2", "make_cfg3", "make_cfg4_layer",
    "make_cfg5_layer", "CFG4_LAYERS", "CFG5_LAYERS", "make_conv_case",
]


# ---------------------------------------------------------------------------
# edit-region shapes
# ---------------------------------------------------------------------------

def rect_mask(rng: np.random.Generator, H: int, W: int, area: float) -> np.ndarray:
    """One axis-aligned rectangle of about ``area * H * W`` pixels at a uniform
    position.  Height ~ U{hmin..hmax} around sqrt(target), width = round(target/h)."""
    target = max(1, int(round(area * H * W)))
    side = math.sqrt(target)
    hmin = max(1, int(side / 1.4))
    hmax = max(hmin, min(H, int(math.ceil(side * 1.4))))
    h = int(rng.integers(hmin, hmax + 1))
    w = int(min(W, max(1, round(target / h))))
    y0 = int(rng.integers(0, H - h + 1))
    x0 = int(rng.integers(0, W - w + 1))
    m = np.zeros((H, W), dtype=bool)
    m[y0:y0 + h, x0:x0 + w] = True
    return m


def _ellipse_union(H, W, cy, cx, ax, ay, th, s):
    yy, xx = np.mgrid[0:H, 0:W].astype(np.float64)
    m = np.zeros((H, W), dtype=bool)
    for i in range(len(cy)):
        dy, dx = yy - cy[i], xx - cx[i]
        u = (dx * math.cos(th[i]) + dy * math.sin(th[i])) / (s * ax[i])
        v = (-dx * math.sin(th[i]) + dy * math.cos(th[i])) / (s * ay[i])
        m |= (u * u + v * v) <= 1.0
    return m


def blob_mask(rng: np.random.Generator, H: int, W: int, area: float,
              kmin: int = 1, kmax: int = 3, ellipse: bool = True) -> np.ndarray:
    """Union of k ~ U{kmin..kmax} seeded ellipses (or discs) covering about
    ``area`` of the image.  Centres are uniform; for ellipses the angle is
    uniform and the axis ratio is drawn from [0.5, 2].  A common scale factor
    is bisected until the union's pixel count is within 10% of the target."""
    k = int(rng.integers(kmin, kmax + 1))
    cy = rng.uniform(0, H, size=k)
    cx = rng.uniform(0, W, size=k)
    th = rng.uniform(0, math.pi, size=k) if ellipse else np.zeros(k)
    ratio = rng.uniform(0.5, 2.0, size=k) if ellipse else np.ones(k)
    wgt = rng.uniform(0.5, 1.5, size=k)
    ax = wgt * np.sqrt(ratio)
    ay = wgt / np.sqrt(ratio)
    target = area * H * W
    lo, hi = 1e-3, float(max(H, W)) * 2
    best = None
    for _ in range(60):
        s = 0.5 * (lo + hi)
        m = _ellipse_union(H, W, cy, cx, ax, ay, th, s)
        c = int(m.sum())
        if best is None or abs(c - target) < abs(int(best.sum()) - target):
            best = m
        if abs(c - target) <= 0.1 * target:
            return m
        if c < target:
            lo = s
        else:
            hi = s
    if best is None or best.sum() == 0:  # degenerate tiny target: one pixel
        best = np.zeros((H, W), dtype=bool)
        best[int(cy[0]) % H, int(cx[0]) % W] = True
    return best


def pool_any(mask: np.ndarray, f: int) -> np.ndarray:
    """Place a full-resolution edit region on a coarser activation grid: a
    coarse pixel is edited when any of its f x f fine pixels is.  This only
    decides where the synthetic edit lands in a lower-resolution layer."""
    H, W = mask.shape
    assert H % f == 0 and W % f == 0
    return mask.reshape(H // f, f, W // f, f).any(axis=(1, 3))


# ---------------------------------------------------------------------------
# parameters
# ---------------------------------------------------------------------------

def kaiming_uniform(rng, c_out, k, c_in) -> np.ndarray:
    """U(-b, b) with b = sqrt(6 / fan_in), fan_in = C_in * k * k; KRSC layout."""
    bound = math.sqrt(6.0 / (c_in * k * k))
    return rng.uniform(-bound, bound, size=(c_out, k, k, c_in)).astype(np.float32)


def bias_uniform(rng, c_out) -> np.ndarray:
    return rng.uniform(-0.1, 0.1, size=(c_out,)).astype(np.float32)


def _to(a: np.ndarray, dtype: torch.dtype) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(a))
    return t.to(dtype) if t.dtype != dtype else t


@dataclass
class ConvLayer:
    """One synthetic conv layer: input activations (original / edited), the
    edit region at the input's resolution, and the layer parameters."""
    x_orig: torch.Tensor          # [N, H, W, C_in]
    x_edit: torch.Tensor          # [N, H, W, C_in]
    edit: np.ndarray              # bool [H, W] where x_edit was changed
    weight: torch.Tensor          # [C_out, k, k, C_in], same dtype as x
    bias: torch.Tensor            # [C_out] float32
    kernel: int = 3
    stride: int = 1
    pad: int = 1
    block: int = 4
    gn_gamma: torch.Tensor | None = None   # [C_in] float32
    gn_beta: torch.Tensor | None = None
    meta: dict = field(default_factory=dict)


def _edited_activation(rng, x: np.ndarray, edit: np.ndarray, mode: str, noise_std: float = 0.5):
    xe = x.copy()
    ys, xs = np.nonzero(edit)
    if mode == "add_noise":
        xe[:, ys, xs, :] += rng.normal(0.0, noise_std, size=(x.shape[0], len(ys), x.shape[3])).astype(np.float32)
    elif mode == "fresh":
        xe[:, ys, xs, :] = rng.normal(0.0, 1.0, size=(x.shape[0], len(ys), x.shape[3])).astype(np.float32)
    else:
        raise ValueError(mode)
    return xe


def make_conv_case(seed: int, H: int, W: int, c_in: int, c_out: int, *, dtype=torch.bfloat16,
                   kernel=3, stride=1, pad=1, block=4, edit=None, area=0.012,
                   mode="fresh", gn=False, N=1, all_edit=False) -> ConvLayer:
    """Generic layer: x_orig ~ N(0,1); x_edit differs from it inside ``edit``
    (a seeded blob mask of ``area`` when not given)."""
    rng = np.random.default_rng(seed)
    x = rng.normal(0.0, 1.0, size=(N, H, W, c_in)).astype(np.float32)
    if all_edit:
        edit = np.ones((H, W), dtype=bool)
    elif edit is None:
        edit = blob_mask(rng, H, W, area)
    xe = _edited_activation(rng, x, edit, mode)
    w = kaiming_uniform(rng, c_out, kernel, c_in)
    b = bias_uniform(rng, c_out)
    layer = ConvLayer(_to(x, dtype), _to(xe, dtype), edit, _to(w, dtype), _to(b, torch.float32),
                      kernel, stride, pad, block)
    if gn:
        layer.gn_gamma = _to((1.0 + 0.1 * rng.normal(size=c_in)).astype(np.float32), torch.float32)
        layer.gn_beta = _to((0.1 * rng.normal(size=c_in)).astype(np.float32), torch.float32)
    return layer


# ---------------------------------------------------------------------------
# the five workloads
# ---------------------------------------------------------------------------

def make_cfg1(seed: int = 0) -> ConvLayer:
    """Single 3x3 s1 p1 conv, fp32, N=1, C_in=C_out=64, 64x64 NHWC.  A_orig ~
    N(0,1); A_edit = A_orig + N(0, std 0.5) inside one rectangle of ~5% area
    (h ~ U{10..20}, w = round(205/h)).  Output block 4 (input block 6)."""
    rng = np.random.default_rng(seed)
    H = W = 64
    x = rng.normal(0.0, 1.0, size=(1, H, W, 64)).astype(np.float32)
    h = int(rng.integers(10, 21))
    w = int(round(205 / h))
    y0 = int(rng.integers(0, H - h + 1))
    x0 = int(rng.integers(0, W - w + 1))
    edit = np.zeros((H, W), dtype=bool)
    edit[y0:y0 + h, x0:x0 + w] = True
    xe = _edited_activation(rng, x, edit, "add_noise", 0.5)
    wt = kaiming_uniform(rng, 64, 3, 64)
    b = bias_uniform(rng, 64)
    return ConvLayer(torch.from_numpy(x), torch.from_numpy(xe), edit, torch.from_numpy(wt),
                     torch.from_numpy(b), 3, 1, 1, 4, meta={"threshold": 1e-3, "dilate": 1})


def make_cfg2(seed: int = 0, H: int = 256, W: int = 256, area: float = 0.012):
    """Two 3xHxW uint8 images (CHW); the edited one differs inside 1-3 seeded
    ellipses covering ~``area``: edited = (orig + U{1..255}) mod 256 on every
    channel there.  Returns (orig, edited, edit_region)."""
    rng = np.random.default_rng(seed)
    orig = rng.integers(0, 256, size=(1, 3, H, W), dtype=np.int64)
    edit = blob_mask(rng, H, W, area, 1, 3, ellipse=True)
    delta = rng.integers(1, 256, size=(1, 3, H, W), dtype=np.int64)
    edited = np.where(edit[None, None], (orig + delta) % 256, orig)
    return (torch.from_numpy(orig.astype(np.uint8)), torch.from_numpy(edited.astype(np.uint8)), edit)


CFG2_SCALES = ((256, 256, 8), (128, 128, 4), (64, 64, 4), (32, 32, 2))


@dataclass
class ResBlock:
    """DDPM-style residual block: GN(32)+SiLU -> conv1 -> GN(32)+SiLU -> conv2 + x."""
    x_orig: torch.Tensor
    x_edit: torch.Tensor
    edit: np.ndarray
    w1: torch.Tensor
    b1: torch.Tensor
    w2: torch.Tensor
    b2: torch.Tensor
    g1: torch.Tensor
    be1: torch.Tensor
    g2: torch.Tensor
    be2: torch.Tensor
    groups: int = 32
    eps: float = 1e-5
    block: int = 8


def make_cfg3(seed: int = 0, H: int = 256, W: int = 256, C: int = 128, area: float = 0.012,
              block: int = 8, all_edit: bool = False, edit=None) -> ResBlock:
    """x_orig ~ N(0,1) bf16 [1,H,W,C]; 1-3 seeded discs totalling ~``area``;
    inside them x_edit is a fresh N(0,1) draw.  GN gamma = 1 + 0.1 N(0,1),
    beta = 0.1 N(0,1); conv weights Kaiming-uniform, biases U(-0.1, 0.1)."""
    rng = np.random.default_rng(seed)
    x = rng.normal(0.0, 1.0, size=(1, H, W, C)).astype(np.float32)
    if all_edit:
        edit = np.ones((H, W), dtype=bool)
    elif edit is None:
        edit = blob_mask(rng, H, W, area, 1, 3, ellipse=False)
    xe = _edited_activation(rng, x, edit, "fresh")
    bf = torch.bfloat16
    w1 = kaiming_uniform(rng, C, 3, C)
    b1 = bias_uniform(rng, C)
    w2 = kaiming_uniform(rng, C, 3, C)
    b2 = bias_uniform(rng, C)
    g1 = (1.0 + 0.1 * rng.normal(size=C)).astype(np.float32)
    be1 = (0.1 * rng.normal(size=C)).astype(np.float32)
    g2 = (1.0 + 0.1 * rng.normal(size=C)).astype(np.float32)
    be2 = (0.1 * rng.normal(size=C)).astype(np.float32)
    return ResBlock(_to(x, bf), _to(xe, bf), edit, _to(w1, bf), _to(b1, torch.float32),
                    _to(w2, bf), _to(b2, torch.float32), _to(g1, torch.float32),
                    _to(be1, torch.float32), _to(g2, torch.float32), _to(be2, torch.float32),
                    32, 1e-5, block)


# Stable-Diffusion-latent-shaped convs: (H, W, C, block)
CFG4_LAYERS = ((64, 64, 320, 4), (32, 32, 640, 2), (16, 16, 1280, 1))
CFG4_AREAS = (0.005, 0.012, 0.05, 0.10, 0.20)


def make_cfg4_layer(seed: int, layer: int, area: float = 0.012, all_edit: bool = False) -> ConvLayer:
    """Masks are drawn at 64x64 (one rectangle plus discs totalling ``area``)
    and placed on the 32x32 / 16x16 grids with ``pool_any``."""
    H, W, C, b = CFG4_LAYERS[layer]
    rng = np.random.default_rng(seed)
    if all_edit:
        edit = np.ones((H, W), dtype=bool)
    else:
        m = rect_mask(rng, 64, 64, area / 2) | blob_mask(rng, 64, 64, area / 2, 1, 3, ellipse=False)
        edit = pool_any(m, 64 // H)
    return make_conv_case(seed + 1000 * (layer + 1), H, W, C, C, block=b, edit=edit)


# GauGAN-generator-shaped layers: (H_in, W_in, C_in, C_out, kernel, stride, block)
CFG5_LAYERS = (
    (8, 16, 1024, 1024, 3, 1, 1),
    (16, 32, 1024, 1024, 3, 1, 2),
    (32, 64, 1024, 512, 3, 1, 2),
    (64, 128, 512, 256, 3, 1, 4),
    (128, 256, 256, 128, 3, 1, 4),
    (256, 512, 128, 64, 3, 1, 8),
    (256, 512, 64, 64, 3, 2, 4),
    (64, 128, 512, 256, 1, 1, 4),
)
CFG5_AREAS = (0.005, 0.012, 0.05, 0.10, 0.20, 0.30)


def make_cfg5_layer(seed: int, layer: int, area: float = 0.012, all_edit: bool = False) -> ConvLayer:
    """Masks are drawn at 256x512 (rectangle plus blobs) and placed on each
    layer's input grid with ``pool_any``."""
    H, W, ci, co, k, s, b = CFG5_LAYERS[layer]
    rng = np.random.default_rng(seed)
    if all_edit:
        edit = np.ones((H, W), dtype=bool)
    else:
        m = rect_mask(rng, 256, 512, area / 2) | blob_mask(rng, 256, 512, area / 2, 1, 3, ellipse=True)
        edit = pool_any(m, 256 // H)
    return make_conv_case(seed + 1000 * (layer + 1), H, W, ci, co, kernel=k, stride=s,
                          pad=k // 2, block=b, edit=edit)


# ---------------------------------------------------------------------------
# GauGAN-style layers beside the plain convs
# ---------------------------------------------------------------------------

# decoder upsampling layers: (input H, W, C_in, C_out, output tile edge); a
# 3x3 transposed conv, stride 2, padding 1, output padding 1 doubles H and W
UPSAMPLE_LAYERS = (
    (32, 64, 512, 256, 4),
    (64, 128, 256, 128, 4),
)
# SPADE-modulated 3x3 convs: (H, W, C_in, C_out, tile edge)
SPADE_LAYERS = (
    (64, 128, 256, 256, 4),
    (128, 256, 128, 128, 8),
)


def make_upsample_layer(seed: int, layer: int, area: float = 0.012, all_edit: bool = False) -> ConvLayer:
    """Input at (H, W), output at (2H, 2W).  The edit is drawn at 256x512,
    placed on the output grid (``meta['edit_out']``) and on the input grid
    with ``pool_any``; x_edit differs from x_orig inside the input's edit."""
    H, W, ci, co, b = UPSAMPLE_LAYERS[layer]
    rng = np.random.default_rng(seed)
    if all_edit:
        out_edit = np.ones((2 * H, 2 * W), dtype=bool)
    else:
        m = rect_mask(rng, 256, 512, area / 2) | blob_mask(rng, 256, 512, area / 2, 1, 3, ellipse=True)
        out_edit = pool_any(m, 256 // (2 * H))
    in_edit = pool_any(out_edit, 2)
    L = make_conv_case(seed + 7000 * (layer + 1), H, W, ci, co, kernel=3, stride=2, pad=1, block=b, edit=in_edit)
    L.meta = {"output_padding": 1, "edit_out": out_edit}
    return L


def make_spade_layer(seed: int, layer: int, area: float = 0.012) -> ConvLayer:
    """A 3x3 conv whose input is modulated per pixel: ``meta`` holds the
    modulation maps gamma / beta of the original and of the edited image
    (N(0, 0.3^2), bf16, fresh values inside the edit, as an edited
    segmentation map changes them there)."""
    H, W, ci, co, b = SPADE_LAYERS[layer]
    rng = np.random.default_rng(seed + 9000 * (layer + 1))
    m = rect_mask(rng, 256, 512, area / 2) | blob_mask(rng, 256, 512, area / 2, 1, 3, ellipse=True)
    edit = pool_any(m, 256 // H)
    L = make_conv_case(seed + 8000 * (layer + 1), H, W, ci, co, kernel=3, stride=1, pad=1, block=b, edit=edit)
    maps = {}
    for name in ("gamma", "beta"):
        orig = rng.normal(0.0, 0.3, size=(1, H, W, ci)).astype(np.float32)
        ed = orig.copy()
        ys, xs = np.nonzero(edit)
        ed[:, ys, xs, :] = rng.normal(0.0, 0.3, size=(1, len(ys), ci)).astype(np.float32)
        maps[name + "_orig"] = _to(orig, torch.bfloat16)
        maps[name + "_edit"] = _to(ed, torch.bfloat16)
    L.meta = maps
    return L
