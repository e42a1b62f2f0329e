"""Pins for the oracle's other layer types (transposed conv, SPADE-style input),
never against the oracle itself.

mer.dev notes on SIGE, section 5 (limitations and scope: GauGAN-style
generators) and the GauGAN-shaped workload: besides plain and stride-2 3x3
convs a generator has learned upsampling (a transposed conv) and spatially
modulated normalisation (per-pixel gamma / beta from the segmentation map).

  * transposed conv: torch.nn.functional.conv_transpose2d in float64 (several
    kernel / stride / padding choices, with input transform, bias, residual);
  * SPADE input: instance normalisation (GroupNorm with one channel per group,
    statistics of the input itself), per-pixel modulation and the activation
    written with torch ops in float64, then torch conv2d;
  * tile masking for both: an empty list returns the cache bit for bit, every
    tile listed gives the dense layer, pixels outside the list keep the cache
    and pixels inside equal the dense layer of the edited input.
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

from helpers import bits, tile_cover


def _t(shape, seed, dtype=torch.float32, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g, dtype=torch.float64) * scale).to(dtype)


def _torch_tconv(x, w, bias, k, s, p, op, gn=None, silu=False, residual=None):
    X = x.double()
    if gn is not None:
        sc, sh = (torch.from_numpy(a) for a in gn)
        X = X * sc[:, None, None, :] + sh[:, None, None, :]
        if silu:
            X = F.silu(X)
        if x.dtype == torch.bfloat16:
            X = X.to(torch.bfloat16).double()
    y = F.conv_transpose2d(X.permute(0, 3, 1, 2), w.double().permute(3, 0, 1, 2),
                           None if bias is None else bias.double(), stride=s, padding=p, output_padding=op)
    y = y.permute(0, 2, 3, 1)
    if residual is not None:
        y = y + residual.double()
    return y.numpy()


@pytest.mark.parametrize("k,s,p,op", [(3, 2, 1, 1), (3, 2, 1, 0), (4, 2, 1, 0), (3, 1, 1, 0), (2, 2, 0, 0)])
def test_conv_transpose_equals_library(orc, k, s, p, op):
    x = _t((2, 5, 7, 8), 1)
    w = _t((6, k, k, 8), 2, scale=0.3)
    b = _t((6,), 3, scale=0.1)
    ref = _torch_tconv(x, w, b, k, s, p, op)
    got = orc.conv_transpose_f64(x, w, b, k, s, p, op)
    assert got.shape == ref.shape
    assert np.abs(got - ref).max() <= 1e-12 * max(1.0, np.abs(ref).max())


def test_conv_transpose_with_transform_residual_bf16(orc):
    x = _t((1, 6, 6, 16), 4, torch.bfloat16)
    w = _t((16, 3, 3, 16), 5, torch.bfloat16, 0.2)
    b = _t((16,), 6, scale=0.1)
    gn = orc.gn_affine(x, 4, _t((16,), 7) * 0.1 + 1.0, _t((16,), 8) * 0.1)
    Ho, Wo = orc.conv_transpose_out_hw(6, 6)
    res = _t((1, Ho, Wo, 16), 9, torch.bfloat16)
    ref = _torch_tconv(x, w, b, 3, 2, 1, 1, gn=gn, silu=True, residual=res)
    got = orc.conv_transpose_f64(x, w, b, gn=gn, silu=True, residual=res)
    assert np.abs(got - ref).max() <= 1e-10 * np.abs(ref).max()


def test_conv_transpose_one_input_pixel_places_the_kernel(orc):
    """A single nonzero input pixel spreads the kernel, flipped into place, onto
    the output at stride 2: out[2i - 1 + r][2j - 1 + c][o] = W[o][r][c][0] * v."""
    x = torch.zeros((1, 4, 4, 1), dtype=torch.float32)
    x[0, 2, 1, 0] = 2.0
    w = _t((3, 3, 3, 1), 10)
    z = orc.conv_transpose_f64(x, w, None)
    exp = np.zeros_like(z)
    for r in range(3):
        for c in range(3):
            exp[0, 2 * 2 - 1 + r, 2 * 1 - 1 + c, :] = 2.0 * w[:, r, c, 0].double().numpy()
    assert np.array_equal(z, exp)


def test_sparse_conv_transpose_invariants(orc):
    x0 = _t((1, 8, 8, 16), 11, torch.bfloat16)
    x1 = x0.clone()
    x1[0, 2:5, 3:6] = _t((3, 3, 16), 12, torch.bfloat16)
    w = _t((8, 3, 3, 16), 13, torch.bfloat16, 0.2)
    b = _t((8,), 14, scale=0.1)
    Ho, Wo = orc.conv_transpose_out_hw(8, 8)
    cache = _t((1, Ho, Wo, 8), 15, torch.bfloat16)
    blk = 4
    empty = np.zeros((0, 2), np.int32)
    assert torch.equal(bits(orc.sparse_conv_transpose(x1, w, b, empty, cache, block=blk)), bits(cache))
    every = np.array([(h, v) for h in range(0, Ho, blk) for v in range(0, Wo, blk)], np.int32)
    dense = orc.round_bf16(orc.conv_transpose_f64(x1, w, b))
    full = orc.sparse_conv_transpose(x1, w, b, every, cache, block=blk)
    assert np.array_equal(full.view(torch.int16).numpy().view(np.uint16), dense)
    some = np.array([(0, 4), (4, 8), (12, 0)], np.int32)
    y = orc.sparse_conv_transpose(x1, w, b, some, cache, block=blk)
    cov = tile_cover(some, blk, 1, Ho, Wo, 8)
    assert torch.equal(bits(y[~cov]), bits(cache[~cov]))
    assert np.array_equal(y.view(torch.int16).numpy().view(np.uint16)[cov.numpy()], dense[cov.numpy()])


def _torch_spade_conv(x, w, bias, gamma, beta, act, eps=1e-5):
    X = x.double().permute(0, 3, 1, 2)
    Xn = F.instance_norm(X, eps=eps)
    t = Xn * (1.0 + gamma.double().permute(0, 3, 1, 2)) + beta.double().permute(0, 3, 1, 2)
    t = {0: lambda v: v, 1: F.silu, 2: lambda v: F.leaky_relu(v, 0.2)}[act](t)
    y = F.conv2d(t, w.double().permute(0, 3, 1, 2), bias.double(), padding=1)
    return y.permute(0, 2, 3, 1).numpy()


@pytest.mark.parametrize("act", [0, 1, 2])
def test_spade_conv_equals_library(orc, act):
    """Instance norm = GroupNorm with one channel per group, statistics of x."""
    x = _t((2, 6, 5, 8), 20)
    w = _t((4, 3, 3, 8), 21, scale=0.3)
    b = _t((4,), 22, scale=0.1)
    gamma = _t((2, 6, 5, 8), 23, scale=0.3)
    beta = _t((2, 6, 5, 8), 24, scale=0.3)
    norm = orc.gn_affine(x, 8, torch.ones(8), torch.zeros(8))
    got = orc.spade_conv(x, w, b, norm, gamma, beta, act=act, rounded=False)
    ref = _torch_spade_conv(x, w, b, gamma, beta, act)
    assert np.abs(got - ref).max() <= 1e-9 * np.abs(ref).max()


def test_spade_conv_negative_slope_and_zero_modulation(orc):
    """gamma = beta = 0 reduces SPADE to the plain normalised input; the leaky
    branch scales negative inputs by 0.2 exactly."""
    x = _t((1, 4, 4, 8), 25)
    w = _t((3, 3, 3, 8), 26, scale=0.3)
    b = torch.zeros(3)
    zero = torch.zeros_like(x)
    norm = orc.gn_affine(x, 8, torch.ones(8), torch.zeros(8))
    plain = orc.dense_conv_f64(x, w, b, gn=norm)
    assert np.abs(orc.spade_conv(x, w, b, norm, zero, zero, act=0, rounded=False) - plain).max() <= 1e-12
    neg = -torch.ones_like(x)                       # (1 + gamma) = 0: the input is beta
    beta = -torch.full_like(x, 2.5)
    z = orc.spade_conv(x, w, b, norm, neg, beta, act=2, rounded=False)
    const = torch.full_like(x, -0.5)                # LeakyReLU(-2.5) = -0.5
    assert np.abs(z - orc.dense_conv_f64(const, w, b)).max() <= 1e-12


def test_spade_sparse_invariants(orc):
    x0 = _t((1, 8, 8, 16), 30, torch.bfloat16)
    x1 = x0.clone()
    x1[0, 1:3, 5:7] = _t((2, 2, 16), 31, torch.bfloat16)
    w = _t((8, 3, 3, 16), 32, torch.bfloat16, 0.2)
    b = _t((8,), 33, scale=0.1)
    gamma = _t((1, 8, 8, 16), 34, torch.bfloat16, 0.3)
    beta = _t((1, 8, 8, 16), 35, torch.bfloat16, 0.3)
    norm = orc.gn_affine(x0, 16, torch.ones(16), torch.zeros(16))
    cache = _t((1, 8, 8, 8), 36, torch.bfloat16)
    blk = 4
    y = orc.spade_conv(x1, w, b, norm, gamma, beta, idx=np.zeros((0, 2), np.int32), block=blk, y_cached=cache)
    assert torch.equal(bits(y), bits(cache))
    dense = orc.spade_conv(x1, w, b, norm, gamma, beta)
    some = np.array([(0, 4)], np.int32)
    y = orc.spade_conv(x1, w, b, norm, gamma, beta, idx=some, block=blk, y_cached=cache)
    cov = tile_cover(some, blk, 1, 8, 8, 8)
    assert torch.equal(bits(y[~cov]), bits(cache[~cov]))
    assert torch.equal(bits(y[cov]), bits(dense[cov]))
