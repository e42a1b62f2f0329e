"""GauGAN-style layers on the GPU against the oracle: the transposed conv
(learned upsampling) and the SPADE-style spatially modulated input.

mer.dev notes on SIGE, section 5: the engine serves GauGAN's generator as
well as diffusion UNets; a generator's decoder upsamples and modulates its
normalised activations per pixel.  Both layers run through
sige_conv_fused_ext on the tensor cores:
  * transposed conv (3x3, stride 2, padding 1, output padding 1) on the tiles
    of the output grid, against ``oracle.sparse_conv_transpose`` with the same
    list; the dense form (no list) against ``oracle.conv_transpose_f64``;
  * SPADE input act((x * s + h) * (1 + gamma) + beta) with LeakyReLU(0.2) or
    SiLU, normalisation statistics of the original (instance norm), against
    ``oracle.spade_conv``;
  * bf16 bar per element (max(2e-2 RMS, one bf16 ulp) of the rounded oracle),
    max(2e-2 RMS, half an ulp) against the unrounded value, every byte outside the tiles
    untouched, an every-tile list equal to the dense layer.
"""
import numpy as np
import pytest
import torch

import spatially_sparse_incremental_b200 as sige
from spatially_sparse_incremental_b200 import inputs
from helpers import assert_close, assert_close_unrounded, bits, rel_err, tile_cover

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _dev_list(idx, cap):
    buf = torch.zeros((max(cap, 1), 2), dtype=torch.int32)
    buf[:len(idx)] = torch.from_numpy(np.asarray(idx, np.int32).reshape(-1, 2))
    return buf.to(DEV), torch.tensor([len(idx)], dtype=torch.int32, device=DEV)


@pytest.mark.parametrize("layer", [0, 1])
def test_transposed_conv_sparse_vs_oracle(orc, layer):
    L = inputs.make_upsample_layer(3, layer, area=0.03)
    op, b = L.meta["output_padding"], L.block
    N, H, W, ci = L.x_orig.shape
    co = L.weight.shape[0]
    cd = sige.conv_desc(3, 2, 1, ci, co, b)
    Ho, Wo = orc.conv_transpose_out_hw(H, W)
    xo, xe, w, bias = L.x_orig.to(DEV), L.x_edit.to(DEV), L.weight.to(DEV), L.bias.to(DEV)
    # the cache: the dense layer of the original (no list)
    y = sige.sige_conv_fused_ext(xo, w, bias, cd, transposed=True, output_padding=op)
    torch.cuda.synchronize()
    dense_ref = orc.conv_transpose_f64(L.x_orig, L.weight, L.bias)
    assert_close_unrounded(y.cpu(), dense_ref, what="dense transposed conv vs unrounded")
    cache = y.clone()
    # tiles at the output resolution, from the output-resolution edit
    idx = orc.reduce_scale(L.meta["edit_out"].astype(np.uint8), Ho, Wo, b, 1)
    cap = -(-Ho // b) * -(-Wo // b)
    di, dc = _dev_list(idx, cap)
    sige.sige_conv_fused_ext(xe, w, bias, cd, y=y, idx=di, count=dc, capacity=cap, transposed=True,
                             output_padding=op)
    torch.cuda.synchronize()
    ref = orc.sparse_conv_transpose(L.x_edit, L.weight, L.bias, idx, cache.cpu(), block=b)
    assert_close(y.cpu(), ref, torch.bfloat16, what="transposed conv")
    cov = tile_cover(idx, b, N, Ho, Wo, co)
    assert torch.equal(bits(y.cpu()[~cov]), bits(cache.cpu()[~cov]))
    r64 = orc.conv_transpose_f64(L.x_edit, L.weight, L.bias)
    assert_close_unrounded(y.cpu(), r64, cov, what="sparse transposed conv vs unrounded")


def test_transposed_conv_with_groupnorm_silu_residual(orc):
    L = inputs.make_upsample_layer(5, 1, area=0.05)
    N, H, W, ci = L.x_orig.shape
    co = L.weight.shape[0]
    b = L.block
    cd = sige.conv_desc(3, 2, 1, ci, co, b)
    Ho, Wo = orc.conv_transpose_out_hw(H, W)
    gamma = torch.linspace(0.8, 1.2, ci)
    beta = torch.linspace(-0.1, 0.1, ci)
    gs, gh = sige.sige_groupnorm_affine(L.x_orig.to(DEV), 32, gamma.to(DEV), beta.to(DEV))
    res = torch.randn((N, Ho, Wo, co), generator=torch.Generator().manual_seed(1)).to(torch.bfloat16)
    y = sige.sige_conv_fused_ext(L.x_edit.to(DEV), L.weight.to(DEV), L.bias.to(DEV), cd, gn_scale=gs, gn_shift=gh,
                                 act=sige.ACT_SILU, transposed=True, output_padding=1, residual=res.to(DEV))
    torch.cuda.synchronize()
    gn = orc.gn_affine(L.x_orig, 32, gamma, beta)
    every = np.array([(h, v) for h in range(0, Ho, b) for v in range(0, Wo, b)], np.int32)
    ref = orc.sparse_conv_transpose(L.x_edit, L.weight, L.bias, every, torch.zeros((N, Ho, Wo, co),
                                    dtype=torch.bfloat16), block=b, gn=gn, silu=True, residual=res)
    assert_close(y.cpu(), ref, torch.bfloat16, what="dense transposed conv with GN+SiLU+residual")


@pytest.mark.parametrize("layer,act", [(0, 2), (1, 2), (0, 1)])
def test_spade_conv_sparse_vs_oracle(orc, layer, act):
    L = inputs.make_spade_layer(4, layer, area=0.03)
    N, H, W, ci = L.x_orig.shape
    co, b = L.weight.shape[0], L.block
    cd = sige.conv_desc(3, 1, 1, ci, co, b)
    m = L.meta
    xo, xe, w, bias = L.x_orig.to(DEV), L.x_edit.to(DEV), L.weight.to(DEV), L.bias.to(DEV)
    # normalisation statistics of the original: instance norm = one channel per group
    ones, zeros = torch.ones(ci), torch.zeros(ci)
    ns, nh = sige.sige_groupnorm_affine(xo, ci, ones.to(DEV), zeros.to(DEV))
    go, bo = m["gamma_orig"].to(DEV), m["beta_orig"].to(DEV)
    ge, be = m["gamma_edit"].to(DEV), m["beta_edit"].to(DEV)
    y = sige.sige_conv_fused_ext(xo, w, bias, cd, gn_scale=ns, gn_shift=nh, spade_gamma=go, spade_beta=bo, act=act)
    torch.cuda.synchronize()
    cache = y.clone()
    norm = orc.gn_affine(L.x_orig, ci, ones, zeros)
    assert_close(cache.cpu(), orc.spade_conv(L.x_orig, L.weight, L.bias, norm, m["gamma_orig"], m["beta_orig"],
                                             act=act), torch.bfloat16, what="dense SPADE conv")
    cap = -(-H // b) * -(-W // b)
    idx = orc.reduce_mask(L.x_orig, L.x_edit, 1e-3, [(H, W, b)], 1)[0]
    di, dc = _dev_list(idx, cap)
    sige.sige_conv_fused_ext(xe, w, bias, cd, y=y, idx=di, count=dc, capacity=cap, gn_scale=ns, gn_shift=nh,
                             spade_gamma=ge, spade_beta=be, act=act)
    torch.cuda.synchronize()
    ref = orc.spade_conv(L.x_edit, L.weight, L.bias, norm, m["gamma_edit"], m["beta_edit"], act=act, idx=idx,
                         block=b, y_cached=cache.cpu())
    assert_close(y.cpu(), ref, torch.bfloat16, what="sparse SPADE conv")
    cov = tile_cover(idx, b, N, H, W, co)
    assert torch.equal(bits(y.cpu()[~cov]), bits(cache.cpu()[~cov]))
    r64 = orc.spade_conv(L.x_edit, L.weight, L.bias, norm, m["gamma_edit"], m["beta_edit"], act=act, rounded=False)
    assert_close_unrounded(y.cpu(), r64, cov, what="sparse SPADE conv vs unrounded")


def test_ext_layer_checks():
    x = torch.zeros((1, 8, 8, 64), dtype=torch.bfloat16, device=DEV)
    w = torch.zeros((64, 3, 3, 64), dtype=torch.bfloat16, device=DEV)
    cd = sige.conv_desc(3, 2, 1, 64, 64, 4)
    with pytest.raises(sige.SigeError) as ei:           # output padding must stay below the stride
        sige.sige_conv_fused_ext(x, w, None, cd, transposed=True, output_padding=2)
    assert ei.value.status == sige.ERR_INVALID_ARG
    xf = torch.zeros((1, 8, 8, 64), dtype=torch.float32, device=DEV)
    with pytest.raises(sige.SigeError) as ei:           # bf16 only
        sige.sige_conv_fused_ext(xf, w.float(), None, cd, transposed=True, output_padding=1)
    assert ei.value.status == sige.ERR_UNSUPPORTED
