"""The fused residual block (sige_resblock_fused) against the oracle.

SIGE project page, "Overview": the layers run on the gathered active blocks
one after the other, each scattering into its cached output; the oracle's
``resblock_sparse`` writes that chain out (conv1 into the cached y1 on the
listed tiles, then conv2 on the updated y1 into the cached out).  The fused
call recomputes y1 on a one-pixel ring around each tile instead of reading
it back, which gives the same values whenever the list covers the edit's
one-pixel neighbourhood (a one-tile dilation does).

Checked through the C ABI, on the same seeded inputs as the oracle:
  * the tile list bit for bit;
  * y1 and out element by element within max(2e-2 RMS, one bf16 ulp) of the
    oracle's rounded values, out also within plain 2e-2 RMS of the oracle's
    unrounded float64 conv2 at the tiles;
  * every byte of y1 and out outside the listed tiles untouched;
  * against the unfused GPU chain (two sige_conv_fused calls);
  * edge cases: an empty list writes nothing, every tile listed gives the
    dense block of the edited input, maps that 8x8 tiles do not divide,
    batch 2 (one list for both items).
"""
import numpy as np
import pytest
import torch

import spatially_sparse_incremental_b200 as sige
from spatially_sparse_incremental_b200 import inputs
from helpers import assert_close, bits, rel_err, tile_cover

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _caches(blk, xo):
    """GPU caches of the original input: GroupNorm affines and the dense y1 / out."""
    C = xo.shape[3]
    cd = sige.conv_desc(3, 1, 1, C, C, blk.block)
    w1, w2, b1, b2 = blk.w1.to(DEV), blk.w2.to(DEV), blk.b1.to(DEV), blk.b2.to(DEV)
    gn1 = sige.sige_groupnorm_affine(xo, 32, blk.g1.to(DEV), blk.be1.to(DEV))
    y1 = sige.sige_dense_conv(xo, w1, b1, cd, gn_scale=gn1[0], gn_shift=gn1[1], silu=True)
    gn2 = sige.sige_groupnorm_affine(y1, 32, blk.g2.to(DEV), blk.be2.to(DEV))
    out = sige.sige_dense_conv(y1, w2, b2, cd, gn_scale=gn2[0], gn_shift=gn2[1], silu=True, residual=xo)
    return cd, (w1, b1, w2, b2), gn1, gn2, y1, out


def _fused(blk, xo, xe, idx, cnt, cap):
    cd, (w1, b1, w2, b2), gn1, gn2, y1c, outc = _caches(blk, xo)
    y1, out = y1c.clone(), outc.clone()
    sige.sige_resblock_fused(xe, w1, b1, gn1, w2, b2, gn2, idx, cnt, cap, y1, out)
    torch.cuda.synchronize()
    return y1, out, y1c, outc


def _oracle_chain(orc, blk, x_orig, x_edit, ref_idx):
    g1 = orc.gn_affine(x_orig, 32, blk.g1, blk.be1)
    oy1 = orc.dense_conv(x_orig, blk.w1, blk.b1, gn=g1, silu=True)
    g2 = orc.gn_affine(oy1, 32, blk.g2, blk.be2)
    oy1, oout = orc.resblock_dense(x_orig, blk, g1, g2)
    ry1, rout = orc.resblock_sparse(x_edit, blk, ref_idx, oy1, oout, g1, g2)
    return g2, ry1, rout


def _check(orc, blk, x_orig, x_edit, ref_idx, y1, out, y1c, outc):
    H, W = x_orig.shape[1:3]
    N, C = x_orig.shape[0], x_orig.shape[3]
    g2, ry1, rout = _oracle_chain(orc, blk, x_orig, x_edit, ref_idx)
    assert_close(y1.cpu(), ry1, torch.bfloat16, what="fused y1")
    assert_close(out.cpu(), rout, torch.bfloat16, what="fused out")
    cov = tile_cover(ref_idx, blk.block, N, H, W, C)
    assert torch.equal(bits(y1.cpu()[~cov]), bits(y1c.cpu()[~cov])), "y1 changed outside the tiles"
    assert torch.equal(bits(out.cpu()[~cov]), bits(outc.cpu()[~cov])), "out changed outside the tiles"
    if cov.any():
        # conv2 at the tiles against the oracle's unrounded float64 value
        r64 = torch.from_numpy(orc.dense_conv_f64(ry1, blk.w2, blk.b2, gn=g2, silu=True, residual=x_edit))
        e = rel_err(out.cpu(), r64, cov)
        assert e <= 2e-2, f"fused out vs unrounded oracle: max|d|/rms = {e:.3g}"


@pytest.mark.parametrize("H,W,area,seed", [(64, 64, 0.05, 40), (256, 256, 0.012, 40), (256, 256, 0.20, 41),
                                           (68, 60, 0.08, 3)])
def test_fused_resblock_vs_oracle(orc, H, W, area, seed):
    blk = inputs.make_cfg3(seed, H=H, W=W, area=area)
    b = blk.block
    cap = -(-H // b) * -(-W // b)
    xo, xe = blk.x_orig.to(DEV), blk.x_edit.to(DEV)
    idx, cnt, _ = sige.sige_reduce_mask(xo, xe, 1e-3, [(H, W, b, cap)], 1)
    y1, out, y1c, outc = _fused(blk, xo, xe, idx, cnt, cap)
    n = int(cnt[0].item())
    ref_idx = orc.reduce_mask(blk.x_orig, blk.x_edit, 1e-3, [(H, W, b)], 1)[0]
    assert np.array_equal(idx[:n].cpu().numpy(), ref_idx)
    assert n > 0
    _check(orc, blk, blk.x_orig, blk.x_edit, ref_idx, y1, out, y1c, outc)


def test_fused_resblock_equals_the_unfused_chain():
    """The fused call and two sige_conv_fused calls on the same list agree
    element by element (the bf16 float bar: the unfused conv may split its K
    loop over a CTA pair, which sums in another order)."""
    blk = inputs.make_cfg3(12, H=128, W=128, area=0.03)
    b, H = blk.block, 128
    cap = (H // b) ** 2
    xo, xe = blk.x_orig.to(DEV), blk.x_edit.to(DEV)
    idx, cnt, _ = sige.sige_reduce_mask(xo, xe, 1e-3, [(H, H, b, cap)], 1)
    y1, out, y1c, outc = _fused(blk, xo, xe, idx, cnt, cap)
    cd, (w1, b1, w2, b2), gn1, gn2, _, _ = _caches(blk, xo)
    uy1, uout = y1c.clone(), outc.clone()
    sige.sige_conv_fused(xe, w1, b1, cd, idx, cnt, cap, uy1, gn1[0], gn1[1], silu=True)
    sige.sige_conv_fused(uy1, w2, b2, cd, idx, cnt, cap, uout, gn2[0], gn2[1], silu=True, residual=xe)
    torch.cuda.synchronize()
    assert_close(y1.cpu(), uy1.cpu(), torch.bfloat16, what="fused vs unfused y1")
    assert_close(out.cpu(), uout.cpu(), torch.bfloat16, what="fused vs unfused out")


def test_fused_resblock_empty_list_writes_nothing():
    blk = inputs.make_cfg3(5, H=64, W=64, area=0.05)
    xo, xe = blk.x_orig.to(DEV), blk.x_edit.to(DEV)
    idx = torch.zeros((64, 2), dtype=torch.int32, device=DEV)
    cnt = torch.zeros(1, dtype=torch.int32, device=DEV)
    y1, out, y1c, outc = _fused(blk, xo, xe, idx, cnt, 64)
    assert torch.equal(bits(y1.cpu()), bits(y1c.cpu())) and torch.equal(bits(out.cpu()), bits(outc.cpu()))


def test_fused_resblock_every_tile_is_the_dense_block(orc):
    blk = inputs.make_cfg3(6, H=64, W=64, area=0.05)
    b, H = blk.block, 64
    every = np.array([(h, w) for h in range(0, H, b) for w in range(0, H, b)], dtype=np.int32)
    idx = torch.from_numpy(every).to(DEV)
    cnt = torch.tensor([len(every)], dtype=torch.int32, device=DEV)
    xo, xe = blk.x_orig.to(DEV), blk.x_edit.to(DEV)
    y1, out, _, _ = _fused(blk, xo, xe, idx, cnt, len(every))
    # GroupNorm statistics stay those of the original; the convs see x_edit everywhere
    g1 = orc.gn_affine(blk.x_orig, 32, blk.g1, blk.be1)
    oy1 = orc.dense_conv(blk.x_orig, blk.w1, blk.b1, gn=g1, silu=True)
    g2 = orc.gn_affine(oy1, 32, blk.g2, blk.be2)
    dy1, dout = orc.resblock_dense(blk.x_edit, blk, g1, g2)
    assert_close(y1.cpu(), dy1, torch.bfloat16, what="all-tile y1")
    assert_close(out.cpu(), dout, torch.bfloat16, what="all-tile out")


def test_fused_resblock_batch_of_two(orc):
    """Two images share one list (the mask is OR-ed over the batch); each has
    its own GroupNorm statistics."""
    a = inputs.make_cfg3(50, H=64, W=64, area=0.04)
    c = inputs.make_cfg3(51, H=64, W=64, area=0.04)
    x_orig = torch.cat([a.x_orig, c.x_orig])
    x_edit = torch.cat([a.x_edit, c.x_edit])
    b, H = a.block, 64
    cap = (H // b) ** 2
    xo, xe = x_orig.to(DEV), x_edit.to(DEV)
    idx, cnt, _ = sige.sige_reduce_mask(xo, xe, 1e-3, [(H, H, b, cap)], 1)
    y1, out, y1c, outc = _fused(a, xo, xe, idx, cnt, cap)
    n = int(cnt[0].item())
    ref_idx = orc.reduce_mask(x_orig, x_edit, 1e-3, [(H, H, b)], 1)[0]
    assert np.array_equal(idx[:n].cpu().numpy(), ref_idx)
    _check(orc, a, x_orig, x_edit, ref_idx, y1, out, y1c, outc)


def test_fused_resblock_argument_checks():
    blk = inputs.make_cfg3(1, H=32, W=32, C=64, area=0.05)
    x = blk.x_orig.to(DEV)
    w = torch.zeros((64, 3, 3, 64), dtype=torch.bfloat16, device=DEV)
    g = (torch.ones((1, 64), device=DEV), torch.zeros((1, 64), device=DEV))
    idx = torch.zeros((16, 2), dtype=torch.int32, device=DEV)
    cnt = torch.zeros(1, dtype=torch.int32, device=DEV)
    with pytest.raises(sige.SigeError) as ei:         # 64 channels: not this kernel's shape
        sige.sige_resblock_fused(x, w, None, g, w, None, g, idx, cnt, 16, x.clone(), x.clone())
    assert ei.value.status == sige.ERR_UNSUPPORTED


# ------------------------------------------------------------------ one-launch step

def _step(blk, xo, xe, cap, ws=None, thr=1e-3):
    cd, (w1, b1, w2, b2), gn1, gn2, y1c, outc = _caches(blk, xo)
    y1, out = y1c.clone(), outc.clone()
    if ws is None:
        ws = sige.zeros_workspace(sige.sige_resblock_step_workspace_bytes(xe), DEV)
    idx, cnt = sige.sige_resblock_step(xo, xe, thr, w1, b1, gn1, w2, b2, gn2, y1, out, cap, workspace=ws)
    torch.cuda.synchronize()
    return idx, cnt, ws, y1, out, y1c, outc


@pytest.mark.parametrize("H,W,area,seed,N", [(64, 64, 0.05, 40, 1), (256, 256, 0.012, 40, 1),
                                             (256, 256, 0.20, 41, 1), (68, 60, 0.08, 3, 1), (64, 64, 0.04, 50, 2)])
def test_step_vs_oracle(orc, H, W, area, seed, N):
    blk = inputs.make_cfg3(seed, H=H, W=W, area=area)
    x_orig, x_edit = blk.x_orig, blk.x_edit
    if N == 2:
        c = inputs.make_cfg3(seed + 1, H=H, W=W, area=area)
        x_orig, x_edit = torch.cat([x_orig, c.x_orig]), torch.cat([x_edit, c.x_edit])
    b = blk.block
    cap = -(-H // b) * -(-W // b)
    xo, xe = x_orig.to(DEV), x_edit.to(DEV)
    idx, cnt, ws, y1, out, y1c, outc = _step(blk, xo, xe, cap)
    n = int(cnt[0].item())
    ref_idx = orc.reduce_mask(x_orig, x_edit, 1e-3, [(H, W, b)], 1)[0]
    assert n == len(ref_idx) and np.array_equal(idx[:n].cpu().numpy(), ref_idx)
    midx, mcnt, _ = sige.sige_reduce_mask(xo, xe, 1e-3, [(H, W, b, cap)], 1)
    assert int(mcnt[0].item()) == n and torch.equal(midx[:n].cpu(), idx[:n].cpu())
    assert sige.sige_get_device_error(ws) == sige.OK
    _check(orc, blk, x_orig, x_edit, ref_idx, y1, out, y1c, outc)


def test_step_twice_on_one_workspace(orc):
    """The second call finds the workspace as the first left it (zero) and
    gives its own edit's list and outputs."""
    a = inputs.make_cfg3(60, H=128, W=128, area=0.02)
    c = inputs.make_cfg3(61, H=128, W=128, area=0.05)
    cap = 256
    ws = sige.zeros_workspace(sige.sige_resblock_step_workspace_bytes(a.x_orig), DEV)
    for blk in (a, c, a):
        xo, xe = blk.x_orig.to(DEV), blk.x_edit.to(DEV)
        idx, cnt, _, y1, out, y1c, outc = _step(blk, xo, xe, cap, ws=ws)
        n = int(cnt[0].item())
        ref_idx = orc.reduce_mask(blk.x_orig, blk.x_edit, 1e-3, [(128, 128, 8)], 1)[0]
        assert np.array_equal(idx[:n].cpu().numpy(), ref_idx)
        _check(orc, blk, blk.x_orig, blk.x_edit, ref_idx, y1, out, y1c, outc)
    assert sige.sige_get_device_error(ws) == sige.OK


def test_step_capacity_overflow_truncates_and_reports(orc):
    """More active tiles than the capacity: the first `capacity` tiles of the
    row-major list are listed and processed, the full count and
    SIGE_ERR_CAPACITY are reported, and nothing outside those tiles changes.
    (Their values are not compared with the chain on the truncated list: the
    ring of y1 next to an unprocessed edited tile is recomputed from the edited
    input, which that chain would have read from the stale cache.)"""
    blk = inputs.make_cfg3(62, H=64, W=64, area=0.08)
    xo, xe = blk.x_orig.to(DEV), blk.x_edit.to(DEV)
    ref_idx = orc.reduce_mask(blk.x_orig, blk.x_edit, 1e-3, [(64, 64, 8)], 1)[0]
    cap = len(ref_idx) // 2
    assert cap >= 1
    idx, cnt, ws, y1, out, y1c, outc = _step(blk, xo, xe, cap)
    assert int(cnt[0].item()) == len(ref_idx)
    assert np.array_equal(idx[:cap].cpu().numpy(), ref_idx[:cap])
    assert sige.sige_get_device_error(ws) == sige.ERR_CAPACITY
    cov = tile_cover(ref_idx[:cap], 8, 1, 64, 64, 128)
    assert torch.equal(bits(y1.cpu()[~cov]), bits(y1c.cpu()[~cov]))
    assert torch.equal(bits(out.cpu()[~cov]), bits(outc.cpu()[~cov]))
    assert not torch.equal(bits(out.cpu()[cov]), bits(outc.cpu()[cov]))   # the listed tiles were rewritten


def test_step_without_an_edit_writes_nothing():
    blk = inputs.make_cfg3(63, H=64, W=64, area=0.05)
    xo = blk.x_orig.to(DEV)
    idx, cnt, ws, y1, out, y1c, outc = _step(blk, xo, xo.clone(), 64)
    assert int(cnt[0].item()) == 0
    assert torch.equal(bits(y1.cpu()), bits(y1c.cpu())) and torch.equal(bits(out.cpu()), bits(outc.cpu()))


def test_step_grid_barrier_timeout_reports_and_the_next_call_is_exact(orc):
    """The failure path of the one-launch step, the allowed way: a wait bound of
    a few cycles makes the grid barrier give up (nothing faults, nothing
    hangs).  The call returns, records SIGE_ERR_TIMEOUT with the barrier's
    wait site (its outputs are then unspecified: the last CTA to arrive still
    sees the barrier complete), and the next call with the default bound, on
    the same workspace, is exact."""
    blk = inputs.make_cfg3(64, H=64, W=64, area=0.05)
    xo, xe = blk.x_orig.to(DEV), blk.x_edit.to(DEV)
    ws = sige.zeros_workspace(sige.sige_resblock_step_workspace_bytes(xe), DEV)
    sige.sige_set_wait_cycles(16)
    try:
        idx, cnt, _, y1, out, y1c, outc = _step(blk, xo, xe, 64, ws=ws)
    finally:
        sige.sige_set_wait_cycles(0)
    detail = int(ws[4:8].cpu().view(torch.int32)[0].item())
    assert sige.sige_get_device_error(ws) == sige.ERR_TIMEOUT
    assert detail == 111                                     # the grid barrier
    idx, cnt, _, y1, out, y1c, outc = _step(blk, xo, xe, 64, ws=ws)
    n = int(cnt[0].item())
    ref_idx = orc.reduce_mask(blk.x_orig, blk.x_edit, 1e-3, [(64, 64, 8)], 1)[0]
    assert n == len(ref_idx) and np.array_equal(idx[:n].cpu().numpy(), ref_idx)
    assert sige.sige_get_device_error(ws) == sige.OK
    _check(orc, blk, blk.x_orig, blk.x_edit, ref_idx, y1, out, y1c, outc)
