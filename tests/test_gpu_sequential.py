"""Sequential edits through the GPU path: tile restore and a second edit on top
of a first one (SIGE project page, "Overview": the cached F_l(A_original) is
updated in place, so an edit session restores the previous edit's tiles before
applying the next)."""
import numpy as np
import pytest
import torch

import spatially_sparse_incremental_b200 as sige
from spatially_sparse_incremental_b200 import inputs

from helpers import bits

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("dtype,C,N,H,W,b", [
    (torch.bfloat16, 128, 1, 64, 64, 8), (torch.float32, 64, 2, 30, 26, 4),
    (torch.uint8, 3, 1, 33, 35, 4), (torch.bfloat16, 20, 2, 17, 19, 2)])
def test_restore_tiles_vs_oracle(orc, dtype, C, N, H, W, b):
    g = torch.Generator().manual_seed(C * 7 + H)
    if dtype == torch.uint8:
        src = torch.randint(0, 256, (N, H, W, C), generator=g, dtype=torch.uint8)
        dst = torch.randint(0, 256, (N, H, W, C), generator=g, dtype=torch.uint8)
    else:
        src = torch.randn((N, H, W, C), generator=g).to(dtype)
        dst = torch.randn((N, H, W, C), generator=g).to(dtype)
    th, tw = -(-H // b), -(-W // b)
    rng = np.random.default_rng(C + W)
    tiles = np.array([(i * b, j * b) for i in range(th) for j in range(tw) if rng.random() < 0.3], np.int32)
    cap = th * tw
    idx = torch.zeros((cap, 2), dtype=torch.int32)
    idx[:len(tiles)] = torch.from_numpy(tiles.reshape(-1, 2))
    # count below capacity: only the first n pairs count (garbage pairs after them must be ignored)
    idx[len(tiles):] = 0
    cnt = torch.tensor([len(tiles)], dtype=torch.int32)
    want = orc.restore_tiles(src, dst, b, tiles)
    d = dst.to(DEV)
    sige.sige_restore_tiles(src.to(DEV), d, b, idx.to(DEV), cnt.to(DEV), cap)
    torch.cuda.synchronize()
    assert torch.equal(bits(d.cpu()), bits(want))


@pytest.mark.parametrize("dtype,C,N,H,W,b,frac,over", [
    (torch.bfloat16, 128, 1, 64, 64, 8, 0.3, False), (torch.float32, 64, 2, 30, 26, 4, 0.3, False),
    (torch.uint8, 16, 1, 33, 35, 4, 0.5, False), (torch.bfloat16, 8, 2, 17, 19, 2, 0.2, True),
    (torch.bfloat16, 64, 1, 16, 16, 8, 0.0, False)])
def test_download_tiles_vs_oracle(orc, dtype, C, N, H, W, b, frac, over):
    """The listed tiles of a device tensor into a host copy (the incremental
    read-back): the host tensor must equal the oracle's tile restore from the
    device values, byte for byte; ragged edge tiles, batch 2, an empty list,
    and a count above the capacity (only the first capacity pairs count)."""
    g = torch.Generator().manual_seed(C * 11 + W)
    if dtype == torch.uint8:
        y = torch.randint(0, 256, (N, H, W, C), generator=g, dtype=torch.uint8)
        host = torch.randint(0, 256, (N, H, W, C), generator=g, dtype=torch.uint8)
    else:
        y = torch.randn((N, H, W, C), generator=g).to(dtype)
        host = torch.randn((N, H, W, C), generator=g).to(dtype)
    th, tw = -(-H // b), -(-W // b)
    rng = np.random.default_rng(C + H)
    tiles = np.array([(i * b, j * b) for i in range(th) for j in range(tw) if rng.random() < frac],
                     np.int32).reshape(-1, 2)
    cap = th * tw
    if over and len(tiles) > 2:
        cap = len(tiles) - 2                                # the device count exceeds the capacity
    idx = torch.zeros((max(cap, len(tiles)), 2), dtype=torch.int32)
    idx[:len(tiles)] = torch.from_numpy(tiles)
    cnt = torch.tensor([len(tiles)], dtype=torch.int32)
    used = tiles[:min(len(tiles), cap)]
    want = orc.restore_tiles(y, host.clone(), b, used)
    host_y = host.clone().pin_memory()
    sige.sige_download_tiles(y.to(DEV), b, idx.to(DEV), cnt.to(DEV), cap, host_y)
    assert torch.equal(bits(host_y), bits(want))


def _apply(xo, xe, blk, cd, cap, y1, out, gs1, gh1, gs2, gh2, w, dev_ws=None):
    idx, cnt, _ = sige.sige_reduce_mask(xo, xe, 1e-3, [(xo.shape[1], xo.shape[2], blk.block, cap)], 1)
    sige.sige_conv_fused(xe, w["w1"], w["b1"], cd, idx, cnt, cap, y1, gs1, gh1, silu=True)
    sige.sige_conv_fused(y1, w["w2"], w["b2"], cd, idx, cnt, cap, out, gs2, gh2, silu=True, residual=xe)
    return idx, cnt


def test_second_edit_after_restore_matches_a_fresh_edit():
    H = 128
    a = inputs.make_cfg3(50, H=H, W=H, area=0.02)
    bblk = inputs.make_cfg3(50, H=H, W=H, area=0.02, edit=np.roll(np.roll(a.edit, 37, 0), 53, 1))
    C = a.x_orig.shape[3]
    cd = sige.conv_desc(3, 1, 1, C, C, a.block)
    cap = (H // a.block) ** 2
    xo = a.x_orig.to(DEV)
    xa, xb = a.x_edit.to(DEV), bblk.x_edit.to(DEV)
    w = {k: getattr(a, k).to(DEV) for k in ("w1", "b1", "w2", "b2")}
    gs1, gh1 = sige.sige_groupnorm_affine(xo, 32, a.g1.to(DEV), a.be1.to(DEV))
    y1o = sige.sige_dense_conv(xo, w["w1"], w["b1"], cd, gn_scale=gs1, gn_shift=gh1, silu=True)
    gs2, gh2 = sige.sige_groupnorm_affine(y1o, 32, a.g2.to(DEV), a.be2.to(DEV))
    outo = sige.sige_dense_conv(y1o, w["w2"], w["b2"], cd, gn_scale=gs2, gn_shift=gh2, silu=True, residual=xo)
    # session: edit A, then restore A's tiles and apply edit B
    y1w, outw = y1o.clone(), outo.clone()
    ia, ca = _apply(xo, xa, a, cd, cap, y1w, outw, gs1, gh1, gs2, gh2, w)
    out_after_a = outw.clone()
    sige.sige_restore_tiles(y1o, y1w, a.block, ia, ca, cap)
    sige.sige_restore_tiles(outo, outw, a.block, ia, ca, cap)
    _apply(xo, xb, a, cd, cap, y1w, outw, gs1, gh1, gs2, gh2, w)
    # reference: edit B applied to untouched caches
    y1f, outf = y1o.clone(), outo.clone()
    _apply(xo, xb, a, cd, cap, y1f, outf, gs1, gh1, gs2, gh2, w)
    torch.cuda.synchronize()
    assert int(ca.item()) > 0
    assert torch.equal(bits(y1w.cpu()), bits(y1f.cpu()))
    assert torch.equal(bits(outw.cpu()), bits(outf.cpu()))
    # the restore mattered: edit A had changed the cache where edit B leaves the original
    assert not torch.equal(bits(out_after_a.cpu()), bits(outf.cpu()))
