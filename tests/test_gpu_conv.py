"""GPU gather / conv / scatter / fused / dense vs the CPU oracle on the same
seeded inputs.  Float outputs: max|GPU - oracle| / RMS(oracle) within 1e-4
(float32 layers) or 2e-2 (bf16 layers); every byte outside the listed tiles
must equal the cached output.

SIGE project page, "Overview": gather the active blocks with their halo from
A_edited, stack them, run F_l, scatter into the cached F_l(A_original)."""
import numpy as np
import pytest
import torch

import spatially_sparse_incremental_b200 as sige
from spatially_sparse_incremental_b200 import inputs
from helpers import TOL, assert_close, bits, rel_err, random_cache, tile_cover

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _idx_dev(idx, cap=None):
    idx = np.asarray(idx, np.int32).reshape(-1, 2)
    cap = len(idx) if cap is None else cap
    buf = torch.zeros((max(cap, 1), 2), dtype=torch.int32)
    buf[:len(idx)] = torch.from_numpy(idx)
    return buf.to(DEV), torch.tensor([len(idx)], dtype=torch.int32, device=DEV), cap


def _out_hw(L):
    H, W = L.x_orig.shape[1:3]
    return (H + 2 * L.pad - L.kernel) // L.stride + 1, (W + 2 * L.pad - L.kernel) // L.stride + 1


def _tiles(orc, L):
    Ho, Wo = _out_hw(L)
    return orc.reduce_mask(L.x_orig, L.x_edit, 1e-3, [(Ho, Wo, L.block)], 1)[0]


def _gn(orc, L):
    if L.gn_gamma is None:
        return None, None, None
    g = orc.gn_affine(L.x_orig, 8 if L.x_orig.shape[3] % 32 else 32, L.gn_gamma, L.gn_beta)
    return g, torch.from_numpy(g[0]).float().to(DEV), torch.from_numpy(g[1]).float().to(DEV)


def _fused_vs_oracle(orc, L, idx, residual=False, seed=0):
    Ho, Wo = _out_hw(L)
    N, Co = L.x_orig.shape[0], L.weight.shape[0]
    cache = random_cache((N, Ho, Wo, Co), L.x_orig.dtype, seed)
    gn, gs, gh = _gn(orc, L)
    res = None
    if residual:
        res = random_cache((N, Ho, Wo, Co), L.x_orig.dtype, seed + 1)
    ref = orc.sparse_conv(L.x_edit, L.weight, L.bias, idx, cache, L.kernel, L.stride, L.pad, L.block,
                          gn=gn, silu=gn is not None, residual=res)
    cd = sige.conv_desc(L.kernel, L.stride, L.pad, L.x_orig.shape[3], Co, L.block)
    di, dc, cap = _idx_dev(idx)
    y = cache.to(DEV)
    sige.sige_conv_fused(L.x_edit.to(DEV), L.weight.to(DEV), L.bias.to(DEV), cd, di, dc, cap, y, gs, gh,
                         silu=gn is not None, residual=None if res is None else res.to(DEV))
    torch.cuda.synchronize()
    got = y.cpu()
    cov = tile_cover(idx, L.block, N, Ho, Wo, Co)
    assert torch.equal(bits(got[~cov]), bits(ref[~cov])), "bytes outside the listed tiles changed"
    return assert_close(got, ref, L.x_orig.dtype, cov)


# ------------------------------------------------------------------ GroupNorm affine

@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_groupnorm_affine(orc, dtype):
    g = torch.Generator().manual_seed(3)
    x = (torch.randn(2, 32, 24, 128, generator=g) * 2 + 0.5).to(dtype)
    gamma, beta = 1 + 0.1 * torch.randn(128, generator=g), 0.1 * torch.randn(128, generator=g)
    sc, sh = orc.gn_affine(x, 32, gamma, beta)
    gs, gh = sige.sige_groupnorm_affine(x.to(DEV), 32, gamma.to(DEV), beta.to(DEV))
    torch.cuda.synchronize()
    assert np.allclose(gs.cpu().double().numpy(), sc, rtol=2e-6, atol=1e-7)
    assert np.allclose(gh.cpu().double().numpy(), sh, rtol=2e-6, atol=1e-6)


# ------------------------------------------------------------------ gather

@pytest.mark.parametrize("dtype,gn", [(torch.float32, False), (torch.bfloat16, False), (torch.bfloat16, True),
                                      (torch.float32, True)])
def test_gather(orc, dtype, gn):
    L = inputs.make_conv_case(21, 20, 28, 64, 64, dtype=dtype, block=4, area=0.08, gn=gn, N=2)
    idx = _tiles(orc, L)
    g, gs, gh = _gn(orc, L)
    ref = orc.gather(L.x_edit, idx, 3, 1, 1, 4, gn=g, silu=gn)
    cd = sige.conv_desc(3, 1, 1, 64, 64, 4)
    di, dc, cap = _idx_dev(idx, len(idx) + 5)
    blocks = sige.sige_gather(L.x_edit.to(DEV), cd, di, dc, cap, gs, gh, silu=gn)
    torch.cuda.synchronize()
    got = blocks[:len(idx)].cpu().double().numpy()
    if not gn:
        assert np.array_equal(got, ref)          # a copy, bit for bit
    elif dtype == torch.float32:
        assert np.allclose(got, ref, rtol=1e-5, atol=1e-6)
    else:
        # transform in float then one rounding to bf16: at most one bf16 step apart
        step = np.abs(ref) * 2.0 ** -7 + 1e-30
        assert np.all(np.abs(got - ref) <= step)
        assert np.mean(got != ref) < 0.01


def test_gather_stride2_and_overlap(orc):
    L = inputs.make_conv_case(22, 17, 19, 16, 16, dtype=torch.bfloat16, block=4, stride=2, area=0.2)
    idx = np.array([(0, 0), (0, 4), (4, 4), (8, 8)], np.int32)
    ref = orc.gather(L.x_edit, idx, 3, 2, 1, 4)
    cd = sige.conv_desc(3, 2, 1, 16, 16, 4)
    di, dc, cap = _idx_dev(idx)
    got = sige.sige_gather(L.x_edit.to(DEV), cd, di, dc, cap).cpu().double().numpy()
    assert np.array_equal(got, ref)


# ------------------------------------------------------------------ stacked-block conv

@pytest.mark.parametrize("dtype,ci,co,b,k,s", [
    (torch.float32, 64, 64, 4, 3, 1), (torch.bfloat16, 128, 128, 8, 3, 1), (torch.bfloat16, 320, 320, 4, 3, 1),
    (torch.bfloat16, 640, 640, 2, 3, 1), (torch.bfloat16, 256, 128, 1, 3, 1), (torch.bfloat16, 64, 64, 4, 3, 2),
    (torch.bfloat16, 512, 256, 4, 1, 1)])
def test_sparse_conv_on_blocks(orc, dtype, ci, co, b, k, s):
    rng = np.random.default_rng(ci + co + b)
    nb = 37
    bin_ = (b - 1) * s + k
    blocks = torch.from_numpy(rng.normal(size=(nb, 1, bin_, bin_, ci)).astype(np.float32)).to(dtype)
    w = torch.from_numpy(inputs.kaiming_uniform(rng, co, k, ci)).to(dtype)
    ref = orc.block_conv(blocks.double().numpy().reshape(nb, bin_, bin_, ci), w, k, s, b)
    cd = sige.conv_desc(k, s, k // 2, ci, co, b)
    cap = nb + 3
    buf = torch.zeros((cap, 1, bin_, bin_, ci), dtype=dtype)
    buf[:nb] = blocks
    cnt = torch.tensor([nb], dtype=torch.int32, device=DEV)
    out = sige.sige_sparse_conv(buf.to(DEV), cd, w.to(DEV), cnt, cap, batch=1)
    torch.cuda.synchronize()
    got = out[:nb].reshape(nb, b, b, co).cpu()
    # float32 accumulators of bf16 (or float32) operands: no output rounding
    err = rel_err(got, torch.from_numpy(ref))
    assert err <= TOL[dtype], err


# ------------------------------------------------------------------ scatter

@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_scatter(orc, dtype):
    rng = np.random.default_rng(5)
    N, Ho, Wo, Co, b = 2, 18, 22, 32, 4
    idx = np.array([(0, 0), (4, 8), (16, 20), (8, 0), (16, 0)], np.int32)   # ragged edge tiles
    out = torch.from_numpy(rng.normal(size=(len(idx), N, b, b, Co)).astype(np.float32))
    bias = torch.from_numpy(rng.normal(size=Co).astype(np.float32))
    res = random_cache((N, Ho, Wo, Co), dtype, 1)
    cache = random_cache((N, Ho, Wo, Co), dtype, 2)
    # expected from the oracle's own rounding of (out + bias + residual)
    exp = cache.clone()
    for t, (h0, w0) in enumerate(idx):
        hi, wi = min(b, Ho - h0), min(b, Wo - w0)
        v = out[t, :, :hi, :wi].double() + bias.double() + res[:, h0:h0 + hi, w0:w0 + wi].double()
        if dtype == torch.bfloat16:
            exp[:, h0:h0 + hi, w0:w0 + wi] = torch.from_numpy(orc.round_bf16(v.numpy()).view(np.int16)).view(torch.bfloat16)
        else:
            exp[:, h0:h0 + hi, w0:w0 + wi] = v.float()
    cd = sige.conv_desc(3, 1, 1, Co, Co, b)
    di, dc, cap = _idx_dev(idx)
    y = cache.to(DEV)
    sige.sige_scatter(out.to(DEV), cd, di, dc, cap, y, bias.to(DEV), res.to(DEV))
    torch.cuda.synchronize()
    got = y.cpu()
    cov = tile_cover(idx, b, N, Ho, Wo, Co)
    assert torch.equal(bits(got[~cov]), bits(cache[~cov]))
    # float32 sum of three terms vs the exactly rounded double sum
    assert rel_err(got, exp, cov) <= (1e-6 if dtype == torch.float32 else 1e-2)


# ------------------------------------------------------------------ unfused pipeline

@pytest.mark.parametrize("dtype,gn,res", [(torch.float32, False, False), (torch.bfloat16, True, True)])
def test_gather_conv_scatter_pipeline(orc, dtype, gn, res):
    L = inputs.make_conv_case(23, 32, 24, 64, 64, dtype=dtype, block=4, area=0.06, gn=gn)
    idx = _tiles(orc, L)
    g, gs, gh = _gn(orc, L)
    Ho, Wo = _out_hw(L)
    cache = random_cache((1, Ho, Wo, 64), dtype, 3)
    resid = random_cache((1, Ho, Wo, 64), dtype, 4) if res else None
    ref = orc.sparse_conv(L.x_edit, L.weight, L.bias, idx, cache, block=4, gn=g, silu=gn, residual=resid)
    cd = sige.conv_desc(3, 1, 1, 64, 64, 4)
    di, dc, cap = _idx_dev(idx, len(idx) + 2)
    blocks = sige.sige_gather(L.x_edit.to(DEV), cd, di, dc, cap, gs, gh, silu=gn)
    outb = sige.sige_sparse_conv(blocks, cd, L.weight.to(DEV), dc, cap)
    y = cache.to(DEV)
    sige.sige_scatter(outb, cd, di, dc, cap, y, L.bias.to(DEV), None if resid is None else resid.to(DEV))
    torch.cuda.synchronize()
    cov = tile_cover(idx, 4, 1, Ho, Wo, 64)
    got = y.cpu()
    assert torch.equal(bits(got[~cov]), bits(cache[~cov]))
    assert_close(got, ref, dtype, cov)


# ------------------------------------------------------------------ fused layer, per config

def test_fused_cfg1_f32(orc):
    for seed in range(3):
        L = inputs.make_cfg1(seed)
        _fused_vs_oracle(orc, L, _tiles(orc, L), seed=seed)


@pytest.mark.parametrize("H", [64, 256])
def test_fused_cfg3_conv(orc, H):
    L = inputs.make_conv_case(24, H, H, 128, 128, dtype=torch.bfloat16, block=8, area=0.012 if H == 256 else 0.05,
                              gn=True)
    idx = _tiles(orc, L)
    _fused_vs_oracle(orc, L, idx, residual=False)
    _fused_vs_oracle(orc, L, idx, residual=True, seed=5)


@pytest.mark.parametrize("layer", [0, 1, 2])
@pytest.mark.parametrize("area", [0.012, 0.05])
def test_fused_cfg4_layers(orc, layer, area):
    L = inputs.make_cfg4_layer(30, layer, area)
    _fused_vs_oracle(orc, L, _tiles(orc, L))


@pytest.mark.parametrize("layer", range(8))
def test_fused_cfg5_layers(orc, layer):
    L = inputs.make_cfg5_layer(31, layer, 0.012)
    _fused_vs_oracle(orc, L, _tiles(orc, L))


@pytest.mark.parametrize("layer", [0, 2, 6, 7])
def test_fused_cfg5_all_ones_equals_dense(orc, layer):
    L = inputs.make_cfg5_layer(32, layer, all_edit=True)
    Ho, Wo = _out_hw(L)
    idx = _tiles(orc, L)
    assert len(idx) == -(-Ho // L.block) * -(-Wo // L.block)
    ref = orc.dense_conv(L.x_edit, L.weight, L.bias, L.kernel, L.stride, L.pad)
    cd = sige.conv_desc(L.kernel, L.stride, L.pad, L.x_orig.shape[3], L.weight.shape[0], L.block)
    di, dc, cap = _idx_dev(idx)
    y = torch.zeros_like(ref).to(DEV)
    sige.sige_conv_fused(L.x_edit.to(DEV), L.weight.to(DEV), L.bias.to(DEV), cd, di, dc, cap, y)
    torch.cuda.synchronize()
    assert_close(y.cpu(), ref, torch.bfloat16)


@pytest.mark.parametrize("block,stride,N", [(4, 1, 1), (4, 1, 2), (2, 1, 2), (3, 1, 1), (4, 2, 1)])
def test_fused_gn_slot_layouts(orc, block, stride, N):
    # GroupNorm affine + SiLU applied while the halo is staged in the slot
    # layouts (row-batched POS for even b, POS otherwise), batch 1 and 2,
    # with a residual; K = 9 x 256 is long enough to be split
    L = inputs.make_conv_case(40 + block + N, 36, 28, 256, 128, dtype=torch.bfloat16, block=block,
                              stride=stride, area=0.08, gn=True, N=N)
    _fused_vs_oracle(orc, L, _tiles(orc, L), residual=True)


def test_fused_ragged_edges_and_batch(orc):
    L = inputs.make_conv_case(25, 30, 26, 64, 64, dtype=torch.bfloat16, block=8, area=0.1, gn=True, N=2)
    _fused_vs_oracle(orc, L, _tiles(orc, L), residual=True)


def test_fused_empty_list_writes_nothing(orc):
    L = inputs.make_conv_case(26, 32, 32, 128, 128, dtype=torch.bfloat16, block=8)
    cache = random_cache((1, 32, 32, 128), torch.bfloat16, 9)
    cd = sige.conv_desc(3, 1, 1, 128, 128, 8)
    di = torch.zeros((16, 2), dtype=torch.int32, device=DEV)
    dc = torch.zeros(1, dtype=torch.int32, device=DEV)
    y = cache.to(DEV)
    sige.sige_conv_fused(L.x_edit.to(DEV), L.weight.to(DEV), L.bias.to(DEV), cd, di, dc, 16, y)
    torch.cuda.synchronize()
    assert torch.equal(bits(y), bits(cache))


# ------------------------------------------------------------------ dense layer

@pytest.mark.parametrize("dtype,H,ci,co,k,s,b", [
    (torch.float32, 64, 64, 64, 3, 1, 4), (torch.bfloat16, 64, 128, 128, 3, 1, 8),
    (torch.bfloat16, 33, 64, 64, 3, 2, 4), (torch.bfloat16, 32, 256, 128, 1, 1, 4)])
def test_dense_conv(orc, dtype, H, ci, co, k, s, b):
    L = inputs.make_conv_case(27, H, H, ci, co, dtype=dtype, kernel=k, stride=s, pad=k // 2, block=b)
    ref = orc.dense_conv(L.x_orig, L.weight, L.bias, k, s, k // 2)
    cd = sige.conv_desc(k, s, k // 2, ci, co, b)
    y = sige.sige_dense_conv(L.x_orig.to(DEV), L.weight.to(DEV), L.bias.to(DEV), cd)
    torch.cuda.synchronize()
    assert_close(y.cpu(), ref, dtype)


# ------------------------------------------------------------------ res block (cfg 3)

def _resblock_gpu(blk, dev_idx, dev_cnt, cap):
    C = blk.x_orig.shape[3]
    cd = sige.conv_desc(3, 1, 1, C, C, blk.block)
    xo, xe = blk.x_orig.to(DEV), blk.x_edit.to(DEV)
    w1, w2, b1, b2 = blk.w1.to(DEV), blk.w2.to(DEV), blk.b1.to(DEV), blk.b2.to(DEV)
    gs1, gh1 = sige.sige_groupnorm_affine(xo, 32, blk.g1.to(DEV), blk.be1.to(DEV))
    y1 = sige.sige_dense_conv(xo, w1, b1, cd, gn_scale=gs1, gn_shift=gh1, silu=True)
    gs2, gh2 = sige.sige_groupnorm_affine(y1, 32, blk.g2.to(DEV), blk.be2.to(DEV))
    out = sige.sige_dense_conv(y1, w2, b2, cd, gn_scale=gs2, gn_shift=gh2, silu=True, residual=xo)
    y1_cache, out_cache = y1.clone(), out.clone()
    sige.sige_conv_fused(xe, w1, b1, cd, dev_idx, dev_cnt, cap, y1, gs1, gh1, silu=True)
    sige.sige_conv_fused(y1, w2, b2, cd, dev_idx, dev_cnt, cap, out, gs2, gh2, silu=True, residual=xe)
    torch.cuda.synchronize()
    return y1, out, y1_cache, out_cache


@pytest.mark.parametrize("H,area", [(64, 0.05), (256, 0.012)])
def test_resblock_cfg3(orc, H, area):
    blk = inputs.make_cfg3(40, H=H, W=H, area=area)
    b = blk.block
    cap = (H // b) ** 2
    idx, cnt, _ = sige.sige_reduce_mask(blk.x_orig.to(DEV), blk.x_edit.to(DEV), 1e-3, [(H, H, b, cap)], 1)
    y1, out, y1c, outc = _resblock_gpu(blk, idx, cnt, cap)
    n = int(cnt[0].item())
    ref_idx = orc.reduce_mask(blk.x_orig, blk.x_edit, 1e-3, [(H, H, b)], 1)[0]
    assert np.array_equal(idx[:n].cpu().numpy(), ref_idx)
    g1 = orc.gn_affine(blk.x_orig, 32, blk.g1, blk.be1)
    oy1 = orc.dense_conv(blk.x_orig, blk.w1, blk.b1, gn=g1, silu=True)
    g2 = orc.gn_affine(oy1, 32, blk.g2, blk.be2)
    oy1, oout = orc.resblock_dense(blk.x_orig, blk, g1, g2)
    assert_close(y1c.cpu(), oy1, torch.bfloat16, what="dense y1")
    # the GPU's y1 cache feeds its conv2, so compare out with the float bar of
    # two chained layers: y1 differs by up to one bf16 ulp per element
    ry1, rout = orc.resblock_sparse(blk.x_edit, blk, ref_idx, oy1, oout, g1, g2)
    assert_close(y1.cpu(), ry1, torch.bfloat16, what="sparse y1")
    assert_close(outc.cpu(), oout, torch.bfloat16, what="dense out")
    assert_close(out.cpu(), rout, torch.bfloat16, what="sparse out")
    cov = tile_cover(ref_idx, b, 1, H, H, blk.x_orig.shape[3])
    assert torch.equal(bits(out.cpu()[~cov]), bits(outc.cpu()[~cov]))


def test_conv_path_selection():
    # bf16 layers whose C_in is a multiple of 64 run on the tensor cores
    for (H, W, ci, co, k, s, b) in inputs.CFG5_LAYERS:
        assert sige.sige_conv_path(sige.conv_desc(k, s, k // 2, ci, co, b), torch.bfloat16) == 1
    for (H, W, C, b) in inputs.CFG4_LAYERS:
        assert sige.sige_conv_path(sige.conv_desc(3, 1, 1, C, C, b), torch.bfloat16) == 1
    assert sige.sige_conv_path(sige.conv_desc(3, 1, 1, 128, 128, 8), torch.bfloat16) == 1
    assert sige.sige_conv_path(sige.conv_desc(3, 1, 1, 64, 64, 4), torch.float32) == 0
    assert sige.sige_conv_path(sige.conv_desc(3, 1, 1, 32, 32, 4), torch.bfloat16) == 0


def test_fused_cuda_core_bf16(orc):
    # C_in = 32 is below the tensor-core kernel's 64-channel chunk
    L = inputs.make_conv_case(28, 24, 24, 32, 32, dtype=torch.bfloat16, block=4, area=0.08, gn=True)
    _fused_vs_oracle(orc, L, _tiles(orc, L), residual=True)


# ------------------------------------------------------------------ 3x3 layers on 8x8 tiles

@pytest.mark.parametrize("H,W,ci,co,N,gn,res", [
    (40, 24, 64, 64, 1, True, False),     # last strip of 8 rows: its second accumulator idles
    (56, 40, 192, 256, 2, True, True),    # C_out 256: one accumulator pair, three K chunks, batch 2
    (48, 48, 128, 96, 1, False, False),   # C_out 96, no input transform
    (30, 26, 64, 32, 2, True, True),      # ragged map, C_out 32
])
def test_conv8_dense(orc, H, W, ci, co, N, gn, res):
    """Every tile of the map: strips of four 8x8 tiles share each weight stage."""
    L = inputs.make_conv_case(60 + H + co, H, W, ci, co, dtype=torch.bfloat16, block=8, gn=gn, N=N)
    g, gs, gh = _gn(orc, L)
    r = random_cache((N, H, W, co), torch.bfloat16, 3) if res else None
    every = np.array([(h, w) for h in range(0, H, 8) for w in range(0, W, 8)], np.int32)
    ref = orc.sparse_conv(L.x_orig, L.weight, L.bias, every, torch.zeros((N, H, W, co), dtype=torch.bfloat16),
                          3, 1, 1, 8, gn=g, silu=gn, residual=r)
    cd = sige.conv_desc(3, 1, 1, ci, co, 8)
    y = sige.sige_dense_conv(L.x_orig.to(DEV), L.weight.to(DEV), L.bias.to(DEV), cd, gn_scale=gs, gn_shift=gh,
                             silu=gn, residual=None if r is None else r.to(DEV))
    torch.cuda.synchronize()
    assert_close(y.cpu(), ref, torch.bfloat16)


@pytest.mark.parametrize("H,W,ci,co,N,area", [
    (64, 64, 256, 256, 1, 0.05),          # C_out 256, four K chunks
    (40, 56, 64, 32, 2, 0.08),            # batch 2: tile pairs across items
    (24, 24, 128, 160, 1, 0.02),          # C_out 160 (not a power of two)
])
def test_conv8_sparse(orc, H, W, ci, co, N, area):
    L = inputs.make_conv_case(70 + H + co, H, W, ci, co, dtype=torch.bfloat16, block=8, area=area, gn=True, N=N)
    _fused_vs_oracle(orc, L, _tiles(orc, L), residual=True, seed=4)


@pytest.mark.parametrize("ntiles", [1, 3])
def test_conv8_odd_tile_count(orc, ntiles):
    """An odd number of listed items: the last unit holds a single tile."""
    L = inputs.make_conv_case(80 + ntiles, 32, 32, 64, 64, dtype=torch.bfloat16, block=8, gn=True)
    idx = np.array([(8, 8), (24, 0), (0, 24)][:ntiles], np.int32)
    _fused_vs_oracle(orc, L, idx, residual=True, seed=6)


# ------------------------------------------------------------------ 1x1 layers (GEMM over gathered pixels)

@pytest.mark.parametrize("H,W,ci,co,b,N,gn,res,area", [
    (64, 128, 512, 256, 4, 1, False, False, 0.012),   # the GauGAN 1x1 layer's shape: two output-channel units
    (36, 28, 128, 48, 4, 2, True, True, 0.08),        # ragged map, batch 2, C_out 48, GN + SiLU, residual
    (32, 32, 64, 128, 8, 1, True, False, 0.05),       # 8x8 tiles: two per unit
    (20, 20, 192, 64, 1, 1, False, True, 0.1),        # one-pixel tiles: 128 per unit
    (30, 26, 64, 16, 3, 1, True, True, 0.1),          # 3x3 tiles: 14 per unit, two padding slots
])
def test_conv1x1_sparse(orc, H, W, ci, co, b, N, gn, res, area):
    L = inputs.make_conv_case(90 + H + co + b, H, W, ci, co, dtype=torch.bfloat16, kernel=1, stride=1, pad=0,
                              block=b, area=area, gn=gn, N=N)
    assert sige.sige_conv_path(sige.conv_desc(1, 1, 0, ci, co, b), torch.bfloat16) == 1
    _fused_vs_oracle(orc, L, _tiles(orc, L), residual=res, seed=7)


@pytest.mark.parametrize("H,W,ci,co,b,N,gn,res", [
    (64, 64, 256, 128, 4, 1, True, True),
    (30, 26, 128, 256, 8, 2, False, False),
])
def test_conv1x1_dense(orc, H, W, ci, co, b, N, gn, res):
    """Every tile of the map through sige_dense_conv (the same kernel)."""
    L = inputs.make_conv_case(95 + H + co, H, W, ci, co, dtype=torch.bfloat16, kernel=1, stride=1, pad=0, block=b,
                              gn=gn, N=N)
    g, gs, gh = _gn(orc, L)
    r = random_cache((N, H, W, co), torch.bfloat16, 5) if res else None
    every = np.array([(h, w) for h in range(0, H, b) for w in range(0, W, b)], np.int32)
    ref = orc.sparse_conv(L.x_orig, L.weight, L.bias, every, torch.zeros((N, H, W, co), dtype=torch.bfloat16),
                          1, 1, 0, b, gn=g, silu=gn, residual=r)
    cd = sige.conv_desc(1, 1, 0, ci, co, b)
    y = sige.sige_dense_conv(L.x_orig.to(DEV), L.weight.to(DEV), L.bias.to(DEV), cd, gn_scale=gs, gn_shift=gh,
                             silu=gn, residual=None if r is None else r.to(DEV))
    torch.cuda.synchronize()
    assert_close(y.cpu(), ref, torch.bfloat16)


@pytest.mark.parametrize("H,W,ci,co,b,N,gn,res,area", [
    (30, 26, 64, 48, 4, 2, False, True, 0.1),         # 4x4 tiles (TMA fill), ragged map, batch 2
    (24, 20, 128, 320, 4, 1, False, False, 0.1),      # C_out 320: five units of 64 output channels
    (64, 64, 320, 320, 4, 1, False, True, 0.012),     # the SD-latent layer's shape (K split 4)
    (24, 24, 64, 48, 8, 1, False, True, 0.1),         # 8x8 tiles with a C_out the 8x8 kernel does not take
    (30, 26, 64, 48, 4, 2, True, True, 0.1),          # GN + SiLU: transformed once into a scratch copy
    (20, 18, 64, 64, 2, 1, True, True, 0.1),          # 2x2, 1x1 and 3x3 tiles: the general tile kernel
    (12, 10, 128, 32, 1, 2, False, True, 0.2),
    (21, 19, 64, 16, 3, 1, True, False, 0.15),
])
def test_tile_gemm_3x3_sparse(orc, H, W, ci, co, b, N, gn, res, area):
    """3x3 stride-1 layers on 4x4 tiles (and 8x8 ones outside the 8x8
    kernel's range) without an input transform: the tile GEMM, one shifted TMA
    box of the tile's pixels per tap (zero outside the map), K split across a
    cluster when the units are few (with GN + SiLU: the transform once per
    input pixel into a scratch copy first); other tile sizes on the general
    kernel."""
    L = inputs.make_conv_case(110 + H + co + b, H, W, ci, co, dtype=torch.bfloat16, block=b, area=area, gn=gn, N=N)
    assert sige.sige_conv_path(sige.conv_desc(3, 1, 1, ci, co, b), torch.bfloat16) == 1
    _fused_vs_oracle(orc, L, _tiles(orc, L), residual=res, seed=9)


@pytest.mark.parametrize("H,W,ci,co,b,N,gn,res,area", [
    (64, 64, 64, 64, 4, 1, False, False, 0.05),      # stride 2: strided TMA boxes, 9 K chunks
    (33, 29, 128, 80, 4, 2, False, True, 0.15),      # odd input map, batch 2, C_out 80, residual
    (40, 48, 64, 32, 8, 1, False, False, 0.2),       # 8x8 output tiles (16x16 strided boxes)
    (33, 29, 128, 80, 4, 2, True, True, 0.15),       # GN + SiLU: transformed once into a scratch copy
])
def test_tile_gemm_3x3_stride2(orc, H, W, ci, co, b, N, gn, res, area):
    """3x3 stride-2 layers on the tile GEMM: tap (dr, dc) of output tile
    (h0, w0) reads every other input pixel from (2 h0 + dr - 1, 2 w0 + dc - 1)."""
    L = inputs.make_conv_case(130 + H + co + b, H, W, ci, co, dtype=torch.bfloat16, stride=2, block=b, area=area,
                              gn=gn, N=N)
    assert sige.sige_conv_path(sige.conv_desc(3, 2, 1, ci, co, b), torch.bfloat16) == 1
    _fused_vs_oracle(orc, L, _tiles(orc, L), residual=res, seed=11)


@pytest.mark.parametrize("H,W,ci,co,b,N,gn", [(28, 36, 64, 64, 4, 1, False), (30, 26, 128, 80, 4, 2, False),
                                               (18, 14, 128, 48, 2, 2, True), (13, 11, 64, 32, 1, 1, False),
                                               (20, 17, 64, 48, 3, 2, False)])
def test_tile_gemm_3x3_dense(orc, H, W, ci, co, b, N, gn):
    """Every tile through sige_dense_conv: the tile GEMM (TMA boxes for 4x4
    tiles, per-thread row copies for 1x1, 2x2 and 3x3 tiles; GN + SiLU through
    the transform pre-pass)."""
    L = inputs.make_conv_case(120 + H + co, H, W, ci, co, dtype=torch.bfloat16, block=b, gn=gn, N=N)
    g, gs, gh = _gn(orc, L)
    r = random_cache((N, H, W, co), torch.bfloat16, 5)
    every = np.array([(h, w) for h in range(0, H, b) for w in range(0, W, b)], np.int32)
    ref = orc.sparse_conv(L.x_orig, L.weight, L.bias, every, torch.zeros((N, H, W, co), dtype=torch.bfloat16),
                          3, 1, 1, b, gn=g, silu=gn, residual=r)
    cd = sige.conv_desc(3, 1, 1, ci, co, b)
    y = sige.sige_dense_conv(L.x_orig.to(DEV), L.weight.to(DEV), L.bias.to(DEV), cd, gn_scale=gs, gn_shift=gh,
                             silu=gn, residual=r.to(DEV))
    torch.cuda.synchronize()
    assert_close(y.cpu(), ref, torch.bfloat16)


def test_conv1x1_empty_list_writes_nothing(orc):
    L = inputs.make_conv_case(98, 16, 16, 64, 64, dtype=torch.bfloat16, kernel=1, stride=1, pad=0, block=4)
    cache = random_cache((1, 16, 16, 64), torch.bfloat16, 8)
    cd = sige.conv_desc(1, 1, 0, 64, 64, 4)
    di = torch.zeros((16, 2), dtype=torch.int32, device=DEV)
    dc = torch.zeros(1, dtype=torch.int32, device=DEV)
    y = cache.to(DEV)
    sige.sige_conv_fused(L.x_edit.to(DEV), L.weight.to(DEV), L.bias.to(DEV), cd, di, dc, 16, y)
    torch.cuda.synchronize()
    assert torch.equal(bits(y.cpu()), bits(cache))
