"""Pins for the CPU oracle: checks against what the pages and the mathematics
fix, never against the oracle itself.

  * hand-derived golden fixtures (tests/golden/*.txt);
  * a library routine for the special cases it covers
    (torch.nn.functional.conv2d / group_norm / silu in float64);
  * brute force with a different formulation on tiny grids (index lists);
  * ground truth known from how the synthetic edit was built;
  * invariants the pages state: unedited pixels reuse the cached output
    (mer.dev notes on SIGE, section 3 "Method"), the conv is linear in its
    input (section 3.1 "Activation Sparsity"), gathered 3x3 stride-1 blocks
    overlap by 2 (SIGE project page, "Overview"), an empty list returns the
    cache and a full list the dense layer.
"""
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from spatially_sparse_incremental_b200 import inputs

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _lines(name):
    with open(os.path.join(GOLD, name)) as f:
        return [ln.strip() for ln in f if ln.strip() and not ln.startswith("#")]


# --------------------------------------------------------------- bf16 rounding

def test_round_bf16_hand_cases(orc):
    for ln in _lines("bf16_rounding.txt"):
        expr, hexbits = [s.strip() for s in ln.split("|")]
        v = float(eval(expr, {"__builtins__": {}}))
        got = orc.round_bf16(np.array([v]))[0]
        assert got == int(hexbits, 16), (expr, hex(got), hexbits)


def test_round_bf16_matches_torch_on_float32_values(orc):
    # For values exactly representable in float32, torch's bf16 conversion
    # (round to nearest even from float) is a single rounding, so it must agree.
    rng = np.random.default_rng(1)
    v = np.concatenate([
        rng.normal(size=20000) * 10.0 ** rng.integers(-40, 38, size=20000),
        rng.uniform(-1, 1, size=5000).astype(np.float32) * 1e-39,   # float subnormals
        np.array([0.0, -0.0, 1.0, -1.0, np.inf, -np.inf, 3.3e38, -3.3e38]),
    ]).astype(np.float32).astype(np.float64)
    ref = torch.from_numpy(v.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = orc.round_bf16(v)
    finite = np.isfinite(v)
    assert np.array_equal(got[finite], ref[finite])
    assert got[v == np.inf][0] == 0x7F80 and got[v == -np.inf][0] == 0xFF80
    assert orc.round_bf16(np.array([np.nan]))[0] & 0x7FFF > 0x7F80


# ------------------------------------------------------------------ pixel mask

@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16, torch.uint8])
@pytest.mark.parametrize("layout", ["NHWC", "NCHW"])
def test_pixel_mask_single_change(orc, dtype, layout):
    # One changed element sets exactly its pixel when |delta| > thr, never when
    # |delta| <= thr (strict), whatever channel, batch item or layout holds it.
    rng = np.random.default_rng(2)
    N, H, W, C = 2, 5, 7, 3
    for trial in range(20):
        if dtype == torch.uint8:
            base = torch.from_numpy(rng.integers(0, 250, size=(N, H, W, C)).astype(np.uint8))
        else:
            base = torch.from_numpy(rng.normal(size=(N, H, W, C)).astype(np.float32)).to(dtype)
        n, y, x, c = (int(rng.integers(0, s)) for s in (N, H, W, C))
        ed = base.clone()
        ed[n, y, x, c] = ed[n, y, x, c] + (3 if dtype == torch.uint8 else 0.5)
        a, b = base, ed
        lay = orc.NHWC
        if layout == "NCHW":
            a, b, lay = base.permute(0, 3, 1, 2).contiguous(), ed.permute(0, 3, 1, 2).contiguous(), orc.NCHW
        m = orc.pixel_mask(a, b, 0.0 if dtype == torch.uint8 else 1e-3, lay)
        exp = np.zeros((H, W), np.uint8)
        exp[y, x] = 1
        assert np.array_equal(m, exp)
        # the stored difference itself as threshold: strict ">" sets nothing;
        # the next float below it sets the pixel again
        d = np.float32(abs(np.float32(ed[n, y, x, c].float().item()) - np.float32(base[n, y, x, c].float().item())))
        assert orc.pixel_mask(a, b, float(d), lay).sum() == 0
        below = float(np.nextafter(d, np.float32(0)))
        assert np.array_equal(orc.pixel_mask(a, b, below, lay), exp)


def test_pixel_mask_identical_inputs_is_empty(orc):
    x = torch.randn(1, 9, 11, 16)
    assert orc.pixel_mask(x, x.clone(), 0.0).sum() == 0


def test_pixel_mask_equals_edit_region_cfg2(orc):
    # cfg 2 builds the edit so that every channel differs inside the ellipses
    # and nothing differs outside: the mask must be exactly that region.
    for seed in range(5):
        o, e, edit = inputs.make_cfg2(seed)
        m = orc.pixel_mask(o, e, 0.0, orc.NCHW)
        assert np.array_equal(m.astype(bool), edit)
        assert 0.009 <= edit.mean() <= 0.015


def test_pixel_mask_equals_edit_region_cfg1(orc):
    for seed in range(3):
        L = inputs.make_cfg1(seed)
        m = orc.pixel_mask(L.x_orig, L.x_edit, 1e-3)
        assert np.array_equal(m.astype(bool), L.edit)


# ------------------------------------------------------------------ index lists

def _brute_tiles(mask, Hs, Ws, b, D):
    """Different formulation: tile (i, j) is active when some set pixel maps
    (through the downsampling floor(y*Hs/H)) into a tile within D tiles."""
    H, W = mask.shape
    th, tw = -(-Hs // b), -(-Ws // b)
    act = np.zeros((th, tw), bool)
    for y, x in zip(*np.nonzero(mask)):
        ti, tj = (y * Hs // H) // b, (x * Ws // W) // b
        act[max(0, ti - D):ti + D + 1, max(0, tj - D):tj + D + 1] = True
    return np.array([(i * b, j * b) for i in range(th) for j in range(tw) if act[i, j]],
                    dtype=np.int32).reshape(-1, 2)


def test_tiles_golden(orc):
    for ln in _lines("tiles_hand.txt"):
        dims, pix, sc, exp = [s.strip() for s in ln.split("|")]
        H, W = map(int, dims.split())
        Hs, Ws, b, D = map(int, sc.split())
        m = np.zeros((H, W), np.uint8)
        if pix != "-":
            for p in pix.split(";"):
                y, x = map(int, p.split(","))
                m[y, x] = 1
        want = np.zeros((0, 2), np.int32) if exp == "-" else np.array(
            [list(map(int, p.split(","))) for p in exp.split(";")], np.int32)
        got = orc.reduce_scale(m, Hs, Ws, b, D)
        assert np.array_equal(got, want), ln


@pytest.mark.parametrize("Hs,b,D", [(4, 1, 1), (4, 2, 1), (2, 1, 1), (4, 3, 1), (4, 2, 0), (2, 2, 2)])
def test_tiles_exhaustive_4x4(orc, Hs, b, D):
    for bits in range(1 << 16):
        m = np.array([(bits >> k) & 1 for k in range(16)], np.uint8).reshape(4, 4)
        got = orc.reduce_scale(m, Hs, Hs, b, D)
        assert np.array_equal(got, _brute_tiles(m, Hs, Hs, b, D)), (bits, Hs, b, D)


def test_tiles_random_grids(orc):
    rng = np.random.default_rng(3)
    for _ in range(300):
        f = int(rng.choice([1, 2, 4]))
        Hs, Ws = int(rng.integers(1, 9)), int(rng.integers(1, 9))
        H, W = Hs * f, Ws * f
        b = int(rng.integers(1, 5))
        D = int(rng.integers(0, 3))
        m = (rng.random((H, W)) < rng.choice([0.01, 0.05, 0.3])).astype(np.uint8)
        got = orc.reduce_scale(m, Hs, Ws, b, D)
        assert np.array_equal(got, _brute_tiles(m, Hs, Ws, b, D))
        # properties: sorted row-major, unique, every set pixel's tile listed
        key = got[:, 0] * 100000 + got[:, 1]
        assert np.all(np.diff(key) > 0)
        listed = {tuple(t) for t in got}
        for y, x in zip(*np.nonzero(m)):
            Y, X = y * Hs // H, x * Ws // W
            assert ((Y // b) * b, (X // b) * b) in listed


def test_downsample_and_dilate_special_cases(orc):
    rng = np.random.default_rng(4)
    m = (rng.random((12, 20)) < 0.1).astype(np.uint8)
    assert np.array_equal(orc.downsample(m, 12, 20), m)            # identity scale
    assert orc.downsample(m, 1, 1)[0, 0] == int(m.any())           # single cell = any
    assert np.array_equal(orc.dilate(m, 0), m)                     # radius 0 = identity
    one = np.zeros((9, 9), np.uint8)
    one[0, 4] = 1
    d = orc.dilate(one, 2)                                          # clipped square
    exp = np.zeros((9, 9), np.uint8)
    exp[0:3, 2:7] = 1
    assert np.array_equal(d, exp)


def test_capacity_truncates_but_counts(orc):
    m = np.ones((16, 16), np.uint8)
    full = orc.reduce_scale(m, 16, 16, 4, 1)
    assert len(full) == 16
    part = orc.reduce_scale(m, 16, 16, 4, 1, capacity=5)
    assert np.array_equal(part, full[:5])


# ------------------------------------------------------------------ GroupNorm / SiLU

@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_gn_affine_matches_torch_group_norm(orc, dtype):
    g = torch.Generator().manual_seed(5)
    N, H, W, C, G = 2, 6, 5, 64, 32
    x = (torch.randn(N, H, W, C, generator=g) * 3 + 1).to(dtype)
    gamma = 1 + 0.1 * torch.randn(C, generator=g)
    beta = 0.1 * torch.randn(C, generator=g)
    sc, sh = orc.gn_affine(x, G, gamma, beta, 1e-5)
    xd = x.double()
    ref = F.group_norm(xd.permute(0, 3, 1, 2), G, gamma.double(), beta.double(), 1e-5).permute(0, 2, 3, 1)
    ours = xd * torch.from_numpy(sc)[:, None, None, :] + torch.from_numpy(sh)[:, None, None, :]
    assert torch.allclose(ours, ref, rtol=0, atol=1e-12)


# ------------------------------------------------------------------ dense layer

def _torch_conv(x, w, bias, k, stride, pad, pre=None, residual=None):
    xd = x.double() if pre is None else pre
    out = F.conv2d(xd.permute(0, 3, 1, 2), w.double().permute(0, 3, 1, 2),
                   None if bias is None else bias.double(), stride=stride, padding=pad).permute(0, 2, 3, 1)
    if residual is not None:
        out = out + residual.double()
    return out


def test_conv_golden(orc):
    x = torch.arange(1, 10, dtype=torch.float32).reshape(1, 3, 3, 1)
    w = torch.ones(1, 3, 3, 1)
    b = torch.tensor([0.5])
    for ln in _lines("conv_hand.txt"):
        s, vals = ln.split("|")
        want = np.array(list(map(float, vals.split())))
        got = orc.dense_conv_f64(x, w, b, 3, int(s), 1).reshape(-1)
        assert np.array_equal(got, want)


@pytest.mark.parametrize("k,stride,pad,N,H,W,ci,co", [
    (3, 1, 1, 1, 9, 7, 16, 8), (3, 2, 1, 2, 10, 9, 8, 24), (1, 1, 0, 1, 6, 6, 32, 16),
    (3, 1, 0, 1, 7, 8, 8, 8), (5, 1, 2, 1, 8, 8, 4, 4)])
def test_dense_conv_matches_torch_conv2d(orc, k, stride, pad, N, H, W, ci, co):
    g = torch.Generator().manual_seed(6)
    x = torch.randn(N, H, W, ci, generator=g)
    w = torch.randn(co, k, k, ci, generator=g) * 0.2
    b = torch.randn(co, generator=g)
    got = orc.dense_conv_f64(x, w, b, k, stride, pad)
    ref = _torch_conv(x, w, b, k, stride, pad).numpy()
    assert np.allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_dense_conv_gn_silu_residual_f32(orc):
    g = torch.Generator().manual_seed(7)
    N, H, W, C = 1, 8, 8, 64
    x = torch.randn(N, H, W, C, generator=g)
    w = torch.randn(C, 3, 3, C, generator=g) * 0.05
    b = torch.randn(C, generator=g) * 0.1
    gamma, beta = 1 + 0.1 * torch.randn(C, generator=g), 0.1 * torch.randn(C, generator=g)
    sc, sh = orc.gn_affine(x, 32, gamma, beta)
    got = orc.dense_conv_f64(x, w, b, 3, 1, 1, gn=(sc, sh), silu=True, residual=x)
    pre = F.silu(F.group_norm(x.double().permute(0, 3, 1, 2), 32, gamma.double(), beta.double(), 1e-5)
                 ).permute(0, 2, 3, 1)
    ref = _torch_conv(x, w, b, 3, 1, 1, pre=pre, residual=x).numpy()
    assert np.allclose(got, ref, rtol=1e-11, atol=1e-11)


def test_dense_conv_bf16_input_rounding(orc):
    # bf16 layers: the transformed input is rounded to bf16 before the conv.
    g = torch.Generator().manual_seed(8)
    N, H, W, C = 1, 6, 6, 64
    x = torch.randn(N, H, W, C, generator=g).to(torch.bfloat16)
    w = (torch.randn(C, 3, 3, C, generator=g) * 0.05).to(torch.bfloat16)
    gamma, beta = 1 + 0.1 * torch.randn(C, generator=g), 0.1 * torch.randn(C, generator=g)
    sc, sh = orc.gn_affine(x, 32, gamma, beta)
    t = x.double() * torch.from_numpy(sc)[:, None, None, :] + torch.from_numpy(sh)[:, None, None, :]
    t = F.silu(t)
    t = torch.from_numpy(orc.bf16_bits_to_f64(orc.round_bf16(t.numpy())))
    got = orc.dense_conv_f64(x, w, None, 3, 1, 1, gn=(sc, sh), silu=True)
    ref = _torch_conv(x, w, None, 3, 1, 1, pre=t).numpy()
    assert np.allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_dense_conv_rounds_once(orc):
    g = torch.Generator().manual_seed(9)
    x = torch.randn(1, 7, 7, 16, generator=g).to(torch.bfloat16)
    w = (torch.randn(8, 3, 3, 16, generator=g) * 0.3).to(torch.bfloat16)
    b = torch.randn(8, generator=g)
    z = orc.dense_conv_f64(x, w, b)
    y = orc.dense_conv(x, w, b)
    assert np.array_equal(y.view(torch.int16).numpy().view(np.uint16), orc.round_bf16(z))
    xf, wf = x.float(), w.float()
    assert np.array_equal(orc.dense_conv(xf, wf, b).numpy(), orc.dense_conv_f64(xf, wf, b).astype(np.float32))


# ------------------------------------------------------------------ sparse layer

def _tile_cover(idx, b, Ho, Wo):
    cov = np.zeros((Ho, Wo), bool)
    for h0, w0 in idx:
        cov[h0:h0 + b, w0:w0 + b] = True
    return cov


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_sparse_conv_invariants(orc, dtype):
    L = inputs.make_conv_case(10, 24, 20, 16, 8, dtype=dtype, block=4, area=0.05)
    yc = orc.dense_conv(L.x_orig, L.weight, L.bias)
    ye = orc.dense_conv(L.x_edit, L.weight, L.bias)
    Ho, Wo = yc.shape[1:3]
    # empty list: the cache, bit for bit
    empty = np.zeros((0, 2), np.int32)
    assert torch.equal(orc.sparse_conv(L.x_edit, L.weight, L.bias, empty, yc, block=4).view(torch.int8),
                       yc.view(torch.int8))
    # all tiles: the dense layer of the edited input
    allt = np.array([(i, j) for i in range(0, Ho, 4) for j in range(0, Wo, 4)], np.int32)
    assert torch.equal(orc.sparse_conv(L.x_edit, L.weight, L.bias, allt, yc, block=4), ye)
    # arbitrary list: cache outside, dense(edited) inside
    rng = np.random.default_rng(0)
    sub = allt[rng.random(len(allt)) < 0.3]
    ys = orc.sparse_conv(L.x_edit, L.weight, L.bias, sub, yc, block=4)
    cov = torch.from_numpy(_tile_cover(sub, 4, Ho, Wo))[None, :, :, None].expand_as(ys)
    assert torch.equal(ys[~cov], yc[~cov]) and torch.equal(ys[cov], ye[cov])


@pytest.mark.parametrize("b,stride,k", [(4, 1, 3), (2, 1, 3), (1, 1, 3), (8, 1, 3), (4, 2, 3), (4, 1, 1)])
def test_single_layer_exact_with_dilation(orc, b, stride, k):
    # With one-tile dilation, the tile-masked layer equals the dense layer of
    # the edited input at every pixel: outside active tiles no input in the
    # receptive field changed, so the cached value is the same double sum.
    pad = k // 2
    L = inputs.make_conv_case(11 + b, 32, 32, 8, 8, kernel=k, stride=stride, pad=pad, block=b, area=0.03)
    yc = orc.dense_conv(L.x_orig, L.weight, L.bias, k, stride, pad)
    ye = orc.dense_conv(L.x_edit, L.weight, L.bias, k, stride, pad)
    Ho, Wo = yc.shape[1:3]
    idx = orc.reduce_mask(L.x_orig, L.x_edit, 1e-3, [(Ho, Wo, b)], 1)[0]
    assert 0 < len(idx) < ((Ho + b - 1) // b) * ((Wo + b - 1) // b)
    ys = orc.sparse_conv(L.x_edit, L.weight, L.bias, idx, yc, k, stride, pad, b)
    assert torch.equal(ys, ye)


def test_linearity_identity(orc):
    # F(A_e) - F(A_o) = W * (A_e - A_o) for a conv without bias (mer.dev notes,
    # section 3.1).  Values on a dyadic grid so every difference is exact.
    rng = np.random.default_rng(12)
    q = 2.0 ** -10
    xo = torch.from_numpy((rng.integers(-4000, 4000, size=(1, 12, 12, 8)) * q).astype(np.float32))
    d = np.zeros((1, 12, 12, 8))
    d[0, 3:7, 5:9] = rng.integers(-500, 500, size=(4, 4, 8)) * q
    xe = xo + torch.from_numpy(d.astype(np.float32))
    w = torch.from_numpy((rng.integers(-64, 64, size=(8, 3, 3, 8)) * 2.0 ** -6).astype(np.float32))
    b = torch.randn(8)
    lhs = orc.dense_conv_f64(xe, w, b) - orc.dense_conv_f64(xo, w, b)
    rhs = orc.dense_conv_f64(xe - xo, w, None)
    assert np.allclose(lhs, rhs, rtol=0, atol=1e-12)
    # the difference vanishes more than one pixel away from the edit
    far = np.ones((12, 12), bool)
    far[2:8, 4:10] = False
    assert np.all(rhs[0][far] == 0)


# ------------------------------------------------------------------ gather / block conv

def test_gather_definition_and_overlap(orc):
    L = inputs.make_conv_case(13, 16, 16, 8, 8, dtype=torch.float32, block=4)
    idx = np.array([(0, 0), (0, 4), (4, 4), (12, 12)], np.int32)
    blk = orc.gather(L.x_edit, idx, 3, 1, 1, 4)
    assert blk.shape == (4, 1, 6, 6, 8)
    xp = F.pad(L.x_edit.double().permute(0, 3, 1, 2), (1, 1, 1, 1)).permute(0, 2, 3, 1).numpy()
    for t, (h0, w0) in enumerate(idx):
        assert np.array_equal(blk[t, 0], xp[0, h0:h0 + 6, w0:w0 + 6])
    # horizontally adjacent tiles share a 2-pixel-wide strip
    assert np.array_equal(blk[0, 0, :, 4:6], blk[1, 0, :, 0:2])


def test_block_conv_then_place_equals_sparse_conv(orc):
    # gather -> valid conv per block -> bias, round, place == tile-masked layer
    L = inputs.make_conv_case(14, 20, 20, 16, 8, dtype=torch.bfloat16, block=4, gn=True)
    gn = orc.gn_affine(L.x_orig, 8, L.gn_gamma, L.gn_beta)
    yc = orc.dense_conv(L.x_orig, L.weight, L.bias, gn=gn, silu=True)
    idx = np.array([(0, 0), (4, 8), (16, 16), (8, 0)], np.int32)
    blk = orc.gather(L.x_edit, idx, 3, 1, 1, 4, gn=gn, silu=True)
    out = orc.block_conv(blk.reshape(-1, 6, 6, 16), L.weight, 3, 1, 4) + L.bias.double().numpy()
    ys = orc.sparse_conv(L.x_edit, L.weight, L.bias, idx, yc, block=4, gn=gn, silu=True)
    for t, (h0, w0) in enumerate(idx):
        want = orc.round_bf16(out[t])
        got = ys[0, h0:h0 + 4, w0:w0 + 4].contiguous().view(torch.int16).numpy().view(np.uint16)
        assert np.array_equal(got, want)


# ------------------------------------------------------------------ res block

def test_resblock_all_and_empty(orc):
    blk = inputs.make_cfg3(0, H=16, W=16, C=64, area=0.05)
    gn1 = orc.gn_affine(blk.x_orig, 32, blk.g1, blk.be1)
    y1o = orc.dense_conv(blk.x_orig, blk.w1, blk.b1, gn=gn1, silu=True)
    gn2 = orc.gn_affine(y1o, 32, blk.g2, blk.be2)
    y1o, outo = orc.resblock_dense(blk.x_orig, blk, gn1, gn2)
    y1e, oute = orc.resblock_dense(blk.x_edit, blk, gn1, gn2)
    allt = np.array([(i, j) for i in range(0, 16, 8) for j in range(0, 16, 8)], np.int32)
    y1s, outs = orc.resblock_sparse(blk.x_edit, blk, allt, y1o, outo, gn1, gn2)
    assert torch.equal(y1s, y1e) and torch.equal(outs, oute)
    y1s, outs = orc.resblock_sparse(blk.x_edit, blk, np.zeros((0, 2), np.int32), y1o, outo, gn1, gn2)
    assert torch.equal(y1s, y1o) and torch.equal(outs, outo)


def test_resblock_dense_matches_torch_f32(orc):
    g = torch.Generator().manual_seed(15)
    C = 64
    x = torch.randn(1, 10, 10, C, generator=g)

    class B:  # f32 copy of a res block's parameters
        pass
    blk = B()
    blk.w1, blk.w2 = torch.randn(C, 3, 3, C, generator=g) * 0.04, torch.randn(C, 3, 3, C, generator=g) * 0.04
    blk.b1, blk.b2 = torch.randn(C, generator=g) * 0.1, torch.randn(C, generator=g) * 0.1
    g1, be1 = 1 + 0.1 * torch.randn(C, generator=g), 0.1 * torch.randn(C, generator=g)
    g2, be2 = 1 + 0.1 * torch.randn(C, generator=g), 0.1 * torch.randn(C, generator=g)
    gn1 = orc.gn_affine(x, 32, g1, be1)
    y1 = orc.dense_conv(x, blk.w1, blk.b1, gn=gn1, silu=True)
    gn2 = orc.gn_affine(y1, 32, g2, be2)
    _, out = orc.resblock_dense(x, blk, gn1, gn2)
    xd = x.double().permute(0, 3, 1, 2)
    h = F.conv2d(F.silu(F.group_norm(xd, 32, g1.double(), be1.double(), 1e-5)),
                 blk.w1.double().permute(0, 3, 1, 2), blk.b1.double(), padding=1)
    h = h.float().double()   # y1 is stored in the layer dtype between the convs
    h2 = F.conv2d(F.silu(F.group_norm(h, 32, g2.double(), be2.double(), 1e-5)),
                  blk.w2.double().permute(0, 3, 1, 2), blk.b2.double(), padding=1) + xd
    ref = h2.permute(0, 2, 3, 1).float()
    assert torch.allclose(out, ref, rtol=1e-5, atol=1e-5)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_sparse_conv_ragged_edge_tiles(orc, dtype):
    # 10x10 output with 4x4 tiles: the last tile row/col is 2 pixels wide and
    # must be clipped at the border (batch of 2, so a spill would land in the
    # next image).
    L = inputs.make_conv_case(16, 10, 10, 8, 8, dtype=dtype, block=4, area=0.05, N=2)
    yc = orc.dense_conv(L.x_orig, L.weight, L.bias)
    ye = orc.dense_conv(L.x_edit, L.weight, L.bias)
    allt = np.array([(i, j) for i in range(0, 10, 4) for j in range(0, 10, 4)], np.int32)
    assert torch.equal(orc.sparse_conv(L.x_edit, L.weight, L.bias, allt, yc, block=4), ye)
    corner = np.array([(8, 8)], np.int32)
    ys = orc.sparse_conv(L.x_edit, L.weight, L.bias, corner, yc, block=4)
    cov = torch.zeros_like(ys, dtype=torch.bool)
    cov[:, 8:10, 8:10, :] = True
    assert torch.equal(ys[cov], ye[cov]) and torch.equal(ys[~cov], yc[~cov])


def test_gather_stride2_definition(orc):
    L = inputs.make_conv_case(17, 15, 13, 8, 8, dtype=torch.float32, block=4, stride=2)
    idx = np.array([(0, 0), (0, 4), (4, 0), (4, 4)], np.int32)
    blk = orc.gather(L.x_edit, idx, 3, 2, 1, 4)
    assert blk.shape == (4, 1, 9, 9, 8)          # b_in = (b - 1) * s + k
    xp = F.pad(L.x_edit.double().permute(0, 3, 1, 2), (1, 10, 1, 10)).permute(0, 2, 3, 1).numpy()
    for t, (h0, w0) in enumerate(idx):
        assert np.array_equal(blk[t, 0], xp[0, 2 * h0:2 * h0 + 9, 2 * w0:2 * w0 + 9])
    # stride-2 neighbours overlap by k - s = 1 pixel
    assert np.array_equal(blk[0, 0, :, 8:9], blk[1, 0, :, 0:1])
    # valid conv of the blocks == the dense stride-2 layer at those tiles
    out = orc.block_conv(blk.reshape(-1, 9, 9, 8), L.weight, 3, 2, 4)
    ref = orc.dense_conv_f64(L.x_edit, L.weight, None, 3, 2, 1)
    for t, (h0, w0) in enumerate(idx):
        hi, wi = min(h0 + 4, ref.shape[1]), min(w0 + 4, ref.shape[2])
        assert np.allclose(out[t, :hi - h0, :wi - w0], ref[0, h0:hi, w0:wi], rtol=0, atol=1e-12)


def test_restore_tiles_copies_listed_regions_only(orc):
    # hand-checkable: a 5x5 image, 2x2 tiles at (0, 0) and the clipped corner (4, 4)
    src = torch.arange(2 * 5 * 5 * 3, dtype=torch.float32).reshape(2, 5, 5, 3)
    dst = -torch.ones_like(src)
    got = orc.restore_tiles(src, dst, 2, np.array([[0, 0], [4, 4]], np.int32))
    want = dst.clone()
    for (y, x) in [(0, 0), (0, 1), (1, 0), (1, 1), (4, 4)]:
        want[:, y, x, :] = src[:, y, x, :]
    assert torch.equal(got, want)
    assert int((got != dst).sum()) == 2 * 5 * 3   # exactly 5 pixels x 2 batch x 3 channels changed
    # an empty list leaves dst as it is; restoring src onto itself is the identity
    assert torch.equal(orc.restore_tiles(src, dst, 2, np.zeros((0, 2), np.int32)), dst)
    assert torch.equal(orc.restore_tiles(src, src, 3, np.array([[0, 3]], np.int32)), src)


# ------------------------------------------------------------------ pixel-level dilation

def _px_tiles_brute(m, Hs, Ws, b, R):
    # a tile is active iff some set pixel of the downsampled mask lies within
    # Chebyshev distance R of one of the tile's pixels (independent of dilate())
    H, W = m.shape
    fy, fx = H // Hs, W // Ws
    ms = m.reshape(Hs, fy, Ws, fx).max(axis=(1, 3))
    ys, xs = np.nonzero(ms)
    out = []
    for i in range(0, Hs, b):
        for j in range(0, Ws, b):
            y1, x1 = min(i + b, Hs) - 1, min(j + b, Ws) - 1
            dy = np.maximum(0, np.maximum(i - ys, ys - y1))
            dx = np.maximum(0, np.maximum(j - xs, xs - x1))
            if len(ys) and (np.maximum(dy, dx) <= R).any():
                out.append((i, j))
    return np.array(out, np.int32).reshape(-1, 2)


@pytest.mark.parametrize("R", [0, 1, 2, 5])
def test_pixel_dilation_lists_brute_force(orc, R):
    rng = np.random.default_rng(100 + R)
    for case in range(60):
        H, W = int(rng.integers(2, 20)) * 2, int(rng.integers(2, 20)) * 2
        a = torch.from_numpy(rng.normal(size=(1, H, W, 4)).astype(np.float32))
        e = a.clone()
        m = rng.random((H, W)) < rng.choice([0.01, 0.05, 0.2])
        e[0, torch.from_numpy(m)] += 1.0
        for (Hs, Ws, b) in [(H, W, int(rng.integers(1, 6))), (H // 2, W // 2, int(rng.integers(1, 4)))]:
            got = orc.reduce_mask_px(a, e, 1e-3, [(Hs, Ws, b)], R)[0]
            want = _px_tiles_brute(m.astype(np.uint8), Hs, Ws, b, R)
            assert np.array_equal(got, want), (case, Hs, Ws, b, R)


def test_pixel_dilation_between_raw_and_tile_dilation(orc):
    L = inputs.make_conv_case(41, 64, 64, 8, 8, block=4, area=0.03)
    sc = [(64, 64, 4)]
    raw = {tuple(t) for t in orc.reduce_mask_px(L.x_orig, L.x_edit, 1e-3, sc, 0)[0]}
    px = {tuple(t) for t in orc.reduce_mask_px(L.x_orig, L.x_edit, 1e-3, sc, 1)[0]}
    tile = {tuple(t) for t in orc.reduce_mask(L.x_orig, L.x_edit, 1e-3, sc, 1)[0]}
    assert raw <= px <= tile and len(px) < len(tile)


@pytest.mark.parametrize("b,k", [(4, 3), (8, 3), (2, 3), (4, 1)])
def test_single_layer_exact_with_pixel_dilation(orc, b, k):
    # dilating by the conv's halo (k // 2 pixels) is enough for the sparse
    # layer to equal the dense layer of the edited input at every pixel
    pad = k // 2
    L = inputs.make_conv_case(13 + b, 32, 32, 8, 8, kernel=k, stride=1, pad=pad, block=b, area=0.03)
    yc = orc.dense_conv(L.x_orig, L.weight, L.bias, k, 1, pad)
    ye = orc.dense_conv(L.x_edit, L.weight, L.bias, k, 1, pad)
    idx = orc.reduce_mask_px(L.x_orig, L.x_edit, 1e-3, [(32, 32, b)], pad)[0]
    ys = orc.sparse_conv(L.x_edit, L.weight, L.bias, idx, yc, k, 1, pad, b)
    assert torch.equal(ys, ye)


def test_resblock_exact_with_two_pixel_dilation(orc):
    # two chained 3x3 convs move the change by 2 pixels; with that dilation the
    # sparse block equals the dense block of the edited input (cached GN stats)
    blk = inputs.make_cfg3(3, H=32, W=32, C=64, area=0.03)
    gn1 = orc.gn_affine(blk.x_orig, 32, blk.g1, blk.be1)
    y1o = orc.dense_conv(blk.x_orig, blk.w1, blk.b1, gn=gn1, silu=True)
    gn2 = orc.gn_affine(y1o, 32, blk.g2, blk.be2)
    y1o, outo = orc.resblock_dense(blk.x_orig, blk, gn1, gn2)
    y1e, oute = orc.resblock_dense(blk.x_edit, blk, gn1, gn2)
    idx = orc.reduce_mask_px(blk.x_orig, blk.x_edit, 1e-3, [(32, 32, blk.block)], 2)[0]
    assert 0 < len(idx) < 16
    y1s, outs = orc.resblock_sparse(blk.x_edit, blk, idx, y1o, outo, gn1, gn2)
    assert torch.equal(outs, oute)
