"""CPU oracle for the SIGE sparse-conv hot path (test infrastructure only).

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg may import this package.  It loads ``liboracle.so`` built from
``sige_oracle.c`` (plain C, double precision) and wraps it for numpy / CPU
torch tensors.  It shares no code with the CUDA library.

Citations name the source page and its section:
  * mer.dev notes on "Efficient Spatially Sparse Inference for Conditional
    GANs and Diffusion Models", sections 3 "Method", 3.1 "Activation
    Sparsity", 3.2 "Sparse Engine SIGE";
  * SIGE project page (dongaigc.com mirror of the project README),
    "Overview" (the tile-based sparse convolution).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sige_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

U8, F32, BF16 = 0, 1, 2
NHWC, NCHW = 0, 1

_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, OpenMP, no FP contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
                               "-fPIC", "-shared", "-std=c11", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        vp, i32, f32, f64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_double
        L.oracle_round_bf16_one.restype = ctypes.c_uint16
        L.oracle_round_bf16_one.argtypes = [f64]
        L.oracle_round_bf16.argtypes = [vp, vp, ctypes.c_long]
        L.oracle_pixel_mask.argtypes = [vp, vp, i32, i32, i32, i32, i32, i32, f32, vp]
        L.oracle_downsample.argtypes = [vp, i32, i32, i32, i32, vp]
        L.oracle_dilate.argtypes = [vp, i32, i32, i32, vp]
        L.oracle_reduce_scale.restype = i32
        L.oracle_reduce_scale.argtypes = [vp, i32, i32, i32, i32, i32, i32, vp, i32]
        L.oracle_gn_affine.argtypes = [vp, i32, i32, i32, i32, i32, i32, vp, vp, f64, vp, vp]
        conv_common = [vp, i32, i32, i32, i32, i32, vp, vp, i32, i32, i32, i32]
        L.oracle_dense_conv_f64.argtypes = conv_common + [vp, vp, i32, vp, vp]
        L.oracle_dense_conv.argtypes = conv_common + [vp, vp, i32, vp, vp]
        L.oracle_sparse_conv.argtypes = conv_common + [i32, vp, i32, vp, vp, i32, vp, vp, vp]
        L.oracle_gather.argtypes = [vp, i32, i32, i32, i32, i32, i32, i32, i32, i32, vp, i32, vp, vp, i32, vp]
        L.oracle_block_conv.argtypes = [vp, i32, i32, vp, i32, i32, i32, i32, i32, vp]
        L.oracle_conv_transpose_f64.argtypes = [vp, i32, i32, i32, i32, i32, vp, vp, i32, i32, i32, i32, i32,
                                                vp, vp, i32, vp, vp]
        L.oracle_sparse_conv_transpose.argtypes = [vp, i32, i32, i32, i32, i32, vp, vp, i32, i32, i32, i32, i32,
                                                   i32, vp, i32, vp, vp, i32, vp, vp, vp]
        L.oracle_spade_conv.argtypes = [vp, i32, i32, i32, i32, i32, vp, vp, i32, i32, i32, i32, vp, vp, vp, vp,
                                        i32, vp, i32, vp, i32, vp, vp, vp]
        _lib = L
    return _lib


def set_threads(n: int) -> None:
    """OpenMP thread count for the oracle's parallel loops."""
    lib()
    try:
        omp = ctypes.CDLL("libgomp.so.1")
        omp.omp_set_num_threads(int(n))
    except OSError:
        os.environ["OMP_NUM_THREADS"] = str(n)


# ----------------------------------------------------------------- marshalling

def _dtype_code(t: torch.Tensor) -> int:
    return {torch.uint8: U8, torch.float32: F32, torch.bfloat16: BF16}[t.dtype]


def _c(t: torch.Tensor) -> torch.Tensor:
    assert t.device.type == "cpu"
    return t.contiguous()


def _p(t):
    if t is None:
        return None
    if isinstance(t, np.ndarray):
        return t.ctypes.data_as(ctypes.c_void_p)
    return ctypes.c_void_p(t.data_ptr())


def round_bf16(values) -> np.ndarray:
    """Round float64 values to bf16 (ties to even) in one step; returns uint16 bits."""
    v = np.ascontiguousarray(np.asarray(values, dtype=np.float64))
    out = np.empty(v.shape, dtype=np.uint16)
    lib().oracle_round_bf16(_p(v), _p(out), v.size)
    return out


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint32) << 16).view(np.float32).astype(np.float64)


def pixel_mask(a_orig: torch.Tensor, a_edit: torch.Tensor, threshold: float, layout: int = NHWC) -> np.ndarray:
    """m[y][x] = OR over n of (max_c |A_edit - A_orig| > threshold), as uint8 [H, W]."""
    a, b = _c(a_orig), _c(a_edit)
    if layout == NHWC:
        N, H, W, C = a.shape
    else:
        N, C, H, W = a.shape
    m = np.zeros((H, W), dtype=np.uint8)
    lib().oracle_pixel_mask(_p(a), _p(b), N, H, W, C, _dtype_code(a), layout, float(threshold), _p(m))
    return m


def downsample(m: np.ndarray, Hs: int, Ws: int) -> np.ndarray:
    m = np.ascontiguousarray(m, dtype=np.uint8)
    out = np.zeros((Hs, Ws), dtype=np.uint8)
    lib().oracle_downsample(_p(m), m.shape[0], m.shape[1], Hs, Ws, _p(out))
    return out


def dilate(m: np.ndarray, R: int) -> np.ndarray:
    m = np.ascontiguousarray(m, dtype=np.uint8)
    out = np.zeros_like(m)
    lib().oracle_dilate(_p(m), m.shape[0], m.shape[1], R, _p(out))
    return out


def reduce_scale(mask: np.ndarray, Hs: int, Ws: int, block: int, dilate_tiles: int = 1,
                 capacity: int | None = None) -> np.ndarray:
    """Active-tile origins (row, col) at scale (Hs, Ws), row-major, int32 [count, 2]."""
    mask = np.ascontiguousarray(mask, dtype=np.uint8)
    H, W = mask.shape
    ntiles = ((Hs + block - 1) // block) * ((Ws + block - 1) // block)
    cap = ntiles if capacity is None else capacity
    idx = np.zeros((max(cap, 1), 2), dtype=np.int32)
    n = lib().oracle_reduce_scale(_p(mask), H, W, Hs, Ws, block, dilate_tiles, _p(idx), cap)
    return idx[:min(n, cap)].copy() if capacity is not None else idx[:n].copy()


def reduce_mask(a_orig, a_edit, threshold, scales, dilate_tiles=1, layout=NHWC):
    """Full reduction: pixel mask, then one index list per (Hs, Ws, block) scale."""
    m = pixel_mask(a_orig, a_edit, threshold, layout)
    return [reduce_scale(m, Hs, Ws, b, dilate_tiles) for (Hs, Ws, b) in scales]


def reduce_mask_px(a_orig, a_edit, threshold, scales, radius=1, layout=NHWC):
    """Pixel-level dilation (mer.dev notes, section 3.2: dilate, then select
    tiles): per scale, OR-downsample the pixel mask, dilate it by a square of
    ``radius`` pixels at that scale, then list the b x b tiles holding a set
    pixel (no tile dilation)."""
    m = pixel_mask(a_orig, a_edit, threshold, layout)
    out = []
    for (Hs, Ws, b) in scales:
        md = dilate(downsample(m, Hs, Ws), radius)
        out.append(reduce_scale(md, Hs, Ws, b, 0))
    return out


def gn_affine(x: torch.Tensor, groups: int, gamma: torch.Tensor, beta: torch.Tensor, eps: float = 1e-5):
    """Per-(n, channel) scale and shift (float64 [N, C]) folding GroupNorm of ``x``."""
    x = _c(x)
    N, H, W, C = x.shape
    sc = np.zeros((N, C), dtype=np.float64)
    sh = np.zeros((N, C), dtype=np.float64)
    lib().oracle_gn_affine(_p(x), N, H, W, C, _dtype_code(x), groups, _p(_c(gamma.float())),
                           _p(_c(beta.float())), float(eps), _p(sc), _p(sh))
    return sc, sh


def _conv_args(x, w, bias, k, stride, pad):
    x, w = _c(x), _c(w)
    N, H, W, Cin = x.shape
    Cout = w.shape[0]
    assert w.shape == (Cout, k, k, Cin) and w.dtype == x.dtype
    Ho = (H + 2 * pad - k) // stride + 1
    Wo = (W + 2 * pad - k) // stride + 1
    b = None if bias is None else _c(bias.float())
    return x, w, b, (N, H, W, Cin, Cout, Ho, Wo)


def _gn(gn):
    if gn is None:
        return None, None
    sc, sh = gn
    return np.ascontiguousarray(sc, dtype=np.float64), np.ascontiguousarray(sh, dtype=np.float64)


def dense_conv_f64(x, w, bias=None, k=3, stride=1, pad=1, gn=None, silu=False, residual=None) -> np.ndarray:
    """Dense layer in double, unrounded: float64 [N, Ho, Wo, C_out]."""
    x, w, b, (N, H, W, Cin, Cout, Ho, Wo) = _conv_args(x, w, bias, k, stride, pad)
    sc, sh = _gn(gn)
    r = None if residual is None else _c(residual)
    z = np.zeros((N, Ho, Wo, Cout), dtype=np.float64)
    lib().oracle_dense_conv_f64(_p(x), N, H, W, Cin, _dtype_code(x), _p(w), _p(b), Cout, k, stride, pad,
                                _p(sc), _p(sh), int(silu), _p(r), _p(z))
    return z


def dense_conv(x, w, bias=None, k=3, stride=1, pad=1, gn=None, silu=False, residual=None) -> torch.Tensor:
    """Dense layer rounded once to x's dtype: [N, Ho, Wo, C_out]."""
    x, w, b, (N, H, W, Cin, Cout, Ho, Wo) = _conv_args(x, w, bias, k, stride, pad)
    sc, sh = _gn(gn)
    r = None if residual is None else _c(residual)
    y = torch.empty((N, Ho, Wo, Cout), dtype=x.dtype)
    lib().oracle_dense_conv(_p(x), N, H, W, Cin, _dtype_code(x), _p(w), _p(b), Cout, k, stride, pad,
                            _p(sc), _p(sh), int(silu), _p(r), _p(y))
    return y


def sparse_conv(x_edit, w, bias, idx: np.ndarray, y_cached: torch.Tensor, k=3, stride=1, pad=1,
                block=4, gn=None, silu=False, residual=None) -> torch.Tensor:
    """Tile-masked layer: the cached output, overwritten at the pixels of the
    listed tiles by the layer applied to ``x_edit`` (SIGE project page, "Overview")."""
    x, w, b, (N, H, W, Cin, Cout, Ho, Wo) = _conv_args(x_edit, w, bias, k, stride, pad)
    sc, sh = _gn(gn)
    r = None if residual is None else _c(residual)
    yc = _c(y_cached)
    assert yc.shape == (N, Ho, Wo, Cout) and yc.dtype == x.dtype
    idx = np.ascontiguousarray(idx, dtype=np.int32).reshape(-1, 2)
    y = torch.empty_like(yc)
    lib().oracle_sparse_conv(_p(x), N, H, W, Cin, _dtype_code(x), _p(w), _p(b), Cout, k, stride, pad,
                             block, _p(idx), len(idx), _p(sc), _p(sh), int(silu), _p(r), _p(yc), _p(y))
    return y


def resblock_dense(x, blk, gn1, gn2):
    """Dense res block: y1 = conv1(silu(gn1(x))) + b1; out = conv2(silu(gn2(y1))) + b2 + x."""
    y1 = dense_conv(x, blk.w1, blk.b1, 3, 1, 1, gn=gn1, silu=True)
    out = dense_conv(y1, blk.w2, blk.b2, 3, 1, 1, gn=gn2, silu=True, residual=x)
    return y1, out


def resblock_sparse(x_edit, blk, idx, y1_cached, out_cached, gn1, gn2):
    """Sparse res block, both convs on the same tile list; y1 is the cached
    y1 overwritten on the listed tiles, and feeds conv2."""
    y1 = sparse_conv(x_edit, blk.w1, blk.b1, idx, y1_cached, 3, 1, 1, blk.block, gn=gn1, silu=True)
    out = sparse_conv(y1, blk.w2, blk.b2, idx, out_cached, 3, 1, 1, blk.block, gn=gn2, silu=True,
                      residual=x_edit)
    return y1, out


def gather(x, idx, k=3, stride=1, pad=1, block=4, gn=None, silu=False) -> np.ndarray:
    """Stacked halo'd blocks, float64 [count, N, b_in, b_in, C_in] (SIGE project page, "Overview")."""
    x = _c(x)
    N, H, W, Cin = x.shape
    idx = np.ascontiguousarray(idx, dtype=np.int32).reshape(-1, 2)
    bin_ = (block - 1) * stride + k
    out = np.zeros((len(idx), N, bin_, bin_, Cin), dtype=np.float64)
    sc, sh = _gn(gn)
    lib().oracle_gather(_p(x), N, H, W, Cin, _dtype_code(x), k, stride, pad, block, _p(idx), len(idx),
                        _p(sc), _p(sh), int(silu), _p(out))
    return out


def block_conv(blocks: np.ndarray, w: torch.Tensor, k=3, stride=1, block=4) -> np.ndarray:
    """Valid conv of each stacked block, float64 [nblocks, b, b, C_out] (no bias)."""
    w = _c(w)
    Cout, Cin = w.shape[0], w.shape[3]
    blocks = np.ascontiguousarray(blocks, dtype=np.float64)
    nb = blocks.size // (((block - 1) * stride + k) ** 2 * Cin)
    out = np.zeros((nb, block, block, Cout), dtype=np.float64)
    lib().oracle_block_conv(_p(blocks), nb, Cin, _p(w), _dtype_code(w), Cout, k, stride, block, _p(out))
    return out


def restore_tiles(src: torch.Tensor, dst: torch.Tensor, block: int, idx: np.ndarray) -> torch.Tensor:
    """Sequential edits (SIGE project page, "Overview": the cache of F_l(A_original)
    is updated in place): the tiles (h0, w0) of ``idx`` are put back from ``src``
    into a copy of ``dst``, clipped at the border; every other element keeps
    dst's value.  A plain copy, written out pixel by pixel."""
    out = dst.clone()
    N, H, W, _ = dst.shape
    for h0, w0 in np.asarray(idx, dtype=np.int64).reshape(-1, 2):
        for i in range(block):
            for j in range(block):
                y, x = int(h0) + i, int(w0) + j
                if y < H and x < W:
                    out[:, y, x, :] = src[:, y, x, :]
    return out


# ------------------------------------------------------- other layer types

def conv_transpose_out_hw(H, W, k=3, stride=2, pad=1, output_padding=1):
    return (H - 1) * stride - 2 * pad + k + output_padding, (W - 1) * stride - 2 * pad + k + output_padding


def conv_transpose_f64(x, w, bias=None, k=3, stride=2, pad=1, output_padding=1, gn=None, silu=False,
                       residual=None) -> np.ndarray:
    """Transposed conv (learned upsampling), unrounded float64 [N, Ho, Wo, C_out].
    ``w`` is [C_out, k, k, C_in]: w[o, r, c, ci] couples input channel ci to
    output channel o at tap (r, c); input pixel (i, j) feeds output pixel
    (i*stride - pad + r, j*stride - pad + c)."""
    x, w = _c(x), _c(w)
    N, H, W, Cin = x.shape
    Cout = w.shape[0]
    assert w.shape == (Cout, k, k, Cin) and w.dtype == x.dtype
    Ho, Wo = conv_transpose_out_hw(H, W, k, stride, pad, output_padding)
    b = None if bias is None else _c(bias.float())
    sc, sh = _gn(gn)
    r = None if residual is None else _c(residual)
    z = np.zeros((N, Ho, Wo, Cout), dtype=np.float64)
    lib().oracle_conv_transpose_f64(_p(x), N, H, W, Cin, _dtype_code(x), _p(w), _p(b), Cout, k, stride, pad,
                                    output_padding, _p(sc), _p(sh), int(silu), _p(r), _p(z))
    return z


def sparse_conv_transpose(x_edit, w, bias, idx, y_cached, k=3, stride=2, pad=1, output_padding=1, block=4,
                          gn=None, silu=False, residual=None) -> torch.Tensor:
    """Tile-masked transposed conv: the cached output, overwritten at the pixels
    of the listed output tiles (output resolution) by the layer on ``x_edit``."""
    x, w = _c(x_edit), _c(w)
    N, H, W, Cin = x.shape
    Cout = w.shape[0]
    yc = _c(y_cached)
    Ho, Wo = conv_transpose_out_hw(H, W, k, stride, pad, output_padding)
    assert yc.shape == (N, Ho, Wo, Cout) and yc.dtype == x.dtype
    b = None if bias is None else _c(bias.float())
    sc, sh = _gn(gn)
    r = None if residual is None else _c(residual)
    idx = np.ascontiguousarray(idx, dtype=np.int32).reshape(-1, 2)
    y = torch.empty_like(yc)
    lib().oracle_sparse_conv_transpose(_p(x), N, H, W, Cin, _dtype_code(x), _p(w), _p(b), Cout, k, stride, pad,
                                       output_padding, block, _p(idx), len(idx), _p(sc), _p(sh), int(silu), _p(r),
                                       _p(yc), _p(y))
    return y


ACT_NONE, ACT_SILU, ACT_LEAKY = 0, 1, 2


def spade_conv(x, w, bias, norm, gamma, beta, act=ACT_LEAKY, k=3, stride=1, pad=1, residual=None, idx=None,
               block=4, y_cached=None, rounded=True):
    """Conv of a SPADE-style input: act((x * scale + shift) * (1 + gamma) + beta)
    with (scale, shift) = ``norm`` per (n, channel) and gamma / beta per pixel
    (NHWC maps of x's shape and dtype).  Dense (idx None) or tile-masked into
    ``y_cached``; rounded once to x's dtype, or unrounded float64 when
    ``rounded`` is False (dense only)."""
    x, w = _c(x), _c(w)
    N, H, W, Cin = x.shape
    Cout = w.shape[0]
    assert w.shape == (Cout, k, k, Cin) and w.dtype == x.dtype
    g, be = _c(gamma), _c(beta)
    assert g.shape == x.shape and be.shape == x.shape and g.dtype == x.dtype and be.dtype == x.dtype
    Ho = (H + 2 * pad - k) // stride + 1
    Wo = (W + 2 * pad - k) // stride + 1
    b = None if bias is None else _c(bias.float())
    sc, sh = _gn(norm)
    r = None if residual is None else _c(residual)
    if idx is None and not rounded:
        z = np.zeros((N, Ho, Wo, Cout), dtype=np.float64)
        lib().oracle_spade_conv(_p(x), N, H, W, Cin, _dtype_code(x), _p(w), _p(b), Cout, k, stride, pad, _p(sc),
                                _p(sh), _p(g), _p(be), int(act), _p(r), block, None, 0, None, _p(z), None)
        return z
    if idx is None:
        y = torch.empty((N, Ho, Wo, Cout), dtype=x.dtype)
        lib().oracle_spade_conv(_p(x), N, H, W, Cin, _dtype_code(x), _p(w), _p(b), Cout, k, stride, pad, _p(sc),
                                _p(sh), _p(g), _p(be), int(act), _p(r), block, None, 0, None, None, _p(y))
        return y
    yc = _c(y_cached)
    assert yc.shape == (N, Ho, Wo, Cout) and yc.dtype == x.dtype
    idx = np.ascontiguousarray(idx, dtype=np.int32).reshape(-1, 2)
    y = torch.empty_like(yc)
    lib().oracle_spade_conv(_p(x), N, H, W, Cin, _dtype_code(x), _p(w), _p(b), Cout, k, stride, pad, _p(sc),
                            _p(sh), _p(g), _p(be), int(act), _p(r), block, _p(idx), len(idx), _p(yc), None, _p(y))
    return y
