"""Python binding of libsige (the C ABI in include/sige.h).

Argument marshalling only: every step of the sparse layer runs in the CUDA
kernels of ``libsige.so``; torch supplies device memory and streams.  The
functions carry the ABI's names and raise ``SigeError`` on any non-OK status.
There is no fallback: if the library is missing, importing a call raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libsige.so")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_CAPACITY, ERR_TIMEOUT, ERR_WORKSPACE = 0, -1, -2, -3, -4, -5, -6
CALL_REDUCE_MASK, CALL_SPARSE_CONV, CALL_CONV_FUSED, CALL_DENSE_CONV, CALL_RESBLOCK = 0, 1, 2, 3, 4
U8, F32, BF16 = 0, 1, 2
NHWC, NCHW = 0, 1
WORKSPACE_HEADER = 256
MAX_SCALES = 8

_DT = {torch.uint8: U8, torch.float32: F32, torch.bfloat16: BF16}


class SigeError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} ({status})")


class TensorDesc(ctypes.Structure):
    _fields_ = [("n", ctypes.c_int32), ("h", ctypes.c_int32), ("w", ctypes.c_int32), ("c", ctypes.c_int32),
                ("dtype", ctypes.c_int32), ("layout", ctypes.c_int32)]


class ConvDesc(ctypes.Structure):
    _fields_ = [("kernel", ctypes.c_int32), ("stride", ctypes.c_int32), ("pad", ctypes.c_int32),
                ("c_in", ctypes.c_int32), ("c_out", ctypes.c_int32), ("block", ctypes.c_int32)]


class LayerExt(ctypes.Structure):
    _fields_ = [("transposed", ctypes.c_int32), ("output_padding", ctypes.c_int32),
                ("spade_gamma", ctypes.c_void_p), ("spade_beta", ctypes.c_void_p), ("act", ctypes.c_int32)]


ACT_NONE, ACT_SILU, ACT_LEAKY = 0, 1, 2


class ScaleDesc(ctypes.Structure):
    _fields_ = [("h", ctypes.c_int32), ("w", ctypes.c_int32), ("block", ctypes.c_int32),
                ("capacity", ctypes.c_int32)]


# Every symbol include/sige.h declares, with its ctypes signature.
_vp, _i32, _f32, _sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_float, ctypes.c_size_t
_TD, _CD, _SD = ctypes.POINTER(TensorDesc), ctypes.POINTER(ConvDesc), ctypes.POINTER(ScaleDesc)
_LE = ctypes.POINTER(LayerExt)
SIGNATURES = {
    "sige_reduce_mask_workspace_bytes": (_sz, [_TD, _i32, _SD]),
    "sige_reduce_mask": (_i32, [_vp, _vp, _TD, _f32, _i32, _i32, _SD, _vp, _vp, _vp, _vp, _sz, _vp]),
    "sige_reduce_mask_px": (_i32, [_vp, _vp, _TD, _f32, _i32, _i32, _SD, _vp, _vp, _vp, _vp, _sz, _vp]),
    "sige_reduce_mask_static": (_i32, [_vp, _vp, _TD, _f32, _i32, _i32, _SD, _vp, _vp, _vp]),
    "sige_gather": (_i32, [_vp, _TD, _CD, _vp, _vp, _i32, _vp, _vp, _i32, _vp, _vp]),
    "sige_sparse_conv": (_i32, [_vp, _CD, _i32, _i32, _vp, _vp, _i32, _vp, _vp, _sz, _vp]),
    "sige_scatter": (_i32, [_vp, _CD, _vp, _vp, _i32, _vp, _vp, _vp, _TD, _vp]),
    "sige_conv_fused": (_i32, [_vp, _TD, _vp, _vp, _CD, _vp, _vp, _i32, _vp, _vp, _i32, _vp, _vp, _TD,
                               _vp, _sz, _vp]),
    "sige_resblock_step_workspace_bytes": (_sz, [_TD, _i32]),
    "sige_resblock_step": (_i32, [_vp, _vp, _TD, _f32, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _vp, _vp,
                                  _i32, _vp, _vp, _vp, _sz, _vp]),
    "sige_conv_fused_ext": (_i32, [_vp, _TD, _vp, _vp, _CD, _LE, _vp, _vp, _i32, _vp, _vp, _vp, _vp, _TD, _vp,
                                   _sz, _vp]),
    "sige_dense_conv": (_i32, [_vp, _TD, _vp, _vp, _CD, _vp, _vp, _i32, _vp, _vp, _TD, _vp, _sz, _vp]),
    "sige_groupnorm_affine": (_i32, [_vp, _TD, _i32, _vp, _vp, _f32, _vp, _vp, _vp]),
    "sige_resblock_fused": (_i32, [_vp, _TD, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _vp, _vp, _i32, _vp,
                                   _vp, _vp, _sz, _vp]),
    "sige_restore_tiles": (_i32, [_vp, _vp, _TD, _i32, _vp, _vp, _i32, _vp]),
    "sige_download_tiles_bytes": (_sz, [_TD, _i32, _i32]),
    "sige_download_tiles": (_i32, [_vp, _TD, _i32, _vp, _vp, _i32, _vp, _vp, _vp, _vp]),
    "sige_conv_workspace_bytes": (_sz, [_CD, _i32, _i32, _i32, _i32]),
    "sige_get_error": (_i32, [_vp, _vp]),
    "sige_get_device_error": (_i32, [_vp, _vp]),
    "sige_workspace_bytes": (_sz, [_i32, _CD, _i32]),
    "sige_set_wait_cycles": (_i32, [ctypes.c_int64]),
    "sige_conv_path": (_i32, [_CD, _i32]),
    "sige_conv_schedule": (_i32, [_CD, _i32, _i32, _i32, _vp, _i32]),
    "sige_attention_core": (_i32, [_vp, _TD, _vp, _vp, _i32, _i32, _i32, _vp, _vp, _i32, _i32, _vp, _vp]),
    "sige_attention_path": (_i32, [_TD, _i32, _i32]),
    "sige_launch_count": (ctypes.c_uint64, []),
    "sige_status_string": (ctypes.c_char_p, [_i32]),
}

_lib = None


def lib() -> ctypes.CDLL:
    """Load libsige.so (built by ``__graft_entry__.build()``); raise if absent."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is not built; run __graft_entry__.build() first")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def status_string(status: int) -> str:
    try:
        return lib().sige_status_string(int(status)).decode()
    except Exception:  # library missing
        return "status"


def _check(st: int, what: str):
    if st != OK:
        raise SigeError(st, what)


def _ptr(t):
    if t is None:
        return None
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def tensor_desc(t: torch.Tensor, layout: int = NHWC) -> TensorDesc:
    if t.dim() != 4:
        raise ValueError("expected a 4-d tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    if layout == NHWC:
        n, h, w, c = t.shape
    else:
        n, c, h, w = t.shape
    return TensorDesc(n, h, w, c, _DT[t.dtype], layout)


def conv_desc(kernel, stride, pad, c_in, c_out, block) -> ConvDesc:
    return ConvDesc(kernel, stride, pad, c_in, c_out, block)


def zeros_workspace(nbytes: int, device) -> torch.Tensor:
    """A zero-filled device workspace (16-byte aligned, as torch allocations are)."""
    return torch.zeros(max(int(nbytes), WORKSPACE_HEADER), dtype=torch.uint8, device=device)


# ------------------------------------------------------------------ calls

def sige_reduce_mask_workspace_bytes(desc: TensorDesc, scales) -> int:
    arr = (ScaleDesc * len(scales))(*[ScaleDesc(*s) for s in scales])
    return int(lib().sige_reduce_mask_workspace_bytes(ctypes.byref(desc), len(scales), arr))


def _host_counts(n, want):
    return (ctypes.c_int32 * n)() if want else None


def sige_reduce_mask(a_orig, a_edit, threshold, scales, dilate=1, layout=NHWC, idx=None, counts=None,
                     workspace=None, stream=None, host_counts=False):
    """Difference mask -> per-scale active-tile lists.  ``scales`` is a list of
    (h, w, block, capacity).  Returns (idx [sum(capacity), 2] int32, counts
    [n_scales] int32, workspace); all on the device, nothing synchronised.
    With ``host_counts=True`` the call also copies the counts to the host
    (the library synchronises the stream) and returns them as a fourth item,
    a list of ints."""
    desc = tensor_desc(a_orig, layout)
    arr = (ScaleDesc * len(scales))(*[ScaleDesc(*s) for s in scales])
    dev = a_orig.device
    if idx is None:
        idx = torch.empty((max(1, sum(s[3] for s in scales)), 2), dtype=torch.int32, device=dev)
    if counts is None:
        counts = torch.empty(len(scales), dtype=torch.int32, device=dev)
    need = int(lib().sige_reduce_mask_workspace_bytes(ctypes.byref(desc), len(scales), arr))
    if workspace is None:
        workspace = zeros_workspace(need, dev)
    hc = _host_counts(len(scales), host_counts)
    st = lib().sige_reduce_mask(_ptr(a_orig), _ptr(a_edit), ctypes.byref(desc), float(threshold), int(dilate),
                                len(scales), arr, _ptr(idx), _ptr(counts), hc, _ptr(workspace),
                                workspace.numel(), _stream(stream))
    _check(st, "sige_reduce_mask")
    if host_counts:
        return idx, counts, workspace, [int(v) for v in hc]
    return idx, counts, workspace


def sige_reduce_mask_px(a_orig, a_edit, threshold, scales, radius=1, layout=NHWC, idx=None, counts=None,
                        workspace=None, stream=None, host_counts=False):
    """As sige_reduce_mask, with the mask dilated by ``radius`` pixels at each
    scale before tiling (no tile dilation)."""
    desc = tensor_desc(a_orig, layout)
    arr = (ScaleDesc * len(scales))(*[ScaleDesc(*s) for s in scales])
    dev = a_orig.device
    if idx is None:
        idx = torch.empty((max(1, sum(s[3] for s in scales)), 2), dtype=torch.int32, device=dev)
    if counts is None:
        counts = torch.empty(len(scales), dtype=torch.int32, device=dev)
    need = int(lib().sige_reduce_mask_workspace_bytes(ctypes.byref(desc), len(scales), arr))
    if workspace is None:
        workspace = zeros_workspace(need, dev)
    hc = _host_counts(len(scales), host_counts)
    st = lib().sige_reduce_mask_px(_ptr(a_orig), _ptr(a_edit), ctypes.byref(desc), float(threshold), int(radius),
                                   len(scales), arr, _ptr(idx), _ptr(counts), hc, _ptr(workspace),
                                   workspace.numel(), _stream(stream))
    _check(st, "sige_reduce_mask_px")
    if host_counts:
        return idx, counts, workspace, [int(v) for v in hc]
    return idx, counts, workspace


def sige_reduce_mask_static(a_orig, a_edit, threshold, scales, dilate=1, layout=NHWC, idx=None, counts=None,
                            stream=None):
    """sige_reduce_mask for callers that cannot allocate a workspace: the
    library's built-in 64 KB scratch is used instead (calls on one device must
    not overlap).  Returns (idx, counts)."""
    desc = tensor_desc(a_orig, layout)
    arr = (ScaleDesc * len(scales))(*[ScaleDesc(*s) for s in scales])
    dev = a_orig.device
    if idx is None:
        idx = torch.empty((max(1, sum(s[3] for s in scales)), 2), dtype=torch.int32, device=dev)
    if counts is None:
        counts = torch.empty(len(scales), dtype=torch.int32, device=dev)
    st = lib().sige_reduce_mask_static(_ptr(a_orig), _ptr(a_edit), ctypes.byref(desc), float(threshold),
                                       int(dilate), len(scales), arr, _ptr(idx), _ptr(counts), _stream(stream))
    _check(st, "sige_reduce_mask_static")
    return idx, counts


def sige_gather(x, cd: ConvDesc, idx, count, capacity, gn_scale=None, gn_shift=None, silu=False,
                blocks=None, stream=None):
    xd = tensor_desc(x)
    bin_ = (cd.block - 1) * cd.stride + cd.kernel
    if blocks is None:
        blocks = torch.empty((max(capacity, 1), x.shape[0], bin_, bin_, cd.c_in), dtype=x.dtype, device=x.device)
    st = lib().sige_gather(_ptr(x), ctypes.byref(xd), ctypes.byref(cd), _ptr(idx), _ptr(count), int(capacity),
                           _ptr(gn_scale), _ptr(gn_shift), int(bool(silu)), _ptr(blocks), _stream(stream))
    _check(st, "sige_gather")
    return blocks


def sige_sparse_conv(blocks, cd: ConvDesc, weight, count, capacity, batch=1, out_blocks=None, workspace=None,
                     stream=None):
    if out_blocks is None:
        out_blocks = torch.empty((max(capacity, 1), batch, cd.block, cd.block, cd.c_out), dtype=torch.float32,
                                 device=blocks.device)
    if workspace is None:
        workspace = zeros_workspace(sige_conv_workspace_bytes(cd, batch, capacity, 0, 0), blocks.device)
    st = lib().sige_sparse_conv(_ptr(blocks), ctypes.byref(cd), _DT[blocks.dtype], int(batch), _ptr(weight),
                                _ptr(count), int(capacity), _ptr(out_blocks), _ptr(workspace), workspace.numel(),
                                _stream(stream))
    _check(st, "sige_sparse_conv")
    return out_blocks


def sige_scatter(out_blocks, cd: ConvDesc, idx, count, capacity, y, bias=None, residual=None, stream=None):
    yd = tensor_desc(y)
    st = lib().sige_scatter(_ptr(out_blocks), ctypes.byref(cd), _ptr(idx), _ptr(count), int(capacity),
                            _ptr(bias), _ptr(residual), _ptr(y), ctypes.byref(yd), _stream(stream))
    _check(st, "sige_scatter")
    return y


def sige_conv_fused(x, weight, bias, cd: ConvDesc, idx, count, capacity, y, gn_scale=None, gn_shift=None,
                    silu=False, residual=None, workspace=None, stream=None):
    xd, yd = tensor_desc(x), tensor_desc(y)
    if workspace is None:
        workspace = zeros_workspace(sige_conv_workspace_bytes(cd, x.shape[0], capacity, y.shape[1], y.shape[2]),
                                    x.device)
    st = lib().sige_conv_fused(_ptr(x), ctypes.byref(xd), _ptr(weight), _ptr(bias), ctypes.byref(cd), _ptr(idx),
                               _ptr(count), int(capacity), _ptr(gn_scale), _ptr(gn_shift), int(bool(silu)),
                               _ptr(residual), _ptr(y), ctypes.byref(yd), _ptr(workspace), workspace.numel(),
                               _stream(stream))
    _check(st, "sige_conv_fused")
    return y


def conv_out_hw(cd: ConvDesc, H: int, W: int, transposed=False, output_padding=0):
    if transposed:
        return ((H - 1) * cd.stride - 2 * cd.pad + cd.kernel + output_padding,
                (W - 1) * cd.stride - 2 * cd.pad + cd.kernel + output_padding)
    return (H + 2 * cd.pad - cd.kernel) // cd.stride + 1, (W + 2 * cd.pad - cd.kernel) // cd.stride + 1


def sige_conv_fused_ext(x, weight, bias, cd: ConvDesc, y=None, idx=None, count=None, capacity=0, gn_scale=None,
                        gn_shift=None, transposed=False, output_padding=0, spade_gamma=None, spade_beta=None,
                        act=ACT_NONE, residual=None, workspace=None, stream=None):
    """A GauGAN-style layer (transposed conv and / or SPADE-style modulated
    input) on the listed tiles of y, or on every tile when ``idx`` is None."""
    N, H, W, _ = x.shape
    Ho, Wo = conv_out_hw(cd, H, W, transposed, output_padding)
    if y is None:
        y = torch.empty((N, Ho, Wo, cd.c_out), dtype=x.dtype, device=x.device)
    xd, yd = tensor_desc(x), tensor_desc(y)
    if workspace is None:
        workspace = zeros_workspace(sige_conv_workspace_bytes(cd, N, max(capacity, 1), Ho, Wo), x.device)
    ext = LayerExt(int(bool(transposed)), int(output_padding), None if spade_gamma is None else spade_gamma.data_ptr(),
                   None if spade_beta is None else spade_beta.data_ptr(), int(act))
    st = lib().sige_conv_fused_ext(_ptr(x), ctypes.byref(xd), _ptr(weight), _ptr(bias), ctypes.byref(cd),
                                   ctypes.byref(ext), _ptr(idx), _ptr(count), int(capacity), _ptr(gn_scale),
                                   _ptr(gn_shift), _ptr(residual), _ptr(y), ctypes.byref(yd), _ptr(workspace),
                                   workspace.numel(), _stream(stream))
    _check(st, "sige_conv_fused_ext")
    return y


def sige_dense_conv(x, weight, bias, cd: ConvDesc, y=None, gn_scale=None, gn_shift=None, silu=False,
                    residual=None, workspace=None, stream=None):
    N, H, W, _ = x.shape
    Ho = (H + 2 * cd.pad - cd.kernel) // cd.stride + 1
    Wo = (W + 2 * cd.pad - cd.kernel) // cd.stride + 1
    if y is None:
        y = torch.empty((N, Ho, Wo, cd.c_out), dtype=x.dtype, device=x.device)
    xd, yd = tensor_desc(x), tensor_desc(y)
    if workspace is None:
        workspace = zeros_workspace(sige_conv_workspace_bytes(cd, N, 0, Ho, Wo), x.device)
    st = lib().sige_dense_conv(_ptr(x), ctypes.byref(xd), _ptr(weight), _ptr(bias), ctypes.byref(cd),
                               _ptr(gn_scale), _ptr(gn_shift), int(bool(silu)), _ptr(residual), _ptr(y),
                               ctypes.byref(yd), _ptr(workspace), workspace.numel(), _stream(stream))
    _check(st, "sige_dense_conv")
    return y


def sige_resblock_fused(x_edit, w1, b1, gn1, w2, b2, gn2, idx, count, capacity, y1, out, block=8,
                        workspace=None, stream=None):
    """The res block on the active tiles in one launch: y1 and out (the caches,
    NHWC bf16) are updated in place at the listed 8x8 tiles.  ``gn1`` / ``gn2``
    are (scale, shift) pairs from sige_groupnorm_affine; biases may be None."""
    xd = tensor_desc(x_edit)
    if workspace is None:
        workspace = zeros_workspace(WORKSPACE_HEADER, x_edit.device)
    st = lib().sige_resblock_fused(_ptr(x_edit), ctypes.byref(xd), _ptr(w1), _ptr(b1), _ptr(gn1[0]), _ptr(gn1[1]),
                                   _ptr(w2), _ptr(b2), _ptr(gn2[0]), _ptr(gn2[1]), int(block), _ptr(idx),
                                   _ptr(count), int(capacity), _ptr(y1), _ptr(out), _ptr(workspace),
                                   workspace.numel(), _stream(stream))
    _check(st, "sige_resblock_fused")
    return y1, out


def sige_resblock_step_workspace_bytes(x, block=8) -> int:
    xd = tensor_desc(x)
    return int(lib().sige_resblock_step_workspace_bytes(ctypes.byref(xd), int(block)))


def sige_resblock_step(x_orig, x_edit, threshold, w1, b1, gn1, w2, b2, gn2, y1, out, capacity, dilate=1, block=8,
                       idx=None, count=None, workspace=None, stream=None):
    """Mask, tile list and the fused res block in one launch.  Returns (idx,
    count) on the device; y1 and out are updated in place."""
    xd = tensor_desc(x_edit)
    dev = x_edit.device
    if idx is None:
        idx = torch.empty((max(int(capacity), 1), 2), dtype=torch.int32, device=dev)
    if count is None:
        count = torch.empty(1, dtype=torch.int32, device=dev)
    if workspace is None:
        workspace = zeros_workspace(sige_resblock_step_workspace_bytes(x_edit, block), dev)
    st = lib().sige_resblock_step(_ptr(x_orig), _ptr(x_edit), ctypes.byref(xd), float(threshold), int(dilate),
                                  _ptr(w1), _ptr(b1), _ptr(gn1[0]), _ptr(gn1[1]), _ptr(w2), _ptr(b2), _ptr(gn2[0]),
                                  _ptr(gn2[1]), int(block), _ptr(idx), _ptr(count), int(capacity), _ptr(y1),
                                  _ptr(out), _ptr(workspace), workspace.numel(), _stream(stream))
    _check(st, "sige_resblock_step")
    return idx, count


def sige_groupnorm_affine(x, groups, gamma, beta, eps=1e-5, scale=None, shift=None, stream=None):
    xd = tensor_desc(x)
    if scale is None:
        scale = torch.empty((x.shape[0], x.shape[3]), dtype=torch.float32, device=x.device)
    if shift is None:
        shift = torch.empty_like(scale)
    st = lib().sige_groupnorm_affine(_ptr(x), ctypes.byref(xd), int(groups), _ptr(gamma), _ptr(beta), float(eps),
                                     _ptr(scale), _ptr(shift), _stream(stream))
    _check(st, "sige_groupnorm_affine")
    return scale, shift


def sige_restore_tiles(src, dst, block, idx, count, capacity, stream=None):
    """dst[n, h0+i, w0+j, :] = src[n, h0+i, w0+j, :] for the listed tiles (in-image
    pixels, i, j < block); every other element of dst is left as it is."""
    if src.shape != dst.shape or src.dtype != dst.dtype:
        raise ValueError("src and dst must have the same shape and dtype")
    d = tensor_desc(dst)
    st = lib().sige_restore_tiles(_ptr(src), _ptr(dst), ctypes.byref(d), int(block), _ptr(idx), _ptr(count),
                                  int(capacity), _stream(stream))
    _check(st, "sige_restore_tiles")
    return dst


def sige_download_tiles_bytes(y, block, capacity) -> int:
    d = tensor_desc(y)
    return int(lib().sige_download_tiles_bytes(ctypes.byref(d), int(block), int(capacity)))


def sige_download_tiles(y, block, idx, count, capacity, host_y, staging=None, host_staging=None, stream=None):
    """host_y[n, h0+i, w0+j, :] = y[n, h0+i, w0+j, :] for the listed tiles of the
    device tensor y (in-image pixels, i, j < block); every other element of the
    host tensor host_y is left as it is.  Returns once host_y is complete."""
    if tuple(host_y.shape) != tuple(y.shape) or host_y.dtype != y.dtype or host_y.device.type != "cpu":
        raise ValueError("host_y must be a host tensor of y's shape and dtype")
    if not host_y.is_contiguous():
        raise ValueError("host_y must be contiguous")
    nbytes = sige_download_tiles_bytes(y, block, capacity)
    if staging is None:
        staging = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=y.device)
    if host_staging is None:
        host_staging = torch.empty(max(nbytes, 16), dtype=torch.uint8).pin_memory()
    if staging.numel() * staging.element_size() < nbytes or host_staging.numel() * host_staging.element_size() < nbytes:
        raise ValueError("staging buffers smaller than sige_download_tiles_bytes")
    d = tensor_desc(y)
    st = lib().sige_download_tiles(_ptr(y), ctypes.byref(d), int(block), _ptr(idx), _ptr(count), int(capacity),
                                   _ptr(staging), ctypes.c_void_p(host_staging.data_ptr()),
                                   ctypes.c_void_p(host_y.data_ptr()), _stream(stream))
    _check(st, "sige_download_tiles")
    return host_y


def sige_conv_workspace_bytes(cd: ConvDesc, batch: int, capacity: int, out_h: int, out_w: int) -> int:
    return int(lib().sige_conv_workspace_bytes(ctypes.byref(cd), int(batch), int(capacity), int(out_h), int(out_w)))


def sige_get_error(workspace, stream=None) -> int:
    return int(lib().sige_get_error(_ptr(workspace), _stream(stream)))


def sige_get_device_error(workspace, stream=None) -> int:
    return int(lib().sige_get_device_error(_ptr(workspace), _stream(stream)))


def sige_workspace_bytes(which_call: int, cd: ConvDesc | None, capacity: int) -> int:
    return int(lib().sige_workspace_bytes(int(which_call), None if cd is None else ctypes.byref(cd),
                                          int(capacity)))


def sige_set_wait_cycles(cycles: int) -> None:
    """Bound of the device waits that report SIGE_ERR_TIMEOUT (0: the kernels'
    own bounds), for launches enqueued from now on, process-wide."""
    _check(lib().sige_set_wait_cycles(int(cycles)), "sige_set_wait_cycles")


def sige_conv_path(cd: ConvDesc, dtype: torch.dtype) -> int:
    return int(lib().sige_conv_path(ctypes.byref(cd), _DT[dtype]))


def sige_attention_path(q, dv: int, heads: int) -> int:
    """Which kernel sige_attention_core runs for queries like ``q`` (an NHWC
    tensor), value width dv and this head count: 1 = tcgen05 tensor cores,
    0 = CUDA cores; negative = a sige_status."""
    qd = tensor_desc(q)
    return int(lib().sige_attention_path(ctypes.byref(qd), int(dv), int(heads)))


def sige_attention_core(q, k, v, heads: int, idx, count, capacity: int, block: int, o=None, stream=None):
    """Attention at the tokens under the tile list: q [N, H, W, D] bf16, k
    [N, Lk, D], v [N, Lk, Dv] (a [N, H, W, *] map is viewed as [N, H*W, *]),
    o [N, H, W, Dv] written at those tokens only (zeros elsewhere when
    allocated here)."""
    N, H, W, D = q.shape
    kk = k.reshape(N, -1, D)
    vv = v.reshape(N, kk.shape[1], -1)
    if o is None:
        o = torch.zeros((N, H, W, vv.shape[2]), dtype=q.dtype, device=q.device)
    qd = tensor_desc(q)
    st = lib().sige_attention_core(_ptr(q), ctypes.byref(qd), _ptr(kk), _ptr(vv), int(kk.shape[1]),
                                   int(vv.shape[2]), int(heads), _ptr(idx), _ptr(count), int(capacity), int(block),
                                   _ptr(o), _stream(stream))
    _check(st, "sige_attention_core")
    return o


def sige_attention_sparse(x, idx, count, capacity: int, block: int, wq, wo, bo, heads: int, k_map, v_map, y,
                          wk=None, wv=None, residual=None, workspace=None, stream=None):
    """One attention layer with pruned queries, in place into the cached output
    ``y`` [N, H, W, Co]: q = x Wq at the tokens under the tile list (sparse 1x1
    conv), the cached key / value maps ``k_map`` [N, H, W, D] / ``v_map``
    updated there from x when ``wk`` / ``wv`` are given (self-attention; a
    cross-attention caller passes the context's key / value sequences
    [N, Lc, *] and no ``wk`` / ``wv``), the attention step, and
    y = o Wo + bo (+ residual) at those tokens (sparse 1x1 conv).  Weights
    are 1x1 conv weights [c_out][1][1][c_in] (the transposed projection
    matrices).  With caches built from the original map and an edit confined to
    the listed tiles, the keys and values equal those of the whole edited map."""
    N, H, W, C = x.shape
    D, Dv, Co = wq.shape[0], v_map.shape[-1], wo.shape[0]
    cd_q = conv_desc(1, 1, 0, C, D, block)
    if workspace is None:
        need = max(sige_conv_workspace_bytes(conv_desc(1, 1, 0, ci, co, block), N, capacity, 0, 0)
                   for ci, co in ((C, D), (C, Dv), (Dv, Co)))
        workspace = zeros_workspace(need, x.device)
    q = torch.empty((N, H, W, D), dtype=x.dtype, device=x.device)
    sige_conv_fused(x, wq, None, cd_q, idx, count, capacity, q, workspace=workspace, stream=stream)
    if wk is not None:
        sige_conv_fused(x, wk, None, cd_q, idx, count, capacity, k_map, workspace=workspace, stream=stream)
    if wv is not None:
        sige_conv_fused(x, wv, None, conv_desc(1, 1, 0, C, Dv, block), idx, count, capacity, v_map,
                        workspace=workspace, stream=stream)
    o = torch.empty((N, H, W, Dv), dtype=x.dtype, device=x.device)
    sige_attention_core(q, k_map, v_map, heads, idx, count, capacity, block, o, stream)
    sige_conv_fused(o, wo, bo, conv_desc(1, 1, 0, Dv, Co, block), idx, count, capacity, y, residual=residual,
                    workspace=workspace, stream=stream)
    return y


SCHEDULE_FIELDS = ("layout", "T", "tile_groups", "splits", "units", "split_sum", "unit_cols", "weight_stages",
                   "halo_bytes", "reduce_scatter_bytes", "cout_tiles", "k_chunks", "cluster_for_sparse",
                   "halo_offset", "smem_bytes")


def sige_conv_schedule(cd: ConvDesc, tiles: int, grid: int, cluster: int) -> dict:
    """Work decomposition of the tensor-core conv for ``tiles`` active tiles
    (times batch) on a launch of ``grid`` CTAs in clusters of ``cluster``;
    host-only.  Keys are SCHEDULE_FIELDS."""
    out = (ctypes.c_int32 * len(SCHEDULE_FIELDS))()
    _check(lib().sige_conv_schedule(ctypes.byref(cd), int(tiles), int(grid), int(cluster),
                                    ctypes.cast(out, ctypes.c_void_p), len(SCHEDULE_FIELDS)), "sige_conv_schedule")
    return dict(zip(SCHEDULE_FIELDS, (int(v) for v in out)))


def sige_launch_count() -> int:
    return int(lib().sige_launch_count())
