"""Host-side checks of the C ABI: the library loads without a GPU, exports
every symbol include/sige.h declares with the signature the binding uses, and
rejects bad arguments before touching the device."""
import ctypes
import os
import re

import pytest

import spatially_sparse_incremental_b200 as sige

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sige.h")


@pytest.fixture(scope="module")
def L():
    import __graft_entry__
    __graft_entry__.build_library()
    return sige.lib()


def _declared():
    txt = open(HEADER).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_ ]*?\**\s*\b(sige_[a-z_]+)\s*\(", txt, flags=re.M)
    return sorted(set(names))


# The calls of the hot path's C boundary: the five steps of the layer (mask
# reduction, gather, block conv, scatter, fused layer) and the workspace /
# status / device-error utilities around them.
BOUNDARY = ("sige_reduce_mask", "sige_gather", "sige_sparse_conv", "sige_scatter", "sige_conv_fused",
            "sige_workspace_bytes", "sige_status_string", "sige_get_device_error")


def test_header_declares_the_calls():
    names = _declared()
    for call in BOUNDARY:
        assert call in names, call


def test_boundary_calls_exported(L):
    for call in BOUNDARY:
        assert hasattr(L, call), call


def test_every_declared_symbol_is_exported_and_bound(L):
    names = _declared()
    assert set(names) == set(sige.SIGNATURES), set(names) ^ set(sige.SIGNATURES)
    for n in names:
        assert hasattr(L, n), n


def test_status_strings(L):
    for st in (0, -1, -2, -3, -4, -5, -6):
        s = sige.status_string(st)
        assert s and s != "unknown status"
    assert sige.status_string(-99) == "unknown status"


def _scales(*s):
    return (sige.ScaleDesc * len(s))(*[sige.ScaleDesc(*q) for q in s])


def test_reduce_mask_validation(L):
    d = sige.TensorDesc(1, 256, 256, 3, sige.U8, sige.NCHW)
    sc = _scales((256, 256, 8, 1024), (128, 128, 4, 1024), (64, 64, 4, 256), (32, 32, 2, 256))
    need = L.sige_reduce_mask_workspace_bytes(ctypes.byref(d), 4, sc)
    # header + one 16-byte-padded flag byte per tile per scale
    assert need == 256 + 1024 + 1024 + 256 + 256
    fake = ctypes.c_void_p(0x1000)
    ws = ctypes.c_void_p(0x2000)
    hc = (ctypes.c_int32 * 4)()
    args = lambda **kw: dict(dict(a=fake, b=fake, d=ctypes.byref(d), thr=0.0, dil=1, ns=4, sc=sc,
                                  idx=fake, cnt=fake, hc=None, ws=ws, wsb=need, st=None), **kw)

    def call(**kw):
        a = args(**kw)
        return L.sige_reduce_mask(a["a"], a["b"], a["d"], a["thr"], a["dil"], a["ns"], a["sc"], a["idx"],
                                  a["cnt"], a["hc"], a["ws"], a["wsb"], a["st"])
    assert call(a=None) == sige.ERR_INVALID_ARG
    assert call(idx=None) == sige.ERR_INVALID_ARG
    assert call(thr=-1.0) == sige.ERR_INVALID_ARG
    assert call(thr=float("nan")) == sige.ERR_INVALID_ARG
    assert call(dil=-1) == sige.ERR_INVALID_ARG
    assert call(ns=0) == sige.ERR_INVALID_ARG
    assert call(ns=9) == sige.ERR_INVALID_ARG
    assert call(wsb=need - 1) == sige.ERR_WORKSPACE
    assert call(ws=None) == sige.ERR_WORKSPACE
    bad = _scales((100, 100, 8, 16))          # 256 is not a multiple of 100
    assert call(ns=1, sc=bad) == sige.ERR_INVALID_ARG
    d16 = sige.TensorDesc(1, 16, 16, 3, 7, sige.NHWC)
    assert call(d=ctypes.byref(d16)) == sige.ERR_UNSUPPORTED
    # with host counts requested, argument errors still come first
    assert call(a=None, hc=hc) == sige.ERR_INVALID_ARG
    assert call(wsb=need - 1, hc=hc) == sige.ERR_WORKSPACE


def test_reduce_mask_static_checks_before_enqueueing(L):
    """Every argument is checked before the static entry point touches the
    device (memsets or the symbol lookup): these calls return the argument
    error on a host with no GPU at all."""
    d = sige.TensorDesc(1, 64, 64, 8, sige.F32, sige.NHWC)
    sc = _scales((64, 64, 8, 64))
    fake = ctypes.c_void_p(0x1000)

    def call(a=fake, idx=fake, cnt=fake, thr=1e-3, dil=1, desc=ctypes.byref(d), scales=sc, ns=1):
        return L.sige_reduce_mask_static(a, fake, desc, thr, dil, ns, scales, idx, cnt, None)
    assert call(a=None) == sige.ERR_INVALID_ARG
    assert call(idx=None) == sige.ERR_INVALID_ARG
    assert call(cnt=None) == sige.ERR_INVALID_ARG
    assert call(idx=ctypes.c_void_p(0x1004)) == sige.ERR_INVALID_ARG      # pairs need 8-byte alignment
    assert call(thr=float("nan")) == sige.ERR_INVALID_ARG
    assert call(dil=-1) == sige.ERR_INVALID_ARG
    assert call(ns=0) == sige.ERR_INVALID_ARG
    dbad = sige.TensorDesc(1, 64, 64, 8, 7, sige.NHWC)
    assert call(desc=ctypes.byref(dbad)) == sige.ERR_UNSUPPORTED
    # more tiles than the 64 KB built-in scratch holds
    dbig = sige.TensorDesc(1, 4096, 4096, 8, sige.F32, sige.NHWC)
    assert call(desc=ctypes.byref(dbig), scales=_scales((4096, 4096, 8, 1 << 18))) == sige.ERR_WORKSPACE


def test_workspace_bytes_by_call(L):
    cd = sige.ConvDesc(3, 1, 1, 128, 128, 8)
    conv = L.sige_conv_workspace_bytes(ctypes.byref(cd), 1, 1024, 0, 0)
    for which in (sige.CALL_SPARSE_CONV, sige.CALL_CONV_FUSED, sige.CALL_DENSE_CONV):
        assert sige.sige_workspace_bytes(which, cd, 1024) == conv
    # the mask bound covers any split of the tiles into scales
    d = sige.TensorDesc(1, 256, 256, 3, sige.U8, sige.NCHW)
    sc = _scales((256, 256, 8, 1024), (128, 128, 4, 1024), (64, 64, 4, 256), (32, 32, 2, 256))
    exact = L.sige_reduce_mask_workspace_bytes(ctypes.byref(d), 4, sc)
    tiles = 1024 + 1024 + 256 + 256
    assert sige.sige_workspace_bytes(sige.CALL_REDUCE_MASK, None, tiles) >= exact
    assert sige.sige_workspace_bytes(sige.CALL_RESBLOCK, None, 0) >= 256
    assert sige.sige_workspace_bytes(99, cd, 16) == 0
    assert sige.sige_workspace_bytes(sige.CALL_CONV_FUSED, cd, -1) == 0
    assert sige.sige_workspace_bytes(sige.CALL_CONV_FUSED, None, 16) == 0


def test_wait_cycles_setting(L):
    assert L.sige_set_wait_cycles(-1) == sige.ERR_INVALID_ARG
    assert L.sige_set_wait_cycles(1000) == sige.OK
    assert L.sige_set_wait_cycles(0) == sige.OK


def test_conv_validation(L):
    cd = sige.ConvDesc(3, 1, 1, 128, 128, 8)
    xd = sige.TensorDesc(1, 64, 64, 128, sige.BF16, sige.NHWC)
    yd = sige.TensorDesc(1, 64, 64, 128, sige.BF16, sige.NHWC)
    fake = ctypes.c_void_p(0x1000)
    ws = ctypes.c_void_p(0x2000)
    wsb = L.sige_conv_workspace_bytes(ctypes.byref(cd), 1, 64, 64, 64)
    assert wsb >= 256

    def fused(**kw):
        a = dict(x=fake, xd=ctypes.byref(xd), w=fake, b=None, cd=ctypes.byref(cd), idx=fake, cnt=fake, cap=64,
                 gs=None, gh=None, silu=0, res=None, y=fake, yd=ctypes.byref(yd), ws=ws, wsb=wsb, st=None)
        a.update(kw)
        return L.sige_conv_fused(*a.values())
    assert fused(x=None) == sige.ERR_INVALID_ARG
    assert fused(cap=-1) == sige.ERR_INVALID_ARG
    assert fused(gs=fake) == sige.ERR_INVALID_ARG               # scale without shift
    ydb = sige.TensorDesc(1, 63, 64, 128, sige.BF16, sige.NHWC)
    assert fused(yd=ctypes.byref(ydb)) == sige.ERR_INVALID_ARG  # wrong output size
    ydf = sige.TensorDesc(1, 64, 64, 128, sige.F32, sige.NHWC)
    assert fused(yd=ctypes.byref(ydf)) == sige.ERR_UNSUPPORTED  # dtype mismatch
    assert fused(ws=None) == sige.ERR_WORKSPACE
    assert fused(wsb=10) == sige.ERR_WORKSPACE
    bad = sige.ConvDesc(3, 1, 3, 128, 128, 8)                   # pad >= kernel
    assert fused(cd=ctypes.byref(bad)) == sige.ERR_INVALID_ARG
    assert fused(x=ctypes.c_void_p(0x1001)) == sige.ERR_UNSUPPORTED  # misaligned


def test_conv_path_selection(L):
    assert sige.sige_conv_path(sige.ConvDesc(3, 1, 1, 64, 64, 4), __import__("torch").float32) == 0
    assert sige.sige_conv_path(sige.ConvDesc(3, 1, 3, 64, 64, 4), __import__("torch").float32) == sige.ERR_INVALID_ARG


def test_gather_scatter_validation(L):
    cd = sige.ConvDesc(3, 1, 1, 64, 64, 4)
    fake = ctypes.c_void_p(0x1000)
    xd = sige.TensorDesc(1, 16, 16, 64, sige.F32, sige.NHWC)
    assert L.sige_gather(None, ctypes.byref(xd), ctypes.byref(cd), fake, fake, 4, None, None, 0, fake, None) \
        == sige.ERR_INVALID_ARG
    xd3 = sige.TensorDesc(1, 16, 16, 3, sige.F32, sige.NHWC)      # C != c_in
    assert L.sige_gather(fake, ctypes.byref(xd3), ctypes.byref(cd), fake, fake, 4, None, None, 0, fake, None) \
        == sige.ERR_INVALID_ARG
    yd = sige.TensorDesc(1, 16, 16, 64, sige.U8, sige.NHWC)
    assert L.sige_scatter(fake, ctypes.byref(cd), fake, fake, 4, None, None, fake, ctypes.byref(yd), None) \
        == sige.ERR_UNSUPPORTED
    # zero capacity is a no-op that launches nothing
    n0 = sige.sige_launch_count()
    yd2 = sige.TensorDesc(1, 16, 16, 64, sige.F32, sige.NHWC)
    assert L.sige_scatter(fake, ctypes.byref(cd), fake, fake, 0, None, None, fake, ctypes.byref(yd2), None) == sige.OK
    assert sige.sige_launch_count() == n0


def test_groupnorm_validation(L):
    fake = ctypes.c_void_p(0x1000)
    xd = sige.TensorDesc(1, 8, 8, 30, sige.F32, sige.NHWC)        # 30 channels, 32 groups
    assert L.sige_groupnorm_affine(fake, ctypes.byref(xd), 32, fake, fake, 1e-5, fake, fake, None) \
        == sige.ERR_INVALID_ARG


def test_reduce_mask_px_validation(L):
    d = sige.TensorDesc(1, 64, 64, 8, sige.F32, sige.NHWC)
    sc = _scales((64, 64, 8, 64))
    need = L.sige_reduce_mask_workspace_bytes(ctypes.byref(d), 1, sc)
    fake, ws = ctypes.c_void_p(0x1000), ctypes.c_void_p(0x2000)

    def call(radius=1, a=fake, wsb=need, thr=1e-3):
        return L.sige_reduce_mask_px(a, fake, ctypes.byref(d), thr, radius, 1, sc, fake, fake, None, ws, wsb, None)
    assert call(radius=-1) == sige.ERR_INVALID_ARG
    assert call(a=None) == sige.ERR_INVALID_ARG
    assert call(thr=float("nan")) == sige.ERR_INVALID_ARG
    assert call(wsb=need - 1) == sige.ERR_WORKSPACE


def test_restore_tiles_validation(L):
    d = sige.TensorDesc(1, 32, 32, 16, sige.BF16, sige.NHWC)
    fake = ctypes.c_void_p(0x1000)

    def call(src=fake, dst=fake, desc=ctypes.byref(d), block=8, idx=fake, cnt=fake, cap=16):
        return L.sige_restore_tiles(src, dst, desc, block, idx, cnt, cap, None)
    assert call(src=None) == sige.ERR_INVALID_ARG
    assert call(dst=None) == sige.ERR_INVALID_ARG
    assert call(idx=None) == sige.ERR_INVALID_ARG
    assert call(block=0) == sige.ERR_INVALID_ARG
    assert call(cap=-1) == sige.ERR_INVALID_ARG
    assert call(cap=0) == sige.OK                      # nothing to restore, no launch
    dn = sige.TensorDesc(1, 32, 32, 16, sige.BF16, sige.NCHW)
    assert call(desc=ctypes.byref(dn)) == sige.ERR_UNSUPPORTED
    assert call(desc=None) == sige.ERR_INVALID_ARG


def test_attention_core_validation(L):
    d = sige.TensorDesc(1, 16, 16, 320, sige.BF16, sige.NHWC)
    fake = ctypes.c_void_p(0x1000)

    def call(q=fake, desc=ctypes.byref(d), k=fake, v=fake, keys=256, dv=320, heads=8, idx=fake, cnt=fake, cap=16,
             block=4, o=fake):
        return L.sige_attention_core(q, desc, k, v, keys, dv, heads, idx, cnt, cap, block, o, None)
    for kw in ({"q": None}, {"k": None}, {"v": None}, {"o": None}, {"idx": None}, {"cnt": None}, {"desc": None}):
        assert call(**kw) == sige.ERR_INVALID_ARG, kw
    assert call(keys=0) == sige.ERR_INVALID_ARG
    assert call(dv=0) == sige.ERR_INVALID_ARG
    assert call(heads=0) == sige.ERR_INVALID_ARG
    assert call(heads=3) == sige.ERR_INVALID_ARG           # 320 not a multiple of 3
    assert call(dv=324) == sige.ERR_INVALID_ARG            # dv not a multiple of heads
    assert call(block=0) == sige.ERR_INVALID_ARG
    assert call(cap=-1) == sige.ERR_INVALID_ARG
    assert call(block=9) == sige.ERR_UNSUPPORTED           # more than 64 queries per tile
    assert call(heads=1) == sige.ERR_UNSUPPORTED           # head width 320 > 256
    df = sige.TensorDesc(1, 16, 16, 320, sige.F32, sige.NHWC)
    assert call(desc=ctypes.byref(df)) == sige.ERR_UNSUPPORTED
    dn = sige.TensorDesc(1, 16, 16, 320, sige.BF16, sige.NCHW)
    assert call(desc=ctypes.byref(dn)) == sige.ERR_UNSUPPORTED
    big = sige.TensorDesc(1 << 16, 16, 16, 320, sige.BF16, sige.NHWC)
    assert call(desc=ctypes.byref(big), keys=1 << 16) == sige.ERR_INVALID_ARG   # keys x batch past 32 bits
    assert call(cap=0) == sige.OK                          # no tiles: no launch


def test_resblock_fused_validation(L):
    xd = sige.TensorDesc(1, 64, 64, 128, sige.BF16, sige.NHWC)
    fake = ctypes.c_void_p(0x1000)
    ws = ctypes.c_void_p(0x2000)

    def call(**kw):
        a = dict(x=fake, xd=ctypes.byref(xd), w1=fake, b1=None, g1s=fake, g1h=fake, w2=fake, b2=None, g2s=fake,
                 g2h=fake, block=8, idx=fake, cnt=fake, cap=64, y1=ctypes.c_void_p(0x10000000),
                 out=ctypes.c_void_p(0x20000000), ws=ws, wsb=256, st=None)
        a.update(kw)
        return L.sige_resblock_fused(*a.values())
    assert call(x=None) == sige.ERR_INVALID_ARG
    assert call(g2h=None) == sige.ERR_INVALID_ARG
    assert call(cap=-1) == sige.ERR_INVALID_ARG
    assert call(idx=ctypes.c_void_p(0x1004)) == sige.ERR_INVALID_ARG      # pairs need 8-byte alignment
    assert call(y1=fake) == sige.ERR_INVALID_ARG                          # y1 overlaps x
    assert call(block=4) == sige.ERR_UNSUPPORTED
    xd64 = sige.TensorDesc(1, 64, 64, 64, sige.BF16, sige.NHWC)
    assert call(xd=ctypes.byref(xd64)) == sige.ERR_UNSUPPORTED
    xdf = sige.TensorDesc(1, 64, 64, 128, sige.F32, sige.NHWC)
    assert call(xd=ctypes.byref(xdf)) == sige.ERR_UNSUPPORTED
    assert call(x=ctypes.c_void_p(0x1008)) == sige.ERR_UNSUPPORTED       # tensors need 16-byte alignment
    assert call(ws=None) == sige.ERR_WORKSPACE
    assert call(wsb=255) == sige.ERR_WORKSPACE
    n0 = sige.sige_launch_count()
    assert call(cap=0) == sige.OK                                        # nothing to do, no launch
    assert sige.sige_launch_count() == n0


def test_conv_fused_ext_validation(L):
    xd = sige.TensorDesc(1, 32, 64, 256, sige.BF16, sige.NHWC)
    cd = sige.ConvDesc(3, 2, 1, 256, 128, 4)
    yd = sige.TensorDesc(1, 64, 128, 128, sige.BF16, sige.NHWC)        # (32 - 1) * 2 - 2 + 3 + 1 = 64
    fake = ctypes.c_void_p(0x1000)
    ws = ctypes.c_void_p(0x2000)
    wsb = L.sige_conv_workspace_bytes(ctypes.byref(cd), 1, 512, 64, 128)

    def call(transposed=1, op=1, act=0, g=None, b=None, **kw):
        ext = sige.LayerExt(transposed, op, g, b, act)
        a = dict(x=fake, xd=ctypes.byref(xd), w=fake, bias=None, cd=ctypes.byref(cd), ext=ctypes.byref(ext),
                 idx=fake, cnt=fake, cap=512, gs=None, gh=None, res=None, y=fake, yd=ctypes.byref(yd), ws=ws,
                 wsb=wsb, st=None)
        a.update(kw)
        return L.sige_conv_fused_ext(*a.values())
    assert call(op=2) == sige.ERR_INVALID_ARG            # output padding >= stride
    assert call(act=3) == sige.ERR_INVALID_ARG
    assert call(b=0x3000) == sige.ERR_INVALID_ARG       # beta without gamma
    assert call(ext=None) == sige.ERR_INVALID_ARG
    assert call(gs=fake) == sige.ERR_INVALID_ARG        # scale without shift
    assert call(idx=ctypes.c_void_p(0x1004)) == sige.ERR_INVALID_ARG
    assert call(op=0) == sige.ERR_INVALID_ARG           # then the output would be 63 x 127
    yd_plain = sige.TensorDesc(1, 16, 32, 128, sige.BF16, sige.NHWC)
    assert call(transposed=0, op=0, yd=ctypes.byref(yd_plain)) != sige.ERR_INVALID_ARG
    assert call(g=0x3008) == sige.ERR_UNSUPPORTED       # misaligned modulation map
    assert call(wsb=16) == sige.ERR_WORKSPACE


def test_resblock_step_validation(L):
    xd = sige.TensorDesc(1, 64, 64, 128, sige.BF16, sige.NHWC)
    need = L.sige_resblock_step_workspace_bytes(ctypes.byref(xd), 8)
    assert need == 256 + 64 * 4                  # header + one 32-bit flag per 8x8 tile
    fake = ctypes.c_void_p(0x1000)
    ws = ctypes.c_void_p(0x2000)

    def call(**kw):
        a = dict(xo=ctypes.c_void_p(0x30000000), x=fake, xd=ctypes.byref(xd), thr=1e-3, dil=1, w1=fake, b1=None,
                 g1s=fake, g1h=fake, w2=fake, b2=None, g2s=fake, g2h=fake, block=8, idx=fake, cnt=fake, cap=64,
                 y1=ctypes.c_void_p(0x10000000), out=ctypes.c_void_p(0x20000000), ws=ws, wsb=need, st=None)
        a.update(kw)
        return L.sige_resblock_step(*a.values())
    assert call(xo=None) == sige.ERR_INVALID_ARG
    assert call(thr=-1.0) == sige.ERR_INVALID_ARG
    assert call(thr=float("nan")) == sige.ERR_INVALID_ARG
    assert call(dil=-1) == sige.ERR_INVALID_ARG
    assert call(block=4) == sige.ERR_UNSUPPORTED
    assert call(wsb=need - 1) == sige.ERR_WORKSPACE
    assert call(y1=ctypes.c_void_p(0x30000000)) == sige.ERR_INVALID_ARG     # y1 overlaps x_orig
    assert call(xo=ctypes.c_void_p(0x30000008)) == sige.ERR_UNSUPPORTED     # x_orig needs 16-byte alignment


def test_attention_path_selection(L):
    """Heads of width 8..64 in steps of 8 take the tensor-core kernel; wider
    heads or widths that are not multiples of 8, the CUDA-core one."""
    import torch
    q = lambda c: torch.empty((1, 8, 8, c), dtype=torch.bfloat16)
    assert sige.sige_attention_path(q(320), 320, 8) == 1      # heads of 40
    assert sige.sige_attention_path(q(64), 32, 1) == 1        # 64 / 32
    assert sige.sige_attention_path(q(32), 32, 4) == 1        # heads of 8
    assert sige.sige_attention_path(q(256), 256, 2) == 0      # heads of 128
    assert sige.sige_attention_path(q(60), 60, 2) == 0        # heads of 30
    assert sige.sige_attention_path(q(320), 320, 3) == sige.ERR_INVALID_ARG
    assert sige.sige_attention_path(torch.empty((1, 8, 8, 64)), 64, 1) == sige.ERR_UNSUPPORTED   # float32
