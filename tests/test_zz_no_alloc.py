"""The allocation-free mask reduction (sige_reduce_mask_static).

It serves callers that cannot give the library a device workspace, such as a
process that reserves all of its device memory up front or a plugin host that
exposes no allocator.  Its scratch is a fixed array inside the library that
every call on a device shares.  This file is named so that pytest collects it
last: if it fails, a run stopping at the first failure has already run every
other test.  It must also pass on its own in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

import spatially_sparse_incremental_b200 as sige
from spatially_sparse_incremental_b200 import inputs

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _lists(idx, cnt, scales):
    idx, cnt = idx.cpu().numpy(), cnt.cpu().numpy()
    out, off = [], 0
    for s, (_, _, _, cap) in enumerate(scales):
        out.append(idx[off:off + min(int(cnt[s]), cap)].copy())
        off += cap
    return out, cnt.copy()


def _static_call(a, b, thr, scales, dilate, layout):
    """Direct C-ABI call of the new entry point (no workspace argument)."""
    L = sige.lib()
    desc = sige.tensor_desc(a, layout)
    arr = (sige.ScaleDesc * len(scales))(*[sige.ScaleDesc(*s) for s in scales])
    idx = torch.full((sum(s[3] for s in scales), 2), -7, dtype=torch.int32, device=DEV)
    cnt = torch.full((len(scales),), -7, dtype=torch.int32, device=DEV)
    st = L.sige_reduce_mask_static(ctypes.c_void_p(a.data_ptr()), ctypes.c_void_p(b.data_ptr()),
                                   ctypes.byref(desc), float(thr), int(dilate), len(scales), arr,
                                   ctypes.c_void_p(idx.data_ptr()), ctypes.c_void_p(cnt.data_ptr()),
                                   ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == sige.OK, sige.status_string(st)
    torch.cuda.synchronize()
    return _lists(idx, cnt, scales)


def test_static_scratch_matches_workspace_entry_point_twice_in_a_row():
    scales = [(h, w, b, -(-h // b) * -(-w // b)) for (h, w, b) in inputs.CFG2_SCALES]
    for seed in (3, 4):      # two calls in a row on different edits share the scratch
        o, e, _ = inputs.make_cfg2(seed)
        o, e = o.to(DEV), e.to(DEV)
        got, gcnt = _static_call(o, e, 0.0, scales, 1, sige.NCHW)
        ref_idx, ref_cnt, _ = sige.sige_reduce_mask(o, e, 0.0, scales, 1, sige.NCHW)
        torch.cuda.synchronize()
        ref, rcnt = _lists(ref_idx, ref_cnt, scales)
        assert np.array_equal(gcnt, rcnt), (seed, gcnt, rcnt)
        for s in range(len(scales)):
            assert np.array_equal(got[s], ref[s]), (seed, s)
    # bf16 activations, one scale, same check
    blk = inputs.make_cfg3(5, H=64, W=64, C=128, area=0.05)
    xo, xe = blk.x_orig.to(DEV), blk.x_edit.to(DEV)
    sc = [(64, 64, 8, 64)]
    for _ in range(2):
        got, gcnt = _static_call(xo, xe, 1e-3, sc, 1, sige.NHWC)
        ri, rc, _ = sige.sige_reduce_mask(xo, xe, 1e-3, sc, 1)
        ref, rcnt = _lists(ri, rc, sc)
        assert np.array_equal(gcnt, rcnt) and np.array_equal(got[0], ref[0])


def test_static_scratch_rejects_oversized_requests():
    x = torch.zeros((1, 256, 512, 8), dtype=torch.float32, device=DEV)
    too_big = [(256, 512, 1, 256 * 512)]          # 131072 tile flags > 64 KB of scratch
    n0 = sige.sige_launch_count()
    with pytest.raises(sige.SigeError) as ei:
        sige.sige_reduce_mask_static(x, x, 0.0, too_big)
    assert ei.value.status == sige.ERR_WORKSPACE
    assert sige.sige_launch_count() == n0


def test_static_scratch_lists_equal_the_oracle(orc):
    """The allocation-free call's lists against the oracle itself, not only
    against the workspace entry point."""
    caps = [(h, w, b, -(-h // b) * -(-w // b)) for (h, w, b) in inputs.CFG2_SCALES]
    for seed in (21, 22):
        o, e, _ = inputs.make_cfg2(seed)
        got, gcnt = _static_call(o.to(DEV), e.to(DEV), 0.0, caps, 1, sige.NCHW)
        ref = orc.reduce_mask(o, e, 0.0, inputs.CFG2_SCALES, 1, orc.NCHW)
        for s in range(len(caps)):
            assert int(gcnt[s]) == len(ref[s]) and np.array_equal(got[s], ref[s]), (seed, s)


def test_static_scratch_marks_an_incomplete_call_with_negative_counts():
    """A call whose reducing CTA gave up (its bounded wait, shortened here to
    one clock cycle, expired) cannot report through a workspace header, so it
    leaves counts of -1; the next call, with the default bound, is exact."""
    blk = inputs.make_cfg3(9)
    xo, xe = blk.x_orig.to(DEV), blk.x_edit.to(DEV)
    sc = [(256, 256, 8, 1024)]
    try:
        sige.sige_set_wait_cycles(1)
        _, cnt = sige.sige_reduce_mask_static(xo, xe, 1e-3, sc)
        torch.cuda.synchronize()
    finally:
        sige.sige_set_wait_cycles(0)
    assert int(cnt.item()) < 0
    got, gcnt = _static_call(xo, xe, 1e-3, sc, 1, sige.NHWC)
    ri, rc, _ = sige.sige_reduce_mask(xo, xe, 1e-3, sc, 1)
    ref, rcnt = _lists(ri, rc, sc)
    assert np.array_equal(gcnt, rcnt) and np.array_equal(got[0], ref[0])
