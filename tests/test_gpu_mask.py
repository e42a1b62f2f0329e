"""GPU mask reduction vs the oracle: bit-exact tile lists and counts.

mer.dev notes on SIGE, section 3.2 "Sparse Engine SIGE" (downsample, dilate,
select tiles); SIGE project page, "Overview" (active block indices)."""
import numpy as np
import pytest
import torch

import spatially_sparse_incremental_b200 as sige
from spatially_sparse_incremental_b200 import inputs

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _gpu_lists(a, b, thr, scales, dilate=1, layout=sige.NHWC, workspace=None):
    idx, cnt, ws = sige.sige_reduce_mask(a.to(DEV), b.to(DEV), thr, scales, dilate, layout, workspace=workspace)
    torch.cuda.synchronize()
    cnt = cnt.cpu().numpy()
    idx = idx.cpu().numpy()
    out, off = [], 0
    for s, (h, w, blk, cap) in enumerate(scales):
        out.append(idx[off:off + min(cnt[s], cap)])
        off += cap
    return out, cnt, ws


def _full_caps(scales):
    return [(h, w, b, -(-h // b) * -(-w // b)) for (h, w, b) in scales]


def test_cfg2_images_100_seeds(orc):
    scales = inputs.CFG2_SCALES
    for seed in range(100):
        o, e, _ = inputs.make_cfg2(seed)
        ref = orc.reduce_mask(o, e, 0.0, scales, 1, orc.NCHW)
        got, cnt, _ = _gpu_lists(o, e, 0.0, _full_caps(scales), 1, sige.NCHW)
        for s in range(len(scales)):
            assert cnt[s] == len(ref[s]), (seed, s)
            assert np.array_equal(got[s], ref[s]), (seed, s)


def test_cfg1_f32_nhwc(orc):
    for seed in range(10):
        L = inputs.make_cfg1(seed)
        sc = [(64, 64, 4)]
        ref = orc.reduce_mask(L.x_orig, L.x_edit, 1e-3, sc, 1)
        got, _, _ = _gpu_lists(L.x_orig, L.x_edit, 1e-3, _full_caps(sc))
        assert np.array_equal(got[0], ref[0])


def test_cfg3_bf16_activations(orc):
    for seed in range(3):
        blk = inputs.make_cfg3(seed)
        sc = [(256, 256, 8), (128, 128, 4), (64, 64, 2)]
        ref = orc.reduce_mask(blk.x_orig, blk.x_edit, 1e-3, sc, 1)
        got, _, _ = _gpu_lists(blk.x_orig, blk.x_edit, 1e-3, _full_caps(sc))
        for s in range(len(sc)):
            assert np.array_equal(got[s], ref[s]), (seed, s)


def test_random_small_cases(orc):
    # covers the scalar path (C*esize not a multiple of 16, odd widths), both
    # layouts, batch > 1, several scales, dilation 0..2, ragged tile grids.
    rng = np.random.default_rng(7)
    for case in range(150):
        dtype = [torch.uint8, torch.float32, torch.bfloat16][case % 3]
        layout = sige.NHWC if rng.random() < 0.5 else sige.NCHW
        N = int(rng.integers(1, 3))
        f = int(rng.choice([1, 2, 4]))
        Hs, Ws = int(rng.integers(1, 12)), int(rng.integers(1, 12))
        H, W = Hs * f, Ws * f
        C = int(rng.choice([1, 3, 8, 16, 64]))
        if dtype == torch.uint8:
            a = torch.from_numpy(rng.integers(0, 256, size=(N, H, W, C)).astype(np.uint8))
        else:
            a = torch.from_numpy(rng.normal(size=(N, H, W, C)).astype(np.float32)).to(dtype)
        b = a.clone()
        m = rng.random((N, H, W)) < rng.choice([0.0, 0.02, 0.1, 1.0])
        if dtype == torch.uint8:
            b[torch.from_numpy(m)] = b[torch.from_numpy(m)] ^ 1
        else:
            b[torch.from_numpy(m)] = b[torch.from_numpy(m)] + 1.0
        if layout == sige.NCHW:
            a, b = a.permute(0, 3, 1, 2).contiguous(), b.permute(0, 3, 1, 2).contiguous()
        thr = 0.0 if dtype == torch.uint8 else 1e-3
        sc = [(H, W, int(rng.integers(1, 5)))]
        if f > 1:
            sc.append((Hs, Ws, int(rng.integers(1, 4))))
        D = int(rng.integers(0, 3))
        ref = orc.reduce_mask(a, b, thr, sc, D, orc.NHWC if layout == sige.NHWC else orc.NCHW)
        got, _, _ = _gpu_lists(a, b, thr, _full_caps(sc), D, layout)
        for s in range(len(sc)):
            assert np.array_equal(got[s], ref[s]), (case, s)


def test_empty_and_full_masks():
    x = torch.randn(1, 64, 64, 32)
    got, cnt, _ = _gpu_lists(x, x.clone(), 1e-3, [(64, 64, 8, 64)])
    assert cnt[0] == 0 and len(got[0]) == 0
    got, cnt, _ = _gpu_lists(x, x + 1, 1e-3, [(64, 64, 8, 64), (32, 32, 4, 64)])
    want = np.array([(i, j) for i in range(0, 64, 8) for j in range(0, 64, 8)], np.int32)
    assert cnt[0] == 64 and np.array_equal(got[0], want)
    want2 = np.array([(i, j) for i in range(0, 32, 4) for j in range(0, 32, 4)], np.int32)
    assert np.array_equal(got[1], want2)


def test_capacity_overflow_reports_and_truncates(orc):
    x = torch.randn(1, 64, 64, 16)
    y = x + 1
    ref = orc.reduce_mask(x, y, 1e-3, [(64, 64, 4)], 1)[0]
    got, cnt, ws = _gpu_lists(x, y, 1e-3, [(64, 64, 4, 100)])
    assert cnt[0] == 256
    assert np.array_equal(got[0], ref[:100])
    assert sige.sige_get_error(ws) == sige.ERR_CAPACITY
    assert sige.sige_get_error(ws) == sige.OK                # cleared
    # the workspace is reusable and left zero-filled past its header
    got, cnt, ws = _gpu_lists(x, y, 1e-3, [(64, 64, 4, 256)], workspace=ws)
    assert cnt[0] == 256 and sige.sige_get_error(ws) == sige.OK
    assert int(ws[256:].sum().item()) == 0


def test_workspace_reuse_across_calls(orc):
    ws = None
    for seed in range(5):
        o, e, _ = inputs.make_cfg2(seed)
        ref = orc.reduce_mask(o, e, 0.0, inputs.CFG2_SCALES, 1, orc.NCHW)
        got, _, ws = _gpu_lists(o, e, 0.0, _full_caps(inputs.CFG2_SCALES), 1, sige.NCHW, workspace=ws)
        for s in range(4):
            assert np.array_equal(got[s], ref[s])


def test_wide_grids_multiword_rows(orc):
    # tile rows wider than 32 tiles span several bit words: dilation must
    # carry across word boundaries (and stay inside the last, partial word)
    rng = np.random.default_rng(11)
    for (H, W, b, D) in [(64, 300, 1, 1), (40, 520, 2, 2), (16, 1000, 1, 5), (48, 96, 1, 1), (8, 2048, 1, 33)]:
        a = torch.from_numpy(rng.normal(size=(1, H, W, 8)).astype(np.float32))
        e = a.clone()
        m = rng.random((H, W)) < 0.01
        m[:, 31] = rng.random(H) < 0.3        # flags right at word boundaries
        m[:, 32] |= rng.random(H) < 0.3
        e[0, torch.from_numpy(m)] += 1.0
        sc = [(H, W, b)]
        ref = orc.reduce_mask(a, e, 1e-3, sc, D)
        got, cnt, _ = _gpu_lists(a, e, 1e-3, _full_caps(sc), D)
        assert cnt[0] == len(ref[0]) and np.array_equal(got[0], ref[0]), (H, W, b, D)


@pytest.mark.parametrize("area", [0.10, 0.20, 0.30, 0.50])
def test_cfg3_large_edits(orc, area):
    # large edits: many chunks hold nothing but differing vectors
    blk = inputs.make_cfg3(0, H=256, W=256, C=128, area=area, block=8)
    sc = [(256, 256, 8)]
    ref = orc.reduce_mask(blk.x_orig, blk.x_edit, 1e-3, sc, 1)
    got, cnt, ws = _gpu_lists(blk.x_orig, blk.x_edit, 1e-3, _full_caps(sc))
    assert sige.sige_get_error(ws) == sige.OK
    assert cnt[0] == len(ref[0]) and np.array_equal(got[0], ref[0])


def test_pixel_dilation_random_cases(orc):
    rng = np.random.default_rng(21)
    for case in range(80):
        dtype = [torch.uint8, torch.float32, torch.bfloat16][case % 3]
        layout = sige.NHWC if rng.random() < 0.6 else sige.NCHW
        f = int(rng.choice([1, 2, 4]))
        Hs, Ws = int(rng.integers(2, 20)), int(rng.integers(2, 20))
        H, W, C = Hs * f, Ws * f, int(rng.choice([3, 8, 16, 64]))
        if dtype == torch.uint8:
            a = torch.from_numpy(rng.integers(0, 256, size=(1, H, W, C)).astype(np.uint8))
        else:
            a = torch.from_numpy(rng.normal(size=(1, H, W, C)).astype(np.float32)).to(dtype)
        b = a.clone()
        m = rng.random((1, H, W)) < rng.choice([0.01, 0.05, 0.3])
        b[torch.from_numpy(m)] = (b[torch.from_numpy(m)] ^ 1) if dtype == torch.uint8 else b[torch.from_numpy(m)] + 1.0
        if layout == sige.NCHW:
            a, b = a.permute(0, 3, 1, 2).contiguous(), b.permute(0, 3, 1, 2).contiguous()
        thr = 0.0 if dtype == torch.uint8 else 1e-3
        sc = [(H, W, int(rng.integers(1, 6))), (Hs, Ws, int(rng.integers(1, 4)))]
        R = int(rng.integers(0, 4))
        ref = orc.reduce_mask_px(a, b, thr, sc, R, orc.NHWC if layout == sige.NHWC else orc.NCHW)
        caps = _full_caps(sc)
        idx, cnt, _ = sige.sige_reduce_mask_px(a.to(DEV), b.to(DEV), thr, caps, R, layout)
        torch.cuda.synchronize()
        cnt, idx, off = cnt.cpu().numpy(), idx.cpu().numpy(), 0
        for s, (h, w, blk, cap) in enumerate(caps):
            assert cnt[s] == len(ref[s]) and np.array_equal(idx[off:off + cnt[s]], ref[s]), (case, s, R)
            off += cap


def test_pixel_dilation_cfg3(orc):
    blk = inputs.make_cfg3(0, H=256, W=256, C=128, area=0.012)
    sc = [(256, 256, 8)]
    for R in (1, 2):
        ref = orc.reduce_mask_px(blk.x_orig, blk.x_edit, 1e-3, sc, R)[0]
        idx, cnt, ws = sige.sige_reduce_mask_px(blk.x_orig.to(DEV), blk.x_edit.to(DEV), 1e-3, _full_caps(sc), R)
        torch.cuda.synchronize()
        n = int(cnt[0].item())
        assert n == len(ref) and np.array_equal(idx[:n].cpu().numpy(), ref)
        assert sige.sige_get_error(ws) == sige.OK


def test_host_counts_equal_device_counts(orc):
    """The opt-in host copy of the counts (the call synchronises the stream)
    holds exactly the device counts, for one and for several scales."""
    blk = inputs.make_cfg3(7)
    xo, xe = blk.x_orig.to(DEV), blk.x_edit.to(DEV)
    sc = [(256, 256, 8, 1024), (128, 128, 4, 1024), (64, 64, 2, 1024)]
    idx, cnt, _, host = sige.sige_reduce_mask(xo, xe, 1e-3, sc, 1, host_counts=True)
    assert host == cnt.cpu().tolist()
    ref = orc.reduce_mask(blk.x_orig, blk.x_edit, 1e-3, [s[:3] for s in sc], 1)
    assert host == [len(r) for r in ref]
    o, e, _ = inputs.make_cfg2(11)
    caps = _full_caps(inputs.CFG2_SCALES)
    _, cnt2, _, host2 = sige.sige_reduce_mask_px(o.to(DEV), e.to(DEV), 0.0, caps, 2, sige.NCHW, host_counts=True)
    assert host2 == cnt2.cpu().tolist()


def test_host_counts_refused_during_capture():
    """A capturing stream cannot be synchronised: the request is refused
    before anything is enqueued, and the capture stays valid."""
    x = torch.zeros((1, 64, 64, 8), dtype=torch.float32, device=DEV)
    sc = [(64, 64, 8, 64)]
    ws = sige.zeros_workspace(4096, DEV)
    sige.sige_reduce_mask(x, x, 0.0, sc, 1, workspace=ws)   # one-time set-up outside the capture
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        with pytest.raises(sige.SigeError) as ei:
            sige.sige_reduce_mask(x, x, 0.0, sc, 1, workspace=ws, stream=s, host_counts=True)
        sige.sige_reduce_mask(x, x, 0.0, sc, 1, workspace=ws, stream=s)
    assert ei.value.status == sige.ERR_INVALID_ARG
    g.replay()
    torch.cuda.synchronize()


def test_expired_wait_reports_timeout_and_the_next_call_is_exact(orc):
    """Failure path of the reducing CTA's bounded wait.  With the bound set to
    one clock cycle it expires while the other CTAs still stream the 33 MB of
    input: the call returns, the workspace header holds SIGE_ERR_TIMEOUT with
    the wait site (-1) in its detail word, and no count is written.  With the
    default bound restored and the workspace zero-filled again, the next call
    gives the oracle's list bit for bit."""
    blk = inputs.make_cfg3(2)
    xo, xe = blk.x_orig.to(DEV), blk.x_edit.to(DEV)
    sc = [(256, 256, 8, 1024)]
    ref = orc.reduce_mask(blk.x_orig, blk.x_edit, 1e-3, [(256, 256, 8)], 1)[0]
    ws = sige.zeros_workspace(sige.sige_reduce_mask_workspace_bytes(sige.tensor_desc(xo), sc), DEV)
    cnt = torch.full((1,), -9, dtype=torch.int32, device=DEV)
    try:
        sige.sige_set_wait_cycles(1)
        sige.sige_reduce_mask(xo, xe, 1e-3, sc, 1, counts=cnt, workspace=ws)
        torch.cuda.synchronize()
    finally:
        sige.sige_set_wait_cycles(0)
    head = ws[:8].view(torch.int32).cpu().tolist()
    assert head == [sige.ERR_TIMEOUT, -1], head
    assert int(cnt.item()) == -9                       # the reducer wrote nothing
    assert sige.sige_get_device_error(ws) == sige.ERR_TIMEOUT
    assert sige.sige_get_device_error(ws) == sige.OK   # read and cleared
    ws.zero_()
    got, cnt2, _ = _gpu_lists(blk.x_orig, blk.x_edit, 1e-3, sc, workspace=ws)
    assert int(cnt2[0]) == len(ref) and np.array_equal(got[0], ref)
    assert sige.sige_get_device_error(ws) == sige.OK
