"""Attention by query-token pruning on the GPU against the oracle.

The nubint.ai review of the SIGE paper ("Proposed method", fourth item; "Main
findings") carries the engine over to attention layers by pruning the query
tokens of unedited regions; the mer.dev notes (abstract) name Stable
Diffusion's attention layers.  The reading (queries only for the tokens under
the active tiles, keys and values dense, every other token keeps its cached
bytes) is the oracle's, ``oracle/attention.py``.

Checked through the C ABI:
  * ``sige_attention_core`` against ``attention_core_tokens`` at the active
    tokens: per element within max(2e-2 RMS, one bf16 ulp) of the oracle's
    value rounded to bf16, and against its unrounded float64 value within
    plain 2e-2 RMS (CUDA-core kernel, fp32 weights) or within the bound that
    the tensor-core kernel's bf16 weights give (``assert_weight_rounding_bound``);
    every other byte of the output untouched;
  * self- and cross-attention, 1/2/4/8 heads, head widths 40/64/128, tiles of
    1/2/4/8 pixels, batch 1 and 2, maps that tiles do not divide, key counts
    that are not a multiple of the kernel's chunk, an empty list;
  * ``sige_attention_sparse`` (q projection, key/value cache update, the step,
    output projection with bias and residual) against ``sparse_attention`` with
    bf16 storage of q, k, v and o.
"""
import numpy as np
import pytest
import torch

import spatially_sparse_incremental_b200 as sige
from helpers import assert_close, bf16_ulp, bits, rel_err
from oracle import attention as att

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _bf16(rng, *shape, scale=1.0):
    return torch.from_numpy(rng.normal(0.0, scale, size=shape)).to(torch.bfloat16)


def _tile_list(rng, H, W, b, frac):
    """A random set of tile origins in row-major order (at least one)."""
    every = [(h, w) for h in range(0, H, b) for w in range(0, W, b)]
    keep = rng.random(len(every)) < frac
    if not keep.any():
        keep[rng.integers(len(every))] = True
    return np.array([t for t, k in zip(every, keep) if k], dtype=np.int32).reshape(-1, 2), len(every)


def _device_list(idx, cap):
    d = torch.zeros((max(cap, 1), 2), dtype=torch.int32)
    d[:len(idx)] = torch.from_numpy(idx)
    return d.to(DEV), torch.tensor([len(idx)], dtype=torch.int32, device=DEV)


def _core_case(seed, N, H, W, D, Dv, heads, b, Lk=None, frac=0.3):
    rng = np.random.default_rng(seed)
    q = _bf16(rng, N, H, W, D)
    Lk = H * W if Lk is None else Lk
    k = _bf16(rng, N, Lk, D)
    v = _bf16(rng, N, Lk, Dv)
    idx, cap = _tile_list(rng, H, W, b, frac)
    o0 = _bf16(rng, N, H, W, Dv)                 # stands for the cached output
    idx_d, cnt = _device_list(idx, cap)
    o = o0.to(DEV)
    sige.sige_attention_core(q.to(DEV), k.to(DEV), v.to(DEV), heads, idx_d, cnt, cap, b, o)
    torch.cuda.synchronize()
    tok, ref = att.attention_core_tokens(q, k, v, heads, idx, b, H, W)
    got = o.cpu().view(N, H * W, Dv)
    touched = torch.zeros(H * W, dtype=torch.bool)
    touched[torch.from_numpy(tok)] = True
    # outside the active tokens: the cached bytes, bit for bit
    assert torch.equal(bits(got[:, ~touched]), bits(o0.view(N, H * W, Dv)[:, ~touched]))
    g = got[:, torch.from_numpy(tok)]
    assert_close(g, att._round_to(ref, torch.bfloat16), torch.bfloat16, what="attention core (rounded ref)")
    if sige.sige_attention_path(q, Dv, heads) == 1:
        _, ref_abs = att.attention_core_tokens(q, k, v.abs(), heads, idx, b, H, W)
        assert_weight_rounding_bound(g, ref, ref_abs)
    else:
        e = rel_err(g, torch.from_numpy(ref))
        assert e <= 2e-2, f"attention core vs unrounded oracle: max|d|/rms = {e:.3g}"
    return len(tok)


def assert_weight_rounding_bound(got, ref, ref_abs):
    """The tensor-core kernel's bound against the unrounded oracle.  It rounds
    each weight p_j = exp(s_j - m) to bf16 (relative error <= 2^-9) before the
    P V product and divides by the sum of the unrounded weights, so its float32
    row is within 2^-9 sum_j p_j |v_j| / sum_j p_j of the exact one (ref_abs
    is the oracle's attention over |v|: that weighted sum); the final rounding
    adds half a bf16 ulp of the output.  A 1% margin on the first term and
    1e-5 RMS cover the float32 sums and the exponent approximation (2^-22)."""
    g = got.double().numpy()
    r = np.asarray(ref, dtype=np.float64)
    rms = float(np.sqrt(np.mean(r * r)))
    allow = 2.0 ** -9 * 1.01 * np.asarray(ref_abs, dtype=np.float64) + 0.5 * bf16_ulp(g) + 1e-5 * rms
    worst = float((np.abs(g - r) / allow).max())
    assert worst <= 1.0, f"tensor-core attention vs unrounded oracle: max |d| / bound = {worst:.3g}"


@pytest.mark.parametrize("N,H,W,D,Dv,heads,b", [
    (1, 16, 16, 64, 64, 1, 4),      # one head of width 64
    (1, 16, 16, 256, 256, 4, 2),    # four heads of 64, 2x2 tiles
    (2, 12, 12, 128, 128, 1, 4),    # batch 2, head width 128
    (1, 16, 16, 320, 320, 8, 4),    # the SD-latent layer's eight heads of 40
    (1, 13, 11, 128, 64, 2, 4),     # ragged map, dv != d
    (1, 8, 8, 64, 64, 1, 8),        # one 8x8 tile = 64 queries
    (1, 9, 7, 32, 32, 4, 1),        # one-pixel tiles, heads of 8
    (2, 16, 16, 256, 256, 2, 8),    # heads of 128, 8x8 tiles
])
def test_attention_core_self(N, H, W, D, Dv, heads, b):
    assert _core_case(100 + H + D + heads + b, N, H, W, D, Dv, heads, b) > 0


@pytest.mark.parametrize("Lk,heads", [(77, 8), (33, 2), (1, 2), (300, 4)])
def test_attention_core_cross(Lk, heads):
    """Keys and values from a context sequence of Lk tokens (not a multiple of
    the 32-key chunk; a single key: weight 1)."""
    _core_case(7 + Lk, 1, 16, 16, 320, 320, heads, 4, Lk=Lk)


def test_attention_core_empty_list_writes_nothing():
    rng = np.random.default_rng(3)
    q = _bf16(rng, 1, 8, 8, 64)
    kv = _bf16(rng, 1, 64, 64)
    o0 = _bf16(rng, 1, 8, 8, 64)
    idx_d = torch.zeros((4, 2), dtype=torch.int32, device=DEV)
    cnt = torch.zeros(1, dtype=torch.int32, device=DEV)
    o = o0.to(DEV)
    sige.sige_attention_core(q.to(DEV), kv.to(DEV), kv.to(DEV), 1, idx_d, cnt, 4, 4, o)
    torch.cuda.synchronize()
    assert torch.equal(bits(o.cpu()), bits(o0))


def test_attention_core_every_tile_is_dense_attention():
    """Every tile listed: the step is plain multi-head attention over the map."""
    rng = np.random.default_rng(5)
    H = W = 8
    idx = np.array([(h, w) for h in range(0, H, 4) for w in range(0, W, 4)], dtype=np.int32)
    q = _bf16(rng, 1, H, W, 128)
    k = _bf16(rng, 1, H * W, 128)
    v = _bf16(rng, 1, H * W, 128)
    idx_d, cnt = _device_list(idx, len(idx))
    o = torch.zeros((1, H, W, 128), dtype=torch.bfloat16, device=DEV)
    sige.sige_attention_core(q.to(DEV), k.to(DEV), v.to(DEV), 2, idx_d, cnt, len(idx), 4, o)
    torch.cuda.synchronize()
    qf, kf, vf = (t.double().reshape(1, -1, 2, 64).transpose(1, 2) for t in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(qf, kf, vf).transpose(1, 2).reshape(1, H, W, 128)
    assert rel_err(o.cpu(), ref) <= 2e-2


def _layer_case(seed, N, H, W, C, D, heads, b, cross=False, Lc=77):
    rng = np.random.default_rng(seed)
    idx, cap = _tile_list(rng, H, W, b, 0.2)
    x0 = _bf16(rng, N, H, W, C)
    x1 = x0.clone()
    for h0, w0 in idx:                           # the edit lies inside the listed tiles
        x1[:, h0:h0 + b, w0:w0 + b] = _bf16(rng, N, min(b, H - h0), min(b, W - w0), C)
    s = C ** -0.5
    wq, wk, wv = (rng.normal(0, s, size=(C, D)) for _ in range(3))
    wo, bo = rng.normal(0, D ** -0.5, size=(D, C)), rng.normal(0, 0.1, size=C)
    as_conv = lambda m: torch.from_numpy(np.ascontiguousarray(m.T)).to(torch.bfloat16).reshape(m.shape[1], 1, 1, -1)
    Wq, Wk, Wv, Wo = (as_conv(m) for m in (wq, wk, wv, wo))
    # the projections the engine stores are bf16: the oracle takes the same
    # bf16 weights
    f = lambda t: t.reshape(t.shape[0], -1).T.double().numpy()
    wq_, wk_, wv_, wo_ = f(Wq), f(Wk), f(Wv), f(Wo)
    y0 = _bf16(rng, N, H, W, C)                  # stands for the cached layer output
    idx_d, cnt = _device_list(idx, cap)
    y = y0.to(DEV)
    if cross:
        ctx = _bf16(rng, N, Lc, C)
        kmap = att._round_to(ctx.double().numpy() @ wk_, torch.bfloat16).view(N, Lc, D).to(DEV)
        vmap = att._round_to(ctx.double().numpy() @ wv_, torch.bfloat16).view(N, Lc, D).to(DEV)
        sige.sige_attention_sparse(x1.to(DEV), idx_d, cnt, cap, b, Wq.to(DEV), Wo.to(DEV),
                                   torch.from_numpy(bo).float().to(DEV), heads, kmap, vmap, y, residual=x1.to(DEV))
        ref = att.sparse_attention(x1, y0, idx, b, wq_, wk_, wv_, wo_, bo, heads, context=ctx, residual=x1,
                                   storage=torch.bfloat16)
    else:
        # caches of the original map's keys and values, then updated at the tokens
        seq0 = x0.double().numpy().reshape(N, H * W, C)
        kmap = att._round_to(seq0 @ wk_, torch.bfloat16).view(N, H, W, D).to(DEV)
        vmap = att._round_to(seq0 @ wv_, torch.bfloat16).view(N, H, W, D).to(DEV)
        sige.sige_attention_sparse(x1.to(DEV), idx_d, cnt, cap, b, Wq.to(DEV), Wo.to(DEV),
                                   torch.from_numpy(bo).float().to(DEV), heads, kmap, vmap, y,
                                   wk=Wk.to(DEV), wv=Wv.to(DEV), residual=x1.to(DEV))
        ref = att.sparse_attention(x1, y0, idx, b, wq_, wk_, wv_, wo_, bo, heads, residual=x1,
                                   storage=torch.bfloat16)
    torch.cuda.synchronize()
    tok = att.active_tokens(idx, b, H, W)
    got = y.cpu().view(N, H * W, C)
    refv = ref.view(N, H * W, C)
    touched = torch.zeros(H * W, dtype=torch.bool)
    touched[torch.from_numpy(tok)] = True
    assert torch.equal(bits(got[:, ~touched]), bits(y0.view(N, H * W, C)[:, ~touched]))
    t = torch.from_numpy(tok)
    assert_close(got[:, t], refv[:, t], torch.bfloat16, what="sparse attention layer")


@pytest.mark.parametrize("heads", [1, 4])
def test_attention_layer_self(heads):
    _layer_case(11 + heads, 1, 16, 16, 128, 128, heads, 4)


def test_attention_layer_sd_latent_shape():
    """C = 320 with eight heads, 4x4 tiles, batch 2."""
    _layer_case(23, 2, 16, 16, 320, 320, 8, 4)


def test_attention_layer_cross():
    _layer_case(31, 1, 16, 16, 320, 320, 8, 4, cross=True)


# ---- the tensor-core kernel (heads of width 8..64, multiples of 8): 128-key
# chunks, key splits over a cluster when the list is short, a running maximum
# that moves the accumulator's base only when it grows by more than 2^8

@pytest.mark.parametrize("N,H,W,D,Dv,heads,b,frac", [
    (1, 64, 64, 320, 320, 8, 4, 0.01),   # the SD-latent layer, 4096 keys, a short list: keys split 8 ways
    (1, 64, 64, 320, 320, 8, 4, 0.15),   # a longer list: fewer splits
    (2, 32, 32, 128, 128, 2, 8, 0.05),   # batch 2, 1024 keys, heads of 64
    (1, 48, 40, 64, 64, 8, 2, 0.03),     # heads of 8 (padded to 16), 1920 keys: a ragged last chunk
    (1, 40, 40, 192, 96, 4, 8, 0.1),     # dv != d (48 / 24), 1600 keys
])
def test_attention_core_tensor_path_long_keys(N, H, W, D, Dv, heads, b, frac):
    assert sige.sige_attention_path(torch.empty((N, H, W, D), dtype=torch.bfloat16), Dv, heads) == 1
    assert _core_case(500 + H + W + D + b, N, H, W, D, Dv, heads, b, frac=frac) > 0


def test_attention_core_tensor_path_every_tile_several_rounds():
    """Every tile of a 48x48 map, batch 2, eight heads of 40: 288 blocks of
    128 queries, more than the launch's CTAs, so each CTA walks several."""
    assert _core_case(77, 2, 48, 48, 320, 320, 8, 4, frac=1.0) == 48 * 48


def test_attention_core_growing_scores():
    """Scores that rise along the key sequence (by ~80 in base-2 exponent
    units over 4096 keys) move the running maximum chunk after chunk and make
    the key splits' maxima differ by far more than 2^8: the rescaled
    accumulator and the weighted merge must still give the softmax of the
    oracle."""
    rng = np.random.default_rng(9)
    N, H, W, D, heads, b = 1, 64, 64, 64, 1, 8
    u = rng.normal(size=D)
    u /= np.linalg.norm(u)
    q = torch.from_numpy(4.0 * u + 0.3 * rng.normal(size=(N, H, W, D))).to(torch.bfloat16)
    ramp = np.linspace(0.0, 1.0, H * W)[None, :, None]
    k = torch.from_numpy(110.0 * ramp * u + 0.3 * rng.normal(size=(N, H * W, D))).to(torch.bfloat16)
    v = _bf16(rng, N, H * W, D)
    idx = np.array([(8, 16), (40, 0), (56, 56)], dtype=np.int32)
    idx_d, cnt = _device_list(idx, 64)
    o0 = _bf16(rng, N, H, W, D)
    o = o0.to(DEV)
    sige.sige_attention_core(q.to(DEV), k.to(DEV), v.to(DEV), heads, idx_d, cnt, 64, b, o)
    torch.cuda.synchronize()
    tok, ref = att.attention_core_tokens(q, k, v, heads, idx, b, H, W)
    got = o.cpu().view(N, H * W, D)
    g = got[:, torch.from_numpy(tok)]
    assert_close(g, att._round_to(ref, torch.bfloat16), torch.bfloat16, what="growing scores (rounded ref)")
    _, ref_abs = att.attention_core_tokens(q, k, v.abs(), heads, idx, b, H, W)
    assert_weight_rounding_bound(g, ref, ref_abs)
    touched = torch.zeros(H * W, dtype=torch.bool)
    touched[torch.from_numpy(tok)] = True
    assert torch.equal(bits(got[:, ~touched]), bits(o0.view(N, H * W, D)[:, ~touched]))
