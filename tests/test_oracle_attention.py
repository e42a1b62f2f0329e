"""Pins for the sparse-attention oracle (query-token pruning), never against the
oracle itself:

  * with every query token active, the result is textbook multi-head attention:
    torch.nn.functional.scaled_dot_product_attention in float64, self- and
    cross-attention, with output projection, bias and residual;
  * closed forms: one key gives softmax weight 1 (output = its value row
    projected); equal keys give uniform weights (output = mean of the values);
  * invariants: permuting the key/value tokens together changes nothing;
    tokens outside the tile list keep the cached bytes; an empty list returns
    the cache;
  * the active token set against the tile-coverage helper the conv tests use.

The reading (queries only for the tokens under the active tiles, keys and
values dense) follows the nubint.ai review of the SIGE paper ("Proposed
method": attention layers by pruning unedited query tokens) and the mer.dev
notes (abstract: attention layers for Stable Diffusion).
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

from helpers import bits, random_cache, tile_cover
from oracle import attention as att


def _rand(rng, *shape, scale=1.0):
    return rng.normal(0.0, scale, size=shape)


def _case(seed, N=2, H=6, W=5, C=32, D=32, Dv=32, Co=24, Ck=None, Lc=None):
    rng = np.random.default_rng(seed)
    x = _rand(rng, N, H, W, C)
    ck = C if Ck is None else Ck
    wq, wk, wv = _rand(rng, C, D, scale=C ** -0.5), _rand(rng, ck, D, scale=ck ** -0.5), _rand(rng, ck, Dv, scale=ck ** -0.5)
    wo, bo = _rand(rng, Dv, Co, scale=Dv ** -0.5), _rand(rng, Co, scale=0.1)
    ctx = _rand(rng, N, Lc, ck) if Lc is not None else None
    res = _rand(rng, N, H, W, Co)
    return x, wq, wk, wv, wo, bo, ctx, res


def _all_tiles(H, W, b):
    return np.array([(h, w) for h in range(0, H, b) for w in range(0, W, b)], dtype=np.int32)


def _library(x, wq, wk, wv, wo, bo, heads, ctx, res):
    t = lambda a: torch.from_numpy(np.asarray(a, dtype=np.float64))
    X = t(x)
    N, H, W, C = X.shape
    seq = X.reshape(N, H * W, C)
    src = seq if ctx is None else t(ctx)
    q, k, v = seq @ t(wq), src @ t(wk), src @ t(wv)
    split = lambda a: a.reshape(N, a.shape[1], heads, -1).transpose(1, 2)
    o = F.scaled_dot_product_attention(split(q), split(k), split(v))
    o = o.transpose(1, 2).reshape(N, H * W, -1) @ t(wo) + t(bo)
    return (o + t(res).reshape(N, H * W, -1)).numpy()


@pytest.mark.parametrize("heads,block", [(1, 2), (4, 2), (2, 4)])
def test_all_tokens_equal_library_self_attention(heads, block):
    x, wq, wk, wv, wo, bo, _, res = _case(1 + heads)
    H, W = x.shape[1:3]
    tok, vals = att.sparse_attention_f64(x, _all_tiles(H, W, block), block, wq, wk, wv, wo, bo, heads,
                                         residual=res)
    assert np.array_equal(tok, np.arange(H * W))
    ref = _library(x, wq, wk, wv, wo, bo, heads, None, res)
    assert np.abs(vals - ref).max() <= 1e-12 * np.abs(ref).max()


def test_all_tokens_equal_library_cross_attention():
    x, wq, wk, wv, wo, bo, ctx, res = _case(7, Ck=20, Lc=9)
    H, W = x.shape[1:3]
    _, vals = att.sparse_attention_f64(x, _all_tiles(H, W, 3), 3, wq, wk, wv, wo, bo, 4, context=ctx, residual=res)
    ref = _library(x, wq, wk, wv, wo, bo, 4, ctx, res)
    assert np.abs(vals - ref).max() <= 1e-12 * np.abs(ref).max()


def test_one_key_gives_its_value():
    # softmax over a single score is 1: every active query returns v0 Wo + bo
    x, wq, wk, wv, wo, bo, ctx, _ = _case(3, Ck=16, Lc=1)
    idx = np.array([[0, 0], [2, 3]], dtype=np.int32)
    tok, vals = att.sparse_attention_f64(x, idx, 2, wq, wk, wv, wo, bo, 2, context=ctx)
    for n in range(x.shape[0]):
        want = ctx[n, 0] @ wv @ wo + bo
        assert np.allclose(vals[n], want[None, :], rtol=0, atol=1e-12)


def test_equal_keys_give_the_mean_value():
    # Wk = 0: every score is 0, the weights are uniform
    x, wq, wk, wv, wo, bo, _, _ = _case(4)
    wk = np.zeros_like(wk)
    H, W = x.shape[1:3]
    tok, vals = att.sparse_attention_f64(x, np.array([[2, 2]], dtype=np.int32), 2, wq, wk, wv, wo, bo, 4)
    for n in range(x.shape[0]):
        want = x[n].reshape(H * W, -1).mean(axis=0) @ wv @ wo + bo
        assert np.abs(vals[n] - want[None, :]).max() <= 1e-12


def test_key_permutation_invariance():
    x, wq, wk, wv, wo, bo, ctx, _ = _case(5, Ck=12, Lc=11)
    perm = np.random.default_rng(0).permutation(ctx.shape[1])
    idx = np.array([[0, 0], [4, 4]], dtype=np.int32)
    _, a = att.sparse_attention_f64(x, idx, 2, wq, wk, wv, wo, bo, 2, context=ctx)
    _, b = att.sparse_attention_f64(x, idx, 2, wq, wk, wv, wo, bo, 2, context=ctx[:, perm])
    assert np.abs(a - b).max() <= 1e-12


def test_untouched_tokens_keep_cached_bytes():
    x, wq, wk, wv, wo, bo, _, res = _case(6, H=9, W=7)
    N, H, W = x.shape[:3]
    cache = random_cache((N, H, W, wo.shape[1]), torch.bfloat16, 11)
    idx = np.array([[0, 4], [4, 0], [8, 4]], dtype=np.int32)   # the last tile is ragged at the bottom
    out = att.sparse_attention(x, cache, idx, 4, wq, wk, wv, wo, bo, 2, residual=res)
    cov = tile_cover(idx, 4, N, H, W, wo.shape[1])
    assert torch.equal(bits(out[~cov]), bits(cache[~cov]))
    assert not torch.equal(bits(out[cov]), bits(cache[cov]))
    # empty list: the cache, byte for byte
    empty = att.sparse_attention(x, cache, np.zeros((0, 2), np.int32), 4, wq, wk, wv, wo, bo, 2)
    assert torch.equal(bits(empty), bits(cache))


def test_active_tokens_match_tile_cover():
    rng = np.random.default_rng(9)
    for _ in range(50):
        H, W, b = int(rng.integers(1, 20)), int(rng.integers(1, 20)), int(rng.integers(1, 6))
        grid = [(h, w) for h in range(0, H, b) for w in range(0, W, b)]
        pick = [t for t in grid if rng.random() < 0.3]
        idx = np.array(pick, dtype=np.int32).reshape(-1, 2)
        cov = tile_cover(idx, b, 1, H, W, 1)[0, :, :, 0].reshape(-1).numpy()
        assert np.array_equal(att.active_tokens(idx, b, H, W), np.nonzero(cov)[0])


def test_dense_attention_is_the_full_list():
    x, wq, wk, wv, wo, bo, _, _ = _case(8, H=4, W=4)
    N, H, W = x.shape[:3]
    dense = att.dense_attention(x, wq, wk, wv, wo, bo, 2)
    cache = torch.zeros((N, H, W, wo.shape[1]), dtype=torch.bfloat16)
    full = att.sparse_attention(x, cache, _all_tiles(H, W, 2), 2, wq, wk, wv, wo, bo, 2)
    assert torch.equal(bits(dense), bits(full))


def test_bf16_storage_rounds_q_k_v_and_o_once():
    # library composition with the same rounding points (q, k, v, o to bf16,
    # ties to even): element-wise equal to float64 noise except where a value
    # of o sits on a bf16 rounding boundary (then within one bf16 ulp of o
    # carried through Wo)
    import oracle
    rb = lambda a: oracle.bf16_bits_to_f64(oracle.round_bf16(a)).reshape(np.shape(a))
    x, wq, wk, wv, wo, bo, _, res = _case(12, H=6, W=6)
    N, H, W, C = x.shape
    heads = 4
    _, got = att.sparse_attention_f64(x, _all_tiles(H, W, 3), 3, wq, wk, wv, wo, bo, heads, residual=res,
                                      storage=torch.bfloat16)
    t = lambda a: torch.from_numpy(np.asarray(a, dtype=np.float64))
    seq = x.reshape(N, H * W, C)
    q, k, v = t(rb(seq @ wq)), t(rb(seq @ wk)), t(rb(seq @ wv))
    split = lambda a: a.reshape(N, H * W, heads, -1).transpose(1, 2)
    o = F.scaled_dot_product_attention(split(q), split(k), split(v)).transpose(1, 2).reshape(N, H * W, -1)
    o = rb(o.numpy())
    ref = o @ wo + bo + res.reshape(N, H * W, -1)
    bound = 2.0 ** -8 * (np.abs(o) @ np.abs(wo)) + 1e-12
    assert np.all(np.abs(got - ref) <= bound)
    exact = np.abs(got - ref) <= 1e-12 * np.abs(ref).max()
    assert exact.mean() >= 0.99
    # and the storage rounding is visible: float64 storage differs
    _, plain = att.sparse_attention_f64(x, _all_tiles(H, W, 3), 3, wq, wk, wv, wo, bo, heads, residual=res)
    assert np.abs(plain - got).max() > 1e-6


def test_core_on_stored_projections_equals_library():
    rng = np.random.default_rng(13)
    N, H, W, D, Dv, Lk, heads = 2, 5, 7, 32, 48, 19, 4
    q, k, v = rng.normal(size=(N, H, W, D)), rng.normal(size=(N, Lk, D)), rng.normal(size=(N, Lk, Dv))
    idx = np.array([[0, 0], [2, 4], [4, 6]], dtype=np.int32)
    tok, o = att.attention_core_tokens(q, k, v, heads, idx, 2, H, W)
    assert np.array_equal(tok, att.active_tokens(idx, 2, H, W))
    t = lambda a: torch.from_numpy(np.asarray(a, dtype=np.float64))
    split = lambda a, L: a.reshape(N, L, heads, -1).transpose(1, 2)
    ref = F.scaled_dot_product_attention(split(t(q).reshape(N, H * W, D), H * W), split(t(k), Lk), split(t(v), Lk))
    ref = ref.transpose(1, 2).reshape(N, H * W, Dv).numpy()[:, tok]
    assert np.abs(o - ref).max() <= 1e-12 * np.abs(ref).max()
