"""CPU oracle for sparse attention by query-token pruning (test infrastructure only).

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg may import this module.  Plain numpy, float64 arithmetic, one rounding of
the result to the output dtype.  It shares no code with the CUDA library.

What it follows.  The nubint.ai review of "Efficient Spatially Sparse
Inference for Conditional GANs and Diffusion Models" ("Proposed method",
fourth item; "Main findings", last item) and the mer.dev notes on the same
paper (abstract: the extension to attention layers for Stable Diffusion) say
that the engine carries over to attention layers by pruning the query tokens
of unedited regions, so that the attention-map work shrinks with the edited
area.  The pages give no formulas for it.  The reading taken here, the plainest
one that matches the conv path:

  * the tokens of an attention layer are the pixels of its H x W feature map,
    row-major;
  * the active query tokens are the pixels covered by the active-tile list of
    that resolution (the list the convs of the same block use), clipped to the
    map;
  * keys and values are computed densely: from every token of the edited map
    (self-attention) or from the context sequence (cross-attention);
  * for an active token i: q_i = x_i Wq; per head h,
    o_i^h = softmax(q_i^h K^h^T / sqrt(d_head)) V^h; out_i = concat_h(o_i^h) Wo
    + bo (+ residual_i), rounded once into the cached output;
  * every other token keeps its cached output byte for byte (its query is
    pruned, so its attention row is not recomputed even though keys and values
    of edited tokens changed: the method's approximation, as for the convs
    outside the dilated mask).

Normalisation layers before the attention (LayerNorm / GroupNorm of the
transformer block) are not part of this function; they are per-token and would
be applied to x and the context before it.

Storage precision.  With ``storage=torch.bfloat16`` the projections q, k, v and
the attention output o (before Wo) are each rounded once to bf16, as a chain
that stores them between its steps does; everything else stays float64.  With
``storage=None`` nothing is rounded before the end.
"""
from __future__ import annotations

import numpy as np
import torch


def _f64(t) -> np.ndarray:
    if isinstance(t, torch.Tensor):
        return t.detach().to(torch.float64).cpu().numpy()
    return np.asarray(t, dtype=np.float64)


def active_tokens(idx: np.ndarray, block: int, H: int, W: int) -> np.ndarray:
    """Row-major token ids of the pixels covered by the tile list ``idx``
    (int32 [M, 2] of tile origins (h0, w0)), clipped to H x W; sorted, unique."""
    hit = np.zeros(H * W, dtype=bool)
    for h0, w0 in np.asarray(idx, dtype=np.int64).reshape(-1, 2):
        for y in range(h0, min(h0 + block, H)):
            row = y * W
            for x in range(w0, min(w0 + block, W)):
                hit[row + x] = True
    return np.nonzero(hit)[0]


def softmax_rows(s: np.ndarray) -> np.ndarray:
    """Row-wise softmax in float64, shifted by the row maximum."""
    m = s.max(axis=-1, keepdims=True)
    e = np.exp(s - m)
    return e / e.sum(axis=-1, keepdims=True)


def attention_core(q: np.ndarray, k: np.ndarray, v: np.ndarray, heads: int) -> np.ndarray:
    """Multi-head scaled dot-product attention, float64.
    q [Lq, D], k [Lk, D], v [Lk, Dv]; D and Dv split evenly over `heads`.
    Returns [Lq, Dv]."""
    Lq, D = q.shape
    Dv = v.shape[1]
    dh, dvh = D // heads, Dv // heads
    out = np.empty((Lq, Dv), dtype=np.float64)
    for h in range(heads):
        qh = q[:, h * dh:(h + 1) * dh]
        kh = k[:, h * dh:(h + 1) * dh]
        vh = v[:, h * dvh:(h + 1) * dvh]
        p = softmax_rows((qh @ kh.T) / np.sqrt(dh))
        out[:, h * dvh:(h + 1) * dvh] = p @ vh
    return out


def _stored(a: np.ndarray, storage) -> np.ndarray:
    """`a` rounded once to the storage dtype (bf16: ties to even, straight
    from double), back in float64; unchanged when storage is None."""
    if storage is None:
        return a
    if storage != torch.bfloat16:
        raise ValueError("storage must be None or torch.bfloat16")
    from oracle import bf16_bits_to_f64, round_bf16
    return bf16_bits_to_f64(round_bf16(a)).reshape(a.shape)


def sparse_attention_f64(x_edit, idx: np.ndarray, block: int, wq, wk, wv, wo, bo=None, heads: int = 1,
                         context=None, residual=None, storage=None):
    """The active tokens' outputs in float64 (before rounding).

    x_edit [N, H, W, C] (edited feature map), wq [C, D], wk [Ck, D], wv [Ck, Dv],
    wo [Dv, Co], bo [Co] or None, context [N, Lc, Ck] or None (self-attention:
    keys and values from x_edit), residual [N, H, W, Co] or None.
    Returns (tokens, values): tokens = active token ids, values [N, len, Co]."""
    x = _f64(x_edit)
    N, H, W, C = x.shape
    tok = active_tokens(idx, block, H, W)
    Wq, Wk, Wv, Wo = _f64(wq), _f64(wk), _f64(wv), _f64(wo)
    b = _f64(bo) if bo is not None else np.zeros(Wo.shape[1])
    ctx = _f64(context) if context is not None else None
    res = _f64(residual) if residual is not None else None
    vals = np.empty((N, len(tok), Wo.shape[1]), dtype=np.float64)
    for n in range(N):
        seq = x[n].reshape(H * W, C)
        src = seq if ctx is None else ctx[n]
        k = _stored(src @ Wk, storage)
        v = _stored(src @ Wv, storage)
        q = _stored(seq[tok] @ Wq, storage)
        o = _stored(attention_core(q, k, v, heads), storage) @ Wo + b
        if res is not None:
            o = o + res[n].reshape(H * W, -1)[tok]
        vals[n] = o
    return tok, vals


def _round_to(vals: np.ndarray, dtype: torch.dtype) -> torch.Tensor:
    """One rounding of float64 values to `dtype` (bf16: round-to-nearest-even
    straight from double, as the conv oracle rounds)."""
    if dtype == torch.bfloat16:
        from oracle import round_bf16
        bits = round_bf16(np.ascontiguousarray(vals)).astype(np.uint16)
        return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16)
    return torch.from_numpy(vals).to(dtype)


def sparse_attention(x_edit, out_cached: torch.Tensor, idx: np.ndarray, block: int, wq, wk, wv, wo, bo=None,
                     heads: int = 1, context=None, residual=None, storage=None) -> torch.Tensor:
    """Cached output [N, H, W, Co] with the active tokens recomputed and rounded
    once to its dtype; every other element is the cached one."""
    tok, vals = sparse_attention_f64(x_edit, idx, block, wq, wk, wv, wo, bo, heads, context, residual, storage)
    out = out_cached.clone()
    N, H, W, Co = out.shape
    flat = out.view(N, H * W, Co)
    if len(tok):
        flat[:, torch.from_numpy(tok)] = _round_to(vals, out.dtype)
    return out


def attention_core_tokens(q, k, v, heads: int, idx: np.ndarray, block: int, H: int, W: int):
    """The attention step alone on stored projections: q [N, H, W, D] (read at
    the active tokens), k [N, Lk, D], v [N, Lk, Dv].  Returns (tokens, o) with
    o [N, len, Dv] in float64 (before rounding)."""
    Q, K, V = _f64(q), _f64(k), _f64(v)
    N = Q.shape[0]
    tok = active_tokens(idx, block, H, W)
    o = np.empty((N, len(tok), V.shape[2]), dtype=np.float64)
    for n in range(N):
        o[n] = attention_core(Q[n].reshape(H * W, -1)[tok], K[n], V[n], heads)
    return tok, o


def dense_attention(x, wq, wk, wv, wo, bo=None, heads: int = 1, context=None, residual=None,
                    dtype=torch.bfloat16) -> torch.Tensor:
    """Every token recomputed (the cache of the original map, or the dense
    baseline), rounded once to `dtype`."""
    N, H, W, _ = x.shape
    every = np.array([(h, w) for h in range(H) for w in range(W)], dtype=np.int32)
    _, vals = sparse_attention_f64(x, every, 1, wq, wk, wv, wo, bo, heads, context, residual)
    return _round_to(vals, dtype).view(N, H, W, -1)
