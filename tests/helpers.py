"""Shared helpers for the GPU parity tests."""
import numpy as np
import torch

TOL = {torch.float32: 1e-4, torch.bfloat16: 2e-2}
MEAN_TOL_BF16 = 2e-3


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    """Spacing of bf16 numbers (8 significant bits) at |x|."""
    a = np.abs(np.asarray(x, dtype=np.float64))
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    return np.where(a >= 2.0 ** -126, 2.0 ** (e - 7), 2.0 ** -133)


def assert_close(got: torch.Tensor, ref: torch.Tensor, dtype, mask=None, what=""):
    """The float parity bar.  float32 outputs: max|d| <= 1e-4 * RMS(ref).
    bf16 outputs: both sides round once to bf16, and where the GPU's float32
    sum and the oracle's exact sum fall on two sides of a rounding midpoint
    they differ by one bf16 ulp -- up to 2^-7 |y|, more than 2e-2 * RMS for
    the largest outputs on its own.  So each element must satisfy
    |d| <= max(2e-2 * RMS, ulp_bf16(ref)), and the mean |d| must stay below
    2e-3 * RMS (a systematic error cannot hide behind the ulp allowance)."""
    g = got.detach().double().cpu().numpy()
    r = ref.detach().double().cpu().numpy()
    rms = float(np.sqrt(np.mean(r * r)))
    d = np.abs(g - r)
    if mask is not None:
        m = mask.cpu().numpy() if isinstance(mask, torch.Tensor) else mask
        d, r = d[m], r[m]
    if d.size == 0:
        return 0.0
    if dtype == torch.float32:
        err = d.max() / rms
        assert err <= TOL[torch.float32], f"{what} max|d|/rms = {err:.3g}"
        return err
    allow = np.maximum(TOL[torch.bfloat16] * rms, bf16_ulp(r))
    worst = (d / allow).max()
    mean = d.mean() / rms
    assert worst <= 1.0, f"{what} max |d|/allowance = {worst:.3g} (max|d|/rms = {d.max() / rms:.3g})"
    assert mean <= MEAN_TOL_BF16, f"{what} mean|d|/rms = {mean:.3g}"
    return d.max() / rms


def assert_close_unrounded(got: torch.Tensor, ref64, mask=None, what=""):
    """bf16 outputs against the oracle's UNROUNDED float64 values: each
    element within max(2e-2 * RMS, half a bf16 ulp of the value) -- the GPU
    rounds its float32 sum once, so a correct result is within half an ulp
    plus the float32 summation error, and for outputs far above the RMS (a
    transposed conv's output phases have 1 to 4 taps, so its largest values
    reach ~10 RMS) the half ulp alone exceeds 2e-2 * RMS -- and the mean
    within 2e-3 * RMS."""
    g = got.detach().double().cpu().numpy()
    r = ref64.detach().double().cpu().numpy() if isinstance(ref64, torch.Tensor) else np.asarray(ref64, np.float64)
    rms = float(np.sqrt(np.mean(r * r)))
    d = np.abs(g - r)
    if mask is not None:
        m = mask.cpu().numpy() if isinstance(mask, torch.Tensor) else mask
        d, r = d[m], r[m]
    if d.size == 0:
        return 0.0
    allow = np.maximum(TOL[torch.bfloat16] * rms, 0.5 * bf16_ulp(r) * (1 + 1e-3))
    worst = (d / allow).max()
    assert worst <= 1.0, f"{what} max |d|/allowance = {worst:.3g} (max|d|/rms = {d.max() / rms:.3g})"
    assert d.mean() / rms <= MEAN_TOL_BF16, f"{what} mean|d|/rms = {d.mean() / rms:.3g}"
    return d.max() / rms


def rel_err(got: torch.Tensor, ref: torch.Tensor, mask=None) -> float:
    """max |got - ref| / RMS(ref), over `mask` when given (RMS over all of ref)."""
    g, r = got.detach().double().cpu(), ref.detach().double().cpu()
    rms = r.pow(2).mean().sqrt().item()
    d = (g - r).abs()
    if mask is not None:
        d = d[mask]
    if d.numel() == 0:
        return 0.0
    return d.max().item() / max(rms, 1e-30)


def tile_cover(idx: np.ndarray, b: int, N: int, Ho: int, Wo: int, C: int) -> torch.Tensor:
    cov = torch.zeros((N, Ho, Wo, C), dtype=torch.bool)
    for h0, w0 in np.asarray(idx).reshape(-1, 2):
        cov[:, h0:h0 + b, w0:w0 + b, :] = True
    return cov


def bits(t: torch.Tensor) -> torch.Tensor:
    """Raw bytes of a tensor, for bit-for-bit comparisons."""
    return t.detach().cpu().contiguous().view(torch.uint8)


def random_cache(shape, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(shape, generator=g).to(dtype)
