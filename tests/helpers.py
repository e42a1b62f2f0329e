"""Shared helpers for the GPU parity tests."""
import numpy as np
import torch

TOL = {torch.float32: 1e-4, torch.bfloat16: 2e-2}


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
