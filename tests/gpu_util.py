"""Helpers shared by the GPU parity tests (no method arithmetic here)."""
import numpy as np
import torch


def dev(a: np.ndarray) -> torch.Tensor:
    """numpy -> CUDA tensor; bf16 bit patterns (uint16) travel as int16."""
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        a = a.view(np.int16)
    return torch.from_numpy(a).cuda()


def host(t: torch.Tensor) -> np.ndarray:
    t = t.detach().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def sample_rows(n: int, k: int, seed: int = 0) -> np.ndarray:
    """Edges plus a seeded random sample of row indices in [0, n)."""
    rng = np.random.default_rng(seed)
    edge = np.r_[0:min(16, n), max(0, n - 16):n]
    pick = rng.choice(n, size=min(k, n), replace=False)
    return np.unique(np.r_[edge, pick])


def bf16_ulp(bits: np.ndarray) -> np.ndarray:
    """Spacing of bf16 numbers at the magnitude of each value (bits as uint16)."""
    e = (np.asarray(bits, np.uint32) >> 7) & 0xFF
    e = np.maximum(e, 1)
    return np.ldexp(1.0, e.astype(np.int64) - 127 - 7)
