"""Float64 helpers of the oracle (test infrastructure only).

bf16 decoding is written out here rather than borrowed: a bf16 value is the
upper 16 bits of an IEEE-754 binary32, so widening the pattern by 16 zero bits
gives the exact binary32, and binary32 -> binary64 is exact.
"""
from __future__ import annotations

import numpy as np


def decode_bf16(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16 / int16) -> float64, exactly."""
    u = np.asarray(bits).view(np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)


def to_f64(x) -> np.ndarray:
    """Host float64 copy of a numpy array or a torch tensor (fp32 or bf16)."""
    try:
        import torch  # plain CPU tensor handling only
        if isinstance(x, torch.Tensor):
            x = x.detach().cpu().contiguous()
            if x.dtype == torch.bfloat16:
                return decode_bf16(x.view(torch.int16).numpy())
            return x.numpy().astype(np.float64)
    except ImportError:  # pragma: no cover
        pass
    x = np.asarray(x)
    if x.dtype == np.uint16:
        return decode_bf16(x)
    return x.astype(np.float64)


def row_log_softmax(Z: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """log pi = z - lse(z) along the last axis, lse = m + log sum exp(z - m).

    Returns (log_pi, lse). A row that is entirely -inf keeps lse = -inf.
    """
    m = np.max(Z, axis=-1, keepdims=True)
    m_safe = np.where(np.isfinite(m), m, 0.0)
    lse = m_safe + np.log(np.sum(np.exp(Z - m_safe), axis=-1, keepdims=True))
    return Z - lse, lse[..., 0]
