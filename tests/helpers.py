"""Test helpers: moving tensors to the oracle and comparing results."""
from __future__ import annotations

import numpy as np
import torch

import oracle

# Per-row normwise tolerance on layer outputs (bf16 data, fp32 accumulation):
#   max_t ||Y_t - Yref_t||_inf / ||Yref_t||_inf <= 2e-2.
OUT_RTOL = 2e-2


def to_oracle(t: torch.Tensor) -> np.ndarray:
    """bf16 -> raw uint16 bits (the oracle widens them exactly); f32 stays f32."""
    t = t.detach().contiguous().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype in (torch.float32, torch.float64, torch.int32, torch.int64):
        return t.numpy()
    raise TypeError(t.dtype)


def rowwise_rel_err(y: np.ndarray, ref: np.ndarray) -> float:
    """max over rows of ||y - ref||_inf / ||ref||_inf."""
    y = np.asarray(y, np.float64)
    ref = np.asarray(ref, np.float64)
    if ref.size == 0:
        return 0.0
    num = np.abs(y - ref).max(axis=1)
    den = np.maximum(np.abs(ref).max(axis=1), 1e-30)
    return float((num / den).max())


def oracle_route(logits: torch.Tensor, k: int, renorm: int):
    return oracle.route(to_oracle(logits.float()), k, renorm)


def expert_at_slot(slot_of: np.ndarray) -> np.ndarray:
    e = np.empty_like(slot_of)
    e[slot_of] = np.arange(len(slot_of), dtype=slot_of.dtype)
    return e
