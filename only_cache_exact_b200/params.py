"""Offline parameter preparation for Slim attention (run once per layer, not per step).

Slim Attention article, section "K-Cache is All You Need": with W_K square
and invertible, the new parameter W_KV = W_K^(-1)·W_V lets the values be
recovered from the cached keys (V = K·W_KV). This is a weight transform done
when a model is loaded, like converting a checkpoint: it is computed here in
float64 by an LU solve of W_K·W_KV = W_V (on whatever device the weights
live) and rounded once to the storage type the decode kernels read. It is
not part of the generation step.
"""
from __future__ import annotations

import numpy as np
import torch


def make_wkv(W_K, W_V, dtype: torch.dtype = torch.bfloat16, device=None) -> torch.Tensor:
    """W_KV = W_K^(-1)·W_V in float64, returned as a contiguous `dtype` tensor on `device`."""
    wk = torch.as_tensor(np.asarray(W_K) if not isinstance(W_K, torch.Tensor) else W_K).to(torch.float64)
    wv = torch.as_tensor(np.asarray(W_V) if not isinstance(W_V, torch.Tensor) else W_V).to(torch.float64)
    if wk.dim() != 2 or wk.shape[0] != wk.shape[1] or wv.shape != wk.shape:
        raise ValueError("W_K and W_V must be square d×d matrices of the same size")
    wkv = torch.linalg.solve(wk, wv)
    return wkv.to(dtype).contiguous().to(device if device is not None else wkv.device)


def cache_bytes(B: int, cap: int, d: int, dtype: torch.dtype, k_only: bool = True) -> int:
    """Context-memory footprint of one layer: K-only (slim) or K+V (standard MHA)."""
    e = torch.finfo(dtype).bits // 8
    return B * cap * d * e * (1 if k_only else 2)
