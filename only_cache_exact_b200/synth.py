"""Seeded synthetic inputs shared by the CUDA path's tests/bench and the oracle.

This module only draws random numbers and rounds them to a storage type. It
holds none of the attention arithmetic: no projection, no softmax, no W_KV.
Both sides receive the arrays it returns; neither side's code lives here.

Recipe (Slim attention, "K-Cache is All You Need": Q, K, V are row-vector
projections X·W of an input X; W_K must be square and invertible):

* X ~ N(0, 1), one independent stream per sequence so a single sequence can be
  regenerated on its own;
* W_Q, W_V ~ N(0, 1/d);
* W_K = G_orth · diag(s), G_orth a Haar-random orthogonal matrix (QR of a
  Gaussian matrix with the sign of diag(R) folded in), s ~ U[0.5, 2], so
  cond(W_K) <= 4 and its inverse is diag(1/s)·G_orthᵀ;
* ragged lengths are integers uniform on [lo, hi] inclusive.

Every matrix that a GPU kernel reads is rounded here to the storage type of its
workload (bf16 or fp32) and handed to *both* sides in that rounded form, so the
oracle and the kernels start from identical numbers. Arrays are returned as
float64 NumPy arrays holding representable values; ``to_storage`` converts
them to the torch dtype a kernel wants.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch

__all__ = [
    "stream",
    "round_to",
    "to_storage",
    "orthogonal",
    "LayerWeights",
    "make_weights",
    "make_tokens",
    "make_tokens_device",
    "make_lengths",
]

_TORCH_DTYPES = {"bf16": torch.bfloat16, "f32": torch.float32, "f64": torch.float64}


def stream(seed: int, *path: int) -> np.random.Generator:
    """Independent NumPy generator for (seed, *path), e.g. (seed, 1, b) for sequence b."""
    return np.random.default_rng(np.random.SeedSequence([int(seed), *[int(p) for p in path]]))


def round_to(a: np.ndarray, dtype: str) -> np.ndarray:
    """Round float64 values to `dtype` ("bf16", "f32" or "f64", nearest-even) and return float64."""
    if dtype == "f64":
        return np.asarray(a, dtype=np.float64)
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float64))
    return t.to(_TORCH_DTYPES[dtype]).to(torch.float64).numpy()


def to_storage(a: np.ndarray, dtype: str) -> torch.Tensor:
    """CPU torch tensor of `a` in storage type `dtype` (values must already be representable)."""
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float64)).to(_TORCH_DTYPES[dtype])


def orthogonal(d: int, rng: np.random.Generator) -> np.ndarray:
    """Haar orthogonal d×d matrix: QR of a Gaussian matrix, columns sign-fixed by diag(R)."""
    g = rng.standard_normal((d, d))
    q, r = np.linalg.qr(g)
    return q * np.sign(np.diag(r))[None, :]


@dataclass
class LayerWeights:
    """One MHA layer's projections (row-vector convention, each d×d)."""

    W_Q: np.ndarray
    W_K: np.ndarray
    W_V: np.ndarray
    G_orth: np.ndarray  # orthogonal factor of W_K before rounding
    s: np.ndarray  # diagonal factor of W_K before rounding
    dtype: str

    @property
    def d(self) -> int:
        return self.W_K.shape[0]


def make_weights(d: int, seed: int, dtype: str = "bf16") -> LayerWeights:
    """Draw W_Q, then G (-> G_orth), then s, then W_V from one stream; W_K = G_orth·diag(s).

    W_K is rounded to `dtype` because the prefill kernel reads it; W_Q and W_V
    stay float64 (no kernel reads them: q is a boundary input and W_V only
    reaches a kernel through W_KV).
    """
    rng = stream(seed, 0)
    w_q = rng.standard_normal((d, d)) / np.sqrt(d)
    g = orthogonal(d, rng)
    s = rng.uniform(0.5, 2.0, size=d)
    w_v = rng.standard_normal((d, d)) / np.sqrt(d)
    w_k = round_to(g * s[None, :], dtype)
    return LayerWeights(W_Q=w_q, W_K=w_k, W_V=w_v, G_orth=g, s=s, dtype=dtype)


def make_tokens(n: int, d: int, seed: int, seq: int, dtype: str = "bf16", part: int = 1) -> np.ndarray:
    """n token rows X ~ N(0,1) of sequence `seq`, rounded to `dtype`.

    `part` separates the prompt rows (1) from the decode-step rows (2) and
    cross-attention encoder rows (3) so each can be regenerated alone.
    """
    rng = stream(seed, part, seq)
    return round_to(rng.standard_normal((n, d)), dtype)


def make_tokens_device(n: int, d: int, seed: int, seq: int, dtype: str = "bf16", part: int = 1,
                       device="cuda") -> torch.Tensor:
    """n token rows X ~ N(0,1) of sequence `seq` drawn by torch's generator on `device`, in `dtype`.

    For workloads whose prompts are too large to draw on the host (tens of
    millions of rows). The stream is seeded from (seed, part, seq) like
    `make_tokens` but is a different stream: a test that needs these rows on
    the host copies them back (they are exact in `dtype`)."""
    g = torch.Generator(device=device)
    g.manual_seed(int(np.random.SeedSequence([int(seed), int(part), int(seq)]).generate_state(1, np.uint64)[0]
                      & 0x7FFFFFFFFFFFFFFF))
    return torch.randn(n, d, generator=g, device=device, dtype=torch.float32).to(_TORCH_DTYPES[dtype])


def make_lengths(batch: int, lo: int, hi: int, seed: int) -> np.ndarray:
    """Ragged cached lengths, integers uniform on [lo, hi] inclusive (int32)."""
    rng = stream(seed, 4)
    return rng.integers(lo, hi + 1, size=batch).astype(np.int32)
