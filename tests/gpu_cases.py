"""Builds seeded decode cases for the GPU parity tests and evaluates the oracle on them.

The GPU side gets its K cache from the library's own prompt-phase
projection (slim_prefill_k) of the synthetic prompt rows; the oracle
recomputes K and V = X·W_V in float64 from the same rows. Inputs come from
only_cache_exact_b200.synth; expected values only from oracle/.
"""
from __future__ import annotations

import functools
from dataclasses import dataclass, field

import numpy as np
import torch

from oracle import slim_oracle as O
from only_cache_exact_b200 import params, synth

TORCH_DT = {"bf16": torch.bfloat16, "f32": torch.float32}


@dataclass
class Case:
    d: int
    H: int
    lens: np.ndarray            # cached rows per sequence before the step
    cap: int
    dtype: str = "bf16"
    append: bool = True
    seed: int = 0
    w: synth.LayerWeights = None
    X: list = field(default_factory=list)   # per-sequence prompt rows (float64, representable)
    x_new: np.ndarray = None                # [B][d] this step's token rows
    q64: np.ndarray = None                  # [B][d] float64 queries
    k_new64: np.ndarray = None              # [B][d] float64 keys of this step

    @property
    def B(self):
        return len(self.lens)


@functools.lru_cache(maxsize=8)
def weights(d, seed, dtype) -> synth.LayerWeights:
    """synth.make_weights, memoised (a d=4096 layer takes seconds to draw)."""
    return synth.make_weights(d, seed, dtype)


def make_case(d, H, lens, cap, dtype="bf16", append=True, seed=0) -> Case:
    c = Case(d=d, H=H, lens=np.asarray(lens, dtype=np.int32), cap=cap, dtype=dtype, append=append, seed=seed)
    c.w = weights(d, seed, dtype)
    c.X = [synth.make_tokens(int(n), d, seed, b, dtype) for b, n in enumerate(c.lens)]
    c.x_new = np.stack([synth.make_tokens(1, d, seed, b, dtype, part=2)[0] for b in range(c.B)])
    c.q64 = c.x_new @ c.w.W_Q
    c.k_new64 = c.x_new @ c.w.W_K
    return c


def oracle_out(c: Case, seqs=None) -> np.ndarray:
    """Standard MHA step per sequence with explicit K and V caches (V = X·W_V)."""
    seqs = range(c.B) if seqs is None else seqs
    res = []
    for b in seqs:
        K = O.project(c.X[b], c.w.W_K)
        V = O.project(c.X[b], c.w.W_V)
        if c.append:
            K = np.vstack([K, c.k_new64[b]])
            V = np.vstack([V, c.x_new[b] @ c.w.W_V])
        res.append(O.mha_decode(c.q64[b], K, V, c.H))
    return np.stack(res)


def oracle_out_stored(c: Case, seqs=None) -> np.ndarray:
    """Option (b) of the generation step evaluated exactly (float64 softmax and products) on the
    operands the device stores: K and W_KV = W_K^(-1)·W_V rounded once to the cache type.
    What remains between this and the device result is the kernels' own rounding (P in the
    cache type, float32 sums); what separates it from oracle_out is the method's storage
    precision, which W_KV amplifies by the conditioning of W_K."""
    seqs = range(c.B) if seqs is None else seqs
    wkv = synth.round_to(O.wkv_solve(c.w.W_K, c.w.W_V), c.dtype)
    res = []
    for b in seqs:
        K = synth.round_to(O.project(c.X[b], c.w.W_K), c.dtype)
        if c.append:
            K = np.vstack([K, synth.round_to(c.k_new64[b], c.dtype)[None]])
        res.append(O.slim_decode_b(c.q64[b], K, wkv, c.H))
    return np.stack(res)


class GpuState:
    """Device buffers of a case: cache filled by slim_prefill_k, W_KV, inputs, workspace."""

    def __init__(self, c: Case, S, variant=None, dev="cuda"):
        tdt = TORCH_DT[c.dtype]
        self.S = S
        self.c = c
        self.K = torch.zeros(c.B, c.cap, c.d, dtype=tdt, device=dev)
        self.lens = torch.zeros(c.B, dtype=torch.int32, device=dev)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        W_K = synth.to_storage(c.w.W_K, c.dtype).to(dev)
        for b in range(c.B):
            n = int(c.lens[b])
            if n == 0:
                continue
            Xb = synth.to_storage(c.X[b], c.dtype).to(dev).view(1, n, c.d)
            S.slim_prefill_k(Xb, W_K, self.K[b:b + 1], self.lens[b:b + 1], self.status)
        self.W_KV = params.make_wkv(c.w.W_K, c.w.W_V, dtype=tdt, device=dev)
        self.q = torch.from_numpy(c.q64).to(torch.float32).to(dev).contiguous()
        self.k_new = synth.to_storage(synth.round_to(c.k_new64, c.dtype), c.dtype).to(dev) if c.append else None
        self.out = torch.full((c.B, c.d), float("nan"), dtype=torch.float32, device=dev)
        self.ws = S.alloc_workspace(S.SLIM_BF16 if c.dtype == "bf16" else S.SLIM_F32, c.B, c.d, c.H, c.cap,
                                    S.SLIM_AUTO, device=dev)
        torch.cuda.synchronize()
        assert int(self.status.item()) == 0
        assert torch.equal(self.lens.cpu(), torch.from_numpy(c.lens))

    def step(self, variant):
        self.S.slim_decode_step(self.q, self.k_new, self.K, self.lens, self.W_KV, self.c.H, self.out, self.ws,
                                self.status, variant=variant)
        torch.cuda.synchronize()
        return self.out.cpu().double().numpy()


def rel_l2_per_head(got: np.ndarray, ref: np.ndarray, H: int) -> np.ndarray:
    B, d = ref.shape
    g = got.reshape(B, H, d // H)
    r = ref.reshape(B, H, d // H)
    return np.linalg.norm(g - r, axis=2) / np.maximum(np.linalg.norm(r, axis=2), 1e-30)


class BigState:
    """A full-size workload: prompt rows drawn on the device (synth.make_tokens_device), the K
    cache filled by slim_prefill_k in chunks, and host copies of the rows of the sequences in
    `sample` only, so the oracle can recompute those sequences one at a time. The Case it
    carries holds X for the sampled sequences alone (oracle_out(c, sample) works on it)."""

    def __init__(self, d, H, lens, cap, S, sample, append=True, seed=0, chunk=8192, dev="cuda"):
        c = Case(d=d, H=H, lens=np.asarray(lens, dtype=np.int32), cap=cap, dtype="bf16", append=append, seed=seed)
        c.w = weights(d, seed, "bf16")
        self.S, self.c, self.sample = S, c, list(sample)
        self.K = torch.empty(c.B, cap, d, dtype=torch.bfloat16, device=dev)
        self.lens = torch.zeros(c.B, dtype=torch.int32, device=dev)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        W_K = synth.to_storage(c.w.W_K, "bf16").to(dev)
        c.X = [None] * c.B
        for b in range(c.B):
            n = int(c.lens[b])
            rows = []
            for r0 in range(0, n, chunk):
                r1 = min(n, r0 + chunk)
                Xd = synth.make_tokens_device(r1 - r0, d, seed + 1000 * (1 + r0 // chunk), b, "bf16", device=dev)
                S.slim_prefill_k(Xd.view(1, r1 - r0, d), W_K, self.K[b:b + 1], self.lens[b:b + 1], self.status)
                if b in self.sample:
                    rows.append(Xd.float().cpu().double().numpy())
            if b in self.sample:
                c.X[b] = np.vstack(rows) if rows else np.zeros((0, d))
        c.x_new = np.stack([synth.make_tokens(1, d, seed, b, "bf16", part=2)[0] for b in range(c.B)])
        c.q64 = c.x_new @ c.w.W_Q
        c.k_new64 = c.x_new @ c.w.W_K
        self.W_KV = params.make_wkv(c.w.W_K, c.w.W_V, dtype=torch.bfloat16, device=dev)
        self.q = torch.from_numpy(c.q64).to(torch.float32).to(dev).contiguous()
        self.k_new = synth.to_storage(synth.round_to(c.k_new64, "bf16"), "bf16").to(dev) if append else None
        self.out = torch.full((c.B, d), float("nan"), dtype=torch.float32, device=dev)
        self.ws = S.alloc_workspace(S.SLIM_BF16, c.B, d, H, cap, S.SLIM_VARIANT_B, device=dev)
        torch.cuda.synchronize()
        assert int(self.status.item()) == 0
        assert torch.equal(self.lens.cpu(), torch.from_numpy(c.lens))

    def step(self, variant):
        self.S.slim_decode_step(self.q, self.k_new, self.K, self.lens, self.W_KV, self.c.H, self.out, self.ws,
                                self.status, variant=variant)
        torch.cuda.synchronize()
        return self.out.cpu().double().numpy()
