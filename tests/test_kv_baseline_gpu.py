"""GPU parity of slim_mha_decode_step, the standard MHA step over explicit K and V caches that
Slim attention rewrites (Slim Attention article, "K-Cache is All You Need": standard MHA caches
both k and v of every token; the K-only step is claimed up to 2x faster when memory-bound).

Both caches are filled by the library's prompt-phase GEMM (K = X·W_K, V = X·W_V with W_V
rounded to bf16, as a bf16 model stores it); the oracle is the same float64 standard MHA as for
the Slim step (V = X·W_V with the unrounded W_V). Tolerance: relative L2 per (sequence, head)
<= 2e-2; lengths, status bits and appended rows exactly.
"""
import numpy as np
import pytest
import torch

from tests.gpu_cases import make_case, oracle_out, rel_l2_per_head
from only_cache_exact_b200 import synth

pytestmark = pytest.mark.gpu

TOL_BF16 = 2e-2


@pytest.fixture(scope="module")
def S():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from only_cache_exact_b200 import slim
    return slim


class KVState:
    def __init__(self, c, S, dev="cuda"):
        self.S, self.c = S, c
        self.K = torch.zeros(c.B, c.cap, c.d, dtype=torch.bfloat16, device=dev)
        self.V = torch.zeros(c.B, c.cap, c.d, dtype=torch.bfloat16, device=dev)
        self.lens = torch.zeros(c.B, dtype=torch.int32, device=dev)
        lens_v = torch.zeros(c.B, dtype=torch.int32, device=dev)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        W_K = synth.to_storage(c.w.W_K, "bf16").to(dev)
        W_V = synth.to_storage(synth.round_to(c.w.W_V, "bf16"), "bf16").to(dev)
        for b in range(c.B):
            n = int(c.lens[b])
            if n == 0:
                continue
            Xb = synth.to_storage(c.X[b], "bf16").to(dev).view(1, n, c.d)
            S.slim_prefill_k(Xb, W_K, self.K[b:b + 1], self.lens[b:b + 1], self.status)
            S.slim_prefill_k(Xb, W_V, self.V[b:b + 1], lens_v[b:b + 1], self.status)
        self.q = torch.from_numpy(c.q64).to(torch.float32).to(dev).contiguous()
        if c.append:
            self.k_new = synth.to_storage(synth.round_to(c.k_new64, "bf16"), "bf16").to(dev)
            self.v_new = synth.to_storage(synth.round_to(c.x_new @ c.w.W_V, "bf16"), "bf16").to(dev)
        else:
            self.k_new = self.v_new = None
        self.out = torch.full((c.B, c.d), float("nan"), dtype=torch.float32, device=dev)
        self.ws = S.alloc_mha_workspace(S.SLIM_BF16, c.B, c.d, c.H, c.cap, device=dev)
        torch.cuda.synchronize()
        assert int(self.status.item()) == 0

    def step(self):
        self.S.slim_mha_decode_step(self.q, self.k_new, self.v_new, self.K, self.V, self.lens, self.c.H, self.out,
                                    self.ws, self.status)
        torch.cuda.synchronize()
        return self.out.cpu().double().numpy()


def _check(got, ref, H):
    assert np.all(np.isfinite(got))
    err = rel_l2_per_head(got, ref, H)
    assert err.max() <= TOL_BF16, (err.max(), np.unravel_index(err.argmax(), err.shape))


@pytest.mark.parametrize("d,H,lens,cap", [
    (1024, 16, [1000, 517, 1, 300, 0], 1100),   # d_h = 64, ragged, an empty and a one-row sequence
    (4096, 32, [700, 333, 64], 800),             # d_h = 128
])
def test_mha_step_matches_oracle_with_append(S, d, H, lens, cap):
    c = make_case(d, H, lens=lens, cap=cap, seed=41)
    g = KVState(c, S)
    _check(g.step(), oracle_out(c), c.H)
    assert torch.equal(g.lens.cpu(), torch.from_numpy(c.lens + 1))
    assert int(g.status.item()) == 0
    for b in range(c.B):  # this step's k and v went to row lens[b] of both caches
        assert torch.equal(g.K[b, int(c.lens[b])].cpu(), g.k_new[b].cpu())
        assert torch.equal(g.V[b, int(c.lens[b])].cpu(), g.v_new[b].cpu())


def test_mha_step_cross_attention_fixed_cache(S):
    c = make_case(1280, 20, lens=[1500, 1499, 700, 33], cap=1500, append=False, seed=42)
    g = KVState(c, S)
    ref = oracle_out(c)
    for _ in range(2):
        _check(g.step(), ref, c.H)
    assert torch.equal(g.lens.cpu(), torch.from_numpy(c.lens))


def test_mha_step_overflow_reported(S):
    c = make_case(1024, 16, lens=[64, 10], cap=64, seed=43)
    g = KVState(c, S)
    got = g.step()
    assert int(g.status.item()) & S.SLIM_DEV_OVERFLOW
    assert np.all(got[0] == 0.0)
    assert g.lens.cpu().tolist() == [64, 11]
    _check(got[1:], oracle_out(c, [1]), c.H)
