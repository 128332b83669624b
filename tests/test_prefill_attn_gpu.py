"""GPU parity of slim_prefill_attention: the prompt phase's attention output over the K-only
cache (Slim Attention article, "K-Cache is All You Need", prompt phase), against the float64
oracle's standard causal MHA with an explicit V = X·W_V cache: query j of a sequence attends
over every cached row up to and including its own.

The keys come from the library's own prompt-phase projection (slim_prefill_k); the queries are
q = x·W_Q rounded once to bf16 (the kernel's input type), and the oracle gets the same rounded
queries. Tolerance: relative L2 per (query, head) <= 2e-2.
"""
import numpy as np
import pytest
import torch

from tests.gpu_cases import weights
from oracle import slim_oracle as O
from only_cache_exact_b200 import params, synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def S():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from only_cache_exact_b200 import slim
    return slim


def _run(S, d, H, prev, n, seed):
    """prev[b] rows cached before the prompt (a chunked prefill's earlier part), then n prompt rows."""
    B = len(prev)
    cap = max(prev) + n + 16
    w = weights(d, seed, "bf16")
    dev = "cuda"
    K = torch.empty(B, cap, d, dtype=torch.bfloat16, device=dev)  # rows past the lengths are scratch
    lens = torch.zeros(B, dtype=torch.int32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    W_K = synth.to_storage(w.W_K, "bf16").to(dev)
    X = []
    for b in range(B):
        Xb = synth.make_tokens(prev[b] + n, d, seed, b, "bf16")
        X.append(Xb)
        if prev[b]:
            S.slim_prefill_k(synth.to_storage(Xb[:prev[b]], "bf16").to(dev).view(1, prev[b], d), W_K,
                             K[b:b + 1], lens[b:b + 1], status)
    Xp = torch.stack([synth.to_storage(X[b][prev[b]:], "bf16") for b in range(B)]).to(dev)
    S.slim_prefill_k(Xp, W_K, K, lens, status)  # the prompt's keys, appended for all sequences at once
    Q64 = [synth.round_to(X[b][prev[b]:] @ w.W_Q, "bf16") for b in range(B)]
    Q = torch.stack([synth.to_storage(q, "bf16") for q in Q64]).to(dev)
    W_KV = params.make_wkv(w.W_K, w.W_V, dtype=torch.bfloat16, device=dev)
    out = torch.full((B, n, d), float("nan"), dtype=torch.float32, device=dev)
    ws = torch.empty(S.slim_prefill_attention_workspace_bytes(S.SLIM_BF16, B, d, H, cap), dtype=torch.uint8,
                     device=dev)
    S.slim_prefill_attention(Q, K, lens, W_KV, H, out, ws, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert lens.cpu().tolist() == [p + n for p in prev]  # not changed by the attention
    got = out.cpu().double().numpy()
    assert np.all(np.isfinite(got))
    worst = 0.0
    for b in range(B):
        Kb = O.project(X[b], w.W_K)
        Vb = O.project(X[b], w.W_V)
        ref = np.stack([O.mha_decode(Q64[b][j], Kb[:prev[b] + j + 1], Vb[:prev[b] + j + 1], H) for j in range(n)])
        g = got[b].reshape(n, H, d // H)
        r = ref.reshape(n, H, d // H)
        err = np.linalg.norm(g - r, axis=2) / np.maximum(np.linalg.norm(r, axis=2), 1e-30)
        worst = max(worst, float(err.max()))
    assert worst <= 2e-2, worst


def test_prompt_attention_d1024(S):
    """d_h = 64, two sequences, one with 77 rows cached before the prompt; 300 queries: several
    64-row query and key tiles and a ragged last tile."""
    _run(S, 1024, 16, [0, 77], 300, seed=51)


def test_prompt_attention_d4096(S):
    """d_h = 128, one sequence of 150 prompt rows."""
    _run(S, 4096, 32, [0], 150, seed=52)


def test_prompt_attention_many_key_tiles(S):
    """d_h = 64, 700 prompt rows after 200 cached ones: up to 8 key tiles of 128 per query tile,
    the S regions and the K and V rings reused several times, a ragged last key tile."""
    _run(S, 1024, 16, [200], 700, seed=53)


def test_prompt_attention_query_tiles_share_the_ragged_key_tile(S):
    """d_h = 128, 140 prompt rows after 10 cached ones: the two 128-query tiles a CTA holds both
    attend key tile 1 (rows 128..255), whose rows from 150 on are past the length; the lower tile
    zeroes them for both."""
    _run(S, 4096, 32, [10], 140, seed=54)


def test_prompt_attention_odd_query_tile_count(S):
    """d_h = 64, 3 sequences with different cached prefixes and 5 query tiles each: the CTA with the
    first tile has no second one."""
    _run(S, 512, 8, [0, 33, 64], 520, seed=55)
