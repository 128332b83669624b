"""Pins for the float64 oracle, each against something other than the oracle itself.

Sources (Slim Attention article, section "K-Cache is All You Need"):
W_KV = W_K^(-1)·W_V; V = X·W_V = K·W_KV; generation step options (a) and (b);
the rewrite is exact. Pins used here:
  * hand-derived worked examples (tests/golden/, closed forms with ln 3 scores);
  * a library routine: torch's scaled_dot_product_attention in float64;
  * brute force with explicit Python loops on tiny inputs, with V = X·W_V;
  * closed form W_K^(-1) = diag(1/s)·G_orthᵀ against an LU solve;
  * invariants and special cases (softmax sums to 1, T=1, q=0, one dominant
    row, row permutations, per-head independence);
  * planted mistakes: mutated copies of oracle functions must fail a pin.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import slim_oracle as O
from oracle.fp32_gemm import gemm_f32_fmaf
from only_cache_exact_b200 import synth


def _load(golden_dir, name):
    with open(os.path.join(golden_dir, name)) as f:
        g = json.load(f)
    return {k: (np.array(v, dtype=np.float64) if isinstance(v, list) else v) for k, v in g.items()}


# ----------------------------------------------------------------------------- worked examples
@pytest.mark.parametrize("name", ["worked_two_rows_one_head.json", "worked_two_rows_two_heads.json"])
def test_worked_example_mha_and_both_slim_orders(golden_dir, name):
    g = _load(golden_dir, name)
    H = g["H"]
    K = O.project(g["X"], g["W_K"])
    V = O.project(g["X"], g["W_V"])
    W_KV = O.wkv_solve(g["W_K"], g["W_V"])
    np.testing.assert_allclose(W_KV, g["expected_W_KV"], rtol=0, atol=1e-14)
    for o in (O.mha_decode(g["q"], K, V, H), O.slim_decode_a(g["q"], K, W_KV, H),
              O.slim_decode_b(g["q"], K, W_KV, H)):
        np.testing.assert_allclose(o, g["expected_o"], rtol=0, atol=1e-12)


def test_worked_example_softmax_weights(golden_dir):
    g = _load(golden_dir, "worked_two_rows_two_heads.json")
    K = O.project(g["X"], g["W_K"])
    d_h = K.shape[1] // g["H"]
    for h in range(g["H"]):
        c = O.head_slice(h, d_h)
        p = O.softmax(K[:, c] @ g["q"][c] / math.sqrt(d_h))
        np.testing.assert_allclose(p, g["expected_softmax"][h], atol=1e-15)


# ----------------------------------------------------------------------------- library routine
@pytest.mark.parametrize("d,H,T", [(8, 1, 5), (16, 4, 9), (64, 2, 33)])
def test_mha_decode_matches_torch_sdpa(d, H, T):
    rng = np.random.default_rng(7)
    q = rng.standard_normal(d)
    K = rng.standard_normal((T, d))
    V = rng.standard_normal((T, d))
    d_h = d // H
    tq = torch.from_numpy(q).view(1, H, 1, d_h)
    tK = torch.from_numpy(K).view(T, H, d_h).permute(1, 0, 2).unsqueeze(0)
    tV = torch.from_numpy(V).view(T, H, d_h).permute(1, 0, 2).unsqueeze(0)
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tK, tV).reshape(d).numpy()
    np.testing.assert_allclose(O.mha_decode(q, K, V, H), ref, rtol=0, atol=1e-13)


# ----------------------------------------------------------------------------- brute force
def _brute_mha(q, X, W_K, W_V, H):
    """Explicit loops: k_t = x_t·W_K, v_t = x_t·W_V, per-head scaled dot, exp, normalise."""
    T, d = len(X), len(W_K)
    d_h = d // H
    k = [[sum(X[t][i] * W_K[i][j] for i in range(d)) for j in range(d)] for t in range(T)]
    v = [[sum(X[t][i] * W_V[i][j] for i in range(d)) for j in range(d)] for t in range(T)]
    o = [0.0] * d
    for h in range(H):
        cols = range(h * d_h, (h + 1) * d_h)
        s = [sum(q[j] * k[t][j] for j in cols) / math.sqrt(d_h) for t in range(T)]
        mx = max(s)
        e = [math.exp(x - mx) for x in s]
        z = sum(e)
        for j in cols:
            o[j] = sum(e[t] / z * v[t][j] for t in range(T))
    return np.array(o)


@pytest.mark.parametrize("d,H,T", [(6, 3, 4), (8, 2, 7), (4, 1, 1)])
def test_slim_orders_equal_bruteforce_mha(d, H, T):
    w = synth.make_weights(d, seed=3, dtype="f64")
    X = synth.make_tokens(T, d, seed=3, seq=0, dtype="f64")
    q = synth.stream(3, 9).standard_normal(d)
    ref = _brute_mha(q.tolist(), X.tolist(), w.W_K.tolist(), w.W_V.tolist(), H)
    K = O.project(X, w.W_K)
    W_KV = O.wkv_closed_form(w.G_orth, w.s, w.W_V)
    for o in (O.slim_decode_a(q, K, W_KV, H), O.slim_decode_b(q, K, W_KV, H),
              O.mha_decode(q, K, O.project(X, w.W_V), H)):
        np.testing.assert_allclose(o, ref, rtol=0, atol=1e-10)


# ----------------------------------------------------------------------------- identity
@pytest.mark.parametrize("d", [16, 64, 256])
def test_wkv_closed_form_equals_lu_solve(d):
    w = synth.make_weights(d, seed=0, dtype="f64")
    closed = O.wkv_closed_form(w.G_orth, w.s, w.W_V)
    lu = O.wkv_solve(w.W_K, w.W_V)
    assert np.max(np.abs(closed - lu)) <= 1e-10 * np.max(np.abs(lu))


@pytest.mark.parametrize("d,T", [(64, 50), (256, 144)])
def test_v_reconstructed_from_k(d, T):
    """[KC-eq2]: K·W_KV reproduces X·W_V to 1e-10 relative in float64."""
    w = synth.make_weights(d, seed=1, dtype="f64")
    X = synth.make_tokens(T, d, seed=1, seq=0, dtype="f64")
    V_direct = O.project(X, w.W_V)
    V_from_k = O.project(O.project(X, w.W_K), O.wkv_closed_form(w.G_orth, w.s, w.W_V))
    assert np.max(np.abs(V_from_k - V_direct)) <= 1e-10 * np.max(np.abs(V_direct))


# ----------------------------------------------------------------------------- invariants
def test_softmax_sums_to_one_and_is_shift_invariant():
    rng = np.random.default_rng(0)
    for n in (1, 2, 17, 1000):
        s = rng.standard_normal(n) * 10
        p = O.softmax(s)
        assert abs(p.sum() - 1.0) <= 1e-12
        assert np.all(p >= 0)
        np.testing.assert_allclose(O.softmax(s + 123.0), p, atol=1e-15)


def _rand_case(d=32, H=4, T=12, seed=5):
    rng = np.random.default_rng(seed)
    return rng.standard_normal(d), rng.standard_normal((T, d)), rng.standard_normal((T, d)), H


def test_single_row_returns_that_value_row():
    q, K, V, H = _rand_case(T=1)
    np.testing.assert_allclose(O.mha_decode(q, K, V, H), V[0], atol=1e-15)


def test_zero_query_averages_value_rows():
    q, K, V, H = _rand_case()
    np.testing.assert_allclose(O.mha_decode(np.zeros_like(q), K, V, H), V.mean(axis=0), atol=1e-14)


def test_dominant_score_selects_its_row():
    q, K, V, H = _rand_case()
    d_h = K.shape[1] // H
    K = K.copy()
    K[7] = 0.0
    for h in range(H):  # row 7 aligned with q in every head, scaled far above the rest
        c = O.head_slice(h, d_h)
        K[7, c] = 1e3 * q[c] / np.linalg.norm(q[c])
    np.testing.assert_allclose(O.mha_decode(q, K, V, H), V[7], atol=1e-12)


def test_row_permutation_invariance():
    q, K, V, H = _rand_case(T=20)
    perm = np.random.default_rng(1).permutation(20)
    np.testing.assert_allclose(O.mha_decode(q, K[perm], V[perm], H), O.mha_decode(q, K, V, H), atol=1e-14)


def test_heads_are_independent():
    """Changing head 1's columns of q and K leaves heads 0, 2, 3 unchanged."""
    q, K, V, H = _rand_case()
    d_h = K.shape[1] // H
    o = O.mha_decode(q, K, V, H)
    q2, K2 = q.copy(), K.copy()
    c = O.head_slice(1, d_h)
    q2[c] *= -3.0
    K2[:, c] += 1.0
    o2 = O.mha_decode(q2, K2, V, H)
    for h in (0, 2, 3):
        np.testing.assert_array_equal(o2[O.head_slice(h, d_h)], o[O.head_slice(h, d_h)])


def test_empty_cache_gives_zeros():
    q, K, V, H = _rand_case()
    np.testing.assert_array_equal(O.mha_decode(q, K[:0], V[:0], H), np.zeros_like(q))


def test_prefill_then_decode_step_includes_own_token():
    """A step attends to its own k/v: with T_prompt=0 the first step returns v_0 = x_0·W_V."""
    d, H = 16, 2
    w = synth.make_weights(d, seed=2, dtype="f64")
    x = synth.make_tokens(3, d, seed=2, seq=0, dtype="f64")
    out = O.run_prefill_then_decode(x[:0], x, w.W_Q, w.W_K, w.W_V, H)
    np.testing.assert_allclose(out[0], x[0] @ w.W_V, atol=1e-13)
    # later steps equal both slim orders on the same cache
    W_KV = O.wkv_closed_form(w.G_orth, w.s, w.W_V)
    K = O.project(x, w.W_K)
    q2 = x[2] @ w.W_Q
    np.testing.assert_allclose(out[2], O.slim_decode_b(q2, K, W_KV, H), atol=1e-11)
    np.testing.assert_allclose(out[2], O.slim_decode_a(q2, K, W_KV, H), atol=1e-11)


# ----------------------------------------------------------------------------- fp32 GEMM oracle
def test_fp32_gemm_exact_on_small_integers():
    rng = np.random.default_rng(0)
    X = rng.integers(-8, 9, size=(37, 53)).astype(np.float32)
    W = rng.integers(-8, 9, size=(53, 29)).astype(np.float32)
    exact = (X.astype(np.int64) @ W.astype(np.int64)).astype(np.float32)
    np.testing.assert_array_equal(gemm_f32_fmaf(X, W), exact)


def test_fp32_gemm_within_rounding_bound():
    """|fl(X·W) - X·W| <= gamma_n · |X|·|W| with gamma_n = n·u/(1-n·u), u = 2^-24."""
    rng = np.random.default_rng(1)
    n = 256
    X = rng.standard_normal((20, n)).astype(np.float32)
    W = rng.standard_normal((n, 30)).astype(np.float32)
    y = gemm_f32_fmaf(X, W).astype(np.float64)
    ref = X.astype(np.float64) @ W.astype(np.float64)
    u = 2.0 ** -24
    bound = (n * u / (1 - n * u)) * (np.abs(X).astype(np.float64) @ np.abs(W).astype(np.float64))
    assert np.all(np.abs(y - ref) <= bound)


def test_fp32_gemm_order_is_k_ascending():
    """Catastrophic cancellation exposes the order: (1e8 + 1) - 1e8 in fp32 with k ascending."""
    X = np.array([[1e8, 1.0, -1e8]], dtype=np.float32)
    W = np.ones((3, 1), dtype=np.float32)
    # ascending: fl(fl(1e8 + 1) - 1e8) = 0 (1e8 + 1 rounds to 1e8 in fp32)
    assert gemm_f32_fmaf(X, W)[0, 0] == 0.0
    X2 = np.array([[1e8, -1e8, 1.0]], dtype=np.float32)
    assert gemm_f32_fmaf(X2, W)[0, 0] == 1.0


# ----------------------------------------------------------------------------- planted mistakes
def _mut_no_scale(q, K, V, H):
    d_h = K.shape[1] // H
    o = np.zeros(K.shape[1])
    for h in range(H):
        c = O.head_slice(h, d_h)
        o[c] = O.softmax(K[:, c] @ q[c]) @ V[:, c]
    return o


def _mut_swapped_heads(q, K, V, H):
    d_h = K.shape[1] // H
    o = np.zeros(K.shape[1])
    for h in range(H):
        c, c2 = O.head_slice(h, d_h), O.head_slice(H - 1 - h, d_h)
        o[c] = O.softmax(K[:, c2] @ q[c2] / math.sqrt(d_h)) @ V[:, c]
    return o


def _mut_b_transposed_wkv(q, K, W_KV, H):
    return O.slim_decode_b(q, K, np.asarray(W_KV).T, H)


def _mut_b_head_slice_of_k(q, K, W_KV, H):
    d_h = K.shape[1] // H
    o = np.zeros(K.shape[1])
    for h in range(H):
        c = O.head_slice(h, d_h)
        p = O.softmax(K[:, c] @ q[c] / math.sqrt(d_h))
        o[c] = (p @ K[:, c]) @ np.asarray(W_KV)[c, c]  # drops the other heads' columns of K
    return o


def _mut_closed_form_s_not_inverted(G, s, W_V):
    return (np.asarray(G).T * np.asarray(s)[:, None]) @ W_V


def test_planted_mistakes_are_caught(golden_dir):
    g = _load(golden_dir, "worked_two_rows_two_heads.json")
    K = O.project(g["X"], g["W_K"])
    V = O.project(g["X"], g["W_V"])
    W_KV = O.wkv_solve(g["W_K"], g["W_V"])
    exp = g["expected_o"]
    assert not np.allclose(_mut_no_scale(g["q"], K, V, 2), exp, atol=1e-6)
    assert not np.allclose(_mut_swapped_heads(g["q"], K, V, 2), exp, atol=1e-6)
    assert not np.allclose(_mut_b_transposed_wkv(g["q"], K, W_KV, 2), exp, atol=1e-6)
    assert not np.allclose(_mut_b_head_slice_of_k(g["q"], K, W_KV, 2), exp, atol=1e-6)
    w = synth.make_weights(16, seed=0, dtype="f64")
    assert not np.allclose(_mut_closed_form_s_not_inverted(w.G_orth, w.s, w.W_V),
                           O.wkv_solve(w.W_K, w.W_V), atol=1e-6)
