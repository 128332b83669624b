"""Oracle for Slim attention decode: plain, slow, obviously correct, float64, CPU.

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
module. It shares no code with the CUDA path and imports nothing from it.

Source: the Slim Attention article (localbendi.com/xw/1329462), section
"K-Cache is All You Need", and the arXiv abstract "Slim attention: cut your
context memory in half without loss -- K-cache is all you need for MHA"
(pulseaugur.com summary). Tags used below:

  [KC-proj]   standard MHA forms Q, K, V from the input X with the square
              projections W_Q, W_K, W_V (row vectors: K = X·W_K).
  [KC-cache]  during inference every token's k and v is kept for later tokens.
  [KC-eq1]    with W_K invertible, W_KV = W_K^(-1)·W_V.
  [KC-eq2]    V = X·W_V = X·W_K·W_K^(-1)·W_V = K·W_KV.
  [KC-prompt] prompt phase: Q and K of all prompt tokens in parallel; K is
              cached, V is not computed.
  [KC-gen]    generation phase, per step: form q, score it against the cached
              K (the softmax input), then either (a) compute V from K and
              multiply the softmax result by V, or (b) multiply the softmax
              result by K first and the product by W_KV ("more efficient for
              long sequences"); finally append this step's k to the K cache.
  [KC-exact]  the rewrite is exact: results equal standard MHA.

Readings where the pages are silent (each is also listed in the design notes):
  * softmax scale 1/sqrt(d_h); head h owns columns [h·d_h, (h+1)·d_h) of q, K,
    V and of W_KV's output;
  * a generation step attends to its own k/v (the append happens before the
    scores), as causal MHA includes the diagonal; cross-attention has no own
    token;
  * no mask, no RoPE, no W_O: the output is the concatenated head outputs.

The main parity definition is ``mha_decode`` over explicit K and V caches with
V = X·W_V (never derived from K). ``slim_decode_a`` / ``slim_decode_b`` are the
two slim orderings in float64, used by the oracle's own pins.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "project",
    "softmax",
    "head_slice",
    "mha_decode",
    "wkv_closed_form",
    "wkv_solve",
    "slim_decode_a",
    "slim_decode_b",
    "run_prefill_then_decode",
]


def project(X: np.ndarray, W: np.ndarray) -> np.ndarray:
    """Row-vector projection X·W in float64 ([KC-proj])."""
    return np.asarray(X, dtype=np.float64) @ np.asarray(W, dtype=np.float64)


def softmax(s: np.ndarray) -> np.ndarray:
    """Softmax of a 1-D score vector (max subtracted for range only)."""
    s = np.asarray(s, dtype=np.float64)
    e = np.exp(s - s.max())
    return e / e.sum()


def head_slice(h: int, d_h: int) -> slice:
    """Columns of head h (reading: contiguous d_h-wide slices)."""
    return slice(h * d_h, (h + 1) * d_h)


def mha_decode(q: np.ndarray, K: np.ndarray, V: np.ndarray, H: int) -> np.ndarray:
    """One standard-MHA generation step for one sequence ([KC-cache], [KC-gen]).

    q: (d,) query of this step; K, V: (T, d) cached keys and values, all rows
    visible. Returns the (d,) concatenation over heads of softmax(q_h·K_hᵀ/sqrt(d_h))·V_h.
    T == 0 returns zeros (reading: nothing to attend to).
    """
    q = np.asarray(q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    T, d = K.shape
    d_h = d // H
    o = np.zeros(d)
    if T == 0:
        return o
    for h in range(H):
        c = head_slice(h, d_h)
        p = softmax(K[:, c] @ q[c] / np.sqrt(d_h))
        o[c] = p @ V[:, c]
    return o


def wkv_closed_form(G_orth: np.ndarray, s: np.ndarray, W_V: np.ndarray) -> np.ndarray:
    """W_KV = W_K^(-1)·W_V ([KC-eq1]) for W_K = G_orth·diag(s): W_K^(-1) = diag(1/s)·G_orthᵀ."""
    return (np.asarray(G_orth).T / np.asarray(s)[:, None]) @ np.asarray(W_V, dtype=np.float64)


def wkv_solve(W_K: np.ndarray, W_V: np.ndarray) -> np.ndarray:
    """W_KV = W_K^(-1)·W_V ([KC-eq1]) by an LU solve of W_K·W_KV = W_V."""
    return np.linalg.solve(np.asarray(W_K, dtype=np.float64), np.asarray(W_V, dtype=np.float64))


def slim_decode_a(q: np.ndarray, K: np.ndarray, W_KV: np.ndarray, H: int) -> np.ndarray:
    """Generation step, option (a) of [KC-gen]: V = K·W_KV ([KC-eq2]), then softmax·V per head."""
    V = project(K, W_KV)
    return mha_decode(q, K, V, H)


def slim_decode_b(q: np.ndarray, K: np.ndarray, W_KV: np.ndarray, H: int) -> np.ndarray:
    """Generation step, option (b) of [KC-gen]: per head u_h = softmax_h·K (a full d-row),
    then o_h = u_h·W_KV[:, head h columns]."""
    q = np.asarray(q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    W_KV = np.asarray(W_KV, dtype=np.float64)
    T, d = K.shape
    d_h = d // H
    o = np.zeros(d)
    if T == 0:
        return o
    for h in range(H):
        c = head_slice(h, d_h)
        p = softmax(K[:, c] @ q[c] / np.sqrt(d_h))
        u = p @ K
        o[c] = u @ W_KV[:, c]
    return o


def run_prefill_then_decode(X_prompt: np.ndarray, X_steps: np.ndarray, W_Q: np.ndarray,
                            W_K: np.ndarray, W_V: np.ndarray, H: int) -> np.ndarray:
    """Standard MHA over a prompt followed by len(X_steps) generation steps, one sequence.

    The prompt's k and v rows are cached ([KC-cache]); at each step t the row
    x_t gives q_t, k_t, v_t ([KC-proj]), k_t and v_t are appended, and q_t
    attends over every cached row including its own. Returns (steps, d).
    """
    K = project(X_prompt, W_K)
    V = project(X_prompt, W_V)
    out = []
    for x in np.asarray(X_steps, dtype=np.float64):
        q = x @ W_Q
        K = np.vstack([K, x @ W_K])
        V = np.vstack([V, x @ W_V])
        out.append(mha_decode(q, K, V, H))
    return np.stack(out)
