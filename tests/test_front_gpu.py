"""GPU parity of the step front end: slim_project_qk (q = x·W_Q, k = x·W_K for the step's input
rows) and slim_decode_step_x (that front end followed by the step). Source: Slim Attention
article, section "K-Cache is All You Need", generation phase (the step's query is formed from
the new token's row and scored against the cache; its key is appended).

Bars:
  * fp32: q and k bitwise equal to the fixed-order fp32 GEMM oracle (oracle/fp32_gemm.c): one
    accumulator per output, reduction index ascending, one fused multiply-add per step.
  * bf16 (tensor cores): the float64 product of the same bf16 operands is the reference. q is an
    fp32 sum of exact products, so rel-L2 per row <= 1e-5; k is that sum rounded once to bf16, so
    each element is within half a bf16 unit (2^-8 relative) plus the fp32 sum's error.
  * slim_decode_step_x equals slim_project_qk + slim_decode_step bit for bit (same kernels, same
    inputs), and meets the decode bars against the exact-MHA oracle: rel-L2 per head <= 2e-2
    for bf16 caches, max-abs <= 2e-3 for the fp32 workload.
"""
import numpy as np
import pytest
import torch

from oracle import fp32_gemm
from oracle import slim_oracle as O
from only_cache_exact_b200 import params, synth
from tests.gpu_cases import GpuState, make_case, oracle_out, rel_l2_per_head, weights

pytestmark = pytest.mark.gpu

TDT = {"bf16": torch.bfloat16, "f32": torch.float32}


@pytest.fixture(scope="module")
def S():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from only_cache_exact_b200 import slim
    return slim


def _project(S, x, WQ, WK, dtype):
    """Runs slim_project_qk on host float64 arrays holding values exact in `dtype`."""
    dev = "cuda"
    B, d = x.shape
    xd = synth.to_storage(x, dtype).to(dev)
    wq = synth.to_storage(WQ, dtype).to(dev)
    wk = synth.to_storage(WK, dtype).to(dev) if WK is not None else None
    q = torch.full((B, d), float("nan"), dtype=torch.float32, device=dev)
    k = torch.full((B, d), float("nan"), dtype=TDT[dtype], device=dev) if WK is not None else None
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    S.slim_project_qk(xd, wq, wk, q, k, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return q.cpu().numpy(), (k.float().cpu().numpy() if k is not None else None)


@pytest.mark.parametrize("d,B,with_k", [(256, 1, True), (256, 10, True), (264, 3, False)])
def test_fp32_projection_bitwise_equals_fixed_order_gemm(S, d, B, with_k):
    """Rows of the fp32 workload's step tokens (d=256) and a ragged column tile (d=264)."""
    w = synth.make_weights(d, 3, "f32")
    WQ = synth.round_to(w.W_Q, "f32")
    x = synth.make_tokens(B, d, 3, 0, "f32", part=2)
    q, k = _project(S, x, WQ, w.W_K if with_k else None, "f32")
    q_ref = fp32_gemm.gemm_f32_fmaf(x.astype(np.float32), WQ.astype(np.float32))
    assert np.array_equal(q.view(np.uint32), q_ref.view(np.uint32))
    if with_k:
        k_ref = fp32_gemm.gemm_f32_fmaf(x.astype(np.float32), w.W_K.astype(np.float32))
        assert np.array_equal(k.view(np.uint32), k_ref.view(np.uint32))


@pytest.mark.parametrize("d,B,with_k", [
    (1024, 8, True),    # 16 column tiles of 128: reduction split over clusters of 8
    (4096, 16, True),   # 64 tiles, clusters of 2
    (1280, 64, False),  # cross-attention (q only): 10 tiles, clusters of 4
    (1280, 64, True),   # 20 tiles, clusters of 4
    (4096, 1, False),   # one row (15 padding rows read as zero): 32 tiles, clusters of 4
    (256, 3, True),     # 4 tiles, clusters of 2 with two chunks each
    (1024, 200, True),  # 208 padded rows (N = 208)
    (1024, 300, True),  # two groups of rows (256 + 44)
    (200, 5, True),     # d not a multiple of 128: the CUDA-core path in bf16
])
def test_bf16_projection_matches_float64_product(S, d, B, with_k):
    w = weights(d, 4, "bf16")
    WQ = synth.round_to(w.W_Q, "bf16")
    x = synth.make_tokens(B, d, 4, 0, "bf16", part=2)
    q, k = _project(S, x, WQ, w.W_K if with_k else None, "bf16")
    q64 = x @ WQ
    err = np.linalg.norm(q - q64, axis=1) / np.linalg.norm(q64, axis=1)
    assert err.max() <= 1e-5, err.max()
    if with_k:
        k64 = x @ w.W_K
        tol = 2.0 ** -8 * np.abs(k64) + 1e-5 * np.abs(k64).max(axis=1, keepdims=True)
        assert np.all(np.abs(k - k64) <= tol), np.max(np.abs(k - k64) - tol)
        # almost every element is the correctly rounded bf16 of the exact product
        assert np.mean(k == synth.round_to(k64, "bf16")) >= 0.99


def test_bf16_projection_is_deterministic(S):
    """The cluster-split reduction adds the partial tiles in rank order: repeated calls agree bitwise."""
    d, B = 1024, 8
    w = weights(d, 4, "bf16")
    x = synth.make_tokens(B, d, 4, 1, "bf16", part=2)
    WQ = synth.round_to(w.W_Q, "bf16")
    a = _project(S, x, WQ, w.W_K, "bf16")
    b = _project(S, x, WQ, w.W_K, "bf16")
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def _x_case(d, H, lens, cap, append, seed, dtype="bf16"):
    """A decode case whose q and k come from the stored (rounded) W_Q and W_K."""
    c = make_case(d, H, lens, cap, dtype=dtype, append=append, seed=seed)
    c.WQr = synth.round_to(c.w.W_Q, dtype)
    c.q64 = c.x_new @ c.WQr
    c.k_new64 = c.x_new @ c.w.W_K
    return c


def _step_x(S, g, c, variant):
    dev = "cuda"
    tdt = TDT[c.dtype]
    x = synth.to_storage(c.x_new, c.dtype).to(dev)
    wq = synth.to_storage(c.WQr, c.dtype).to(dev)
    wk = synth.to_storage(c.w.W_K, c.dtype).to(dev) if c.append else None
    dt = S.SLIM_BF16 if c.dtype == "bf16" else S.SLIM_F32
    ws = torch.empty(S.slim_decode_step_x_workspace_bytes(dt, c.B, c.d, c.H, c.cap, variant), dtype=torch.uint8,
                     device=dev)
    S.slim_decode_step_x(x, wq, wk, g.K, g.lens, g.W_KV, c.H, g.out, ws, g.status, variant=variant)
    torch.cuda.synchronize()
    return x, wq, wk, tdt


@pytest.mark.parametrize("variant", ["B", "A"])
def test_step_x_equals_front_end_then_step_and_matches_oracle(S, variant):
    """d=1024, 8 ragged sequences with append: bitwise equal to the two calls, within tolerance of
    the exact MHA step."""
    v = S.SLIM_VARIANT_B if variant == "B" else S.SLIM_VARIANT_A
    c = _x_case(1024, 16, [300, 77, 1024, 5, 640, 1, 900, 129], 1100, True, seed=21)
    g1 = GpuState(c, S)
    x, wq, wk, tdt = _step_x(S, g1, c, v)
    got = g1.out.cpu().double().numpy()
    assert int(g1.status.item()) == 0
    assert g1.lens.cpu().tolist() == [n + 1 for n in c.lens]
    # the same step through the two public calls
    g2 = GpuState(c, S)
    q = torch.empty(c.B, c.d, dtype=torch.float32, device="cuda")
    k = torch.empty(c.B, c.d, dtype=tdt, device="cuda")
    S.slim_project_qk(x, wq, wk, q, k, g2.status)
    S.slim_decode_step(q, k, g2.K, g2.lens, g2.W_KV, c.H, g2.out, g2.ws, g2.status, variant=v)
    torch.cuda.synchronize()
    assert torch.equal(g1.out, g2.out)
    assert torch.equal(g1.K, g2.K) and torch.equal(g1.lens, g2.lens)
    err = rel_l2_per_head(got, oracle_out(c), c.H)
    assert err.max() <= 2e-2, err.max()


def test_step_x_cross_attention(S):
    """W_K = NULL: q only, no append; d=1280 (20 heads of 64), 8 sequences."""
    c = _x_case(1280, 20, [1500, 700, 1500, 33, 1200, 1500, 64, 999], 1500, False, seed=22)
    g = GpuState(c, S)
    _step_x(S, g, c, S.SLIM_VARIANT_B)
    got = g.out.cpu().double().numpy()
    assert int(g.status.item()) == 0
    assert g.lens.cpu().tolist() == c.lens.tolist()
    err = rel_l2_per_head(got, oracle_out(c), c.H)
    assert err.max() <= 2e-2, err.max()


def test_step_x_d4096(S):
    """d=4096, 32 heads of 128, three sequences (the 7B-style layer)."""
    c = _x_case(4096, 32, [2000, 517, 3000], 3100, True, seed=23)
    g = GpuState(c, S)
    _step_x(S, g, c, S.SLIM_VARIANT_B)
    got = g.out.cpu().double().numpy()
    assert int(g.status.item()) == 0
    err = rel_l2_per_head(got, oracle_out(c), c.H)
    assert err.max() <= 2e-2, err.max()


def test_fp32_prompt_then_16_steps_from_input_rows(S):
    """The fp32 workload (d=256, H=4, 128-token prompt, 16 steps) driven from the token rows: every
    step forms q and k on the device."""
    d, H, n_prompt, steps = 256, 4, 128, 16
    w = synth.make_weights(d, 0, "f32")
    WQ = synth.round_to(w.W_Q, "f32")
    X = synth.make_tokens(n_prompt + steps, d, 0, 0, "f32")
    ref = O.run_prefill_then_decode(X[:n_prompt], X[n_prompt:], WQ, w.W_K, w.W_V, H)
    dev = "cuda"
    cap = n_prompt + steps
    K = torch.zeros(1, cap, d, dtype=torch.float32, device=dev)
    lens = torch.zeros(1, dtype=torch.int32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    W_K = synth.to_storage(w.W_K, "f32").to(dev)
    W_Q = synth.to_storage(WQ, "f32").to(dev)
    S.slim_prefill_k(synth.to_storage(X[:n_prompt], "f32").to(dev).view(1, n_prompt, d), W_K, K, lens, status)
    W_KV = params.make_wkv(w.W_K, w.W_V, dtype=torch.float32, device=dev)
    ws = torch.empty(S.slim_decode_step_x_workspace_bytes(S.SLIM_F32, 1, d, H, cap, S.SLIM_VARIANT_B),
                     dtype=torch.uint8, device=dev)
    out = torch.empty(1, d, dtype=torch.float32, device=dev)
    errs = []
    for t in range(steps):
        x = synth.to_storage(X[n_prompt + t][None], "f32").to(dev)
        S.slim_decode_step_x(x, W_Q, W_K, K, lens, W_KV, H, out, ws, status, variant=S.SLIM_VARIANT_B)
        torch.cuda.synchronize()
        errs.append(np.max(np.abs(out.cpu().double().numpy()[0] - ref[t])))
    assert int(status.item()) == 0
    assert int(lens.item()) == cap
    assert max(errs) <= 2e-3, max(errs)
    # the appended keys are the fixed-order fp32 products, bit for bit
    k_ref = fp32_gemm.gemm_f32_fmaf(X[n_prompt:].astype(np.float32), w.W_K.astype(np.float32))
    assert np.array_equal(K[0, n_prompt:].cpu().numpy().view(np.uint32), k_ref.view(np.uint32))
