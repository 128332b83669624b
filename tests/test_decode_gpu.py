"""GPU parity of slim_decode_step (both orderings) and slim_prefill_k against the float64 oracle.

Tolerances: bf16 caches, relative L2 per (sequence, head) <= 2e-2 against exact
MHA, or <= 1e-2 against option (b) evaluated exactly on the stored operands; fp32
cache (the fp32 workload), max-abs <= 2e-3. Integer/byte results (lengths,
appended cache rows, status bits) are compared exactly.
"""
import numpy as np
import pytest
import torch

from tests.gpu_cases import GpuState, make_case, oracle_out, oracle_out_stored, rel_l2_per_head
from oracle import slim_oracle as O
from only_cache_exact_b200 import synth

pytestmark = pytest.mark.gpu

TOL_BF16 = 2e-2
TOL_F32 = 2e-3
TOL_STORED = 1e-2  # bf16 P and float32 sums against float64 on the same stored operands


@pytest.fixture(scope="module")
def S():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from only_cache_exact_b200 import slim
    return slim


def _check_bf16(got, ref, H):
    err = rel_l2_per_head(got, ref, H)
    assert np.all(np.isfinite(got))
    assert err.max() <= TOL_BF16, (err.max(), np.unravel_index(err.argmax(), err.shape))
    return err.max()


@pytest.mark.parametrize("variant", ["B", "A"])
def test_self_attention_ragged_d1024(S, variant):
    c = make_case(1024, 16, lens=[1000, 517, 1, 300, 0], cap=1100, seed=1)
    g = GpuState(c, S)
    v = S.SLIM_VARIANT_B if variant == "B" else S.SLIM_VARIANT_A
    got = g.step(v)
    _check_bf16(got, oracle_out(c), c.H)
    assert torch.equal(g.lens.cpu(), torch.from_numpy(c.lens + 1))
    assert int(g.status.item()) == 0
    for b in range(c.B):  # appended rows are the k_new bytes
        assert torch.equal(g.K[b, int(c.lens[b])].cpu(), g.k_new[b].cpu())


def test_cross_attention_fixed_cache_d1280(S):
    c = make_case(1280, 20, lens=[1500, 1500, 1499, 700, 33, 1500], cap=1500, append=False, seed=2)
    g = GpuState(c, S)
    for _ in range(3):  # the cache is fixed: repeated steps give the same answer, lens unchanged
        got = g.step(S.SLIM_VARIANT_B)
        _check_bf16(got, oracle_out(c), c.H)
    assert torch.equal(g.lens.cpu(), torch.from_numpy(c.lens))


def test_long_single_sequence_merged_in_rounds(S):
    # One 6000-row sequence at d=1024 is cut into ~47 work items, more than the one-sequence
    # merge stages in shared memory at once, so its U rows arrive in several rounds.
    c = make_case(1024, 16, lens=[6000], cap=6100, seed=12)
    g = GpuState(c, S)
    _check_bf16(g.step(S.SLIM_VARIANT_B), oracle_out(c), c.H)
    assert int(g.status.item()) == 0


def test_d4096_four_cta_cluster(S):
    c = make_case(4096, 32, lens=[700, 333, 64], cap=800, seed=3)
    g = GpuState(c, S)
    _check_bf16(g.step(S.SLIM_VARIANT_B), oracle_out(c), c.H)


@pytest.mark.parametrize("d,H", [(1024, 16), (1280, 20), (4096, 32)])
def test_rising_scores_force_rescale(S, d, H):
    """Later rows scaled up so each head's running max grows by far more than 2^8 across tiles
    (one CTA per item at d=1024; clusters of 2 and 4 CTAs exchanging P and alpha above).

    The softmax is sharply peaked here, so the bf16 cache's rounding, amplified through W_KV,
    moves some heads by a few percent from exact MHA whatever the kernel does (3.6% and 6.6%
    at d=1280 and d=4096 with float64 arithmetic on the stored operands). The kernels are
    therefore held to the stored-operand evaluation of option (b) at a tighter bound."""
    c = make_case(d, H, lens=[600, 257], cap=700, seed=4)
    for b in range(c.B):
        n = len(c.X[b])
        scale = np.linspace(0.2, 6.0, n)[:, None]
        c.X[b] = synth.round_to(c.X[b] * scale, "bf16")
    c.x_new = synth.round_to(c.x_new * 3.0, "bf16")
    c.q64 = c.x_new @ c.w.W_Q
    c.k_new64 = c.x_new @ c.w.W_K
    ref = oracle_out_stored(c)
    for v in (S.SLIM_VARIANT_B, S.SLIM_VARIANT_A):
        err = rel_l2_per_head(GpuState(c, S).step(v), ref, c.H)
        assert err.max() <= TOL_STORED, (v, err.max(), np.unravel_index(err.argmax(), err.shape))


def test_empty_and_single_row(S):
    c = make_case(1024, 16, lens=[0, 1, 0], cap=64, seed=5)
    g = GpuState(c, S)
    ref = oracle_out(c)
    got = g.step(S.SLIM_VARIANT_B)
    _check_bf16(got, ref, c.H)
    # no append over an empty cache: nothing to attend to, output is zero
    c2 = make_case(1024, 16, lens=[0, 5], cap=64, append=False, seed=5)
    g2 = GpuState(c2, S)
    got2 = g2.step(S.SLIM_VARIANT_B)
    assert np.all(got2[0] == 0.0)
    _check_bf16(got2[1:], oracle_out(c2, [1]), c2.H)


def test_device_status_overflow_and_badlen(S):
    c = make_case(1024, 16, lens=[64, 10, 20], cap=64, seed=6)
    g = GpuState(c, S)
    g.lens[2] = -3
    torch.cuda.synchronize()
    got = g.step(S.SLIM_VARIANT_B)
    st = int(g.status.item())
    assert st & S.SLIM_DEV_OVERFLOW and st & S.SLIM_DEV_BADLEN and not st & S.SLIM_DEV_TIMEOUT
    assert np.all(got[0] == 0.0) and np.all(got[2] == 0.0)
    assert g.lens.cpu().tolist() == [64, 11, -3]
    _check_bf16(got[1:2], oracle_out(c, [1]), c.H)


@pytest.mark.parametrize("variant", ["B", "A"])
def test_fp32_prompt_then_16_steps(S, variant):
    """The fp32 workload: d=256, H=4, one sequence, 128-token prompt then 16 generation steps."""
    d, H, n_prompt, steps = 256, 4, 128, 16
    w = synth.make_weights(d, 0, "f32")
    X = synth.make_tokens(n_prompt + steps, d, 0, 0, "f32")
    ref = O.run_prefill_then_decode(X[:n_prompt], X[n_prompt:], w.W_Q, w.W_K, w.W_V, H)
    dev = "cuda"
    K = torch.zeros(1, n_prompt + steps, d, dtype=torch.float32, device=dev)
    lens = torch.zeros(1, dtype=torch.int32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    W_K = synth.to_storage(w.W_K, "f32").to(dev)
    S.slim_prefill_k(synth.to_storage(X[:n_prompt], "f32").to(dev).view(1, n_prompt, d), W_K, K, lens, status)
    from only_cache_exact_b200 import params
    W_KV = params.make_wkv(w.W_K, w.W_V, dtype=torch.float32, device=dev)
    ws = S.alloc_workspace(S.SLIM_F32, 1, d, H, n_prompt + steps)
    out = torch.empty(1, d, dtype=torch.float32, device=dev)
    v = S.SLIM_VARIANT_B if variant == "B" else S.SLIM_VARIANT_A
    errs = []
    for t in range(steps):
        x = X[n_prompt + t]
        q = torch.from_numpy((x @ w.W_Q)[None]).float().to(dev)
        k = torch.from_numpy((x @ w.W_K)[None]).float().to(dev)
        S.slim_decode_step(q, k, K, lens, W_KV, H, out, ws, status, variant=v)
        torch.cuda.synchronize()
        errs.append(np.max(np.abs(out.cpu().double().numpy()[0] - ref[t])))
    assert int(status.item()) == 0 and int(lens.item()) == n_prompt + steps
    assert max(errs) <= TOL_F32, errs


def test_fp32_prefill_bitwise_equals_fixed_order_gemm(S):
    from oracle.fp32_gemm import gemm_f32_fmaf
    d, n = 256, 128
    w = synth.make_weights(d, 0, "f32")
    X = synth.make_tokens(n, d, 0, 0, "f32")
    K = torch.zeros(1, n + 5, d, dtype=torch.float32, device="cuda")
    lens = torch.tensor([3], dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    S.slim_prefill_k(synth.to_storage(X, "f32").cuda().view(1, n, d), synth.to_storage(w.W_K, "f32").cuda(), K,
                     lens, status)
    torch.cuda.synchronize()
    ref = gemm_f32_fmaf(X.astype(np.float32), w.W_K.astype(np.float32))
    np.testing.assert_array_equal(K[0, 3:3 + n].cpu().numpy(), ref)
    assert int(lens.item()) == 3 + n and int(status.item()) == 0
    # a prefill that does not fit is skipped and reported
    S.slim_prefill_k(synth.to_storage(X[:8], "f32").cuda().view(1, 8, d), synth.to_storage(w.W_K, "f32").cuda(), K,
                     lens, status)
    torch.cuda.synchronize()
    assert int(status.item()) & S.SLIM_DEV_OVERFLOW and int(lens.item()) == 3 + n


def test_bf16_prefill_within_tolerance(S):
    d, n = 1024, 300
    w = synth.make_weights(d, 1, "bf16")
    X = synth.make_tokens(n, d, 1, 0, "bf16")
    K = torch.zeros(2, 400, d, dtype=torch.bfloat16, device="cuda")
    lens = torch.tensor([0, 17], dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    Xt = synth.to_storage(X, "bf16").cuda()
    S.slim_prefill_k(torch.stack([Xt, Xt]), synth.to_storage(w.W_K, "bf16").cuda(), K, lens, status)
    torch.cuda.synchronize()
    ref = X @ w.W_K
    for b, off in ((0, 0), (1, 17)):
        got = K[b, off:off + n].float().cpu().double().numpy()
        rel = np.linalg.norm(got - ref) / np.linalg.norm(ref)
        assert rel <= 4e-3, rel  # bf16 output rounding is 2^-9 relative
    assert lens.cpu().tolist() == [300, 317]


def test_host_buffer_entry_point(S):
    c = make_case(1024, 16, lens=[400, 129], cap=600, seed=7)
    g = GpuState(c, S)
    q_h = g.q.cpu().pin_memory()
    k_h = g.k_new.cpu().pin_memory()
    out_h = torch.empty(c.B, c.d, dtype=torch.float32).pin_memory()
    S.slim_decode_step_host(q_h, k_h, g.K, g.lens, g.W_KV, c.H, out_h, g.ws, g.status, variant=S.SLIM_VARIANT_B)
    torch.cuda.synchronize()
    _check_bf16(out_h.double().numpy(), oracle_out(c), c.H)
    assert g.lens.cpu().tolist() == [401, 130]


def test_repeated_steps_advance(S):
    """Four appended steps in a row match the oracle run with the growing cache."""
    c = make_case(1024, 16, lens=[250, 97], cap=300, seed=8)
    g = GpuState(c, S)
    for step in range(4):
        x = np.stack([synth.make_tokens(1, c.d, 100 + step, b, "bf16", part=2)[0] for b in range(c.B)])
        c.x_new, c.q64, c.k_new64 = x, x @ c.w.W_Q, x @ c.w.W_K
        g.q.copy_(torch.from_numpy(c.q64).float())
        g.k_new.copy_(synth.to_storage(synth.round_to(c.k_new64, "bf16"), "bf16"))
        got = g.step(S.SLIM_VARIANT_B)
        _check_bf16(got, oracle_out(c), c.H)
        # grow the oracle's prompt by the appended row for the next step
        c.X = [np.vstack([c.X[b], x[b:b + 1]]) for b in range(c.B)]
        c.lens = c.lens + 1
    assert g.lens.cpu().tolist() == [254, 101]


def test_bench_workload_sampled(S):
    """d=1024, H=16, B=8, T=4096 (the timed workload): sequences 0 and 7 against the oracle."""
    c = make_case(1024, 16, lens=[4096] * 8, cap=4096 + 64, seed=0)
    g = GpuState(c, S)
    got = g.step(S.SLIM_VARIANT_B)
    _check_bf16(got[[0, 7]], oracle_out(c, [0, 7]), c.H)
    assert np.all(np.isfinite(got))


def test_bf16_prefill_d4096_tensor_core_gemm(S):
    """tcgen05 GEMM path: K = X·W_K for 300 rows at d=4096, two sequences at different offsets."""
    d, n = 4096, 300
    w = synth.make_weights(d, 2, "bf16")
    X = synth.make_tokens(n, d, 2, 0, "bf16")
    K = torch.zeros(2, 700, d, dtype=torch.bfloat16, device="cuda")
    lens = torch.tensor([5, 390], dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    Xt = synth.to_storage(X, "bf16").cuda()
    S.slim_prefill_k(torch.stack([Xt, Xt]), synth.to_storage(w.W_K, "bf16").cuda(), K, lens, status)
    torch.cuda.synchronize()
    ref = X @ w.W_K
    for b, off in ((0, 5), (1, 390)):
        got = K[b, off:off + n].float().cpu().double().numpy()
        rel = np.linalg.norm(got - ref) / np.linalg.norm(ref)
        assert rel <= 4e-3, rel
    # rows outside the written range are untouched
    assert float(K[0, :5].abs().max()) == 0.0 and float(K[1, 390 + n:].abs().max()) == 0.0
    assert lens.cpu().tolist() == [305, 690] and int(status.item()) == 0


def test_ordering_a_d4096(S):
    c = make_case(4096, 32, lens=[200, 37], cap=300, seed=12)
    g = GpuState(c, S)
    _check_bf16(g.step(S.SLIM_VARIANT_A), oracle_out(c), c.H)


def test_selector_tunes_then_auto_step_matches(S):
    """slim_tune measures both orderings at several T, restores lens, and SLIM_AUTO then runs the
    recorded winner; the step it runs still matches the oracle."""
    c = make_case(1024, 16, lens=[900, 900], cap=1200, append=False, seed=11)
    g = GpuState(c, S)
    dt = S.SLIM_BF16
    S.slim_tune_clear()
    assert S.slim_select_variant(dt, c.B, c.d, c.H, 900) == S.SLIM_VARIANT_B  # empty table: (b)
    Ts = [16, 128, 900]
    S.slim_tune(g.q, g.K, g.lens, torch.from_numpy(c.lens), g.W_KV, c.H, Ts, 3, g.out, g.ws, g.status)
    torch.cuda.synchronize()
    assert torch.equal(g.lens.cpu(), torch.from_numpy(c.lens))  # restored
    assert int(g.status.item()) == 0
    picks = [S.slim_select_variant(dt, c.B, c.d, c.H, t) for t in Ts]
    assert all(v in (S.SLIM_VARIANT_A, S.SLIM_VARIANT_B) for v in picks)
    # which ordering wins is measured, not assumed (at this small batch ordering (a) on tensor
    # cores can win); a recorded point changes the choice near its own T only
    S.slim_tune_record(dt, c.B, c.d, c.H, 16, 0.001, 1.0)
    assert S.slim_select_variant(dt, c.B, c.d, c.H, 16) == S.SLIM_VARIANT_A
    S.slim_tune_record(dt, c.B, c.d, c.H, 128, 1.0, 0.001)
    assert S.slim_select_variant(dt, c.B, c.d, c.H, 128) == S.SLIM_VARIANT_B
    assert S.slim_select_variant(dt, c.B, c.d, c.H, 900) == picks[-1]
    got = g.step(S.SLIM_AUTO)
    _check_bf16(got, oracle_out(c), c.H)
    S.slim_tune_clear()


@pytest.mark.parametrize("d,H,lens", [(1024, 16, [6000, 4097, 5000, 129]), (4096, 32, [2000, 1537])])
def test_ordering_a_many_tiles_per_cta(S, d, H, lens):
    """Ordering (a) with several 128-row x 256-column V tiles per persistent CTA (both TMEM
    accumulators in turn) and a ragged last tile per sequence, against the oracle."""
    c = make_case(d, H, lens=lens, cap=max(lens) + 8, seed=13)
    g = GpuState(c, S)
    _check_bf16(g.step(S.SLIM_VARIANT_A), oracle_out(c), c.H)
    assert torch.equal(g.lens.cpu(), torch.from_numpy(c.lens + 1))
    assert int(g.status.item()) == 0


def test_bounded_wait_runs_out_and_context_recovers(S):
    """The failure path of a split launch: the test hook makes the MMA warp wait on a barrier that
    nothing completes, with every wait limited to 2 ms. The call returns, the status word carries
    SLIM_DEV_TIMEOUT, and the next ordinary step on the same buffers (cross-attention: the cache and
    lengths are not touched by the failed step) matches the oracle."""
    c = make_case(1024, 16, lens=[600, 300, 45], cap=640, append=False, seed=14)
    g = GpuState(c, S)
    S.slim_debug_stall_next(2_000_000)
    g.step(S.SLIM_VARIANT_B)
    st = int(g.status.item())
    assert st & S.SLIM_DEV_TIMEOUT, st
    assert torch.equal(g.lens.cpu(), torch.from_numpy(c.lens))
    g.status.zero_()
    got = g.step(S.SLIM_VARIANT_B)
    assert int(g.status.item()) == 0
    _check_bf16(got, oracle_out(c), c.H)
