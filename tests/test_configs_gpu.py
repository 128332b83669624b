"""GPU parity of slim_decode_step on the shapes of the five benchmark workloads, at full size.

Each workload's own launch configuration is exercised: the work split over the
SMs (ragged lengths, clusters of 1, 2 and 4 CTAs), the merge of the split
partials for many sequences (B > 4, B·H above the SM count, more sequences than
one merge launch takes) and the projection by W_KV. Full-size cases compare
sampled sequences with the float64 oracle (standard MHA with explicit K and V
caches, V = X·W_V), one sequence at a time; every output is checked for
finiteness and the lengths and status word exactly.

Tolerance: relative L2 error per (sequence, head) <= 2e-2 against exact MHA
for bf16 caches (Slim attention article, "K-Cache is All You Need": the
rewrite is exact, so only storage and arithmetic rounding separate the two).
"""
import numpy as np
import pytest
import torch

from tests.gpu_cases import BigState, GpuState, make_case, oracle_out, rel_l2_per_head
from only_cache_exact_b200 import synth

pytestmark = pytest.mark.gpu

TOL_BF16 = 2e-2


@pytest.fixture(scope="module")
def S():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from only_cache_exact_b200 import slim
    return slim


def _check(got, ref, H):
    assert np.all(np.isfinite(got))
    err = rel_l2_per_head(got, ref, H)
    assert err.max() <= TOL_BF16, (err.max(), np.unravel_index(err.argmax(), err.shape))
    return err.max()


# ------------------------------------------------------------------ many sequences, short caches
@pytest.mark.parametrize("lens", [[300, 17, 512, 129, 64], list(range(100, 420, 20))],
                         ids=["B5", "B16"])
def test_d4096_h32_many_sequences(S, lens):
    """d=4096, H=32 (d_h=128) with B=5 and B=16: more than four sequences per merge launch."""
    c = make_case(4096, 32, lens=lens, cap=600, seed=31)
    g = GpuState(c, S)
    _check(g.step(S.SLIM_VARIANT_B), oracle_out(c), c.H)
    assert torch.equal(g.lens.cpu(), torch.from_numpy(c.lens + 1))
    assert int(g.status.item()) == 0


def test_d1280_h20_b8_more_heads_than_sms(S):
    """d=1280, H=20, B=8: B·H = 160 (sequence, head) pairs, more than the 148 SMs."""
    c = make_case(1280, 20, lens=[200, 333, 600, 17, 1, 450, 512, 90], cap=700, seed=32)
    g = GpuState(c, S)
    _check(g.step(S.SLIM_VARIANT_B), oracle_out(c), c.H)
    assert torch.equal(g.lens.cpu(), torch.from_numpy(c.lens + 1))


@pytest.mark.parametrize("d,H,B", [(1280, 20, 130), (4096, 32, 66)])
def test_batch_beyond_one_merge_launch(S, d, H, B):
    """More sequences than one merge launch holds (128 at d_h = 64, 64 at d_h = 128)."""
    lens = synth.make_lengths(B, 8, 40, 33)
    c = make_case(d, H, lens=lens, cap=48, seed=33)
    g = GpuState(c, S)
    _check(g.step(S.SLIM_VARIANT_B), oracle_out(c), c.H)
    assert torch.equal(g.lens.cpu(), torch.from_numpy(c.lens + 1))
    assert int(g.status.item()) == 0


# ------------------------------------------------------------------ the workloads at full size
def test_7b_style_ragged_b16_full_size(S):
    """d=4096, H=32, B=16, ragged cached lengths uniform in [16384, 32768]: the shortest, the
    longest and a middle sequence against the oracle."""
    lens = synth.make_lengths(16, 16384, 32768, 0)
    order = np.argsort(lens)
    sample = sorted({int(order[0]), int(order[-1]), int(order[len(order) // 2])})
    g = BigState(4096, 32, lens, int(lens.max()) + 16, S, sample, append=True, seed=0)
    got = g.step(S.SLIM_VARIANT_B)
    assert np.all(np.isfinite(got))
    _check(got[sample], oracle_out(g.c, sample), g.c.H)
    assert torch.equal(g.lens.cpu(), torch.from_numpy(lens + 1))
    assert int(g.status.item()) == 0


def test_cross_attention_b64_full_size(S):
    """d=1280, H=20, B=64, a fixed 1500-row encoder cache per sequence, no append: four sampled
    sequences on three repeated steps (the cache and lengths do not change)."""
    lens = np.full(64, 1500, dtype=np.int32)
    sample = [0, 21, 42, 63]
    g = BigState(1280, 20, lens, 1500, S, sample, append=False, seed=1)
    ref = oracle_out(g.c, sample)
    for _ in range(3):
        got = g.step(S.SLIM_VARIANT_B)
        assert np.all(np.isfinite(got))
        _check(got[sample], ref, g.c.H)
    assert torch.equal(g.lens.cpu(), torch.from_numpy(lens))
    assert int(g.status.item()) == 0


def test_long_context_b1_full_size(S):
    """d=4096, H=32, B=1, 131008 cached rows plus the appended one in a 131072-row cache: every
    head against the oracle."""
    lens = np.array([131072 - 64], dtype=np.int32)
    g = BigState(4096, 32, lens, 131072, S, [0], append=True, seed=2)
    got = g.step(S.SLIM_VARIANT_B)
    _check(got, oracle_out(g.c, [0]), g.c.H)
    assert int(g.lens.item()) == 131072 - 63 and int(g.status.item()) == 0
