"""The allocation-free entry point, slim_decode_step_noalloc.

Some callers cannot allocate device memory: a plug-in whose host runtime owns
all device memory under a plan fixed at start-up and hands it only the tensors
it computes on, or a decode loop that cannot afford cudaMalloc's implicit
device synchronisation. They cannot pass the workspace slim_decode_step needs,
so this entry point takes its scratch from a buffer compiled into the library.

Checked here through the C ABI: the step it runs is the step the workspace
entry point runs, bit for bit (the same kernels in the same order read the same
inputs), on two calls in a row with a call of another shape in between, so the
shared scratch, which keeps the previous call's contents, cannot leak a stale
plan or partial into a later call; both orderings; and sizes that need more
scratch than the buffer holds are refused. The file name keeps it last in
collection order, so a run that stops at the first failure has run every other
test first; it also passes alone in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

from tests.gpu_cases import GpuState, make_case, oracle_out, rel_l2_per_head

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def S():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from only_cache_exact_b200 import slim
    return slim


def _raw_noalloc(S, g, variant):
    c = g.c
    fn = S.raw_lib().slim_decode_step_noalloc
    p = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())  # noqa: E731
    return fn(p(g.q), p(g.k_new), p(g.K), p(g.lens), p(g.W_KV), S.SLIM_BF16, c.B, c.d, c.H, c.cap, variant, 0,
              p(g.out), p(g.status), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _raw_workspace(S, g, variant):
    c = g.c
    p = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())  # noqa: E731
    return S.raw_lib().slim_decode_step(p(g.q), p(g.k_new), p(g.K), p(g.lens), p(g.W_KV), S.SLIM_BF16, c.B, c.d,
                                        c.H, c.cap, variant, 0, p(g.out), p(g.ws), g.ws.numel(), p(g.status),
                                        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _same_step(S, ref, nal, variant, call):
    """One call of each entry point on identical buffers; everything they write must agree exactly."""
    c = ref.c
    assert _raw_workspace(S, ref, variant) == S.SLIM_OK
    assert _raw_noalloc(S, nal, variant) == S.SLIM_OK
    torch.cuda.synchronize()
    assert torch.equal(nal.out, ref.out), (variant, call)
    assert torch.equal(nal.lens, ref.lens), (variant, call)
    assert int(nal.status.item()) == 0 and int(ref.status.item()) == 0
    if c.append:
        for bi in range(c.B):
            row = int(c.lens[bi]) + call
            assert torch.equal(nal.K[bi, row], ref.K[bi, row]), (variant, call, bi)
    return nal.out.cpu().double().numpy()


@pytest.mark.parametrize("variant", ["B", "A"])
def test_noalloc_matches_workspace_entry_on_two_calls(S, variant):
    v = S.SLIM_VARIANT_B if variant == "B" else S.SLIM_VARIANT_A
    c = make_case(1024, 16, lens=[700, 333, 64], cap=800, seed=21)
    ref, nal = GpuState(c, S), GpuState(c, S)  # same inputs, one per entry point
    # a call of another shape (cross-attention, d=1280, H=20, six sequences) leaves its own plan and
    # partials in the shared scratch between the two calls compared below
    c2 = make_case(1280, 20, lens=[900, 1500, 17, 640, 1, 1200], cap=1500, append=False, seed=22)
    ref2, nal2 = GpuState(c2, S), GpuState(c2, S)
    first = _same_step(S, ref, nal, v, 0)
    # the first call is also the right answer, not merely the same one
    assert rel_l2_per_head(first, oracle_out(c), c.H).max() <= 2e-2
    _same_step(S, ref2, nal2, v, 0)
    _same_step(S, ref, nal, v, 1)


def test_noalloc_rejects_sizes_beyond_its_scratch(S):
    need = S.slim_decode_workspace_bytes(S.SLIM_BF16, 16, 4096, 32, 40000, S.SLIM_VARIANT_B)
    assert need > S.SLIM_NOALLOC_SCRATCH_BYTES
    dummy = torch.zeros(16, dtype=torch.int32, device="cuda")
    lib = S.raw_lib()
    rc = lib.slim_decode_step_noalloc(ctypes.c_void_p(dummy.data_ptr()), None, ctypes.c_void_p(dummy.data_ptr()),
                                      ctypes.c_void_p(dummy.data_ptr()), ctypes.c_void_p(dummy.data_ptr()),
                                      S.SLIM_BF16, 16, 4096, 32, 40000, S.SLIM_VARIANT_B, 0,
                                      ctypes.c_void_p(dummy.data_ptr()), ctypes.c_void_p(dummy.data_ptr()), None)
    assert rc == S.SLIM_EWORKSPACE
    torch.cuda.synchronize()
    assert int(dummy.abs().sum().item()) == 0  # nothing was enqueued
