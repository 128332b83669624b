"""The allocation-free entry point, slim_decode_step_noalloc, for callers that
cannot allocate device memory (code that must not call cudaMalloc while, for
example, a framework captures a CUDA graph or runs under a fixed memory plan).

It must give the same step as slim_decode_step with a caller workspace, on
two calls in a row (the built-in scratch keeps the previous call's contents),
and refuse sizes that need more scratch than it holds. The file name keeps it
last in collection order so that a run stopping at the first failure has run
everything else first; it also passes alone in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

from tests.gpu_cases import GpuState, make_case, rel_l2_per_head

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


def test_noalloc_matches_workspace_entry_on_two_calls(S):
    c = make_case(1024, 16, lens=[700, 333, 64], cap=800, seed=21)
    ref = GpuState(c, S)   # existing entry point, caller workspace
    nal = GpuState(c, S)   # allocation-free entry point, same inputs
    for call in range(2):
        S.slim_decode_step(ref.q, ref.k_new, ref.K, ref.lens, ref.W_KV, c.H, ref.out, ref.ws, ref.status,
                           variant=S.SLIM_VARIANT_B)
        assert _raw_noalloc(S, nal, S.SLIM_VARIANT_B) == S.SLIM_OK
        torch.cuda.synchronize()
        a = ref.out.cpu().double().numpy()
        b = nal.out.cpu().double().numpy()
        assert np.all(np.isfinite(b))
        assert rel_l2_per_head(b, a, c.H).max() <= 2e-2, call
        assert torch.equal(nal.lens.cpu(), ref.lens.cpu()), call
        assert int(nal.status.item()) == 0 and int(ref.status.item()) == 0
        # the appended rows agree too
        for bi in range(c.B):
            row = int(c.lens[bi]) + call
            assert torch.equal(nal.K[bi, row].cpu(), ref.K[bi, row].cpu())


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
