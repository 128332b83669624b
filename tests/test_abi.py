"""Host-side tests of the C ABI (no GPU): the library loads, exports every
entry point include/slim.h declares, and rejects bad arguments before any
launch; the ordering table behaves as documented."""
import ctypes
import os
import re
import subprocess

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def S():
    from only_cache_exact_b200 import build
    build.build()
    from only_cache_exact_b200 import slim
    return slim


def _declared():
    src = open(os.path.join(ROOT, "include", "slim.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(slim_[a-z_0-9]+)\s*\(", src)))


def test_every_declared_symbol_is_exported(S):
    names = _declared()
    assert "slim_decode_step" in names and "slim_prefill_k" in names
    out = subprocess.run(["nm", "-D", "--defined-only", S.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (slim_\w+)", out))
    missing = [n for n in names if n not in exported]
    assert not missing, missing
    for n in names:
        assert getattr(S.raw_lib(), n) is not None
    assert set(S.EXPORTS) == set(names)


def test_version_and_strerror(S):
    assert S.slim_version() == 100
    for code in (0, -1, -2, -3, -4, 1, 2, 4, 3):
        assert len(S.slim_strerror(code)) > 5
    assert "unknown" in S.slim_strerror(-99)


def test_workspace_size_rules(S):
    n_b = S.slim_decode_workspace_bytes(S.SLIM_BF16, 8, 1024, 16, 4160, S.SLIM_VARIANT_B)
    n_a = S.slim_decode_workspace_bytes(S.SLIM_BF16, 8, 1024, 16, 4160, S.SLIM_VARIANT_A)
    n_auto = S.slim_decode_workspace_bytes(S.SLIM_BF16, 8, 1024, 16, 4160, S.SLIM_AUTO)
    assert n_b > 0 and n_a > 0 and n_auto >= max(n_a, n_b)
    # bf16 ordering (a) keeps each V tile in tensor memory: its workspace holds no V, only one
    # partial per 128-row x 256-column tile, far less than the B*cap*d*2 bytes of a materialised V
    assert n_a < 8 * 4160 * 1024 * 2 // 8
    # the CUDA-core ordering (a) (fp32 caches) still materialises V = K*W_KV: B*cap*d*4 bytes at least
    assert S.slim_decode_workspace_bytes(S.SLIM_F32, 1, 256, 4, 144, S.SLIM_VARIANT_A) >= 144 * 256 * 4
    assert S.slim_decode_workspace_bytes(S.SLIM_BF16, 8, 1000, 16, 4160, S.SLIM_VARIANT_B) == 0  # d % H
    assert S.slim_decode_workspace_bytes(7, 8, 1024, 16, 4160, 0) == 0
    assert S.slim_decode_workspace_bytes(S.SLIM_BF16, 0, 1024, 16, 4160, 0) == 0
    assert S.slim_decode_workspace_bytes(S.SLIM_BF16, 8, 1024, 16, 4160, 3) == 0


def test_decode_rejects_bad_arguments_without_launch(S):
    L = S.raw_lib()
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced: validation fails first
    args = dict(q=fake, k=None, K=fake, lens=fake, w=fake, dt=S.SLIM_BF16, B=8, d=1024, H=16, cap=4160, v=0, th=0,
                out=fake, ws=fake, wsb=1 << 40, st=fake, stream=None)

    def call(**kw):
        a = dict(args, **kw)
        return L.slim_decode_step(a["q"], a["k"], a["K"], a["lens"], a["w"], a["dt"], a["B"], a["d"], a["H"],
                                  a["cap"], a["v"], a["th"], a["out"], a["ws"], a["wsb"], a["st"], a["stream"])

    assert call(q=None) == S.SLIM_EINVAL
    assert call(K=None) == S.SLIM_EINVAL
    assert call(out=None) == S.SLIM_EINVAL
    assert call(st=None) == S.SLIM_EINVAL
    assert call(d=1000) == S.SLIM_EINVAL
    assert call(dt=5) == S.SLIM_EINVAL
    assert call(v=9) == S.SLIM_EINVAL
    assert call(B=0) == S.SLIM_EINVAL
    assert call(cap=0) == S.SLIM_EINVAL
    assert call(q=ctypes.c_void_p((1 << 20) + 4)) == S.SLIM_EINVAL  # q not 16-byte aligned
    assert call(ws=None) == S.SLIM_EWORKSPACE
    assert call(ws=ctypes.c_void_p((1 << 20) + 16)) == S.SLIM_EWORKSPACE
    assert call(wsb=1024) == S.SLIM_EWORKSPACE


def test_prefill_rejects_bad_arguments(S):
    L = S.raw_lib()
    f = ctypes.c_void_p(1 << 20)
    assert L.slim_prefill_k(None, f, f, f, S.SLIM_BF16, 1, 8, 256, 64, f, None) == S.SLIM_EINVAL
    assert L.slim_prefill_k(f, f, f, f, S.SLIM_BF16, 1, 0, 256, 64, f, None) == S.SLIM_EINVAL
    assert L.slim_prefill_k(f, f, f, f, S.SLIM_BF16, 1, 65, 256, 64, f, None) == S.SLIM_EINVAL  # n > cap
    assert L.slim_prefill_k(f, f, f, f, 3, 1, 8, 256, 64, f, None) == S.SLIM_EINVAL


def test_front_end_rejects_bad_arguments_without_launch(S):
    """slim_project_qk and slim_decode_step_x check every argument before launching anything."""
    L = S.raw_lib()
    f = ctypes.c_void_p(1 << 20)
    odd = ctypes.c_void_p((1 << 20) + 8)

    def proj(x=f, wq=f, wk=f, dt=S.SLIM_BF16, B=8, d=1024, q=f, k=f, st=f):
        return L.slim_project_qk(x, wq, wk, dt, B, d, q, k, st, None)

    assert proj(x=None) == S.SLIM_EINVAL
    assert proj(wq=None) == S.SLIM_EINVAL
    assert proj(q=None) == S.SLIM_EINVAL
    assert proj(st=None) == S.SLIM_EINVAL
    assert proj(k=None) == S.SLIM_EINVAL  # W_K without k_out
    assert proj(wk=None) == S.SLIM_EINVAL  # k_out without W_K
    assert proj(dt=4) == S.SLIM_EINVAL
    assert proj(B=0) == S.SLIM_EINVAL
    assert proj(x=odd) == S.SLIM_EINVAL
    assert proj(d=1020) == S.SLIM_EUNSUPPORTED  # a bf16 row of 2040 bytes is not a 16-byte multiple

    def step(x=f, wq=f, wk=f, K=f, lens=f, w=f, d=1024, H=16, v=0, out=f, ws=f, wsb=1 << 40, st=f):
        return L.slim_decode_step_x(x, wq, wk, K, lens, w, S.SLIM_BF16, 8, d, H, 4160, v, 0, out, ws, wsb, st, None)

    assert step(x=None) == S.SLIM_EINVAL
    assert step(wq=None) == S.SLIM_EINVAL
    assert step(K=None) == S.SLIM_EINVAL
    assert step(w=None) == S.SLIM_EINVAL
    assert step(out=None) == S.SLIM_EINVAL
    assert step(d=1000) == S.SLIM_EINVAL
    assert step(v=5) == S.SLIM_EINVAL
    assert step(wk=odd) == S.SLIM_EINVAL
    assert step(ws=None) == S.SLIM_EWORKSPACE
    need = S.slim_decode_step_x_workspace_bytes(S.SLIM_BF16, 8, 1024, 16, 4160, S.SLIM_AUTO)
    assert step(wsb=need - 1) == S.SLIM_EWORKSPACE
    # the step's scratch plus q (fp32) and k (cache dtype), each rounded up to 256 bytes
    base = S.slim_decode_workspace_bytes(S.SLIM_BF16, 8, 1024, 16, 4160, S.SLIM_AUTO)
    assert need == base + 8 * 1024 * 4 + 8 * 1024 * 2
    assert S.slim_decode_step_x_workspace_bytes(S.SLIM_BF16, 8, 1000, 16, 4160, 0) == 0


def test_host_entry_rejects_bad_arguments_before_any_copy(S):
    """Every argument check precedes the host-to-device copies: with fake device pointers that
    would fault if a copy were enqueued, a bad call returns its error code and does nothing."""
    L = S.raw_lib()
    f = ctypes.c_void_p(1 << 20)
    h = ctypes.c_void_p(2 << 20)

    def call(q=h, K=f, lens=f, w=f, v=0, d=1024, st=f):
        return L.slim_decode_step_host(q, None, K, lens, w, S.SLIM_BF16, 8, d, 16, 4160, v, 0, h, f, 1 << 40,
                                       st, None)

    assert call(q=None) == S.SLIM_EINVAL
    assert call(K=None) == S.SLIM_EINVAL
    assert call(lens=None) == S.SLIM_EINVAL
    assert call(w=None) == S.SLIM_EINVAL
    assert call(st=None) == S.SLIM_EINVAL
    assert call(v=7) == S.SLIM_EINVAL
    assert call(v=-1) == S.SLIM_EINVAL
    assert call(d=1000) == S.SLIM_EINVAL
    assert call(K=ctypes.c_void_p((1 << 20) + 8)) == S.SLIM_EINVAL  # cache not 16-byte aligned


def test_binding_constants_match_the_header(S):
    """The Python constants restate include/slim.h's #defines; a changed header must not drift."""
    src = open(os.path.join(ROOT, "include", "slim.h")).read()
    defs = {}
    for name, val in re.findall(r"#define[ \t]+(SLIM_[A-Z_0-9]+)[ \t]+(.+)", src):
        val = re.sub(r"/\*.*?\*/", "", val).strip()
        defs[name] = eval(val, {})  # integer literals and products only
    assert defs, "no #define found"
    for name, val in defs.items():
        assert hasattr(S, name), name
        assert getattr(S, name) == val, (name, getattr(S, name), val)


def test_ordering_table(S):
    S.slim_tune_clear()
    key = (S.SLIM_BF16, 1, 4096, 32)
    assert S.slim_select_variant(*key, 1024) == S.SLIM_VARIANT_B  # empty table: (b)
    S.slim_tune_record(*key, 1024, 0.010, 0.020)   # (a) faster at 1K
    S.slim_tune_record(*key, 65536, 0.900, 0.100)  # (b) faster at 64K
    assert S.slim_select_variant(*key, 1000) == S.SLIM_VARIANT_A
    assert S.slim_select_variant(*key, 2048) == S.SLIM_VARIANT_A   # nearest on a log scale
    assert S.slim_select_variant(*key, 16384) == S.SLIM_VARIANT_B
    assert S.slim_select_variant(S.SLIM_BF16, 2, 4096, 32, 1000) == S.SLIM_VARIANT_B  # other key
    S.slim_tune_record(*key, 1024, 0.030, 0.030)   # overwrite; tie -> (b)
    assert S.slim_select_variant(*key, 1024) == S.SLIM_VARIANT_B
    with pytest.raises(S.SlimError):
        S.slim_tune_record(*key, 10, -1.0, 1.0)
    S.slim_tune_clear()
    assert S.slim_select_variant(*key, 1000) == S.SLIM_VARIANT_B


def test_make_wkv_matches_closed_form():
    """The offline W_KV solve agrees with the closed form diag(1/s)·G_orthᵀ·W_V."""
    from oracle import slim_oracle as O
    from only_cache_exact_b200 import params, synth
    w = synth.make_weights(128, seed=4, dtype="f64")
    got = params.make_wkv(w.W_K, w.W_V, dtype=torch.float64).numpy()
    ref = O.wkv_closed_form(w.G_orth, w.s, w.W_V)
    assert np.max(np.abs(got - ref)) <= 1e-10 * np.max(np.abs(ref))


def test_cache_footprint_is_half():
    from only_cache_exact_b200 import params
    for dt in (torch.bfloat16, torch.float32):
        assert 2 * params.cache_bytes(8, 4096, 1024, dt) == params.cache_bytes(8, 4096, 1024, dt, k_only=False)
    assert params.cache_bytes(1, 144, 256, torch.float32) == 147456


def test_debug_stall_hook_rejects_out_of_range_limits(S):
    """The failure-path test hook only takes wait limits between 1 us and the usual second."""
    with pytest.raises(S.SlimError):
        S.slim_debug_stall_next(10)
    with pytest.raises(S.SlimError):
        S.slim_debug_stall_next(10**10)
    assert S.raw_lib().slim_debug_stall_next(1_000_000) == S.SLIM_OK
