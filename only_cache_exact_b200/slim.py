"""ctypes binding of libslim.so (C ABI in include/slim.h), same names as the C entry points.

Argument marshalling only: torch tensors are checked (device, dtype,
contiguity, shape) and passed as raw pointers with the current CUDA stream;
every step of the path runs in the library's kernels. There is no fallback:
if libslim.so cannot be loaded, importing this module raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libslim.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"libslim.so not built at {LIB_PATH}; run `python -m only_cache_exact_b200.build`")
_lib = ctypes.CDLL(LIB_PATH)

SLIM_OK, SLIM_EINVAL, SLIM_EWORKSPACE, SLIM_ECUDA, SLIM_EUNSUPPORTED = 0, -1, -2, -3, -4
SLIM_DEV_OVERFLOW, SLIM_DEV_BADLEN, SLIM_DEV_TIMEOUT = 1, 2, 4
SLIM_F32, SLIM_BF16 = 0, 1
SLIM_AUTO, SLIM_VARIANT_A, SLIM_VARIANT_B = 0, 1, 2

EXPORTS = [
    "slim_prefill_k", "slim_decode_workspace_bytes", "slim_decode_step", "slim_decode_step_host", "slim_tune",
    "slim_tune_record", "slim_select_variant", "slim_tune_clear", "slim_strerror", "slim_last_launch_count",
    "slim_version", "slim_timing_enable", "slim_timing_read", "slim_decode_step_noalloc",
    "slim_mha_decode_workspace_bytes", "slim_mha_decode_step", "slim_debug_stall_next",
    "slim_prefill_attention_workspace_bytes", "slim_prefill_attention", "slim_project_qk",
    "slim_decode_step_x_workspace_bytes", "slim_decode_step_x", "slim_noalloc_scratch_bytes",
]

_vp, _i32, _i64, _sz, _f32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t, ctypes.c_float
_SIGS = {
    "slim_prefill_k": (_i32, [_vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i64, _vp, _vp]),
    "slim_decode_workspace_bytes": (_sz, [_i32, _i32, _i32, _i32, _i64, _i32]),
    "slim_decode_step": (_i32, [_vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i64, _i32, _i64, _vp, _vp, _sz,
                                _vp, _vp]),
    "slim_decode_step_host": (_i32, [_vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i64, _i32, _i64, _vp, _vp,
                                     _sz, _vp, _vp]),
    "slim_tune": (_i32, [_vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i64, _vp, _i32, _i32, _vp, _vp, _sz, _vp,
                         _vp]),
    "slim_tune_record": (_i32, [_i32, _i32, _i32, _i32, _i64, _f32, _f32]),
    "slim_select_variant": (_i32, [_i32, _i32, _i32, _i32, _i64]),
    "slim_tune_clear": (None, []),
    "slim_strerror": (ctypes.c_char_p, [_i32]),
    "slim_last_launch_count": (_i32, []),
    "slim_version": (_i32, []),
    "slim_timing_enable": (_i32, [_i32]),
    "slim_timing_read": (_i32, [_vp, _i32]),
    "slim_decode_step_noalloc": (_i32, [_vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i64, _i32, _i64, _vp, _vp,
                                        _vp]),
    "slim_mha_decode_workspace_bytes": (_sz, [_i32, _i32, _i32, _i32, _i64]),
    "slim_debug_stall_next": (_i32, [_i64]),
    "slim_prefill_attention_workspace_bytes": (_sz, [_i32, _i32, _i32, _i32, _i64]),
    "slim_prefill_attention": (_i32, [_vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _i64, _vp, _vp, _sz, _vp,
                                      _vp]),
    "slim_mha_decode_step": (_i32, [_vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i64, _vp, _vp, _sz, _vp,
                                    _vp]),
    "slim_project_qk": (_i32, [_vp, _vp, _vp, _i32, _i32, _i32, _vp, _vp, _vp, _vp]),
    "slim_decode_step_x_workspace_bytes": (_sz, [_i32, _i32, _i32, _i32, _i64, _i32]),
    "slim_decode_step_x": (_i32, [_vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i64, _i32, _i64, _vp, _vp,
                                  _sz, _vp, _vp]),
    "slim_noalloc_scratch_bytes": (_sz, []),
}
for _name, (_res, _args) in _SIGS.items():
    _fn = getattr(_lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args
# the scratch size compiled into the library, read from it rather than restated
SLIM_NOALLOC_SCRATCH_BYTES = int(_lib.slim_noalloc_scratch_bytes())

_DT = {torch.bfloat16: SLIM_BF16, torch.float32: SLIM_F32}


class SlimError(RuntimeError):
    def __init__(self, code: int, where: str):
        super().__init__(f"{where}: {slim_strerror(code)} ({code})")
        self.code = code


def _check(code: int, where: str) -> None:
    if code != SLIM_OK:
        raise SlimError(code, where)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _cuda(t: torch.Tensor, name: str) -> None:
    if not (t.is_cuda and t.is_contiguous()):
        raise ValueError(f"{name} must be a contiguous CUDA tensor")


def slim_strerror(code: int) -> str:
    return _lib.slim_strerror(int(code)).decode()


def slim_version() -> int:
    return _lib.slim_version()


def slim_last_launch_count() -> int:
    return _lib.slim_last_launch_count()


def slim_decode_workspace_bytes(dtype: int, B: int, d: int, H: int, cap: int, variant: int = SLIM_AUTO) -> int:
    return int(_lib.slim_decode_workspace_bytes(dtype, B, d, H, cap, variant))


def alloc_workspace(dtype: int, B: int, d: int, H: int, cap: int, variant: int = SLIM_AUTO,
                    device=None) -> torch.Tensor:
    """Caller-owned scratch for slim_decode_step (a uint8 CUDA tensor, 256-byte aligned by torch)."""
    n = slim_decode_workspace_bytes(dtype, B, d, H, cap, variant)
    if n == 0:
        raise SlimError(SLIM_EINVAL, "slim_decode_workspace_bytes")
    return torch.empty(n, dtype=torch.uint8, device=device or torch.device("cuda"))


def slim_prefill_k(X: torch.Tensor, W_K: torch.Tensor, Kcache: torch.Tensor, lens: torch.Tensor,
                   status: torch.Tensor, stream=None) -> None:
    """K = X·W_K for X [B][n][d], written at rows lens[b].. of Kcache [B][cap][d]; lens += n."""
    for t, nm in ((X, "X"), (W_K, "W_K"), (Kcache, "Kcache"), (lens, "lens"), (status, "status")):
        _cuda(t, nm)
    B, n, d = X.shape
    cap = Kcache.shape[1]
    if Kcache.shape != (B, cap, d) or W_K.shape != (d, d) or X.dtype != Kcache.dtype or W_K.dtype != X.dtype:
        raise ValueError("shape/dtype mismatch")
    _check(_lib.slim_prefill_k(_ptr(X), _ptr(W_K), _ptr(Kcache), _ptr(lens), _DT[X.dtype], B, n, d, cap,
                               _ptr(status), _stream(stream)), "slim_prefill_k")


def slim_decode_step(q: torch.Tensor, k_new, Kcache: torch.Tensor, lens: torch.Tensor, W_KV: torch.Tensor, H: int,
                     out: torch.Tensor, workspace: torch.Tensor, status: torch.Tensor, variant: int = SLIM_AUTO,
                     t_hint: int = 0, stream=None) -> None:
    """One generation step for B sequences: q [B][d] fp32, k_new [B][d] or None, out [B][d] fp32."""
    for t, nm in ((q, "q"), (Kcache, "Kcache"), (lens, "lens"), (W_KV, "W_KV"), (out, "out"),
                  (workspace, "workspace"), (status, "status")):
        _cuda(t, nm)
    B, cap, d = Kcache.shape
    if q.shape != (B, d) or out.shape != (B, d) or q.dtype != torch.float32 or out.dtype != torch.float32:
        raise ValueError("q/out must be float32 [B][d]")
    if k_new is not None:
        _cuda(k_new, "k_new")
        if k_new.shape != (B, d) or k_new.dtype != Kcache.dtype:
            raise ValueError("k_new must be [B][d] in the cache dtype")
    _check(_lib.slim_decode_step(_ptr(q), _ptr(k_new), _ptr(Kcache), _ptr(lens), _ptr(W_KV), _DT[Kcache.dtype],
                                 B, d, H, cap, variant, t_hint, _ptr(out), _ptr(workspace), workspace.numel(),
                                 _ptr(status), _stream(stream)), "slim_decode_step")


def slim_project_qk(x: torch.Tensor, W_Q: torch.Tensor, W_K, q_out: torch.Tensor, k_out, status: torch.Tensor,
                    stream=None) -> None:
    """Step front end: q_out = x·W_Q (fp32 [B][d]) and, with W_K, k_out = x·W_K ([B][d] in x's dtype)."""
    for t, nm in ((x, "x"), (W_Q, "W_Q"), (q_out, "q_out"), (status, "status")):
        _cuda(t, nm)
    B, d = x.shape
    if W_Q.shape != (d, d) or W_Q.dtype != x.dtype or q_out.shape != (B, d) or q_out.dtype != torch.float32:
        raise ValueError("shape/dtype mismatch")
    if (W_K is None) != (k_out is None):
        raise ValueError("W_K and k_out go together")
    if W_K is not None:
        _cuda(W_K, "W_K")
        _cuda(k_out, "k_out")
        if W_K.shape != (d, d) or W_K.dtype != x.dtype or k_out.shape != (B, d) or k_out.dtype != x.dtype:
            raise ValueError("shape/dtype mismatch")
    _check(_lib.slim_project_qk(_ptr(x), _ptr(W_Q), _ptr(W_K), _DT[x.dtype], B, d, _ptr(q_out), _ptr(k_out),
                                _ptr(status), _stream(stream)), "slim_project_qk")


def slim_decode_step_x_workspace_bytes(dtype: int, B: int, d: int, H: int, cap: int, variant: int = SLIM_AUTO) -> int:
    return int(_lib.slim_decode_step_x_workspace_bytes(dtype, B, d, H, cap, variant))


def slim_decode_step_x(x: torch.Tensor, W_Q: torch.Tensor, W_K, Kcache: torch.Tensor, lens: torch.Tensor,
                       W_KV: torch.Tensor, H: int, out: torch.Tensor, workspace: torch.Tensor, status: torch.Tensor,
                       variant: int = SLIM_AUTO, t_hint: int = 0, stream=None) -> None:
    """One generation step from the input rows x [B][d] (cache dtype): q = x·W_Q, k = x·W_K (W_K None: no
    append), then the step as slim_decode_step."""
    for t, nm in ((x, "x"), (W_Q, "W_Q"), (Kcache, "Kcache"), (lens, "lens"), (W_KV, "W_KV"), (out, "out"),
                  (workspace, "workspace"), (status, "status")):
        _cuda(t, nm)
    B, cap, d = Kcache.shape
    if x.shape != (B, d) or x.dtype != Kcache.dtype or W_Q.shape != (d, d) or W_Q.dtype != x.dtype:
        raise ValueError("x/W_Q must be [B][d]/[d][d] in the cache dtype")
    if W_K is not None:
        _cuda(W_K, "W_K")
        if W_K.shape != (d, d) or W_K.dtype != x.dtype:
            raise ValueError("W_K must be [d][d] in the cache dtype")
    if out.shape != (B, d) or out.dtype != torch.float32:
        raise ValueError("out must be float32 [B][d]")
    _check(_lib.slim_decode_step_x(_ptr(x), _ptr(W_Q), _ptr(W_K), _ptr(Kcache), _ptr(lens), _ptr(W_KV),
                                   _DT[Kcache.dtype], B, d, H, cap, variant, t_hint, _ptr(out), _ptr(workspace),
                                   workspace.numel(), _ptr(status), _stream(stream)), "slim_decode_step_x")


def slim_decode_step_noalloc(q: torch.Tensor, k_new, Kcache: torch.Tensor, lens: torch.Tensor, W_KV: torch.Tensor,
                             H: int, out: torch.Tensor, status: torch.Tensor, variant: int = SLIM_AUTO,
                             t_hint: int = 0, stream=None) -> None:
    """slim_decode_step for callers that cannot allocate: scratch comes from a buffer built into the library."""
    for t, nm in ((q, "q"), (Kcache, "Kcache"), (lens, "lens"), (W_KV, "W_KV"), (out, "out"), (status, "status")):
        _cuda(t, nm)
    B, cap, d = Kcache.shape
    _check(_lib.slim_decode_step_noalloc(_ptr(q), _ptr(k_new), _ptr(Kcache), _ptr(lens), _ptr(W_KV),
                                         _DT[Kcache.dtype], B, d, H, cap, variant, t_hint, _ptr(out), _ptr(status),
                                         _stream(stream)), "slim_decode_step_noalloc")


def slim_prefill_attention_workspace_bytes(dtype: int, B: int, d: int, H: int, cap: int) -> int:
    return int(_lib.slim_prefill_attention_workspace_bytes(dtype, B, d, H, cap))


def slim_prefill_attention(Q: torch.Tensor, Kcache: torch.Tensor, lens: torch.Tensor, W_KV: torch.Tensor, H: int,
                           out: torch.Tensor, workspace: torch.Tensor, status: torch.Tensor, stream=None) -> None:
    """Causal attention output of the n prompt queries Q [B][n][d] (bf16) over the K-only cache; out [B][n][d]."""
    for t, nm in ((Q, "Q"), (Kcache, "Kcache"), (lens, "lens"), (W_KV, "W_KV"), (out, "out"),
                  (workspace, "workspace"), (status, "status")):
        _cuda(t, nm)
    B, n, d = Q.shape
    cap = Kcache.shape[1]
    if Kcache.shape != (B, cap, d) or out.shape != (B, n, d) or out.dtype != torch.float32:
        raise ValueError("shape/dtype mismatch")
    _check(_lib.slim_prefill_attention(_ptr(Q), _ptr(Kcache), _ptr(lens), _ptr(W_KV), _DT[Q.dtype], B, n, d, H,
                                       cap, _ptr(out), _ptr(workspace), workspace.numel(), _ptr(status),
                                       _stream(stream)), "slim_prefill_attention")


def slim_mha_decode_workspace_bytes(dtype: int, B: int, d: int, H: int, cap: int) -> int:
    return int(_lib.slim_mha_decode_workspace_bytes(dtype, B, d, H, cap))


def alloc_mha_workspace(dtype: int, B: int, d: int, H: int, cap: int, device=None) -> torch.Tensor:
    """Caller-owned scratch for slim_mha_decode_step."""
    n = slim_mha_decode_workspace_bytes(dtype, B, d, H, cap)
    if n == 0:
        raise SlimError(SLIM_EUNSUPPORTED, "slim_mha_decode_workspace_bytes")
    return torch.empty(n, dtype=torch.uint8, device=device or torch.device("cuda"))


def slim_mha_decode_step(q: torch.Tensor, k_new, v_new, Kcache: torch.Tensor, Vcache: torch.Tensor,
                         lens: torch.Tensor, H: int, out: torch.Tensor, workspace: torch.Tensor, status: torch.Tensor,
                         stream=None) -> None:
    """Standard MHA generation step over explicit K and V caches [B][cap][d] (the comparison baseline)."""
    for t, nm in ((q, "q"), (Kcache, "Kcache"), (Vcache, "Vcache"), (lens, "lens"), (out, "out"),
                  (workspace, "workspace"), (status, "status")):
        _cuda(t, nm)
    B, cap, d = Kcache.shape
    if Vcache.shape != Kcache.shape or Vcache.dtype != Kcache.dtype:
        raise ValueError("Vcache must match Kcache")
    if q.shape != (B, d) or out.shape != (B, d) or q.dtype != torch.float32 or out.dtype != torch.float32:
        raise ValueError("q/out must be float32 [B][d]")
    for t, nm in ((k_new, "k_new"), (v_new, "v_new")):
        if t is not None:
            _cuda(t, nm)
            if t.shape != (B, d) or t.dtype != Kcache.dtype:
                raise ValueError(f"{nm} must be [B][d] in the cache dtype")
    _check(_lib.slim_mha_decode_step(_ptr(q), _ptr(k_new), _ptr(v_new), _ptr(Kcache), _ptr(Vcache), _ptr(lens),
                                     _DT[Kcache.dtype], B, d, H, cap, _ptr(out), _ptr(workspace), workspace.numel(),
                                     _ptr(status), _stream(stream)), "slim_mha_decode_step")


def slim_decode_step_host(q_host: torch.Tensor, k_new_host, Kcache: torch.Tensor, lens: torch.Tensor,
                          W_KV: torch.Tensor, H: int, out_host: torch.Tensor, workspace: torch.Tensor,
                          status: torch.Tensor, variant: int = SLIM_AUTO, t_hint: int = 0, stream=None) -> None:
    """slim_decode_step with q, k_new and out in (pinned) host memory; enqueues copies and the step."""
    B, cap, d = Kcache.shape
    if q_host.is_cuda or out_host.is_cuda or (k_new_host is not None and k_new_host.is_cuda):
        raise ValueError("host tensors expected")
    _check(_lib.slim_decode_step_host(_ptr(q_host), _ptr(k_new_host), _ptr(Kcache), _ptr(lens), _ptr(W_KV),
                                      _DT[Kcache.dtype], B, d, H, cap, variant, t_hint, _ptr(out_host),
                                      _ptr(workspace), workspace.numel(), _ptr(status), _stream(stream)),
           "slim_decode_step_host")


def slim_tune(q, Kcache, lens, lens_restore: torch.Tensor, W_KV, H: int, Ts, reps: int, out, workspace, status,
              stream=None) -> None:
    B, cap, d = Kcache.shape
    ts = (ctypes.c_int64 * len(Ts))(*[int(t) for t in Ts])
    lr = lens_restore.to(torch.int32).cpu().contiguous()
    _check(_lib.slim_tune(_ptr(q), _ptr(Kcache), _ptr(lens), ctypes.c_void_p(lr.data_ptr()), _ptr(W_KV),
                          _DT[Kcache.dtype], B, d, H, cap, ts, len(Ts), reps, _ptr(out), _ptr(workspace),
                          workspace.numel(), _ptr(status), _stream(stream)), "slim_tune")


def slim_tune_record(dtype: int, B: int, d: int, H: int, T: int, ms_a: float, ms_b: float) -> None:
    _check(_lib.slim_tune_record(dtype, B, d, H, T, ms_a, ms_b), "slim_tune_record")


def slim_select_variant(dtype: int, B: int, d: int, H: int, T: int) -> int:
    return int(_lib.slim_select_variant(dtype, B, d, H, T))


def slim_tune_clear() -> None:
    _lib.slim_tune_clear()


def slim_timing_enable(n: int) -> None:
    _check(_lib.slim_timing_enable(int(n)), "slim_timing_enable")


def slim_timing_read(n: int) -> list:
    buf = (ctypes.c_float * max(n, 1))()
    cnt = _lib.slim_timing_read(buf, int(n))
    if cnt < 0:
        raise SlimError(cnt, "slim_timing_read")
    return [float(buf[i]) for i in range(cnt)]


def slim_debug_stall_next(wait_ns: int) -> None:
    """Test hook: the next tcgen05 split launch on this thread stalls until its waits (wait_ns) run out."""
    _check(_lib.slim_debug_stall_next(int(wait_ns)), "slim_debug_stall_next")


def raw_lib() -> ctypes.CDLL:
    """The loaded library handle (tests call entry points with raw arguments through it)."""
    return _lib
