"""Thin ctypes binding of libjetlong.so (C ABI in include/jetlong.h).

Argument marshalling only: every function checks tensor dtypes, devices and
shapes, allocates outputs with torch when the caller passes none, and forwards
raw device pointers plus the current CUDA stream to the C entry point of the
same name.  All attention arithmetic runs in the library's CUDA kernels; there
is no CPU fallback.  Importing this module loads the library and raises
``ImportError`` if it has not been built (``python -m
rope_context_extension_sm_b200.build``).
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libjetlong.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"libjetlong.so is not built ({LIB_PATH}); run python -m rope_context_extension_sm_b200.build")

_lib = ctypes.CDLL(LIB_PATH)

JL_OK, JL_ERR_INVALID, JL_ERR_UNSUPPORTED, JL_ERR_CUDA, JL_ERR_TIMEOUT = range(5)
_NAMES = {0: "JL_OK", 1: "JL_ERR_INVALID", 2: "JL_ERR_UNSUPPORTED", 3: "JL_ERR_CUDA", 4: "JL_ERR_TIMEOUT"}

_vp, _i32, _i64, _f32, _f64, _sz = (ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float,
                                    ctypes.c_double, ctypes.c_size_t)

# Every symbol include/jetlong.h declares, with its C signature.
SIGNATURES = {
    "jl_last_error": (ctypes.c_char_p, []),
    "jl_group_size": (_i64, [_i64, _i64]),
    "jl_sync_status": (ctypes.c_int, [_vp]),
    "jl_debug_bounds_enabled": (ctypes.c_int, []),
    "jl_decode_single_launch_enabled": (ctypes.c_int, []),
    "jl_rope_tables": (ctypes.c_int, [_vp, _vp, _i64, _i32, _f64, _vp]),
    "jl_bifocal_prefill": (ctypes.c_int, [_vp, _vp, _vp, _vp, _i32, _i64, _i32, _i32, _i32, _i32, _i32, _i32,
                                          _vp, _vp, _i64, _f32, _vp, _vp, _vp, _sz, _vp]),
    "jl_bifocal_prefill_workspace_size": (_sz, [_i64, _i32, _i32]),
    "jl_bifocal_prefill_and_cache": (ctypes.c_int, [_vp, _vp, _vp, _vp, _i32, _i64, _i32, _i32, _i32, _i32, _i32,
                                                    _i32, _vp, _vp, _i64, _f32, _vp, _vp, _vp, _vp, _i64, _vp, _sz,
                                                    _vp]),
    "jl_plain_prefill": (ctypes.c_int, [_vp, _vp, _vp, _vp, _i32, _i64, _i32, _i32, _i32, _i32, _vp, _vp, _i64,
                                        _f32, _vp, _vp, _vp, _sz, _vp]),
    "jl_bifocal_decode": (ctypes.c_int, [_vp, _vp, _vp, _vp, _i32, _i64, _i32, _i32, _i32, _i32, _i32, _i32, _vp,
                                         _vp, _i64, _f32, _vp, _vp, _vp, _sz, _vp]),
    "jl_bifocal_decode_workspace_size": (_sz, [_i32, _i32, _i32, _i32]),
    "jl_plain_decode": (ctypes.c_int, [_vp, _vp, _vp, _vp, _i32, _i64, _i32, _i32, _i32, _i32, _vp, _vp, _i64,
                                       _f32, _vp, _vp, _vp, _sz, _vp]),
    "jl_bifocal_decode_noalloc": (ctypes.c_int, [_vp, _vp, _vp, _vp, _i32, _i64, _i32, _i32, _i32, _i32, _i32, _i32,
                                                 _vp, _vp, _i64, _f32, _vp, _vp, _vp]),
    "jl_bifocal_decode_noalloc_scratch_bytes": (_sz, []),
    "jl_selftest_wait_timeout": (ctypes.c_int, [_i64, _vp]),
    "jl_rope_tables_scaled": (ctypes.c_int, [_vp, _vp, _i64, _i32, _f64, _vp, _vp]),
    "jl_interp_prefill": (ctypes.c_int, [_vp, _vp, _vp, _vp, _i32, _i64, _i32, _i32, _i32, _i32, _i32, _vp, _vp, _i64,
                                         _vp, _vp, _i64, _f32, _vp, _vp, _vp, _sz, _vp]),
    "jl_bifocal_decode_paged": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _i32, _i32,
                                               _i32, _i32, _i32, _vp, _vp, _i64, _f32, _vp, _vp, _vp, _sz, _vp]),
    "jl_kv_cache_fill_paged": (ctypes.c_int, [_vp, _vp, _vp, _vp, _i32, _i64, _i32, _i32, _vp, _vp, _i64, _vp, _vp,
                                              _vp, _i32, _i32, _i32, _vp]),
    "jl_decode_append_paged": (ctypes.c_int, [_vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _vp, _vp, _i64, _vp, _vp,
                                              _vp, _vp, _i32, _i32, _i32, _vp]),
    "jl_bifocal_prefill_chunk": (ctypes.c_int, [_vp, _vp, _vp, _i32, _i64, _i32, _i32, _vp, _vp, _i64, _i32, _i32,
                                                _i32, _i32, _i32, _vp, _vp, _i64, _f32, _vp, _vp, _vp]),
    "jl_bifocal_prefill_three_pass": (ctypes.c_int, [_vp, _vp, _vp, _vp, _i32, _i64, _i32, _i32, _i32, _i32, _i32,
                                                     _i32, _vp, _vp, _i64, _f32, _vp, _vp, _vp, _sz, _vp]),
    "jl_bifocal_prefill_three_pass_workspace_size": (_sz, [_i64, _i32, _i32]),
    "jl_kv_cache_fill": (ctypes.c_int, [_vp, _vp, _vp, _vp, _i32, _i64, _i32, _i32, _vp, _vp, _i64, _vp, _vp,
                                        _i64, _vp]),
    "jl_decode_append": (ctypes.c_int, [_vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _vp, _vp, _i64, _vp, _vp, _vp,
                                        _i64, _vp]),
}

for _name, (_res, _args) in SIGNATURES.items():
    _fn = getattr(_lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args


class JetLongError(RuntimeError):
    def __init__(self, status: int, where: str):
        msg = _lib.jl_last_error().decode(errors="replace")
        super().__init__(f"{where}: {_NAMES.get(status, status)}: {msg}")
        self.status = status


def _check(status: int, where: str) -> None:
    if status != JL_OK:
        raise JetLongError(status, where)


def _ptr(t: torch.Tensor | None) -> int | None:
    return None if t is None else t.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _need(t: torch.Tensor, dtype, name: str, ndim: int | None = None) -> None:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype} (got {t.dtype})")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dimensions (got {t.dim()})")


def jl_last_error() -> str:
    return _lib.jl_last_error().decode(errors="replace")


def jl_group_size(L: int, w_pretrained: int) -> int:
    return int(_lib.jl_group_size(L, w_pretrained))


def jl_sync_status(stream=None) -> None:
    """Synchronise the stream and raise JetLongError if a kernel's bounded wait ran out."""
    _check(_lib.jl_sync_status(_stream(stream)), "jl_sync_status")


def jl_selftest_wait_timeout(limit_cycles: int, stream=None) -> None:
    """Launch the bounded-wait self-test; jl_sync_status() then raises JL_ERR_TIMEOUT."""
    _check(_lib.jl_selftest_wait_timeout(int(limit_cycles), _stream(stream)), "jl_selftest_wait_timeout")


def jl_rope_tables(n_pos: int, head_dim: int, rope_base: float, *, device="cuda", cos=None, sin=None, stream=None):
    """fp32 [n_pos][head_dim/2] cos/sin tables (allocated unless given)."""
    if cos is None:
        cos = torch.empty((n_pos, head_dim // 2), dtype=torch.float32, device=device)
    if sin is None:
        sin = torch.empty((n_pos, head_dim // 2), dtype=torch.float32, device=device)
    _need(cos, torch.float32, "cos", 2)
    _need(sin, torch.float32, "sin", 2)
    _check(_lib.jl_rope_tables(_ptr(cos), _ptr(sin), n_pos, head_dim, float(rope_base), _stream(stream)),
           "jl_rope_tables")
    return cos, sin


def jl_rope_tables_scaled(n_pos: int, head_dim: int, rope_base: float, freq_scale, *, device="cuda", stream=None):
    """fp32 tables of cos/sin(p * theta_c * freq_scale[c]) for the interpolation variant."""
    import numpy as _np
    lam = _np.ascontiguousarray(_np.asarray(freq_scale, dtype=_np.float64))
    if lam.shape != (head_dim // 2,):
        raise ValueError("freq_scale must have head_dim/2 entries")
    cos = torch.empty((n_pos, head_dim // 2), dtype=torch.float32, device=device)
    sin = torch.empty_like(cos)
    _check(_lib.jl_rope_tables_scaled(_ptr(cos), _ptr(sin), n_pos, head_dim, float(rope_base), lam.ctypes.data,
                                      _stream(stream)), "jl_rope_tables_scaled")
    return cos, sin


def jl_interp_prefill(q, k, v, cu_seqlens, max_seqlen: int, w0: int, cos, sin, cos_rem, sin_rem, *,
                      softmax_scale: float = 0.0, out=None, lse=None, want_lse: bool = True, workspace=None,
                      rotate_keys_in_kernel: bool = False, stream=None):
    """Frequency-interpolation variant of the remote window (local pairs base RoPE).
    Key workspace as for jl_bifocal_prefill."""
    T, hq, hkv, d, out, lse = _prefill_args(q, k, v, cu_seqlens, cos, sin, out, lse, want_lse)
    _need(cos_rem, torch.float32, "cos_rem", 2)
    _need(sin_rem, torch.float32, "sin_rem", 2)
    batch = cu_seqlens.shape[0] - 1
    ws, ws_bytes = _key_workspace(workspace, rotate_keys_in_kernel, T, hkv, d, q.device)
    _check(_lib.jl_interp_prefill(_ptr(q), _ptr(k), _ptr(v), _ptr(cu_seqlens), batch, T, max_seqlen, hq, hkv, d, w0,
                                  _ptr(cos), _ptr(sin), cos.shape[0], _ptr(cos_rem), _ptr(sin_rem), cos_rem.shape[0],
                                  softmax_scale, _ptr(out), _ptr(lse), _ptr(ws), ws_bytes, _stream(stream)),
           "jl_interp_prefill")
    return out, lse


def _prefill_args(q, k, v, cu_seqlens, cos, sin, out, lse, want_lse):
    _need(q, torch.bfloat16, "q", 3)
    _need(k, torch.bfloat16, "k", 3)
    _need(v, torch.bfloat16, "v", 3)
    _need(cu_seqlens, torch.int32, "cu_seqlens", 1)
    _need(cos, torch.float32, "cos", 2)
    _need(sin, torch.float32, "sin", 2)
    T, hq, d = q.shape
    if k.shape != v.shape or k.shape[0] != T or k.shape[2] != d:
        raise ValueError("k and v must be [T][Hkv][d] matching q")
    if out is None:
        out = torch.empty_like(q)
    _need(out, torch.bfloat16, "out", 3)
    if lse is None and want_lse:
        lse = torch.empty((hq, T), dtype=torch.float32, device=q.device)
    if lse is not None:
        _need(lse, torch.float32, "lse", 2)
    return T, hq, k.shape[1], d, out, lse


def jl_bifocal_prefill_workspace_size(total_tokens: int, n_kv_heads: int, head_dim: int) -> int:
    return int(_lib.jl_bifocal_prefill_workspace_size(total_tokens, n_kv_heads, head_dim))


def _key_workspace(workspace, rotate_keys_in_kernel, T, hkv, d, device):
    """(pointer, bytes) of the prefill's key workspace: the caller's tensor, a new one
    (workspace=None), or none at all when the kernel is to rotate the keys itself."""
    if rotate_keys_in_kernel:
        return None, 0
    if workspace is None:
        workspace = torch.empty(jl_bifocal_prefill_workspace_size(T, hkv, d), dtype=torch.uint8, device=device)
    if not workspace.is_cuda or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous CUDA tensor")
    return workspace, workspace.numel() * workspace.element_size()


def jl_bifocal_prefill(q, k, v, cu_seqlens, max_seqlen: int, w0: int, w_pretrained: int, cos, sin, *,
                       softmax_scale: float = 0.0, out=None, lse=None, want_lse: bool = True, workspace=None,
                       rotate_keys_in_kernel: bool = False, stream=None):
    """Bifocal prefill over packed sequences. q [T][Hq][d], k/v [T][Hkv][d] raw bf16.

    The keys are rotated once into a workspace (workspace=None allocates one) unless
    rotate_keys_in_kernel is set.  Returns (out bf16 [T][Hq][d], lse fp32 [Hq][T] or None)."""
    T, hq, hkv, d, out, lse = _prefill_args(q, k, v, cu_seqlens, cos, sin, out, lse, want_lse)
    batch = cu_seqlens.shape[0] - 1
    ws, ws_bytes = _key_workspace(workspace, rotate_keys_in_kernel, T, hkv, d, q.device)
    _check(_lib.jl_bifocal_prefill(_ptr(q), _ptr(k), _ptr(v), _ptr(cu_seqlens), batch, T, max_seqlen, hq, hkv, d,
                                   w0, w_pretrained, _ptr(cos), _ptr(sin), cos.shape[0], softmax_scale, _ptr(out),
                                   _ptr(lse), _ptr(ws), ws_bytes, _stream(stream)), "jl_bifocal_prefill")
    return out, lse


def jl_bifocal_prefill_chunk(q, cu_seqlens, past_lens, max_seqlen: int, max_total: int, k_cache, v_cache, w0: int,
                             w_pretrained: int, cos, sin, *, softmax_scale: float = 0.0, out=None, lse=None,
                             want_lse: bool = True, stream=None):
    """Chunked bifocal prefill: chunk queries (raw, packed by cu_seqlens) against base-RoPE
    caches that already hold past_lens[b] tokens plus this chunk.  Returns (out, lse)."""
    _need(q, torch.bfloat16, "q", 3)
    _need(cu_seqlens, torch.int32, "cu_seqlens", 1)
    _need(past_lens, torch.int32, "past_lens", 1)
    _need(k_cache, torch.bfloat16, "k_cache", 4)
    _need(v_cache, torch.bfloat16, "v_cache", 4)
    T, hq, d = q.shape
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((hq, T), dtype=torch.float32, device=q.device)
    batch = cu_seqlens.shape[0] - 1
    _check(_lib.jl_bifocal_prefill_chunk(_ptr(q), _ptr(cu_seqlens), _ptr(past_lens), batch, T, max_seqlen, max_total,
                                         _ptr(k_cache), _ptr(v_cache), k_cache.shape[1], hq, k_cache.shape[2], d, w0,
                                         w_pretrained, _ptr(cos), _ptr(sin), cos.shape[0], softmax_scale, _ptr(out),
                                         _ptr(lse), _stream(stream)), "jl_bifocal_prefill_chunk")
    return out, lse


def jl_bifocal_prefill_three_pass(q, k, v, cu_seqlens, max_seqlen: int, w0: int, w_pretrained: int, cos, sin, *,
                                  softmax_scale: float = 0.0, out=None, lse=None, workspace=None,
                                  want_lse: bool = True, stream=None):
    """The literal three-pass inclusion-exclusion prefill; returns (out, lse, workspace).

    The workspace holds the passes afterwards: O_p fp32 [3][T][Hq][d], then lse_p fp32 [3][Hq][T]."""
    T, hq, hkv, d, out, lse = _prefill_args(q, k, v, cu_seqlens, cos, sin, out, lse, want_lse)
    need = int(_lib.jl_bifocal_prefill_three_pass_workspace_size(T, hq, d))
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    batch = cu_seqlens.shape[0] - 1
    _check(_lib.jl_bifocal_prefill_three_pass(_ptr(q), _ptr(k), _ptr(v), _ptr(cu_seqlens), batch, T, max_seqlen,
                                              hq, hkv, d, w0, w_pretrained, _ptr(cos), _ptr(sin), cos.shape[0],
                                              softmax_scale, _ptr(out), _ptr(lse), _ptr(workspace),
                                              workspace.numel() * workspace.element_size(), _stream(stream)),
           "jl_bifocal_prefill_three_pass")
    return out, lse, workspace


def jl_bifocal_prefill_and_cache(q, k, v, cu_seqlens, max_seqlen: int, w0: int, w_pretrained: int, cos, sin, k_cache,
                                 v_cache, *, softmax_scale: float = 0.0, out=None, lse=None, want_lse: bool = True,
                                 workspace=None, rotate_keys_in_kernel: bool = False, stream=None):
    """jl_bifocal_prefill that also writes the base-RoPE cache: k_cache[b][j] = R(j) k_j,
    v_cache[b][j] = v_j, caches [batch][stride][Hkv][d] bf16.  Key workspace as for
    jl_bifocal_prefill.  Returns (out, lse)."""
    T, hq, hkv, d, out, lse = _prefill_args(q, k, v, cu_seqlens, cos, sin, out, lse, want_lse)
    _need(k_cache, torch.bfloat16, "k_cache", 4)
    _need(v_cache, torch.bfloat16, "v_cache", 4)
    if k_cache.shape != v_cache.shape or k_cache.shape[2:] != (hkv, d):
        raise ValueError("k_cache and v_cache must both be [batch][stride][Hkv][d]")
    batch = cu_seqlens.shape[0] - 1
    ws, ws_bytes = _key_workspace(workspace, rotate_keys_in_kernel, T, hkv, d, q.device)
    _check(_lib.jl_bifocal_prefill_and_cache(_ptr(q), _ptr(k), _ptr(v), _ptr(cu_seqlens), batch, T, max_seqlen, hq,
                                             hkv, d, w0, w_pretrained, _ptr(cos), _ptr(sin), cos.shape[0],
                                             softmax_scale, _ptr(out), _ptr(lse), _ptr(k_cache), _ptr(v_cache),
                                             k_cache.shape[1], _ptr(ws), ws_bytes, _stream(stream)),
           "jl_bifocal_prefill_and_cache")
    return out, lse


def jl_plain_prefill(q, k, v, cu_seqlens, max_seqlen: int, cos, sin, *, softmax_scale: float = 0.0, out=None,
                     lse=None, want_lse: bool = True, workspace=None, rotate_keys_in_kernel: bool = False,
                     stream=None):
    """Plain causal RoPE prefill (comparator), same layout and key workspace as jl_bifocal_prefill."""
    T, hq, hkv, d, out, lse = _prefill_args(q, k, v, cu_seqlens, cos, sin, out, lse, want_lse)
    batch = cu_seqlens.shape[0] - 1
    ws, ws_bytes = _key_workspace(workspace, rotate_keys_in_kernel, T, hkv, d, q.device)
    _check(_lib.jl_plain_prefill(_ptr(q), _ptr(k), _ptr(v), _ptr(cu_seqlens), batch, T, max_seqlen, hq, hkv, d,
                                 _ptr(cos), _ptr(sin), cos.shape[0], softmax_scale, _ptr(out), _ptr(lse),
                                 _ptr(ws), ws_bytes, _stream(stream)), "jl_plain_prefill")
    return out, lse


def jl_kv_cache_fill(k, v, cu_seqlens, cos, sin, k_cache, v_cache, *, past_lens=None, stream=None):
    """Write R(p) k and v of every token into base-RoPE caches [B][stride][Hkv][d] at
    positions p = past_lens[b] + (token index within its sequence)."""
    if past_lens is not None:
        _need(past_lens, torch.int32, "past_lens", 1)
    _need(k, torch.bfloat16, "k", 3)
    _need(v, torch.bfloat16, "v", 3)
    _need(cu_seqlens, torch.int32, "cu_seqlens", 1)
    _need(k_cache, torch.bfloat16, "k_cache", 4)
    _need(v_cache, torch.bfloat16, "v_cache", 4)
    T, hkv, d = k.shape
    _check(_lib.jl_kv_cache_fill(_ptr(k), _ptr(v), _ptr(cu_seqlens), _ptr(past_lens), cu_seqlens.shape[0] - 1, T,
                                 hkv, d, _ptr(cos),
                                 _ptr(sin), cos.shape[0], _ptr(k_cache), _ptr(v_cache), k_cache.shape[1],
                                 _stream(stream)), "jl_kv_cache_fill")
    return k_cache, v_cache


def jl_decode_append(q, k, v, seqlens, cos, sin, k_cache, v_cache, *, q_out=None, stream=None):
    """Rotate one new raw token per entry by R(seqlens-1): returns q~ and appends k~, v to the caches."""
    _need(q, torch.bfloat16, "q", 3)
    _need(k, torch.bfloat16, "k", 3)
    _need(v, torch.bfloat16, "v", 3)
    _need(seqlens, torch.int32, "seqlens", 1)
    if q_out is None:
        q_out = torch.empty_like(q)
    B, hq, d = q.shape
    _check(_lib.jl_decode_append(_ptr(q), _ptr(k), _ptr(v), _ptr(seqlens), B, hq, k.shape[1], d, _ptr(cos),
                                 _ptr(sin), cos.shape[0], _ptr(q_out), _ptr(k_cache), _ptr(v_cache),
                                 k_cache.shape[1], _stream(stream)), "jl_decode_append")
    return q_out


def jl_bifocal_decode_workspace_size(B: int, Hq: int, head_dim: int, max_seqlen: int) -> int:
    return int(_lib.jl_bifocal_decode_workspace_size(B, Hq, head_dim, max_seqlen))


def _decode_args(q, k_cache, v_cache, seqlens, cos, sin, max_seqlen, out, lse, workspace, want_lse):
    _need(q, torch.bfloat16, "q", 3)
    _need(k_cache, torch.bfloat16, "k_cache", 4)
    _need(v_cache, torch.bfloat16, "v_cache", 4)
    _need(seqlens, torch.int32, "seqlens", 1)
    _need(cos, torch.float32, "cos", 2)
    _need(sin, torch.float32, "sin", 2)
    B, hq, d = q.shape
    if k_cache.shape != v_cache.shape or k_cache.shape[0] != B or k_cache.shape[3] != d:
        raise ValueError("k_cache and v_cache must be [B][cache_stride][Hkv][d] matching q")
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((B, hq), dtype=torch.float32, device=q.device)
    need = jl_bifocal_decode_workspace_size(B, hq, d, max_seqlen)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    return B, hq, k_cache.shape[2], d, out, lse, workspace


def jl_bifocal_decode(q, k_cache, v_cache, seqlens, max_seqlen: int, w0: int, w_pretrained: int, cos, sin, *,
                      softmax_scale: float = 0.0, out=None, lse=None, workspace=None, want_lse: bool = True,
                      stream=None):
    """Single-query bifocal decode on a base-RoPE cache (cache is only read).

    q [B][Hq][d] already rotated by R(seqlens[b]-1); caches [B][stride][Hkv][d].
    Returns (out bf16 [B][Hq][d], lse fp32 [B][Hq] or None)."""
    B, hq, hkv, d, out, lse, ws = _decode_args(q, k_cache, v_cache, seqlens, cos, sin, max_seqlen, out, lse,
                                               workspace, want_lse)
    _check(_lib.jl_bifocal_decode(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(seqlens), B, k_cache.shape[1],
                                  max_seqlen, hq, hkv, d, w0, w_pretrained, _ptr(cos), _ptr(sin), cos.shape[0],
                                  softmax_scale, _ptr(out), _ptr(lse), _ptr(ws), ws.numel() * ws.element_size(),
                                  _stream(stream)), "jl_bifocal_decode")
    return out, lse


def jl_plain_decode(q, k_cache, v_cache, seqlens, max_seqlen: int, cos, sin, *, softmax_scale: float = 0.0,
                    out=None, lse=None, workspace=None, want_lse: bool = True, stream=None):
    """Plain causal decode (comparator), same layout as jl_bifocal_decode."""
    B, hq, hkv, d, out, lse, ws = _decode_args(q, k_cache, v_cache, seqlens, cos, sin, max_seqlen, out, lse,
                                               workspace, want_lse)
    _check(_lib.jl_plain_decode(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(seqlens), B, k_cache.shape[1],
                                max_seqlen, hq, hkv, d, _ptr(cos), _ptr(sin), cos.shape[0], softmax_scale,
                                _ptr(out), _ptr(lse), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "jl_plain_decode")
    return out, lse


def jl_bifocal_decode_paged(q, k_pool, v_pool, block_table, seqlens, max_seqlen: int, w0: int, w_pretrained: int,
                            cos, sin, *, softmax_scale: float = 0.0, out=None, lse=None, workspace=None,
                            want_lse: bool = True, stream=None):
    """Bifocal decode over paged caches: pools [num_pages][page_size][Hkv][d], block_table [B][max_pages]."""
    _need(q, torch.bfloat16, "q", 3)
    _need(k_pool, torch.bfloat16, "k_pool", 4)
    _need(v_pool, torch.bfloat16, "v_pool", 4)
    _need(block_table, torch.int32, "block_table", 2)
    _need(seqlens, torch.int32, "seqlens", 1)
    B, hq, d = q.shape
    num_pages, page_size, hkv, _ = k_pool.shape
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((B, hq), dtype=torch.float32, device=q.device)
    need = jl_bifocal_decode_workspace_size(B, hq, d, max_seqlen)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    _check(_lib.jl_bifocal_decode_paged(_ptr(q), _ptr(k_pool), _ptr(v_pool), _ptr(block_table), _ptr(seqlens), B,
                                        block_table.shape[1], page_size, num_pages, max_seqlen, hq, hkv, d, w0,
                                        w_pretrained, _ptr(cos), _ptr(sin), cos.shape[0], softmax_scale, _ptr(out),
                                        _ptr(lse), _ptr(workspace), workspace.numel() * workspace.element_size(),
                                        _stream(stream)), "jl_bifocal_decode_paged")
    return out, lse


def jl_kv_cache_fill_paged(k, v, cu_seqlens, cos, sin, k_pool, v_pool, block_table, *, past_lens=None, stream=None):
    """jl_kv_cache_fill into paged pools through a block table."""
    T, hkv, d = k.shape
    _check(_lib.jl_kv_cache_fill_paged(_ptr(k), _ptr(v), _ptr(cu_seqlens), _ptr(past_lens), cu_seqlens.shape[0] - 1,
                                       T, hkv, d, _ptr(cos), _ptr(sin), cos.shape[0], _ptr(k_pool), _ptr(v_pool),
                                       _ptr(block_table), block_table.shape[1], k_pool.shape[1], k_pool.shape[0],
                                       _stream(stream)), "jl_kv_cache_fill_paged")


def jl_decode_append_paged(q, k, v, seqlens, cos, sin, k_pool, v_pool, block_table, *, q_out=None, stream=None):
    """jl_decode_append into paged pools through a block table; returns q~."""
    if q_out is None:
        q_out = torch.empty_like(q)
    B, hq, d = q.shape
    _check(_lib.jl_decode_append_paged(_ptr(q), _ptr(k), _ptr(v), _ptr(seqlens), B, hq, k.shape[1], d, _ptr(cos),
                                       _ptr(sin), cos.shape[0], _ptr(q_out), _ptr(k_pool), _ptr(v_pool),
                                       _ptr(block_table), block_table.shape[1], k_pool.shape[1], k_pool.shape[0],
                                       _stream(stream)), "jl_decode_append_paged")
    return q_out


def jl_bifocal_decode_noalloc_scratch_bytes() -> int:
    return int(_lib.jl_bifocal_decode_noalloc_scratch_bytes())


def jl_bifocal_decode_noalloc(q, k_cache, v_cache, seqlens, max_seqlen: int, w0: int, w_pretrained: int, cos, sin,
                              *, out, lse=None, softmax_scale: float = 0.0, stream=None):
    """jl_bifocal_decode for callers that cannot allocate: the library uses its own
    static per-device scratch, so the caller passes only inputs and outputs (out and
    lse are caller-owned; lse may be None).  Calls that overlap on the GPU race on
    the shared scratch."""
    _need(q, torch.bfloat16, "q", 3)
    _need(k_cache, torch.bfloat16, "k_cache", 4)
    _need(v_cache, torch.bfloat16, "v_cache", 4)
    _need(seqlens, torch.int32, "seqlens", 1)
    _need(out, torch.bfloat16, "out", 3)
    B, hq, d = q.shape
    _check(_lib.jl_bifocal_decode_noalloc(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(seqlens), B, k_cache.shape[1],
                                          max_seqlen, hq, k_cache.shape[2], d, w0, w_pretrained, _ptr(cos),
                                          _ptr(sin), cos.shape[0], softmax_scale, _ptr(out), _ptr(lse),
                                          _stream(stream)), "jl_bifocal_decode_noalloc")
    return out, lse


def default_scale(head_dim: int) -> float:
    return 1.0 / math.sqrt(head_dim)
