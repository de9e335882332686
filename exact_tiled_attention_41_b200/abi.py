"""ctypes binding of libfa.so with the C-ABI's own names (argument marshalling only).

Every function here takes the same arguments as its C counterpart in
include/fa.h; device buffers may be given as torch tensors (their data_ptr()
is passed) or as raw integer addresses, and ``stream`` as a torch.cuda.Stream,
a raw cudaStream_t integer, or None for the current torch stream.  Nothing is
computed in Python: the library must be built (``python -m
exact_tiled_attention_41_b200.build``) and is loaded from the package
directory; when it is missing the first call raises.
"""

from __future__ import annotations

import ctypes
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "lib", "libfa.so")

FA_OK = 0
FA_ERR_INVALID_ARG = 1
FA_ERR_UNSUPPORTED = 2
FA_ERR_ALIGNMENT = 3
FA_ERR_WORKSPACE = 4
FA_ERR_CUDA = 5
FA_ERR_TIMEOUT = 6

EXPORTS = (
    "fa_fwd", "fa_fwd_workspace_size", "fa_bwd", "fa_bwd_workspace_size",
    "fa_varlen_fwd", "fa_varlen_fwd_workspace_size", "fa_varlen_bwd", "fa_varlen_bwd_workspace_size",
    "fa_fwd_kvcache", "fa_fwd_kvcache_workspace_size", "fa_status_string", "fa_get_device_status",
    "fa_set_wait_timeout_ns", "fa_debug_wait_timeout_selftest", "fa_debug_umma_selftest",
    "fa_profile_begin", "fa_profile_read",
    "fa_fwd_kvcache_noalloc", "fa_fwd_kvcache_noalloc_scratch_bytes", "fa_debug_exp2_selftest",
    "fa_fwd_ex", "fa_bwd_ex", "fa_varlen_fwd_ex", "fa_varlen_bwd_ex",
    "fa_fwd_kvcache_ex", "fa_fwd_kvcache_ex_workspace_size", "fa_merge_lse",
)

FA_KERNEL_FWD = 0
FA_KERNEL_BWD = 1
FA_KERNEL_DECODE = 2
FA_KERNEL_BWD_DQ = 3
FA_KERNEL_BWD_ALL = 4

_P = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float
_Z = ctypes.c_size_t
_U64 = ctypes.c_ulonglong

_SIGS = {
    "fa_fwd_workspace_size": (_Z, [_I] * 6),
    "fa_fwd": (_I, [_P] * 5 + [_I] * 6 + [_F, _I, _P, _Z, _P]),
    "fa_bwd_workspace_size": (_Z, [_I] * 6),
    "fa_bwd": (_I, [_P] * 9 + [_I] * 6 + [_F, _I, _P, _Z, _P]),
    "fa_varlen_fwd_workspace_size": (_Z, [_I] * 6),
    "fa_varlen_fwd": (_I, [_P] * 7 + [_I] * 8 + [_F, _I, _P, _Z, _P]),
    "fa_varlen_bwd_workspace_size": (_Z, [_I] * 6),
    "fa_varlen_bwd": (_I, [_P] * 11 + [_I] * 8 + [_F, _I, _P, _Z, _P]),
    "fa_fwd_kvcache_workspace_size": (_Z, [_I] * 7),
    "fa_fwd_kvcache": (_I, [_P] * 6 + [_I] * 6 + [_F, _I, _I, _P, _Z, _P]),
    "fa_status_string": (ctypes.c_char_p, [_I]),
    "fa_get_device_status": (_I, [_P]),
    "fa_set_wait_timeout_ns": (_U64, [_U64]),
    "fa_debug_wait_timeout_selftest": (_I, [_U64, _P]),
    "fa_debug_umma_selftest": (_I, [_P, _P, _P, _I, _P]),
    "fa_profile_begin": (_I, [_I]),
    "fa_profile_read": (_I, [_I, ctypes.POINTER(_I), ctypes.POINTER(_F)]),
    "fa_fwd_kvcache_noalloc": (_I, [_P] * 6 + [_I] * 6 + [_F, _I, _I, _P]),
    "fa_fwd_kvcache_noalloc_scratch_bytes": (_Z, []),
    "fa_debug_exp2_selftest": (_I, [_P, _P, _I, _P]),
    "fa_fwd_ex": (_I, [_P] * 5 + [_I] * 6 + [_F, _I, _I, _I, _P, _Z, _P]),
    "fa_bwd_ex": (_I, [_P] * 9 + [_I] * 6 + [_F, _I, _I, _I, _I, _P, _Z, _P]),
    "fa_varlen_fwd_ex": (_I, [_P] * 7 + [_I] * 8 + [_F, _I, _I, _I, _P, _Z, _P]),
    "fa_varlen_bwd_ex": (_I, [_P] * 11 + [_I] * 8 + [_F, _I, _I, _I, _I, _P, _Z, _P]),
    "fa_fwd_kvcache_ex_workspace_size": (_Z, [_I] * 8),
    "fa_merge_lse": (_I, [_P, _P] + [_I] * 6 + [_P, _P, _I, _P]),
    "fa_fwd_kvcache_ex": (_I, [_P] * 6 + [_I] + [_P] * 2 + [_I] * 3 + [_P] * 2 + [_I] * 5 + [_F] + [_I] * 4
                          + [_P, _Z, _P]),
}

_lib = None


def load():
    """Load libfa.so (once) and declare every signature; raises if it is missing."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m exact_tiled_attention_41_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


class FAError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(s):
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(s, int):
        return s
    return s.cuda_stream


def status_string(status: int) -> str:
    return load().fa_status_string(int(status)).decode()


def fa_fwd_workspace_size(B, Hq, Hkv, Sq, Sk, D) -> int:
    return load().fa_fwd_workspace_size(B, Hq, Hkv, Sq, Sk, D)


def fa_fwd(q, k, v, out, lse, B, Hq, Hkv, Sq, Sk, D, softmax_scale, causal, workspace=None,
           workspace_bytes=0, stream=None) -> int:
    return load().fa_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, Hq, Hkv, Sq, Sk, D,
                         float(softmax_scale), int(bool(causal)), _ptr(workspace), workspace_bytes, _stream(stream))


def fa_bwd_workspace_size(B, Hq, Hkv, Sq, Sk, D) -> int:
    return load().fa_bwd_workspace_size(B, Hq, Hkv, Sq, Sk, D)


def fa_bwd(q, k, v, out, dout, lse, dq, dk, dv, B, Hq, Hkv, Sq, Sk, D, softmax_scale, causal, workspace,
           workspace_bytes, stream=None) -> int:
    return load().fa_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(dout), _ptr(lse), _ptr(dq), _ptr(dk), _ptr(dv),
                         B, Hq, Hkv, Sq, Sk, D, float(softmax_scale), int(bool(causal)), _ptr(workspace),
                         workspace_bytes, _stream(stream))


def fa_varlen_fwd_workspace_size(num_seqs, total_q, total_k, Hq, Hkv, D) -> int:
    return load().fa_varlen_fwd_workspace_size(num_seqs, total_q, total_k, Hq, Hkv, D)


def fa_varlen_fwd(q, k, v, out, lse, cu_seqlens_q, cu_seqlens_k, num_seqs, max_seqlen_q, max_seqlen_k, total_q,
                  total_k, Hq, Hkv, D, softmax_scale, causal, workspace=None, workspace_bytes=0, stream=None) -> int:
    return load().fa_varlen_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(cu_seqlens_q),
                                _ptr(cu_seqlens_k), num_seqs, max_seqlen_q, max_seqlen_k, total_q, total_k, Hq, Hkv, D,
                                float(softmax_scale), int(bool(causal)), _ptr(workspace), workspace_bytes,
                                _stream(stream))


def fa_varlen_bwd_workspace_size(num_seqs, total_q, total_k, Hq, Hkv, D) -> int:
    return load().fa_varlen_bwd_workspace_size(num_seqs, total_q, total_k, Hq, Hkv, D)


def fa_varlen_bwd(q, k, v, out, dout, lse, dq, dk, dv, cu_seqlens_q, cu_seqlens_k, num_seqs, max_seqlen_q,
                  max_seqlen_k, total_q, total_k, Hq, Hkv, D, softmax_scale, causal, workspace, workspace_bytes,
                  stream=None) -> int:
    return load().fa_varlen_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(dout), _ptr(lse), _ptr(dq), _ptr(dk),
                                _ptr(dv), _ptr(cu_seqlens_q), _ptr(cu_seqlens_k), num_seqs, max_seqlen_q, max_seqlen_k,
                                total_q, total_k, Hq, Hkv, D, float(softmax_scale), int(bool(causal)), _ptr(workspace),
                                workspace_bytes, _stream(stream))


def fa_fwd_kvcache_workspace_size(B, Hq, Hkv, Sq, cache_capacity, D, num_splits) -> int:
    return load().fa_fwd_kvcache_workspace_size(B, Hq, Hkv, Sq, cache_capacity, D, num_splits)


def fa_fwd_kvcache(q, k_cache, v_cache, cache_seqlens, out, lse, B, Hq, Hkv, Sq, cache_capacity, D, softmax_scale,
                   causal, num_splits, workspace, workspace_bytes, stream=None) -> int:
    return load().fa_fwd_kvcache(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(cache_seqlens), _ptr(out), _ptr(lse),
                                 B, Hq, Hkv, Sq, cache_capacity, D, float(softmax_scale), int(bool(causal)),
                                 int(num_splits), _ptr(workspace), workspace_bytes, _stream(stream))


def fa_fwd_ex(q, k, v, out, lse, B, Hq, Hkv, Sq, Sk, D, softmax_scale, causal, window_left, window_right,
              workspace=None, workspace_bytes=0, stream=None) -> int:
    return load().fa_fwd_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, Hq, Hkv, Sq, Sk, D,
                            float(softmax_scale), int(bool(causal)), int(window_left), int(window_right),
                            _ptr(workspace), workspace_bytes, _stream(stream))


def fa_bwd_ex(q, k, v, out, dout, lse, dq, dk, dv, B, Hq, Hkv, Sq, Sk, D, softmax_scale, causal, window_left,
              window_right, deterministic, workspace, workspace_bytes, stream=None) -> int:
    return load().fa_bwd_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(dout), _ptr(lse), _ptr(dq), _ptr(dk),
                            _ptr(dv), B, Hq, Hkv, Sq, Sk, D, float(softmax_scale), int(bool(causal)),
                            int(window_left), int(window_right), int(bool(deterministic)), _ptr(workspace),
                            workspace_bytes, _stream(stream))


def fa_varlen_fwd_ex(q, k, v, out, lse, cu_seqlens_q, cu_seqlens_k, num_seqs, max_seqlen_q, max_seqlen_k, total_q,
                     total_k, Hq, Hkv, D, softmax_scale, causal, window_left, window_right, workspace=None,
                     workspace_bytes=0, stream=None) -> int:
    return load().fa_varlen_fwd_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(cu_seqlens_q),
                                   _ptr(cu_seqlens_k), num_seqs, max_seqlen_q, max_seqlen_k, total_q, total_k, Hq,
                                   Hkv, D, float(softmax_scale), int(bool(causal)), int(window_left),
                                   int(window_right), _ptr(workspace), workspace_bytes, _stream(stream))


def fa_varlen_bwd_ex(q, k, v, out, dout, lse, dq, dk, dv, cu_seqlens_q, cu_seqlens_k, num_seqs, max_seqlen_q,
                     max_seqlen_k, total_q, total_k, Hq, Hkv, D, softmax_scale, causal, window_left, window_right,
                     deterministic, workspace, workspace_bytes, stream=None) -> int:
    return load().fa_varlen_bwd_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(dout), _ptr(lse), _ptr(dq), _ptr(dk),
                                   _ptr(dv), _ptr(cu_seqlens_q), _ptr(cu_seqlens_k), num_seqs, max_seqlen_q,
                                   max_seqlen_k, total_q, total_k, Hq, Hkv, D, float(softmax_scale),
                                   int(bool(causal)), int(window_left), int(window_right), int(bool(deterministic)),
                                   _ptr(workspace), workspace_bytes, _stream(stream))


def fa_fwd_kvcache_ex_workspace_size(B, Hq, Hkv, Sq, D, cache_capacity, max_blocks_per_seq, num_splits) -> int:
    return load().fa_fwd_kvcache_ex_workspace_size(B, Hq, Hkv, Sq, D, cache_capacity, max_blocks_per_seq, num_splits)


def fa_fwd_kvcache_ex(q, k_cache, v_cache, cache_seqlens, k_new, v_new, seqlen_new, cache_batch_idx, block_table,
                      max_blocks_per_seq, cache_batch, cache_capacity, out, lse, B, Hq, Hkv, Sq, D, softmax_scale,
                      causal, window_left, window_right, num_splits, workspace, workspace_bytes, stream=None) -> int:
    return load().fa_fwd_kvcache_ex(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(cache_seqlens), _ptr(k_new),
                                    _ptr(v_new), int(seqlen_new), _ptr(cache_batch_idx), _ptr(block_table),
                                    int(max_blocks_per_seq), int(cache_batch), int(cache_capacity), _ptr(out),
                                    _ptr(lse), B, Hq, Hkv, Sq, D, float(softmax_scale), int(bool(causal)),
                                    int(window_left), int(window_right), int(num_splits), _ptr(workspace),
                                    workspace_bytes, _stream(stream))


def fa_merge_lse(o_parts, lse_parts, num_parts, B, S, H, D, parts_fp32, out, lse, out_fp32, stream=None) -> int:
    return load().fa_merge_lse(_ptr(o_parts), _ptr(lse_parts), int(num_parts), B, S, H, D, int(bool(parts_fp32)),
                               _ptr(out), _ptr(lse), int(bool(out_fp32)), _stream(stream))


def fa_get_device_status(stream=None) -> int:
    return load().fa_get_device_status(_stream(stream))


def fa_set_wait_timeout_ns(ns: int) -> int:
    return load().fa_set_wait_timeout_ns(int(ns))


def fa_debug_wait_timeout_selftest(timeout_ns: int, stream=None) -> int:
    return load().fa_debug_wait_timeout_selftest(int(timeout_ns), _stream(stream))


def fa_debug_umma_selftest(a, b, c, mode: int, stream=None) -> int:
    return load().fa_debug_umma_selftest(_ptr(a), _ptr(b), _ptr(c), int(mode), _stream(stream))


def fa_debug_exp2_selftest(x, y, n: int, stream=None) -> int:
    return load().fa_debug_exp2_selftest(_ptr(x), _ptr(y), int(n), _stream(stream))


def fa_profile_begin(enable: int) -> int:
    return load().fa_profile_begin(int(enable))


def fa_profile_read(kernel_id: int):
    """Returns (status, launches, total_ms) for the recorded launches of one kernel."""
    n = _I(0)
    ms = _F(0.0)
    st = load().fa_profile_read(int(kernel_id), ctypes.byref(n), ctypes.byref(ms))
    return st, n.value, ms.value


def fa_fwd_kvcache_noalloc(q, k_cache, v_cache, cache_seqlens, out, lse, B, Hq, Hkv, Sq, cache_capacity, D,
                           softmax_scale, causal, num_splits, stream=None) -> int:
    """Decode for callers that cannot allocate: scratch lives in an array inside the library."""
    return load().fa_fwd_kvcache_noalloc(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(cache_seqlens), _ptr(out),
                                         _ptr(lse), B, Hq, Hkv, Sq, cache_capacity, D, float(softmax_scale),
                                         int(bool(causal)), int(num_splits), _stream(stream))


def fa_fwd_kvcache_noalloc_scratch_bytes() -> int:
    return load().fa_fwd_kvcache_noalloc_scratch_bytes()
