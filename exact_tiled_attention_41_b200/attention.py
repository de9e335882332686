"""Torch-tensor entry points over the C ABI: allocation of outputs and workspace
(PyTorch's caching allocator) and argument marshalling; every step of the
computation runs in libfa.so's CUDA kernels.  Inputs must be contiguous bf16
CUDA tensors; anything else raises -- there is no CPU path.

Shapes follow the flash-attention README (flash_attn_func, flash_attn_varlen_func,
flash_attn_with_kvcache docstrings): q (B, Sq, Hq, D), k/v (B, Sk, Hkv, D); varlen
q (total_q, Hq, D) with int32 cu_seqlens; caches (B, capacity, Hkv, D).
softmax_scale defaults to 1/sqrt(D) (README, "How to use FlashAttention").
window_size = (left, right) is the sliding window of the flash_attn_func docstring
(-1 = unbounded side); deterministic selects the backward whose dq does not depend
on the order of float additions.
"""

from __future__ import annotations

import math

import torch

from . import abi


def _check(t: torch.Tensor, name: str, dtype=torch.bfloat16):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device.type != "cuda":
        raise ValueError(f"{name} must be a CUDA tensor (no CPU path)")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _raise(status: int, where: str):
    if status != abi.FA_OK:
        raise abi.FAError(status, where)


def _workspace(nbytes: int, device) -> torch.Tensor | None:
    if nbytes == 0:
        return None
    # torch's allocator returns >= 512-byte aligned blocks
    return torch.empty(nbytes, dtype=torch.uint8, device=device)


def _window(window_size):
    left, right = window_size
    return int(left), int(right)


def flash_attn_func(q, k, v, softmax_scale=None, causal=False, window_size=(-1, -1)):
    """Forward: returns (out (B, Sq, Hq, D) bf16, lse (B, Hq, Sq) fp32)."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _check(t, n)
    B, Sq, Hq, D = q.shape
    Sk, Hkv = k.shape[1], k.shape[2]
    scale = 1.0 / math.sqrt(D) if softmax_scale is None else softmax_scale
    out = torch.empty_like(q)
    lse = torch.empty((B, Hq, Sq), dtype=torch.float32, device=q.device)
    nb = abi.fa_fwd_workspace_size(B, Hq, Hkv, Sq, Sk, D)
    ws = _workspace(nb, q.device)
    _raise(abi.fa_fwd_ex(q, k, v, out, lse, B, Hq, Hkv, Sq, Sk, D, scale, causal, *_window(window_size), ws, nb),
           "fa_fwd")
    return out, lse


def flash_attn_backward(dout, q, k, v, out, lse, softmax_scale=None, causal=False, window_size=(-1, -1),
                        deterministic=False):
    """Backward: returns (dq, dk, dv) shaped like q, k, v."""
    for t, n in ((dout, "dout"), (q, "q"), (k, "k"), (v, "v"), (out, "out")):
        _check(t, n)
    _check(lse, "lse", torch.float32)
    B, Sq, Hq, D = q.shape
    Sk, Hkv = k.shape[1], k.shape[2]
    scale = 1.0 / math.sqrt(D) if softmax_scale is None else softmax_scale
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    nb = abi.fa_bwd_workspace_size(B, Hq, Hkv, Sq, Sk, D)
    ws = _workspace(nb, q.device)
    _raise(abi.fa_bwd_ex(q, k, v, out, dout, lse, dq, dk, dv, B, Hq, Hkv, Sq, Sk, D, scale, causal,
                         *_window(window_size), deterministic, ws, nb), "fa_bwd")
    return dq, dk, dv


def flash_attn_varlen_func(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k, softmax_scale=None,
                           causal=False, window_size=(-1, -1)):
    """Packed forward: returns (out (total_q, Hq, D), lse (Hq, total_q))."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _check(t, n)
    _check(cu_seqlens_q, "cu_seqlens_q", torch.int32)
    _check(cu_seqlens_k, "cu_seqlens_k", torch.int32)
    total_q, Hq, D = q.shape
    total_k, Hkv = k.shape[0], k.shape[1]
    nseq = cu_seqlens_q.numel() - 1
    scale = 1.0 / math.sqrt(D) if softmax_scale is None else softmax_scale
    out = torch.empty_like(q)
    lse = torch.empty((Hq, total_q), dtype=torch.float32, device=q.device)
    nb = abi.fa_varlen_fwd_workspace_size(nseq, total_q, total_k, Hq, Hkv, D)
    ws = _workspace(nb, q.device)
    _raise(abi.fa_varlen_fwd_ex(q, k, v, out, lse, cu_seqlens_q, cu_seqlens_k, nseq, max_seqlen_q, max_seqlen_k,
                                total_q, total_k, Hq, Hkv, D, scale, causal, *_window(window_size), ws, nb),
           "fa_varlen_fwd")
    return out, lse


def flash_attn_varlen_backward(dout, q, k, v, out, lse, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k,
                               softmax_scale=None, causal=False, window_size=(-1, -1), deterministic=False):
    for t, n in ((dout, "dout"), (q, "q"), (k, "k"), (v, "v"), (out, "out")):
        _check(t, n)
    _check(lse, "lse", torch.float32)
    total_q, Hq, D = q.shape
    total_k, Hkv = k.shape[0], k.shape[1]
    nseq = cu_seqlens_q.numel() - 1
    scale = 1.0 / math.sqrt(D) if softmax_scale is None else softmax_scale
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    nb = abi.fa_varlen_bwd_workspace_size(nseq, total_q, total_k, Hq, Hkv, D)
    ws = _workspace(nb, q.device)
    _raise(abi.fa_varlen_bwd_ex(q, k, v, out, dout, lse, dq, dk, dv, cu_seqlens_q, cu_seqlens_k, nseq, max_seqlen_q,
                                max_seqlen_k, total_q, total_k, Hq, Hkv, D, scale, causal, *_window(window_size),
                                deterministic, ws, nb), "fa_varlen_bwd")
    return dq, dk, dv


def flash_attn_with_kvcache(q, k_cache, v_cache, cache_seqlens, softmax_scale=None, causal=False, num_splits=0,
                            return_lse=True, k=None, v=None, cache_batch_idx=None, block_table=None,
                            window_size=(-1, -1)):
    """Attention of new queries against a KV cache (README, flash_attn_with_kvcache docstring).

    q (B, Sq, Hq, D); caches (B_cache, capacity, Hkv, D), or pages (num_blocks, page_block_size, Hkv, D)
    with block_table (B, max_blocks_per_seq) int32; cache_seqlens int32 (B,) or an int.  If k / v
    (B, seqlen_new, Hkv, D) are given they are written into the caches in place at cache_seqlens first.
    Returns (out (B, Sq, Hq, D), lse (B, Hq, Sq) or None).
    """
    for t, n in ((q, "q"), (k_cache, "k_cache"), (v_cache, "v_cache")):
        _check(t, n)
    B, Sq, Hq, D = q.shape
    if isinstance(cache_seqlens, int):
        cache_seqlens = torch.full((B,), cache_seqlens, dtype=torch.int32, device=q.device)
    _check(cache_seqlens, "cache_seqlens", torch.int32)
    if (k is None) != (v is None):
        raise ValueError("k and v must be given together")
    sn = 0
    if k is not None:
        _check(k, "k")
        _check(v, "v")
        sn = k.shape[1]
    if cache_batch_idx is not None:
        _check(cache_batch_idx, "cache_batch_idx", torch.int32)
    max_blocks = 0
    if block_table is not None:
        _check(block_table, "block_table", torch.int32)
        max_blocks = block_table.shape[1]
    cache_batch, cap, Hkv = k_cache.shape[0], k_cache.shape[1], k_cache.shape[2]
    scale = 1.0 / math.sqrt(D) if softmax_scale is None else softmax_scale
    out = torch.empty_like(q)
    lse = torch.empty((B, Hq, Sq), dtype=torch.float32, device=q.device) if return_lse else None
    nb = abi.fa_fwd_kvcache_ex_workspace_size(B, Hq, Hkv, Sq, D, cap, max_blocks, num_splits)
    ws = _workspace(nb, q.device)
    left, right = _window(window_size)
    _raise(abi.fa_fwd_kvcache_ex(q, k_cache, v_cache, cache_seqlens, k, v, sn, cache_batch_idx, block_table,
                                 max_blocks, cache_batch, cap, out, lse, B, Hq, Hkv, Sq, D, scale, causal, left, right,
                                 num_splits, ws, nb), "fa_fwd_kvcache_ex")
    return out, lse


def merge_attention_parts(o_parts, lse_parts, out_dtype=torch.bfloat16, out=None):
    """Merge results over disjoint key sets: o_parts (C, B, S, H, D) bf16 or fp32 and lse_parts (C, B, H, S)
    fp32, as fa_fwd writes them per key set.  Returns (out (B, S, H, D), lse (B, H, S))."""
    if o_parts.dtype not in (torch.bfloat16, torch.float32):
        raise TypeError("o_parts must be bfloat16 or float32")
    _check(o_parts, "o_parts", o_parts.dtype)
    _check(lse_parts, "lse_parts", torch.float32)
    C, B, S, H, D = o_parts.shape
    if tuple(lse_parts.shape) != (C, B, H, S):
        raise ValueError("lse_parts must be (C, B, H, S)")
    if out is None:
        out = torch.empty((B, S, H, D), dtype=out_dtype, device=o_parts.device)
    _check(out, "out", out.dtype)
    lse = torch.empty((B, H, S), dtype=torch.float32, device=o_parts.device)
    _raise(abi.fa_merge_lse(o_parts, lse_parts, C, B, S, H, D, o_parts.dtype == torch.float32, out, lse,
                            out.dtype == torch.float32), "fa_merge_lse")
    return out, lse


class FlashAttnFunction(torch.autograd.Function):
    """Autograd wrapper: forward = fa_fwd_ex, backward = fa_bwd_ex."""

    @staticmethod
    def forward(ctx, q, k, v, softmax_scale=None, causal=False, window_size=(-1, -1), deterministic=False):
        out, lse = flash_attn_func(q, k, v, softmax_scale, causal, window_size)
        ctx.save_for_backward(q, k, v, out, lse)
        ctx.softmax_scale, ctx.causal = softmax_scale, causal
        ctx.window_size, ctx.deterministic = window_size, deterministic
        return out

    @staticmethod
    def backward(ctx, dout):
        q, k, v, out, lse = ctx.saved_tensors
        dq, dk, dv = flash_attn_backward(dout.contiguous(), q, k, v, out, lse, ctx.softmax_scale, ctx.causal,
                                         ctx.window_size, ctx.deterministic)
        return dq, dk, dv, None, None, None, None
