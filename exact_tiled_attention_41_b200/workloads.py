"""Seeded synthetic inputs for the five attention workloads.

This module only draws random numbers; it holds none of the attention
arithmetic, and both the CUDA path and the fp64 oracle consume what it
returns.  Every tensor comes from ``torch.Generator('cpu').manual_seed(seed)``
in a fixed order -- integer lengths first, then Q, K, V, dO -- as
``torch.randn(..., dtype=float32)`` rounded to bfloat16 (i.i.d. N(0, 1)).
Random lengths are inclusive integer draws (``randint(lo, hi + 1)``).

The shapes mirror the workloads on the source pages (flash-attention README,
"Performance" section: head dims 64/128, long sequences; ``flash_attn_with_kvcache``
docstring: contiguous cache with per-row ``cache_seqlens``).
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

BF16_NAN = float("nan")


@dataclass
class Workload:
    name: str
    kind: str                      # "dense" | "varlen" | "kvcache"
    causal: bool
    scale: float
    tensors: dict = field(default_factory=dict)
    meta: dict = field(default_factory=dict)
    window: tuple = (-1, -1)       # sliding window (left, right); -1 = unbounded side


def _randn(g, shape):
    return torch.randn(shape, generator=g, dtype=torch.float32, device=g.device).to(torch.bfloat16)


def dense(B, Sq, Sk, Hq, Hkv, D, causal, seed=0, with_grad=True, name=None) -> Workload:
    """(B, S, H, D) tensors; dO drawn after Q, K, V."""
    g = torch.Generator("cpu").manual_seed(seed)
    q = _randn(g, (B, Sq, Hq, D))
    k = _randn(g, (B, Sk, Hkv, D))
    v = _randn(g, (B, Sk, Hkv, D))
    t = dict(q=q, k=k, v=v)
    if with_grad:
        t["do"] = _randn(g, (B, Sq, Hq, D))
    meta = dict(B=B, Sq=Sq, Sk=Sk, Hq=Hq, Hkv=Hkv, D=D)
    return Workload(name or f"dense_B{B}_Sq{Sq}_Sk{Sk}_Hq{Hq}_Hkv{Hkv}_D{D}", "dense", causal,
                    1.0 / math.sqrt(D), t, meta)


def varlen(lengths_q, lengths_k, Hq, Hkv, D, causal, seed=0, with_grad=True, name=None, g=None) -> Workload:
    """Packed (total, H, D) tensors with int32 cu_seqlens (cu[0] = 0)."""
    g = g if g is not None else torch.Generator("cpu").manual_seed(seed)
    lq = torch.as_tensor(lengths_q, dtype=torch.int64)
    lk = torch.as_tensor(lengths_k, dtype=torch.int64)
    cu_q = torch.zeros(len(lq) + 1, dtype=torch.int32)
    cu_k = torch.zeros(len(lk) + 1, dtype=torch.int32)
    cu_q[1:] = torch.cumsum(lq, 0).to(torch.int32)
    cu_k[1:] = torch.cumsum(lk, 0).to(torch.int32)
    tq, tk = int(cu_q[-1]), int(cu_k[-1])
    q = _randn(g, (tq, Hq, D))
    k = _randn(g, (tk, Hkv, D))
    v = _randn(g, (tk, Hkv, D))
    t = dict(q=q, k=k, v=v, cu_q=cu_q, cu_k=cu_k)
    if with_grad:
        t["do"] = _randn(g, (tq, Hq, D))
    meta = dict(num_seqs=len(lq), max_q=int(lq.max()), max_k=int(lk.max()), total_q=tq, total_k=tk,
                Hq=Hq, Hkv=Hkv, D=D)
    return Workload(name or f"varlen_n{len(lq)}_Hq{Hq}_D{D}", "varlen", causal, 1.0 / math.sqrt(D), t, meta)


def varlen_random(num_seqs, lo, hi, H, D, causal, seed=0, with_grad=True, name=None) -> Workload:
    """Sequence lengths uniform in [lo, hi] (inclusive) from the seed; Sq = Sk per sequence."""
    g = torch.Generator("cpu").manual_seed(seed)
    lens = torch.randint(lo, hi + 1, (num_seqs,), generator=g, dtype=torch.int64)
    return varlen(lens, lens, H, H, D, causal, seed, with_grad, name, g=g)


def kvcache(B, Hq, Hkv, D, capacity, lo, hi, seed=0, Sq=1, nan_guard=True, name=None, lengths=None,
            device="cpu") -> Workload:
    """Contiguous cache (B, capacity, Hkv, D); rows >= cache_seqlens[b] hold NaN guards.

    Only the valid rows are drawn from the generator (K for every batch row,
    then V for every batch row), so the guard rows cost no random numbers.
    Lengths always come from the CPU generator; ``device="cuda"`` draws the
    tensors with a CUDA generator of the same seed (faster for multi-GB caches).
    """
    g = torch.Generator("cpu").manual_seed(seed)
    if lengths is None:
        lens = torch.randint(lo, hi + 1, (B,), generator=g, dtype=torch.int64)
    else:
        lens = torch.as_tensor(lengths, dtype=torch.int64)
    if device != "cpu":
        g = torch.Generator(device).manual_seed(seed)
    q = _randn(g, (B, Sq, Hq, D))
    fill = BF16_NAN if nan_guard else 0.0
    kc = torch.full((B, capacity, Hkv, D), fill, dtype=torch.bfloat16, device=device)
    vc = torch.full((B, capacity, Hkv, D), fill, dtype=torch.bfloat16, device=device)
    for b in range(B):
        L = int(lens[b])
        kc[b, :L] = _randn(g, (L, Hkv, D))
    for b in range(B):
        L = int(lens[b])
        vc[b, :L] = _randn(g, (L, Hkv, D))
    t = dict(q=q, k_cache=kc, v_cache=vc, cache_seqlens=lens.to(torch.int32))
    meta = dict(B=B, Sq=Sq, Hq=Hq, Hkv=Hkv, D=D, capacity=capacity)
    return Workload(name or f"kvcache_B{B}_Hq{Hq}_Hkv{Hkv}_D{D}", "kvcache", False, 1.0 / math.sqrt(D), t, meta)


def kvcache_update(B, Sq, Hq, Hkv, D, capacity, lengths, seqlen_new=0, page=0, seed=0, cache_batch_idx=None,
                   cache_batch=None, spare_blocks=3, name=None) -> Workload:
    """A cache for one flash_attn_with_kvcache call: Sq new queries, optional k / v to append.

    Contiguous (page = 0): caches (cache_batch or B, capacity, Hkv, D); sequence b lives in cache row
    cache_batch_idx[b] (b without an index).  Paged (page > 0, capacity a multiple of page): caches
    (num_blocks, page, Hkv, D) with num_blocks = B * capacity / page + spare_blocks, and a block table
    (B, capacity / page) drawn as a random permutation of the blocks.  Logical rows below
    lengths[b] hold N(0, 1) values, every other row NaN (nothing may read them).  Draw order: block
    permutation, q, K rows, V rows, k_new, v_new.
    """
    g = torch.Generator("cpu").manual_seed(seed)
    lens = torch.as_tensor(lengths, dtype=torch.int64)
    t = {}
    if page > 0:
        assert capacity % page == 0
        nblk_seq = capacity // page
        nblk = B * nblk_seq + spare_blocks
        perm = torch.randperm(nblk, generator=g)[:B * nblk_seq]
        table = perm.reshape(B, nblk_seq).to(torch.int32)
        kc = torch.full((nblk, page, Hkv, D), BF16_NAN, dtype=torch.bfloat16)
        vc = torch.full((nblk, page, Hkv, D), BF16_NAN, dtype=torch.bfloat16)
        t["block_table"] = table

        def rows(cache, b, L, vals):
            for p0 in range(0, L, page):
                n = min(page, L - p0)
                cache[int(table[b, p0 // page]), :n] = vals[p0:p0 + n]
    else:
        nb = cache_batch if cache_batch is not None else B
        kc = torch.full((nb, capacity, Hkv, D), BF16_NAN, dtype=torch.bfloat16)
        vc = torch.full((nb, capacity, Hkv, D), BF16_NAN, dtype=torch.bfloat16)
        idx = torch.arange(B) if cache_batch_idx is None else torch.as_tensor(cache_batch_idx, dtype=torch.int64)
        if cache_batch_idx is not None:
            t["cache_batch_idx"] = idx.to(torch.int32)

        def rows(cache, b, L, vals):
            cache[int(idx[b]), :L] = vals
    q = _randn(g, (B, Sq, Hq, D))
    for b in range(B):
        rows(kc, b, int(lens[b]), _randn(g, (int(lens[b]), Hkv, D)))
    for b in range(B):
        rows(vc, b, int(lens[b]), _randn(g, (int(lens[b]), Hkv, D)))
    if seqlen_new > 0:
        t["k_new"] = _randn(g, (B, seqlen_new, Hkv, D))
        t["v_new"] = _randn(g, (B, seqlen_new, Hkv, D))
    t.update(q=q, k_cache=kc, v_cache=vc, cache_seqlens=lens.to(torch.int32))
    meta = dict(B=B, Sq=Sq, Hq=Hq, Hkv=Hkv, D=D, capacity=capacity, page=page, seqlen_new=seqlen_new)
    return Workload(name or f"kvcache_update_B{B}_Sq{Sq}_Hq{Hq}_Hkv{Hkv}_D{D}", "kvcache", False,
                    1.0 / math.sqrt(D), t, meta)


# The five workloads: sizes as stated for each configuration.
def tiny(causal: bool, seed=0) -> Workload:
    """B=1, Hq=Hkv=2, Sq=Sk=128, D=64."""
    return dense(1, 128, 128, 2, 2, 64, causal, seed, name=f"tiny_B1_H2_S128_D64_{'causal' if causal else 'full'}")


def dense_prefill(seed=0) -> Workload:
    """B=4, Hq=Hkv=16, Sq=Sk=2048, D=128, causal."""
    return dense(4, 2048, 2048, 16, 16, 128, True, seed, name="dense_B4_H16_S2048_D128_causal")


def gqa_long(seed=0) -> Workload:
    """B=2, Hq=32, Hkv=8, Sq=Sk=8192, D=128, causal."""
    return dense(2, 8192, 8192, 32, 8, 128, True, seed, name="gqa_B2_Hq32_Hkv8_S8192_D128_causal")


def varlen_packed(D: int, seed=0) -> Workload:
    """16 sequences, lengths uniform in [128, 4096], Hq=Hkv=16, causal."""
    return varlen_random(16, 128, 4096, 16, D, True, seed, name=f"varlen_16seq_L128-4096_H16_D{D}_causal")


def decode(seed=0, nan_guard=True, device="cpu") -> Workload:
    """B=64, Hq=32, Hkv=8, Sq=1, cache lengths uniform in [1024, 16384], capacity 16384, D=128."""
    return kvcache(64, 32, 8, 128, 16384, 1024, 16384, seed, 1, nan_guard,
                   name="decode_B64_Hq32_Hkv8_cap16384_D128", device=device)
