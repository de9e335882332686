"""fp64 reference of exact softmax attention (forward, backward, varlen, KV cache).

TEST INFRASTRUCTURE ONLY -- see the package docstring.  No blocking, no
online softmax, no fusion: S and P are materialised for one (sequence, query
head) at a time and every step is the textbook formula.

Sources (page titles as published; section named in brackets):

* flash-attention README, "How to use FlashAttention": the main function
  computes softmax(Q @ K^T * softmax_scale) @ V; softmax_scale defaults to
  1/sqrt(headdim).
* flash-attention README, ``flash_attn_func`` docstring: MQA/GQA -- the number
  of query heads must be divisible by the number of KV heads; with 6 query heads
  over 2 KV heads, query heads 0-2 read KV head 0 and 3-5 read KV head 1.
* flash-attention README, ``flash_attn_with_kvcache`` docstring and changelog
  entry 2.1: the causal mask is aligned to the bottom-right corner of the
  attention matrix (key j is kept for query i iff j <= i + seqlen_k - seqlen_q);
  a query row whose mask is all zero produces an output of zero.
* flash-attention README, ``flash_attn_func`` docstring (sliding window local
  attention, changelog 2.3): with window_size = (left, right) other than
  (-1, -1), query i attends only to the keys j with
  i + seqlen_k - seqlen_q - left <= j <= i + seqlen_k - seqlen_q + right;
  -1 means that side of the window is unbounded.
* flash-attention README, ``flash_attn_with_kvcache`` docstring: the cache is
  (batch, seqlen_cache, nheads_k, headdim) and ``cache_seqlens`` gives the
  number of valid keys per batch row.
* kernels-community/flash-attn2 Hub card, "Low-level ops": the low-level ops
  return the softmax log-sum-exp next to the output.
* FlashAttention fork v1.4 release notes, section 4 (``softmax.h``): a row max of
  -inf means every score of the row was masked; it is replaced by 0 so that
  (-inf) - (-inf) never produces NaN.

Readings where the pages are silent:

* LSE is the natural log of sum_j exp(scale * q_i . k_j) over the allowed keys
  (scale included), -inf for a fully masked row.
* The backward is the textbook softmax Jacobian: dV = P^T dO, dP = dO V^T,
  Delta_i = sum_j P_ij dP_ij, dS = P * (dP - Delta), dQ = scale dS K,
  dK = scale dS^T Q.  Rows that are fully masked contribute nothing.
* A causal mask and a window given together keep the keys that both keep
  (the causal rule caps the right side of the window at 0).  Any negative
  window side is unbounded, like -1.
* Varlen packing: tokens of sequence s occupy rows cu[s] .. cu[s+1]-1 of a
  (total, heads, headdim) array; each sequence is an independent problem.
"""

from __future__ import annotations

import numpy as np


def kv_head_of(h: int, n_heads_q: int, n_heads_kv: int) -> int:
    """KV head read by query head ``h`` (README, ``flash_attn_func``: GQA).

    Consecutive blocks of n_heads_q / n_heads_kv query heads share one KV head.
    """
    if n_heads_q % n_heads_kv != 0:
        raise ValueError("number of query heads must be divisible by number of KV heads")
    group = n_heads_q // n_heads_kv
    return h // group


def allowed_mask(len_q: int, len_k: int, causal: bool, window=(-1, -1)) -> np.ndarray:
    """Boolean (len_q, len_k) matrix, True where query i may attend to key j.

    README, ``flash_attn_with_kvcache`` docstring / changelog 2.1: the causal
    mask is aligned to the bottom-right corner, so key j is kept iff
    j <= i + len_k - len_q.  Without ``causal`` every key is kept.
    README, ``flash_attn_func`` docstring: a sliding window (left, right) keeps
    only keys in [i + len_k - len_q - left, i + len_k - len_q + right]; a
    negative side is unbounded.  Both rules together keep the intersection.
    """
    i = np.arange(len_q)[:, None]
    j = np.arange(len_k)[None, :]
    off = len_k - len_q
    keep = np.ones((len_q, len_k), dtype=bool)
    if causal:
        keep &= j <= i + off
    left, right = window
    if left >= 0:
        keep &= j >= i + off - left
    if right >= 0:
        keep &= j <= i + off + right
    return keep


def _scores(q: np.ndarray, k: np.ndarray, scale: float, mask: np.ndarray) -> np.ndarray:
    s = scale * (q @ k.T)
    return np.where(mask, s, -np.inf)


def head_forward(q, k, v, scale, mask):
    """One query head against one KV head: returns (O, LSE, P).

    q (Lq, D), k (Lk, D), v (Lk, Dv) float64; mask (Lq, Lk) bool.
    O = softmax(scale q k^T + mask) v  (README, "How to use FlashAttention");
    fully masked rows give O = 0 (README, causal-mask note) and LSE = -inf.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    s = _scores(q, k, scale, mask)
    m = s.max(axis=1, initial=-np.inf, keepdims=True)
    empty = ~np.isfinite(m)                      # whole row masked
    m_safe = np.where(empty, 0.0, m)             # -inf max replaced by 0 (fork notes, section 4)
    e = np.exp(s - m_safe)                       # exp(-inf) = 0 on masked entries
    l = e.sum(axis=1, keepdims=True)
    p = np.where(empty, 0.0, e / np.where(empty, 1.0, l))
    o = p @ v
    lse = np.where(empty[:, 0], -np.inf, m_safe[:, 0] + np.log(np.where(empty[:, 0], 1.0, l[:, 0])))
    return o, lse, p


def head_backward(q, k, v, do, scale, mask):
    """Gradients (dQ, dK, dV) of sum(O * dO) for one head pair, textbook Jacobian.

    dV = P^T dO; dP = dO V^T; Delta_i = sum_j P_ij dP_ij; dS = P (dP - Delta);
    dQ = scale dS K; dK = scale dS^T Q.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    do = np.asarray(do, dtype=np.float64)
    _, _, p = head_forward(q, k, v, scale, mask)
    dv = p.T @ do
    dp = do @ v.T
    delta = (p * dp).sum(axis=1, keepdims=True)
    ds = p * (dp - delta)
    dq = scale * (ds @ k)
    dk = scale * (ds.T @ q)
    return dq, dk, dv


def _check_heads(hq: int, hkv: int) -> int:
    if hq % hkv != 0:
        raise ValueError("number of query heads must be divisible by number of KV heads")
    return hq // hkv


def mha_forward(q, k, v, scale, causal, window=(-1, -1)):
    """Dense batched attention.

    q (B, Sq, Hq, D), k/v (B, Sk, Hkv, D) -> O (B, Sq, Hq, D), LSE (B, Hq, Sq).
    """
    B, Sq, Hq, D = q.shape
    _, Sk, Hkv, _ = k.shape
    _check_heads(Hq, Hkv)
    mask = allowed_mask(Sq, Sk, causal, window)
    o = np.zeros(q.shape[:3] + (v.shape[3],), dtype=np.float64)
    lse = np.zeros((B, Hq, Sq), dtype=np.float64)
    for b in range(B):
        for h in range(Hq):
            hk = kv_head_of(h, Hq, Hkv)
            o[b, :, h, :], lse[b, h, :], _ = head_forward(q[b, :, h, :], k[b, :, hk, :], v[b, :, hk, :], scale, mask)
    return o, lse


def mha_backward(q, k, v, do, scale, causal, window=(-1, -1)):
    """Dense batched backward: returns dQ (like q), dK, dV (like k, v).

    With GQA the gradients of a KV head are the sums over the query heads
    that read it (README, ``flash_attn_func``: GQA mapping).
    """
    B, Sq, Hq, D = q.shape
    _, Sk, Hkv, _ = k.shape
    _check_heads(Hq, Hkv)
    mask = allowed_mask(Sq, Sk, causal, window)
    dq = np.zeros(q.shape, dtype=np.float64)
    dk = np.zeros(k.shape, dtype=np.float64)
    dv = np.zeros(v.shape, dtype=np.float64)
    for b in range(B):
        for h in range(Hq):
            hk = kv_head_of(h, Hq, Hkv)
            gq, gk, gv = head_backward(q[b, :, h, :], k[b, :, hk, :], v[b, :, hk, :], do[b, :, h, :], scale, mask)
            dq[b, :, h, :] = gq
            dk[b, :, hk, :] += gk
            dv[b, :, hk, :] += gv
    return dq, dk, dv


def _spans(cu):
    cu = np.asarray(cu, dtype=np.int64)
    return [(int(cu[s]), int(cu[s + 1])) for s in range(len(cu) - 1)]


def varlen_forward(q, k, v, cu_q, cu_k, scale, causal, window=(-1, -1)):
    """Packed variable-length batch.

    q (total_q, Hq, D), k/v (total_k, Hkv, D); sequence s spans rows
    cu_q[s]..cu_q[s+1]-1 of q and cu_k[s]..cu_k[s+1]-1 of k/v.
    Returns O (total_q, Hq, D) and LSE (Hq, total_q).
    """
    total_q, Hq, D = q.shape
    Hkv = k.shape[1]
    _check_heads(Hq, Hkv)
    o = np.zeros((total_q, Hq, v.shape[2]), dtype=np.float64)
    lse = np.zeros((Hq, total_q), dtype=np.float64)
    for (q0, q1), (k0, k1) in zip(_spans(cu_q), _spans(cu_k)):
        mask = allowed_mask(q1 - q0, k1 - k0, causal, window)
        for h in range(Hq):
            hk = kv_head_of(h, Hq, Hkv)
            oo, ll, _ = head_forward(q[q0:q1, h, :], k[k0:k1, hk, :], v[k0:k1, hk, :], scale, mask)
            o[q0:q1, h, :] = oo
            lse[h, q0:q1] = ll
    return o, lse


def varlen_backward(q, k, v, do, cu_q, cu_k, scale, causal, window=(-1, -1)):
    """Backward of :func:`varlen_forward`; returns dQ, dK, dV in the packed layouts."""
    total_q, Hq, D = q.shape
    Hkv = k.shape[1]
    _check_heads(Hq, Hkv)
    dq = np.zeros(q.shape, dtype=np.float64)
    dk = np.zeros(k.shape, dtype=np.float64)
    dv = np.zeros(v.shape, dtype=np.float64)
    for (q0, q1), (k0, k1) in zip(_spans(cu_q), _spans(cu_k)):
        mask = allowed_mask(q1 - q0, k1 - k0, causal, window)
        for h in range(Hq):
            hk = kv_head_of(h, Hq, Hkv)
            gq, gk, gv = head_backward(q[q0:q1, h, :], k[k0:k1, hk, :], v[k0:k1, hk, :], do[q0:q1, h, :], scale, mask)
            dq[q0:q1, h, :] = gq
            dk[k0:k1, hk, :] += gk
            dv[k0:k1, hk, :] += gv
    return dq, dk, dv


def kvcache_forward(q, k_cache, v_cache, cache_seqlens, scale, causal, rows=None, window=(-1, -1)):
    """Attention of new queries against a contiguous KV cache.

    README, ``flash_attn_with_kvcache`` docstring: q (B, Sq, Hq, D); caches
    (B, capacity, Hkv, D); batch row b uses keys 0 .. cache_seqlens[b]-1; the
    causal mask (if any) is bottom-right aligned.  Returns O (B, Sq, Hq, D) and
    LSE (B, Hq, Sq).  ``rows`` optionally restricts the work to a list of
    (b, h) pairs (other entries are left as NaN) so that large caches can be
    sampled.
    """
    B, Sq, Hq, D = q.shape
    Hkv = k_cache.shape[2]
    _check_heads(Hq, Hkv)
    o = np.full((B, Sq, Hq, v_cache.shape[3]), np.nan)
    lse = np.full((B, Hq, Sq), np.nan)
    pairs = rows if rows is not None else [(b, h) for b in range(B) for h in range(Hq)]
    for b, h in pairs:
        L = int(cache_seqlens[b])
        hk = kv_head_of(h, Hq, Hkv)
        kk = np.asarray(k_cache[b, :L, hk, :], dtype=np.float64)
        vv = np.asarray(v_cache[b, :L, hk, :], dtype=np.float64)
        mask = allowed_mask(Sq, L, causal, window)
        oo, ll, _ = head_forward(q[b, :, h, :], kk, vv, scale, mask)
        o[b, :, h, :] = oo
        lse[b, h, :] = ll
    return o, lse


def logical_cache_rows(cache, b, n, cache_batch_idx=None, block_table=None):
    """(block, row) address of logical cache rows 0..n-1 of sequence b, and the rows themselves.

    README, ``flash_attn_with_kvcache`` docstring: without a block table the
    cache is (batch_size_cache, seqlen_cache, nheads_k, headdim) and sequence b
    reads batch row cache_batch_idx[b] (b itself when no index is given); with a
    block table the cache is (num_blocks, page_block_size, nheads_k, headdim).
    Reading where the docstring stops: block_table[b, i] is the physical block
    that holds logical rows i * page_block_size .. (i + 1) * page_block_size - 1
    of sequence b, so logical row p sits at (block_table[b, p // page], p % page).
    """
    if block_table is not None:
        page = cache.shape[1]
        addr = [(int(block_table[b][p // page]), p % page) for p in range(n)]
    else:
        bc = b if cache_batch_idx is None else int(cache_batch_idx[b])
        addr = [(bc, p) for p in range(n)]
    rows = np.stack([np.asarray(cache[blk, r], dtype=np.float64) for blk, r in addr]) if n > 0 else \
        np.zeros((0,) + tuple(cache.shape[2:]), dtype=np.float64)
    return addr, rows


def kvcache_update_forward(q, k_cache, v_cache, cache_seqlens, scale, causal, window=(-1, -1), k_new=None,
                           v_new=None, cache_batch_idx=None, block_table=None):
    """The full flash_attn_with_kvcache computation (README docstring), without rotary embedding.

    1. If k_new / v_new (B, seqlen_new, nheads_k, headdim) are given, they are
       written into the caches at logical rows cache_seqlens[b] ..
       cache_seqlens[b] + seqlen_new - 1 of sequence b ("k is concatenated with
       k_cache starting at the indices specified by cache_seqlens"; the caches
       are updated in place, here in copies that are returned).
    2. Sequence b then attends to its first cache_seqlens[b] + seqlen_new
       logical rows (addressing: :func:`logical_cache_rows`).
    3. Attention by the definition, with the bottom-right aligned causal mask
       and sliding window of :func:`allowed_mask`.
    Returns O (B, Sq, Hq, headdim), LSE (B, Hq, Sq), k_cache_after, v_cache_after.
    """
    B, Sq, Hq, D = q.shape
    Hkv = k_cache.shape[2]
    _check_heads(Hq, Hkv)
    k_after = np.array(k_cache, dtype=np.float64, copy=True)
    v_after = np.array(v_cache, dtype=np.float64, copy=True)
    sn = 0 if k_new is None else k_new.shape[1]
    for b in range(B):
        start = int(cache_seqlens[b])
        addr, _ = logical_cache_rows(k_after, b, start + sn, cache_batch_idx, block_table)
        for s in range(sn):
            blk, r = addr[start + s]
            k_after[blk, r] = k_new[b, s]
            v_after[blk, r] = v_new[b, s]
    o = np.zeros((B, Sq, Hq, v_cache.shape[3]), dtype=np.float64)
    lse = np.zeros((B, Hq, Sq), dtype=np.float64)
    for b in range(B):
        L = int(cache_seqlens[b]) + sn
        _, kk = logical_cache_rows(k_after, b, L, cache_batch_idx, block_table)
        _, vv = logical_cache_rows(v_after, b, L, cache_batch_idx, block_table)
        mask = allowed_mask(Sq, L, causal, window)
        for h in range(Hq):
            hk = kv_head_of(h, Hq, Hkv)
            o[b, :, h, :], lse[b, h, :], _ = head_forward(q[b, :, h, :], kk[:, hk, :], vv[:, hk, :], scale, mask)
    return o, lse, k_after, v_after


def merge_lse_partials(lse_parts, o_parts):
    """Merge attention results computed over disjoint key sets.

    For key blocks c with normalised outputs O_c and log-sum-exps LSE_c, the
    attention over the union is O = sum_c exp(LSE_c - LSE) O_c with
    LSE = log sum_c exp(LSE_c).  This is the algebra behind splitting the
    KV-cache load across thread blocks and combining the pieces in a separate
    step (README changelog 2.2); it follows from the definition of softmax.
    lse_parts (C, ...) and o_parts (C, ..., Dv).  Blocks with LSE = -inf are empty.
    """
    lse_parts = np.asarray(lse_parts, dtype=np.float64)
    o_parts = np.asarray(o_parts, dtype=np.float64)
    m = lse_parts.max(axis=0)
    m_safe = np.where(np.isfinite(m), m, 0.0)
    w = np.exp(lse_parts - m_safe)
    tot = w.sum(axis=0)
    lse = np.where(tot > 0, m_safe + np.log(np.where(tot > 0, tot, 1.0)), -np.inf)
    wn = np.where(tot > 0, w / np.where(tot > 0, tot, 1.0), 0.0)
    o = (wn[..., None] * o_parts).sum(axis=0)
    return o, lse
