"""Plant plausible mistakes in the oracle (on the CPU) and check that its pins catch each one.

Every mutant below is a one-line slip somebody could make writing the oracle: a
dropped term, a wrong sign or index, a transposed operand, the wrong mask
alignment.  Each must make at least one pin in tests/test_oracle.py fail.
"""

import numpy as np
import pytest

import oracle
import oracle.attention as A
from tests import test_oracle as pins


def _mask_top_left(len_q, len_k, causal, window=(-1, -1)):
    i = np.arange(len_q)[:, None]
    j = np.arange(len_k)[None, :]
    return np.ones((len_q, len_k), bool) if not causal else (j <= i)


def _window_left_off_by_one(len_q, len_k, causal, window=(-1, -1)):
    # the left edge of the window taken one key too far
    left, right = window
    return _ORIG_MASK(len_q, len_k, causal, (left + 1 if left >= 0 else left, right))


def _window_top_left(len_q, len_k, causal, window=(-1, -1)):
    # the window anchored at the diagonal i = j instead of the bottom-right corner
    m = _ORIG_MASK(len_q, len_k, causal)
    i = np.arange(len_q)[:, None]
    j = np.arange(len_k)[None, :]
    left, right = window
    if left >= 0:
        m &= j >= i - left
    if right >= 0:
        m &= j <= i + right
    return m


def _gqa_modulo(h, hq, hkv):
    return h % hkv


def _fwd_no_scale(q, k, v, scale, mask):
    return _ORIG_FWD(q, k, v, 1.0, mask)


def _fwd_lse_without_max(q, k, v, scale, mask):
    o, lse, p = _ORIG_FWD(q, k, v, scale, mask)
    s = np.where(mask, scale * (np.asarray(q) @ np.asarray(k).T), -np.inf)
    m = s.max(axis=1, initial=-np.inf)
    return o, np.where(np.isfinite(m), lse - m, lse), p


def _bwd_drop_delta(q, k, v, do, scale, mask):
    _, _, p = _ORIG_FWD(q, k, v, scale, mask)
    dv = p.T @ do
    ds = p * (do @ v.T)
    return scale * (ds @ k), scale * (ds.T @ q), dv


def _bwd_sign_flip(q, k, v, do, scale, mask):
    dq, dk, dv = _ORIG_BWD(q, k, v, do, scale, mask)
    return -dq, dk, dv


def _bwd_transposed_dk(q, k, v, do, scale, mask):
    dq, dk, dv = _ORIG_BWD(q, k, v, do, scale, mask)
    _, _, p = _ORIG_FWD(q, k, v, scale, mask)
    dp = do @ v.T
    ds = p * (dp - (p * dp).sum(axis=1, keepdims=True))
    if ds.shape[0] == ds.shape[1]:
        dk = scale * (ds @ q)          # should be ds^T @ q
    return dq, dk, dv


def _bwd_dv_from_do_transposed(q, k, v, do, scale, mask):
    dq, dk, dv = _ORIG_BWD(q, k, v, do, scale, mask)
    _, _, p = _ORIG_FWD(q, k, v, scale, mask)
    if p.shape[0] == p.shape[1]:
        dv = p @ do                    # should be p^T @ do
    return dq, dk, dv


_ORIG_FWD = A.head_forward
_ORIG_MASK = A.allowed_mask
_ORIG_BWD = A.head_backward


def _fails(fn, *args, **kw):
    with pytest.raises(AssertionError):
        fn(*args, **kw)


def test_top_left_causal_mask_is_caught(monkeypatch):
    monkeypatch.setattr(A, "allowed_mask", _mask_top_left)
    monkeypatch.setattr(oracle, "allowed_mask", _mask_top_left)
    _fails(pins.test_causal_mask_matches_pages_q2_k5)


def test_modulo_gqa_mapping_is_caught(monkeypatch):
    monkeypatch.setattr(A, "kv_head_of", _gqa_modulo)
    monkeypatch.setattr(oracle, "kv_head_of", _gqa_modulo)
    _fails(pins.test_gqa_mapping_matches_pages)


def test_missing_scale_is_caught(monkeypatch):
    monkeypatch.setattr(A, "head_forward", _fwd_no_scale)
    _fails(pins.test_forward_matches_torch_sdpa, False, 16, 16, 2, 2)


def test_lse_missing_max_is_caught(monkeypatch):
    monkeypatch.setattr(A, "head_forward", _fwd_lse_without_max)
    monkeypatch.setattr(oracle, "head_forward", _fwd_lse_without_max)
    _fails(pins.test_lse_is_log_sum_exp_fsum)


@pytest.mark.parametrize("mutant", [_bwd_drop_delta, _bwd_sign_flip, _bwd_transposed_dk, _bwd_dv_from_do_transposed])
def test_backward_mutants_are_caught(monkeypatch, mutant):
    monkeypatch.setattr(A, "head_backward", mutant)
    _fails(pins.test_backward_matches_torch_autograd, False, 9, 9, 2, 2)


@pytest.mark.parametrize("mutant", [_window_left_off_by_one, _window_top_left])
def test_window_mask_mutants_are_caught(monkeypatch, mutant):
    monkeypatch.setattr(A, "allowed_mask", mutant)
    monkeypatch.setattr(oracle, "allowed_mask", mutant)
    caught = 0
    for args in (("window_mask_q4_k6_l1_r0.txt", 4, 6, (1, 0)), ("window_mask_q5_k3_l0_r1.txt", 5, 3, (0, 1)),
                 ("window_mask_q5_k5_l2_unbounded.txt", 5, 5, (2, -1))):
        try:
            pins.test_window_mask_matches_hand_derived_interval(*args)
        except AssertionError:
            caught += 1
    assert caught > 0
    _fails(pins.test_window_forward_matches_sliced_sdpa, 9, 14, (2, 1))


_ORIG_ROWS = A.logical_cache_rows


def _paged_rows_swapped(cache, b, n, cache_batch_idx=None, block_table=None):
    # page index and offset exchanged
    if block_table is None:
        return _ORIG_ROWS(cache, b, n, cache_batch_idx, block_table)
    page = cache.shape[1]
    addr = [(int(block_table[b][p % page]), p // page) for p in range(n)]
    rows = np.stack([np.asarray(cache[k, r], dtype=np.float64) for k, r in addr])
    return addr, rows


def _append_one_row_late(cache, b, n, cache_batch_idx=None, block_table=None):
    # every logical row addressed one row further on (kept inside the capacity)
    addr, _ = _ORIG_ROWS(cache, b, n, cache_batch_idx, block_table)
    addr = [(k, min(r + 1, cache.shape[1] - 1)) for k, r in addr]
    rows = np.stack([np.asarray(cache[k, r], dtype=np.float64) for k, r in addr]) if n > 0 else \
        np.zeros((0,) + tuple(cache.shape[2:]))
    return addr, rows


def test_paged_address_mutant_is_caught(monkeypatch):
    monkeypatch.setattr(A, "logical_cache_rows", _paged_rows_swapped)
    monkeypatch.setattr(oracle, "logical_cache_rows", _paged_rows_swapped)
    _fails(pins.test_paged_cache_address_matches_hand_derived_rows)


def test_append_offset_mutant_is_caught(monkeypatch):
    monkeypatch.setattr(A, "logical_cache_rows", _append_one_row_late)
    _fails(pins.test_kvcache_update_equals_dense_on_the_concatenation)
