"""GPU parity of the full KV-cache call (flash-attention README, flash_attn_with_kvcache docstring)
against the fp64 oracle: several new query tokens with the bottom-right causal mask and sliding
windows, k / v appended in place at cache_seqlens, paged caches through a block table (pages of
256 keys), and cache_batch_idx.  Cache rows nobody may read hold NaN."""

import numpy as np
import pytest
import torch

import oracle
from exact_tiled_attention_41_b200 import abi, attention as A, workloads as W
from tests import gpu_helpers as H

pytestmark = pytest.mark.gpu


def run_and_check(w, causal, window=(-1, -1), num_splits=0):
    t = w.tensors
    dev = {n: x.cuda() for n, x in t.items()}
    out, lse = A.flash_attn_with_kvcache(dev["q"], dev["k_cache"], dev["v_cache"], dev["cache_seqlens"], w.scale,
                                         causal, num_splits, True, dev.get("k_new"), dev.get("v_new"),
                                         dev.get("cache_batch_idx"), dev.get("block_table"), window)
    torch.cuda.synchronize()
    assert abi.fa_get_device_status() == 0
    f = H.f64
    o_ref, l_ref, k_after, v_after = oracle.kvcache_update_forward(
        f(t["q"]), f(t["k_cache"]), f(t["v_cache"]), t["cache_seqlens"].numpy(), w.scale, causal, window,
        f(t["k_new"]) if "k_new" in t else None, f(t["v_new"]) if "v_new" in t else None,
        t["cache_batch_idx"].numpy() if "cache_batch_idx" in t else None,
        t["block_table"].numpy() if "block_table" in t else None)
    H.check_o(out, o_ref)
    H.check_lse(lse, l_ref)
    # the caches after the call: appended rows written exactly, every other row untouched (NaN stays NaN)
    for name, after in (("k_cache", k_after), ("v_cache", v_after)):
        got = f(dev[name])
        np.testing.assert_array_equal(np.isnan(got), np.isnan(after))
        fin = ~np.isnan(after)
        np.testing.assert_array_equal(got[fin], after[fin])
    return out, lse


@pytest.mark.parametrize("D", [64, 128, 256])
@pytest.mark.parametrize("Sq", [2, 5, 16])
def test_multi_query_causal(D, Sq):
    lens = [Sq, 63, 64, 65, 700, 1023]
    w = W.kvcache_update(len(lens), Sq, 8, 2, D, 1024, lens, seed=Sq + D)
    run_and_check(w, True)
    run_and_check(w, False)


@pytest.mark.parametrize("num_splits", [0, 1, 5])
def test_append_then_attend(num_splits):
    lens = [0, 1, 250, 777]
    w = W.kvcache_update(len(lens), 3, 8, 2, 128, 1024, lens, seqlen_new=3, seed=40 + num_splits)
    run_and_check(w, True, num_splits=num_splits)


@pytest.mark.parametrize("D", [64, 128, 256])
def test_paged_cache_with_append(D):
    lens = [0, 255, 256, 257, 900, 1400]
    w = W.kvcache_update(len(lens), 4, 8, 2, D, 1536, lens, seqlen_new=4, page=256, seed=50 + D)
    run_and_check(w, True)


def test_paged_cache_single_query():
    lens = [1, 511, 512, 1000]
    run_and_check(W.kvcache_update(4, 1, 16, 4, 128, 1024, lens, page=256, seed=60), False)


def test_cache_batch_index():
    lens = [300, 5, 1022]
    w = W.kvcache_update(3, 2, 4, 4, 128, 1024, lens, seqlen_new=2, seed=70, cache_batch_idx=[4, 0, 2],
                         cache_batch=5)
    run_and_check(w, True)


@pytest.mark.parametrize("window", [(100, 0), (0, 0), (300, -1), (64, 3)])
def test_windows(window):
    lens = [10, 400, 1000]
    w = W.kvcache_update(3, 6, 8, 1, 128, 1024, lens, seqlen_new=2, seed=80 + window[0])
    run_and_check(w, False, window)
    run_and_check(w, True, window)          # causal and window together: the keys both keep


def test_large_group_and_many_tokens():
    # 32 query heads over 2 KV heads with 3 tokens: 48 rows per KV head, three blocks of 16
    lens = [70, 600]
    w = W.kvcache_update(2, 3, 32, 2, 128, 1024, lens, seed=90)
    run_and_check(w, True)


def test_bad_block_id_is_reported_not_read():
    lens = [300]
    w = W.kvcache_update(1, 1, 4, 1, 128, 512, lens, page=256, seed=91, spare_blocks=0)
    t = {n: x.cuda() for n, x in w.tensors.items()}
    t["block_table"][0, 1] = 1 << 20           # a block far outside the cache
    out, _ = A.flash_attn_with_kvcache(t["q"], t["k_cache"], t["v_cache"], t["cache_seqlens"], w.scale, False, 0,
                                       True, block_table=t["block_table"])
    torch.cuda.synchronize()
    assert abi.fa_get_device_status() == abi.FA_ERR_INVALID_ARG
    assert abi.fa_get_device_status() == 0


@pytest.mark.parametrize("num_splits", [0, 1, 3])
def test_head_dim_256_single_token(num_splits):
    # README: head dims up to 256; NaN guards in every cache row past the lengths
    lens = [1, 63, 64, 65, 1000, 2047, 0]
    w = W.kvcache_update(len(lens), 1, 16, 4, 256, 2048, lens, seed=100 + num_splits)
    run_and_check(w, False, num_splits=num_splits)


def test_head_dim_256_paged_single_token():
    lens = [1, 511, 512, 1000]
    run_and_check(W.kvcache_update(4, 1, 8, 2, 256, 1024, lens, page=256, seed=110), False)
