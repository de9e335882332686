"""fa_fwd_kvcache_noalloc: KV-cache decode for callers that cannot allocate device
memory when they decode (plugins or runtimes that plan their device memory ahead of
time and only receive the tensors they own, C programs without an allocator).  Its
partial results live in a fixed array inside the library instead of a caller
workspace.  Where it uses the same split as fa_fwd_kvcache the results must be
bit-identical to that entry point's, here on two calls in a row with different
inputs, so leftovers of the first call cannot leak into the second; where the fixed
array forces a coarser split the result must match fa_fwd_kvcache run with that
split, and the fp64 oracle within the stated tolerances.

This file is named to be collected last: a run that stops at the first failure
has then already run every other test.
"""

import numpy as np
import pytest
import torch

import oracle
from exact_tiled_attention_41_b200 import abi, workloads as W
from tests import gpu_helpers as H

pytestmark = pytest.mark.gpu

FAKE = 0x10000


def _reference(t, B, Hq, Hkv, cap, D, scale, num_splits=0, Sq=1, causal=0):
    out = torch.empty_like(t["q"])
    lse = torch.empty((B, Hq, Sq), dtype=torch.float32, device="cuda")
    nb = abi.fa_fwd_kvcache_workspace_size(B, Hq, Hkv, Sq, cap, D, num_splits)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    assert abi.fa_fwd_kvcache(t["q"], t["k_cache"], t["v_cache"], t["cache_seqlens"], out, lse, B, Hq, Hkv, Sq, cap,
                              D, scale, causal, num_splits, ws, nb) == 0
    return out, lse


def _noalloc(t, B, Hq, Hkv, cap, D, scale, Sq=1, causal=0):
    out = torch.full_like(t["q"], float("nan"))
    lse = torch.full((B, Hq, Sq), float("nan"), dtype=torch.float32, device="cuda")
    st = abi.fa_fwd_kvcache_noalloc(t["q"], t["k_cache"], t["v_cache"], t["cache_seqlens"], out, lse, B, Hq, Hkv,
                                    Sq, cap, D, scale, causal, 0)
    assert st == 0, abi.status_string(st)
    torch.cuda.synchronize()
    assert abi.fa_get_device_status() == 0
    return out, lse


@pytest.mark.parametrize("D", [128, 64])
def test_noalloc_matches_workspace_entry_point_on_two_calls(D):
    B, Hq, Hkv, cap = 6, 32, 8, 4096
    for call, (seed, lengths) in enumerate(((31, [1, 64, 65, 1000, 4096, 2500]), (32, [4096, 3, 777, 128, 0, 2049]))):
        w = W.kvcache(B, Hq, Hkv, D, cap, 0, 0, seed=seed + D, lengths=lengths)
        t = {n: x.cuda() for n, x in w.tensors.items()}
        ref_out, ref_lse = _reference(t, B, Hq, Hkv, cap, D, w.scale)
        out, lse = _noalloc(t, B, Hq, Hkv, cap, D, w.scale)
        # same split, same kernels: the same bits (an empty row gives 0 / -inf in both)
        assert torch.equal(out, ref_out), f"call {call}: output differs from fa_fwd_kvcache"
        assert torch.equal(lse, ref_lse), f"call {call}: LSE differs from fa_fwd_kvcache"


def _partial_bytes(B, Hkv, rows, D, cap, n):
    # the partials of n splits: the split length is ceil(cap / n) rounded up to 64 keys
    chunk = -(-(-(-cap // n)) // 64) * 64
    chunks = -(-cap // chunk)
    r = B * Hkv * chunks * rows
    return (r * D * 4 + 255) // 256 * 256 + r * 4


def test_noalloc_coarsens_the_split_until_the_partials_fit():
    # 64 rows x 8 KV heads x 16 query rows (4 heads per KV head x 4 causal tokens), capacity 4096: four
    # splits of 1024 keys need 16.9 MB of partials > 16 MiB, three splits of 1408 keys 12.7 MB, so the call
    # runs the split fa_fwd_kvcache takes with num_splits = 3 (the automatic split has more than three)
    B, Hq, Hkv, D, cap, Sq = 64, 32, 8, 128, 4096, 4
    limit = abi.fa_fwd_kvcache_noalloc_scratch_bytes()
    n_fit = max(n for n in range(1, 9) if _partial_bytes(B, Hkv, Sq * Hq // Hkv, D, cap, n) <= limit)
    assert n_fit == 3
    g = torch.Generator("cpu").manual_seed(40)
    lengths = torch.randint(Sq, 200, (B,), generator=g).tolist()
    lengths[3], lengths[17], lengths[40] = cap, 2049, 2048
    w = W.kvcache(B, Hq, Hkv, D, cap, 0, 0, seed=41, Sq=Sq, lengths=lengths)
    t = {n: x.cuda() for n, x in w.tensors.items()}
    for _ in range(2):
        out, lse = _noalloc(t, B, Hq, Hkv, cap, D, w.scale, Sq, 1)
        ref_out, ref_lse = _reference(t, B, Hq, Hkv, cap, D, w.scale, n_fit, Sq, 1)
        assert torch.equal(out, ref_out) and torch.equal(lse, ref_lse)
    # and against the fp64 oracle on the rows' valid keys (bottom-right causal tokens)
    L = max(lengths)
    tt = w.tensors
    o_ref, l_ref = oracle.kvcache_forward(H.f64(tt["q"]), H.f64(tt["k_cache"][:, :L]), H.f64(tt["v_cache"][:, :L]),
                                          tt["cache_seqlens"].numpy(), w.scale, True)
    H.check_o(out, o_ref)
    H.check_lse(lse, l_ref)
    assert np.isfinite(H.f64(out)).all()


def test_noalloc_rejects_partials_beyond_the_fixed_array():
    cap_bytes = abi.fa_fwd_kvcache_noalloc_scratch_bytes()
    assert cap_bytes == 16 << 20
    # one split per row already needs B * Hq * (D + 1) * 4 bytes > 16 MiB
    st = abi.fa_fwd_kvcache_noalloc(FAKE, FAKE, FAKE, FAKE, FAKE, None, 1024, 32, 8, 1, 4096, 128, 0.1, 0, 0, 0)
    assert st == abi.FA_ERR_WORKSPACE
    # an explicit split count whose partials do not fit is refused rather than coarsened
    st = abi.fa_fwd_kvcache_noalloc(FAKE, FAKE, FAKE, FAKE, FAKE, None, 64, 32, 8, 1, 16384, 128, 0.1, 0, 256, 0)
    assert st == abi.FA_ERR_WORKSPACE
