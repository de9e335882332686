"""CPU checks of the C-ABI boundary: the library loads, exports every symbol the
header declares, and rejects bad arguments before touching the GPU."""

import os
import re

import pytest

from exact_tiled_attention_41_b200 import abi
from tests.conftest import ROOT

HEADER = os.path.join(ROOT, "include", "fa.h")
FAKE = 0x10000        # a 16-byte aligned address that is never dereferenced (validation fails first)
S0 = 0                # default stream handle


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^FA_API\s+[\w\s\*]+?\b(fa_\w+)\s*\(", text, flags=re.M)))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(abi.LIB_PATH):
        from exact_tiled_attention_41_b200 import build
        build.build()
    return abi.load()


def test_header_declares_the_five_entry_points():
    syms = declared_symbols()
    for name in ("fa_fwd", "fa_bwd", "fa_varlen_fwd", "fa_varlen_bwd", "fa_fwd_kvcache"):
        assert name in syms


def test_library_exports_every_declared_symbol(lib):
    syms = declared_symbols()
    assert len(syms) >= 15
    for name in syms:
        assert hasattr(lib, name), name
    assert set(syms) == set(abi.EXPORTS)


def test_status_strings(lib):
    assert abi.status_string(0) == "ok"
    assert "timed out" in abi.status_string(abi.FA_ERR_TIMEOUT)
    assert abi.status_string(99) == "unknown status"


def _fwd(**kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, out=FAKE, lse=FAKE, B=1, Hq=4, Hkv=2, Sq=128, Sk=128, D=128,
             softmax_scale=0.1, causal=1, stream=S0)
    a.update(kw)
    return abi.fa_fwd(**a)


@pytest.mark.parametrize("kw,want", [
    (dict(q=None), abi.FA_ERR_INVALID_ARG),
    (dict(out=None), abi.FA_ERR_INVALID_ARG),
    (dict(lse=None), abi.FA_ERR_INVALID_ARG),
    (dict(B=0), abi.FA_ERR_INVALID_ARG),
    (dict(Sq=0), abi.FA_ERR_INVALID_ARG),
    (dict(Sk=-1), abi.FA_ERR_INVALID_ARG),
    (dict(Hq=3, Hkv=2), abi.FA_ERR_INVALID_ARG),        # README: Hq must be divisible by Hkv
    (dict(softmax_scale=0.0), abi.FA_ERR_INVALID_ARG),
    (dict(softmax_scale=float("nan")), abi.FA_ERR_INVALID_ARG),
    (dict(D=96), abi.FA_ERR_UNSUPPORTED),
    (dict(D=512), abi.FA_ERR_UNSUPPORTED),                # README: head dims up to 256
    (dict(q=FAKE + 8), abi.FA_ERR_ALIGNMENT),
    (dict(out=FAKE + 2), abi.FA_ERR_ALIGNMENT),
])
def test_fwd_rejects_bad_arguments(lib, kw, want):
    assert _fwd(**kw) == want


def test_bwd_checks_workspace_before_launch(lib):
    need = abi.fa_bwd_workspace_size(2, 4, 2, 300, 300, 128)
    assert need >= 2 * 300 * 4 * 128 * 4       # fp32 dq accumulator at least
    st = abi.fa_bwd(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 2, 4, 2, 300, 300, 128, 0.1, 1,
                    FAKE, need - 1, S0)
    assert st == abi.FA_ERR_WORKSPACE
    st = abi.fa_bwd(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 2, 4, 2, 300, 300, 128, 0.1, 1,
                    FAKE + 16, need, S0)
    assert st == abi.FA_ERR_ALIGNMENT          # workspace must be 256-byte aligned
    st = abi.fa_bwd(FAKE, FAKE, FAKE, FAKE, None, FAKE, FAKE, FAKE, FAKE, 2, 4, 2, 300, 300, 128, 0.1, 1,
                    FAKE, need, S0)
    assert st == abi.FA_ERR_INVALID_ARG


def test_ex_entry_points_validate_like_the_plain_calls(lib):
    # window sides and the deterministic flag never make a bad call valid
    st = abi.fa_fwd_ex(None, FAKE, FAKE, FAKE, FAKE, 1, 4, 2, 128, 128, 128, 0.1, 1, 64, -1, stream=S0)
    assert st == abi.FA_ERR_INVALID_ARG
    st = abi.fa_fwd_ex(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 3, 2, 128, 128, 128, 0.1, 0, 5, 5, stream=S0)
    assert st == abi.FA_ERR_INVALID_ARG
    st = abi.fa_fwd_ex(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 4, 2, (1 << 30) + 1, 128, 128, 0.1, 0, -1, -1, stream=S0)
    assert st == abi.FA_ERR_UNSUPPORTED          # sequences are limited to 2^30 tokens
    need = abi.fa_bwd_workspace_size(2, 4, 2, 300, 300, 128)
    for det in (0, 1):
        st = abi.fa_bwd_ex(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 2, 4, 2, 300, 300, 128, 0.1, 1,
                           32, -1, det, FAKE, need - 1, S0)
        assert st == abi.FA_ERR_WORKSPACE
    st = abi.fa_varlen_fwd_ex(FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, 2, 10, 10, 20, 20, 2, 2, 64, 0.1, 1, 4, 0,
                              stream=S0)
    assert st == abi.FA_ERR_INVALID_ARG
    nv = abi.fa_varlen_bwd_workspace_size(2, 20, 20, 2, 2, 64)
    st = abi.fa_varlen_bwd_ex(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 2, 10, 10, 20, 20,
                              2, 2, 64, 0.1, 1, 4, 0, 1, FAKE + 16, nv, S0)
    assert st == abi.FA_ERR_ALIGNMENT


def test_varlen_rejects_missing_cu_seqlens(lib):
    st = abi.fa_varlen_fwd(FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, 2, 10, 10, 20, 20, 2, 2, 64, 0.1, 1, stream=S0)
    assert st == abi.FA_ERR_INVALID_ARG
    st = abi.fa_varlen_fwd(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE + 2, 2, 10, 10, 20, 20, 2, 2, 64, 0.1, 1, stream=S0)
    assert st == abi.FA_ERR_ALIGNMENT
    assert abi.fa_varlen_fwd_workspace_size(2, 20, 20, 2, 2, 64) == 256
    assert abi.fa_varlen_bwd_workspace_size(2, 20, 20, 2, 2, 64) > 0


def test_forward_workspace_is_optional_but_checked(lib):
    # 256 bytes for the dynamic schedule's unit counter; NULL selects the static schedule, and a given
    # workspace must follow the usual rules (size, 256-byte alignment) -- checked before any launch
    assert abi.fa_fwd_workspace_size(2, 4, 2, 100, 100, 64) == 256
    args = (FAKE, FAKE, FAKE, FAKE, FAKE, 2, 4, 2, 100, 100, 64, 0.1, 1)
    assert abi.fa_fwd(*args, FAKE, 255, S0) == abi.FA_ERR_WORKSPACE
    assert abi.fa_fwd(*args, FAKE + 16, 256, S0) == abi.FA_ERR_ALIGNMENT
    vargs = (FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 2, 10, 10, 20, 20, 2, 2, 64, 0.1, 1)
    assert abi.fa_varlen_fwd(*vargs, FAKE, 100, S0) == abi.FA_ERR_WORKSPACE


def test_kvcache_argument_rules(lib):
    need = abi.fa_fwd_kvcache_workspace_size(64, 32, 8, 1, 16384, 128, 0)
    assert need > 0
    args = [FAKE, FAKE, FAKE, FAKE, FAKE, None, 64, 32, 8, 1, 16384, 128, 0.1, 0, 0, FAKE, need, S0]
    bad_sq = list(args)
    bad_sq[9] = 0                                 # at least one query token per row
    assert abi.fa_fwd_kvcache(*bad_sq) == abi.FA_ERR_INVALID_ARG
    small = list(args)
    small[16] = need - 1
    assert abi.fa_fwd_kvcache(*small) == abi.FA_ERR_WORKSPACE
    no_seqlens = list(args)
    no_seqlens[3] = None
    assert abi.fa_fwd_kvcache(*no_seqlens) == abi.FA_ERR_INVALID_ARG
    # more splits need more partial storage
    assert abi.fa_fwd_kvcache_workspace_size(64, 32, 8, 1, 16384, 128, 64) > abi.fa_fwd_kvcache_workspace_size(
        64, 32, 8, 1, 16384, 128, 4)


def _kv_ex(**kw):
    a = dict(q=FAKE, k_cache=FAKE, v_cache=FAKE, cache_seqlens=FAKE, k_new=None, v_new=None, seqlen_new=0,
             cache_batch_idx=None, block_table=None, max_blocks_per_seq=0, cache_batch=8, cache_capacity=1024,
             out=FAKE, lse=None, B=8, Hq=16, Hkv=4, Sq=3, D=128, softmax_scale=0.1, causal=1, window_left=-1,
             window_right=-1, num_splits=0, workspace=FAKE, workspace_bytes=1 << 40, stream=S0)
    a.update(kw)
    return abi.fa_fwd_kvcache_ex(**a)


@pytest.mark.parametrize("kw,want", [
    (dict(k_new=FAKE), abi.FA_ERR_INVALID_ARG),                                  # k without v
    (dict(k_new=FAKE, v_new=FAKE), abi.FA_ERR_INVALID_ARG),                      # new keys but seqlen_new = 0
    (dict(seqlen_new=2), abi.FA_ERR_INVALID_ARG),                                # seqlen_new without k / v
    (dict(block_table=FAKE, max_blocks_per_seq=4, cache_capacity=100), abi.FA_ERR_INVALID_ARG),  # page % 256
    (dict(block_table=FAKE, max_blocks_per_seq=0, cache_capacity=256), abi.FA_ERR_INVALID_ARG),
    (dict(block_table=FAKE, max_blocks_per_seq=4, cache_capacity=256, cache_batch_idx=FAKE), abi.FA_ERR_INVALID_ARG),
    (dict(cache_batch=0), abi.FA_ERR_INVALID_ARG),
    (dict(D=512), abi.FA_ERR_UNSUPPORTED),
    (dict(workspace_bytes=0), abi.FA_ERR_WORKSPACE),
    (dict(block_table=FAKE + 2, max_blocks_per_seq=4, cache_capacity=256), abi.FA_ERR_ALIGNMENT),
])
def test_kvcache_ex_argument_rules(lib, kw, want):
    assert _kv_ex(**kw) == want


def test_kvcache_ex_workspace_sizes(lib):
    one = abi.fa_fwd_kvcache_ex_workspace_size(8, 16, 4, 1, 128, 4096, 0, 0)
    four = abi.fa_fwd_kvcache_ex_workspace_size(8, 16, 4, 4, 128, 4096, 0, 0)
    assert 0 < one < four                         # partials per query row
    paged = abi.fa_fwd_kvcache_ex_workspace_size(8, 16, 4, 1, 128, 256, 16, 0)
    assert paged == abi.fa_fwd_kvcache_ex_workspace_size(8, 16, 4, 1, 128, 4096, 0, 0)   # 16 pages of 256 keys
    assert abi.fa_fwd_kvcache_ex_workspace_size(8, 16, 4, 1, 128, 100, 16, 0) == 0         # bad page size
    assert abi.fa_fwd_kvcache_workspace_size(8, 16, 4, 1, 4096, 128, 0) == one


def test_product_path_has_no_oracle_or_cpu_fallback():
    pkg = os.path.join(ROOT, "exact_tiled_attention_41_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in text and "from oracle" not in text, f


def test_merge_lse_argument_rules(lib):
    ok = dict(o_parts=FAKE, lse_parts=FAKE, num_parts=2, B=1, S=8, H=2, D=128, parts_fp32=0, out=FAKE, lse=None,
              out_fp32=0, stream=S0)
    for kw, want in ((dict(o_parts=None), abi.FA_ERR_INVALID_ARG), (dict(num_parts=0), abi.FA_ERR_INVALID_ARG),
                     (dict(D=96), abi.FA_ERR_UNSUPPORTED), (dict(out=FAKE + 4), abi.FA_ERR_ALIGNMENT)):
        a = dict(ok)
        a.update(kw)
        assert abi.fa_merge_lse(**a) == want
