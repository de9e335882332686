"""fa_fwd_kvcache_noalloc: KV-cache decode for callers that cannot allocate device
memory when they decode (code inside a CUDA-graph capture that must not grow a
memory pool, plugins or runtimes that only receive the tensors they own).  Its
partial results live in a fixed array inside the library instead of a caller
workspace; the results must match fa_fwd_kvcache's, here on two calls in a row
with different inputs, so leftovers of the first call cannot leak into the second.

This file is named to be collected last: a run that stops at the first failure
has then already run every other test.
"""

import pytest
import torch

from exact_tiled_attention_41_b200 import abi, workloads as W
from tests import gpu_helpers as H

pytestmark = pytest.mark.gpu

FAKE = 0x10000


def _reference(t, B, Hq, Hkv, cap, D, scale):
    out = torch.empty_like(t["q"])
    lse = torch.empty((B, Hq, 1), dtype=torch.float32, device="cuda")
    nb = abi.fa_fwd_kvcache_workspace_size(B, Hq, Hkv, 1, cap, D, 0)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    assert abi.fa_fwd_kvcache(t["q"], t["k_cache"], t["v_cache"], t["cache_seqlens"], out, lse, B, Hq, Hkv, 1, cap,
                              D, scale, 0, 0, ws, nb) == 0
    return out, lse


@pytest.mark.parametrize("D", [128, 64])
def test_noalloc_matches_workspace_entry_point_on_two_calls(D):
    B, Hq, Hkv, cap = 6, 32, 8, 4096
    for call, (seed, lengths) in enumerate(((31, [1, 64, 65, 1000, 4096, 2500]), (32, [4096, 3, 777, 128, 0, 2049]))):
        w = W.kvcache(B, Hq, Hkv, D, cap, 0, 0, seed=seed + D, lengths=lengths)
        t = {n: x.cuda() for n, x in w.tensors.items()}
        ref_out, ref_lse = _reference(t, B, Hq, Hkv, cap, D, w.scale)
        out = torch.full_like(t["q"], float("nan"))
        lse = torch.full((B, Hq, 1), float("nan"), dtype=torch.float32, device="cuda")
        st = abi.fa_fwd_kvcache_noalloc(t["q"], t["k_cache"], t["v_cache"], t["cache_seqlens"], out, lse, B, Hq, Hkv,
                                        1, cap, D, w.scale, 0, 0)
        assert st == 0, abi.status_string(st)
        torch.cuda.synchronize()
        assert abi.fa_get_device_status() == 0
        H.check_o(out, H.f64(ref_out))
        H.check_lse(lse, H.f64(ref_lse))


def test_noalloc_rejects_partials_beyond_the_fixed_array():
    cap_bytes = abi.fa_fwd_kvcache_noalloc_scratch_bytes()
    assert cap_bytes == 16 << 20
    # one split per row already needs B * Hq * (D + 1) * 4 bytes > 16 MiB
    st = abi.fa_fwd_kvcache_noalloc(FAKE, FAKE, FAKE, FAKE, FAKE, None, 1024, 32, 8, 1, 4096, 128, 0.1, 0, 0, 0)
    assert st == abi.FA_ERR_WORKSPACE
    # an explicit split count whose partials do not fit is refused rather than coarsened
    st = abi.fa_fwd_kvcache_noalloc(FAKE, FAKE, FAKE, FAKE, FAKE, None, 64, 32, 8, 1, 16384, 128, 0.1, 0, 256, 0)
    assert st == abi.FA_ERR_WORKSPACE
