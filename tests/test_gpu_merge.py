"""GPU parity of fa_merge_lse (attention over the union of disjoint key sets from the result over each
set: LSE = ln sum_c exp(LSE_c), O = sum_c exp(LSE_c - LSE) O_c) against the oracle's merge, and the
context-parallel use: attention over key shards, merged, equals attention over all keys."""

import numpy as np
import pytest
import torch

import oracle
from exact_tiled_attention_41_b200 import attention as A, workloads as W
from tests import gpu_helpers as H

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("D", [64, 128, 256])
@pytest.mark.parametrize("parts_fp32,out_fp32", [(False, False), (True, True), (True, False)])
def test_merge_matches_oracle(D, parts_fp32, out_fp32):
    g = torch.Generator("cpu").manual_seed(D)
    C, B, S, Hh = 3, 2, 37, 4
    o = torch.randn((C, B, S, Hh, D), generator=g)
    lse = torch.randn((C, B, Hh, S), generator=g) * 3
    lse[1, 0, 1, :5] = -float("inf")          # some empty parts
    lse[:, 1, 2, 7] = -float("inf")           # one row with every part empty
    o = o.to(torch.float32 if parts_fp32 else torch.bfloat16)
    out, lm = A.merge_attention_parts(o.cuda(), lse.cuda(), torch.float32 if out_fp32 else torch.bfloat16)
    torch.cuda.synchronize()
    # the oracle merges row-major (C, rows) views: rows (b, s, h) of O, (b, h, s) of LSE
    on = o.double().numpy()
    ln = lse.double().numpy().transpose(0, 1, 3, 2)           # (C, B, S, H)
    o_ref, l_ref = oracle.merge_lse_partials(ln, on)
    # bf16 output: one rounding of values up to |O| (these synthetic parts are N(0, 1), not attention
    # outputs bounded by 1), i.e. at most max|O| * 2^-8
    tol = 1e-5 if out_fp32 else float(np.abs(o_ref).max()) * 2.0 ** -8
    H.check_o(out, o_ref, tol=tol)
    H.check_lse(lm.permute(0, 2, 1), l_ref, tol=1e-5)
    assert torch.all(out[1, 7, 2] == 0)


def test_key_shards_merged_equal_full_attention():
    # ring / context-parallel: each shard of the keys is attended separately, then merged
    w = W.dense(2, 300, 900, 4, 2, 128, False, seed=33, with_grad=False)
    t = {n: x.cuda() for n, x in w.tensors.items()}
    full_o, full_l = A.flash_attn_func(t["q"], t["k"], t["v"], w.scale, False)
    shards = [(0, 250), (250, 640), (640, 900)]
    parts = [A.flash_attn_func(t["q"], t["k"][:, a:b].contiguous(), t["v"][:, a:b].contiguous(), w.scale, False)
             for a, b in shards]
    o_parts = torch.stack([p[0] for p in parts])
    l_parts = torch.stack([p[1] for p in parts])
    out, lse = A.merge_attention_parts(o_parts, l_parts)
    torch.cuda.synchronize()
    assert (out.float() - full_o.float()).abs().max().item() <= 2e-2
    assert (lse - full_l).abs().max().item() <= 1e-4


def test_merge_in_place_into_the_first_part():
    g = torch.Generator("cpu").manual_seed(3)
    o = torch.randn((2, 1, 64, 2, 128), generator=g).to(torch.bfloat16).cuda()
    lse = torch.randn((2, 1, 2, 64), generator=g).cuda()
    ref, lref = A.merge_attention_parts(o.clone(), lse.clone())
    out, _ = A.merge_attention_parts(o, lse, out=o[0])
    torch.cuda.synchronize()
    assert torch.equal(o[0], ref)
