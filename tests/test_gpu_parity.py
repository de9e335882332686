"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on the
same seeded inputs, at sizes the oracle finishes in seconds that still span
several tiles and a ragged tail, plus the degenerate cases of the method."""

import math

import numpy as np
import pytest
import torch

import oracle
from exact_tiled_attention_41_b200 import abi, workloads as W
from tests import gpu_helpers as H

pytestmark = pytest.mark.gpu


# ----------------------------------------------------------------------------- building blocks


@pytest.mark.parametrize("mode", [0, 1, 2])
def test_tensor_core_selftest(mode):
    g = torch.Generator("cpu").manual_seed(7)
    a = torch.randn(128, 128, generator=g).to(torch.bfloat16)
    b = torch.randn(128, 128, generator=g).to(torch.bfloat16)
    c = torch.full((128, 128), float("nan"), dtype=torch.float32, device="cuda")
    assert abi.fa_debug_umma_selftest(a.cuda(), b.cuda(), c, mode) == 0
    torch.cuda.synchronize()
    a64, b64 = a.double().numpy(), b.double().numpy()
    ref = a64 @ b64.T if mode == 0 else a64 @ b64
    np.testing.assert_allclose(c.cpu().double().numpy(), ref, rtol=0, atol=1e-3)


def test_fma_pipe_exp2_matches_cuda_exp2f():
    # the softmax kernels take part of their exponentials off the multi-function unit; that
    # polynomial must be as accurate as CUDA's own exp2f (about 2 ulp) over the range they use
    x = torch.cat([torch.linspace(-125.0, 8.0, 1 << 20), torch.rand(1 << 20) * 16 - 12,
                   torch.tensor([0.0, 0.5, -0.5, 1.0, -1.0, 7.99, -124.9, -125.0, 8.0, 3.0])]).float()
    x = x[: (x.numel() // 2) * 2].contiguous()
    xd = x.cuda()
    y = torch.empty_like(xd)
    assert abi.fa_debug_exp2_selftest(xd, y, x.numel()) == 0
    ref_cuda = torch.exp2(xd)                       # CUDA exp2f
    torch.cuda.synchronize()
    ref64 = torch.exp2(x.double())
    rel = ((y.cpu().double() - ref64) / ref64).abs()
    rel_cuda = ((ref_cuda.cpu().double() - ref64) / ref64).abs()
    assert rel.max().item() <= 2.5e-7
    assert rel.max().item() <= 2.5 * max(rel_cuda.max().item(), 6e-8)
    # below -125 (the kernels only call it on tiles without masked scores) the result stays a
    # non-negative number under 2^-125: never negative, NaN or large
    z = torch.tensor([-125.5, -126.0, -200.0, -1e30, float("-inf"), -125.9], dtype=torch.float32).cuda()
    yz = torch.full_like(z, 1.0)
    assert abi.fa_debug_exp2_selftest(z, yz, z.numel()) == 0
    torch.cuda.synchronize()
    assert torch.all(yz >= 0) and torch.all(yz <= 2.0 ** -125)


def test_bounded_wait_reports_timeout_instead_of_hanging():
    assert abi.fa_get_device_status() == 0
    assert abi.fa_debug_wait_timeout_selftest(20_000_000) == 0      # 20 ms
    assert abi.fa_get_device_status() == abi.FA_ERR_TIMEOUT
    assert abi.fa_get_device_status() == 0                          # reading clears it


# ----------------------------------------------------------------------------- dense forward + backward


@pytest.mark.parametrize("causal", [False, True])
def test_tiny_config(causal):
    # B=1, Hq=Hkv=2, S=128, D=64 (the smallest of the five workloads)
    H.check_dense(W.tiny(causal))


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("Sq,Sk", [(300, 300), (517, 517), (200, 333), (333, 200), (1, 77)])
def test_dense_ragged_gqa(D, causal, Sq, Sk):
    w = W.dense(2, Sq, Sk, 4, 2, D, causal, seed=Sq * 7 + Sk + D)
    H.check_dense(w)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("Sq,Sk", [(300, 300), (129, 257), (200, 70)])
def test_dense_d256(causal, Sq, Sk):
    w = W.dense(1, Sq, Sk, 4, 1, 256, causal, seed=11)
    H.check_dense(w)


def test_mqa_and_wide_group():
    H.check_dense(W.dense(1, 260, 260, 8, 1, 128, True, seed=3))


def test_fully_masked_rows_give_zero_output_and_grads():
    # README: Sq > Sk under the bottom-right causal rule leaves rows with no key; their output is 0
    w = W.dense(1, 300, 100, 2, 2, 128, True, seed=5)
    errs = H.check_dense(w)
    res = H.run_dense(w)
    assert torch.all(res["out"][0, :200] == 0)
    assert torch.all(torch.isneginf(res["lse"][0, :, :200]))
    assert torch.all(res["dq"][0, :200] == 0)
    assert errs["o"] <= H.O_TOL


def test_large_logits_are_stable():
    w = W.dense(1, 256, 256, 2, 2, 128, True, seed=9)
    w.tensors["q"] = (w.tensors["q"].float() * 8).to(torch.bfloat16)
    H.check_dense(w)


def test_forward_is_deterministic():
    w = W.dense(2, 384, 384, 4, 2, 128, True, seed=1, with_grad=False)
    a = H.run_dense(w, backward=False)
    b = H.run_dense(w, backward=False)
    assert torch.equal(a["out"], b["out"]) and torch.equal(a["lse"], b["lse"])


def test_dk_dv_are_deterministic():
    w = W.dense(1, 384, 384, 4, 2, 128, True, seed=2)
    a = H.run_dense(w)
    b = H.run_dense(w)
    assert torch.equal(a["dk"], b["dk"]) and torch.equal(a["dv"], b["dv"])


# ----------------------------------------------------------------------------- varlen


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_varlen_ragged(D, causal):
    lens = [1, 127, 128, 129, 300, 64, 2]
    w = W.varlen(lens, lens, 4, 2, D, causal, seed=D + causal)
    H.check_varlen(w)


def test_varlen_unequal_q_and_k_lengths():
    lq, lk = [5, 200, 130], [40, 150, 300]
    w = W.varlen(lq, lk, 4, 4, 128, True, seed=4)
    H.check_varlen(w)


def test_varlen_d256():
    lens = [1, 200, 129, 64]
    w = W.varlen(lens, lens, 4, 2, 256, True, seed=6)
    H.check_varlen(w)


def test_varlen_matches_dense_layout():
    # a packed batch of equal lengths is the dense batch
    w = W.dense(3, 200, 200, 4, 2, 64, True, seed=8)
    t = w.tensors
    d = H.run_dense(w)
    cu = torch.arange(0, 601, 200, dtype=torch.int32).cuda()
    from exact_tiled_attention_41_b200 import attention as A
    out, lse = A.flash_attn_varlen_func(t["q"].reshape(600, 4, 64).cuda(), t["k"].reshape(600, 2, 64).cuda(),
                                        t["v"].reshape(600, 2, 64).cuda(), cu, cu, 200, 200, w.scale, True)
    assert torch.equal(out.reshape(3, 200, 4, 64), d["out"])
    assert torch.equal(lse.reshape(4, 3, 200).permute(1, 0, 2), d["lse"])


# ----------------------------------------------------------------------------- KV-cache decode


@pytest.mark.parametrize("num_splits", [0, 1, 3])
def test_kvcache_decode_with_nan_guards(num_splits):
    lens = [1, 63, 64, 65, 1000, 777]
    w = W.kvcache(len(lens), 8, 2, 128, 1024, 0, 0, seed=12, lengths=lens)
    out, lse = H.run_kvcache(w, num_splits)
    t = w.tensors
    o_ref, l_ref = oracle.kvcache_forward(H.f64(t["q"]), H.f64(t["k_cache"]), H.f64(t["v_cache"]),
                                          t["cache_seqlens"].numpy(), w.scale, False)
    H.check_o(out, o_ref)
    H.check_lse(lse, l_ref)


def test_kvcache_gqa_group_of_four_and_d64():
    lens = [2000, 4096, 1, 3000]
    w = W.kvcache(4, 32, 8, 64, 4096, 0, 0, seed=13, lengths=lens)
    out, lse = H.run_kvcache(w)
    t = w.tensors
    o_ref, l_ref = oracle.kvcache_forward(H.f64(t["q"]), H.f64(t["k_cache"]), H.f64(t["v_cache"]),
                                          t["cache_seqlens"].numpy(), w.scale, False)
    H.check_o(out, o_ref)
    H.check_lse(lse, l_ref)


def test_kvcache_empty_cache_row():
    lens = [0, 300]
    w = W.kvcache(2, 4, 4, 128, 512, 0, 0, seed=14, lengths=lens)
    out, lse = H.run_kvcache(w)
    assert torch.all(out[0] == 0)
    assert torch.all(torch.isneginf(lse[0]))
    t = w.tensors
    o_ref, l_ref = oracle.kvcache_forward(H.f64(t["q"]), H.f64(t["k_cache"]), H.f64(t["v_cache"]),
                                          t["cache_seqlens"].numpy(), w.scale, False)
    H.check_o(out[1:], o_ref[1:])


def test_kvcache_equals_dense_forward_on_valid_prefix():
    lens = [333]
    w = W.kvcache(1, 4, 2, 128, 512, 0, 0, seed=15, lengths=lens, nan_guard=False)
    out, lse = H.run_kvcache(w)
    t = w.tensors
    from exact_tiled_attention_41_b200 import attention as A
    o2, l2 = A.flash_attn_func(t["q"].cuda(), t["k_cache"][:, :333].contiguous().cuda(),
                               t["v_cache"][:, :333].contiguous().cuda(), w.scale, False)
    assert (out.float() - o2.float()).abs().max().item() <= 2 ** -7
    assert (lse - l2).abs().max().item() <= 1e-4
