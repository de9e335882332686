"""GPU parity of sliding-window local attention (flash-attention README, flash_attn_func
docstring: query i keeps the keys j with i + Sk - Sq - left <= j <= i + Sk - Sq + right,
-1 = unbounded side; causal caps the right side at 0) against the fp64 oracle, forward and
backward, dense and varlen, at sizes spanning several tiles with ragged tails, and at the
size of the long-context GQA workload on a sampled KV group."""

import numpy as np
import pytest
import torch

import oracle
from exact_tiled_attention_41_b200 import abi, attention as A, workloads as W
from tests import gpu_helpers as H

pytestmark = pytest.mark.gpu

WINDOWS = [(False, (100, 50)), (True, (130, -1)), (False, (0, 0)), (False, (-1, 200)), (True, (300, 7)),
           (False, (257, 0))]


@pytest.mark.parametrize("causal,window", WINDOWS)
@pytest.mark.parametrize("Sq,Sk", [(517, 517), (300, 650), (650, 300)])
@pytest.mark.parametrize("D", [64, 128])
def test_dense_window(D, Sq, Sk, causal, window):
    w = W.dense(1, Sq, Sk, 4, 2, D, causal, seed=Sq + 3 * Sk + D + window[0])
    w.window = window
    H.check_dense(w)


@pytest.mark.parametrize("causal,window", [(False, (100, 50)), (True, (130, -1)), (False, (0, 0))])
@pytest.mark.parametrize("Sq,Sk", [(300, 300), (129, 400), (400, 129)])
def test_dense_window_d256(Sq, Sk, causal, window):
    w = W.dense(1, Sq, Sk, 4, 1, 256, causal, seed=Sq + Sk + window[0])
    w.window = window
    H.check_dense(w)


def test_rows_left_without_keys_are_zero():
    # Sq > Sk with window (0, 1): row i keeps j in [i - 350, i - 349], so rows 0..348 keep nothing
    w = W.dense(1, 650, 300, 2, 2, 128, False, seed=21)
    w.window = (0, 1)
    H.check_dense(w)
    res = H.run_dense(w)
    assert torch.all(res["out"][0, :349] == 0)
    assert torch.all(torch.isneginf(res["lse"][0, :, :349]))
    assert torch.all(res["dq"][0, :349] == 0)


def test_window_reductions_are_bit_identical():
    w = W.dense(2, 520, 520, 4, 2, 128, False, seed=22)
    full = H.run_dense(w)
    w.window = (5000, 5000)                 # wider than the sequence: the full mask
    wide = H.run_dense(w)
    for n in ("out", "lse", "dk", "dv"):
        assert torch.equal(full[n], wide[n]), n
    causal = H.run_dense(W.dense(2, 520, 520, 4, 2, 128, True, seed=22))
    w.window = (-1, 0)                      # an unbounded left side and right side 0: the causal mask
    right0 = H.run_dense(w)
    for n in ("out", "lse", "dk", "dv"):
        assert torch.equal(causal[n], right0[n]), n


def test_window_sides_beyond_2_to_30_are_unbounded():
    w = W.dense(1, 260, 260, 2, 2, 64, False, seed=23, with_grad=False)
    t = w.tensors
    q, k, v = t["q"].cuda(), t["k"].cuda(), t["v"].cuda()
    ref, lref = A.flash_attn_func(q, k, v, w.scale, False)
    out, lse = torch.empty_like(ref), torch.empty_like(lref)
    st = abi.fa_fwd_ex(q, k, v, out, lse, 1, 2, 2, 260, 260, 64, w.scale, 0, 2 ** 31 - 1, 2 ** 30)
    assert st == abi.FA_OK
    torch.cuda.synchronize()
    assert torch.equal(out, ref) and torch.equal(lse, lref)


@pytest.mark.parametrize("causal,window", [(True, (64, -1)), (False, (100, 30)), (False, (0, 0))])
@pytest.mark.parametrize("D", [64, 128, 256])
def test_varlen_window(D, causal, window):
    lens = [1, 127, 128, 129, 300, 64, 2]
    w = W.varlen(lens, lens, 4, 2, D, causal, seed=D + window[0])
    w.window = window
    H.check_varlen(w)


def test_varlen_window_unequal_lengths():
    w = W.varlen([5, 200, 130, 400], [40, 150, 300, 90], 4, 4, 128, True, seed=24)
    w.window = (70, -1)
    H.check_varlen(w)


def test_gqa_long_context_sliding_window_full_size():
    # the long-context GQA workload (B=2, Hq=32, Hkv=8, S=8192, D=128, causal) with a 4096-key window
    w = W.gqa_long(seed=0)
    w.window = (4096, 0)
    res = H.run_dense(w)
    t = w.tensors
    f = H.f64
    b, hk = 0, 3
    qs = slice(4 * hk, 4 * hk + 4)
    q, do = f(t["q"][b:b + 1, :, qs]), f(t["do"][b:b + 1, :, qs])
    k, v = f(t["k"][b:b + 1, :, hk:hk + 1]), f(t["v"][b:b + 1, :, hk:hk + 1])
    o_ref, l_ref = oracle.mha_forward(q, k, v, w.scale, True, w.window)
    H.check_o(res["out"][b:b + 1, :, qs], o_ref)
    H.check_lse(res["lse"][b:b + 1, qs], l_ref)
    dq, dk, dv = oracle.mha_backward(q, k, v, do, w.scale, True, w.window)
    H.check_grad(res["dq"][b:b + 1, :, qs], dq, "dQ")
    H.check_grad(res["dk"][b:b + 1, :, hk:hk + 1], dk, "dK")
    H.check_grad(res["dv"][b:b + 1, :, hk:hk + 1], dv, "dV")
    og = res["out"].float()
    assert torch.isfinite(og).all() and torch.isfinite(res["dq"].float()).all()
