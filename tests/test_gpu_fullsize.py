"""Parity at the full sizes of the five workloads, in the launch configuration the
benchmark times: the GPU computes everything; the fp64 oracle recomputes sampled
heads / sequences / cache rows one by one, and properties that hold at any size
(sum_j dK_j = 0, sum_j dV_j = sum_i dO_i) are checked on every head."""

import numpy as np
import pytest
import torch

import oracle
from exact_tiled_attention_41_b200 import attention as A, workloads as W
from tests import gpu_helpers as H

pytestmark = pytest.mark.gpu


def _grad_invariants(dk, dv, do, group, rel=1e-2):
    # per (batch, KV head): sum over keys of dK is 0; sum over keys of dV equals sum over the group's rows of dO
    dk64, dv64, do64 = dk.double(), dv.double(), do.double()
    B, S, Hkv, D = dk.shape
    sk = dk64.sum(dim=1)                                                # (B, Hkv, D)
    scale_k = dk64.abs().sum(dim=1)
    assert (sk.abs() <= rel * scale_k + 1e-3).all(), "sum_j dK_j != 0"
    # sum_j dV_j = sum_i (sum_j P_ij) dO_i; the kernel rounds P to bf16 before the dV product (row sums
    # then differ from 1 by at most 2^-9) and rounds each dV element to bf16 (relative error <= 2^-9),
    # so the two sides differ by at most 2^-9 (sum_i |dO_i| + sum_j |dV_j|) per column; twice that
    # leaves room for the fp32 accumulation
    sv = dv64.sum(dim=1)
    do_g = do64.reshape(B, do.shape[1], Hkv, group, D)
    so = do_g.sum(dim=(1, 3))
    bound = 2.0 * 2.0 ** -9 * (do_g.abs().sum(dim=(1, 3)) + dv64.abs().sum(dim=1)) + 1e-3
    assert ((sv - so).abs() <= bound).all(), "sum_j dV_j != sum_i dO_i"


def _fwd_last_round_head(B, H, S, rows_per_unit=256, ctas=148):
    """(b, h) of the unit dealt last by the forward's heaviest-first persistent schedule: units are
    (query block m, b, h) with the blocks that see the most keys first, one per CTA per round."""
    m_blocks = (S + rows_per_unit - 1) // rows_per_unit
    n = m_blocks * B * H
    first_of_last_round = (n - 1) // ctas * ctas
    r = first_of_last_round % (B * H)
    return divmod(r, H)


def _check_heads(w, res, pairs):
    t = w.tensors
    f = H.f64
    for b, h in pairs:
        q, k, v, do = (f(t[n][b:b + 1, :, h:h + 1]) for n in ("q", "k", "v", "do"))
        o_ref, l_ref = oracle.mha_forward(q, k, v, w.scale, True)
        H.check_o(res["out"][b:b + 1, :, h:h + 1], o_ref)
        H.check_lse(res["lse"][b:b + 1, h:h + 1], l_ref)
        dq, dk, dv = oracle.mha_backward(q, k, v, do, w.scale, True)
        H.check_grad(res["dq"][b:b + 1, :, h:h + 1], dq, "dQ")
        H.check_grad(res["dk"][b:b + 1, :, h:h + 1], dk, "dK")
        H.check_grad(res["dv"][b:b + 1, :, h:h + 1], dv, "dV")


def test_dense_prefill_full_size():
    w = W.dense_prefill(seed=0)              # B=4, H=16, S=2048, D=128, causal
    res = H.run_dense(w)
    t = w.tensors
    # three fixed heads and the head whose query block the forward's schedule deals last
    last = _fwd_last_round_head(4, 16, 2048)
    assert last == (3, 12)
    _check_heads(w, res, [(0, 0), (3, 15), (1, 7), last])
    _grad_invariants(res["dk"].cpu(), res["dv"].cpu(), t["do"], 1)


def _check_group(w, res, b, hk, G):
    t = w.tensors
    f = H.f64
    qs = slice(G * hk, G * hk + G)
    q, do = f(t["q"][b:b + 1, :, qs]), f(t["do"][b:b + 1, :, qs])
    k, v = f(t["k"][b:b + 1, :, hk:hk + 1]), f(t["v"][b:b + 1, :, hk:hk + 1])
    o_ref, l_ref = oracle.mha_forward(q, k, v, w.scale, True)
    H.check_o(res["out"][b:b + 1, :, qs], o_ref)
    H.check_lse(res["lse"][b:b + 1, qs], l_ref)
    dq, dk, dv = oracle.mha_backward(q, k, v, do, w.scale, True)
    H.check_grad(res["dq"][b:b + 1, :, qs], dq, "dQ")
    H.check_grad(res["dk"][b:b + 1, :, hk:hk + 1], dk, "dK")
    H.check_grad(res["dv"][b:b + 1, :, hk:hk + 1], dv, "dV")


def test_gqa_long_context_full_size():
    w = W.gqa_long(seed=0)                   # B=2, Hq=32, Hkv=8, S=8192, D=128, causal
    res = H.run_dense(w)
    t = w.tensors
    # KV group 5 of batch 1 (query heads 20..23), and the group of the head whose query block the
    # forward's schedule deals last (batch 0, query head 4: KV head 1, query heads 4..7)
    last_b, last_h = _fwd_last_round_head(2, 32, 8192)
    assert (last_b, last_h) == (0, 4)
    for b, hk in ((1, 5), (last_b, last_h // 4)):
        _check_group(w, res, b, hk, 4)
    _grad_invariants(res["dk"].cpu(), res["dv"].cpu(), t["do"], 4)


@pytest.mark.parametrize("D", [64, 256])
def test_varlen_packed_full_size(D):
    w = W.varlen_packed(D, seed=0)           # 16 sequences, L ~ U[128, 4096], H=16, causal
    t, m = w.tensors, w.meta
    q, k, v = t["q"].cuda(), t["k"].cuda(), t["v"].cuda()
    cq, ck = t["cu_q"].cuda(), t["cu_k"].cuda()
    out, lse = A.flash_attn_varlen_func(q, k, v, cq, ck, m["max_q"], m["max_k"], w.scale, True)
    backward = True
    if backward:
        dq, dk, dv = A.flash_attn_varlen_backward(t["do"].cuda(), q, k, v, out, lse, cq, ck, m["max_q"], m["max_k"],
                                                  w.scale, True)
    torch.cuda.synchronize()
    cu = t["cu_q"].numpy()
    lens = np.diff(cu)
    f = H.f64
    for s in (int(np.argmin(lens)), int(np.argmax(lens)), 7):
        a, e = int(cu[s]), int(cu[s + 1])
        for h in (0, 11):
            qq, kk, vv = (f(t[n][a:e, h:h + 1])[None] for n in ("q", "k", "v"))
            o_ref, l_ref = oracle.mha_forward(qq, kk, vv, w.scale, True)
            H.check_o(out[a:e, h:h + 1][None], o_ref)
            H.check_lse(lse[h:h + 1, a:e][None], l_ref)
            if backward:
                gq, gk, gv = oracle.mha_backward(qq, kk, vv, f(t["do"][a:e, h:h + 1])[None], w.scale, True)
                H.check_grad(dq[a:e, h:h + 1][None], gq, "dQ")
                H.check_grad(dk[a:e, h:h + 1][None], gk, "dK")
                H.check_grad(dv[a:e, h:h + 1][None], gv, "dV")


def test_decode_full_size():
    w = W.decode(seed=0)                     # B=64, Hq=32, Hkv=8, cap 16384, L ~ U[1024, 16384], NaN guards
    out, lse = H.run_kvcache(w)
    t = w.tensors
    lens = t["cache_seqlens"].numpy()
    rng = np.random.default_rng(0)
    rows = [(int(b), int(h)) for b, h in zip(rng.integers(0, 64, 24), rng.integers(0, 32, 24))]
    rows += [(int(np.argmin(lens)), 0), (int(np.argmax(lens)), 31)]
    og, lg = H.f64(out), H.f64(lse)
    qn = H.f64(t["q"])
    for b, h in rows:
        L = int(lens[b])
        hk = oracle.kv_head_of(h, 32, 8)
        kk = H.f64(t["k_cache"][b, :L, hk])
        vv = H.f64(t["v_cache"][b, :L, hk])
        o_ref, l_ref, _ = oracle.head_forward(qn[b, :, h], kk, vv, w.scale, oracle.allowed_mask(1, L, False))
        assert np.abs(og[b, :, h] - o_ref).max() <= H.O_TOL
        assert np.abs(lg[b, h] - l_ref).max() <= H.LSE_TOL
    assert np.isfinite(og).all()
