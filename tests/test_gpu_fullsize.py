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
    sv = dv64.sum(dim=1)
    so = do64.reshape(B, do.shape[1], Hkv, group, D).sum(dim=(1, 3))
    assert torch.allclose(sv, so, rtol=rel, atol=0.5), "sum_j dV_j != sum_i dO_i"


def test_dense_prefill_full_size():
    w = W.dense_prefill(seed=0)              # B=4, H=16, S=2048, D=128, causal
    res = H.run_dense(w)
    t = w.tensors
    f = H.f64
    for b, h in ((0, 0), (3, 15), (1, 7)):
        q, k, v, do = (f(t[n][b:b + 1, :, h:h + 1]) for n in ("q", "k", "v", "do"))
        o_ref, l_ref = oracle.mha_forward(q, k, v, w.scale, True)
        H.check_o(res["out"][b:b + 1, :, h:h + 1], o_ref)
        H.check_lse(res["lse"][b:b + 1, h:h + 1], l_ref)
        dq, dk, dv = oracle.mha_backward(q, k, v, do, w.scale, True)
        H.check_grad(res["dq"][b:b + 1, :, h:h + 1], dq, "dQ")
        H.check_grad(res["dk"][b:b + 1, :, h:h + 1], dk, "dK")
        H.check_grad(res["dv"][b:b + 1, :, h:h + 1], dv, "dV")
    _grad_invariants(res["dk"].cpu(), res["dv"].cpu(), t["do"], 1)


def test_gqa_long_context_full_size():
    w = W.gqa_long(seed=0)                   # B=2, Hq=32, Hkv=8, S=8192, D=128, causal
    res = H.run_dense(w)
    t = w.tensors
    f = H.f64
    b, hk = 1, 5                             # one KV group: query heads 20..23 read KV head 5
    qs = slice(4 * hk, 4 * hk + 4)
    q, do = f(t["q"][b:b + 1, :, qs]), f(t["do"][b:b + 1, :, qs])
    k, v = f(t["k"][b:b + 1, :, hk:hk + 1]), f(t["v"][b:b + 1, :, hk:hk + 1])
    o_ref, l_ref = oracle.mha_forward(q, k, v, w.scale, True)
    H.check_o(res["out"][b:b + 1, :, qs], o_ref)
    H.check_lse(res["lse"][b:b + 1, qs], l_ref)
    dq, dk, dv = oracle.mha_backward(q, k, v, do, w.scale, True)
    H.check_grad(res["dq"][b:b + 1, :, qs], dq, "dQ")
    H.check_grad(res["dk"][b:b + 1, :, hk:hk + 1], dk, "dK")
    H.check_grad(res["dv"][b:b + 1, :, hk:hk + 1], dv, "dV")
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
