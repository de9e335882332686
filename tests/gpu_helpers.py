"""Shared helpers for the GPU parity tests: run the CUDA path through the C ABI
(via the torch-tensor wrappers) and the fp64 oracle on the same seeded inputs,
and compare with the tolerances stated for this method:
  forward O: max-abs <= 1e-2; LSE: max-abs <= 1e-3 (bf16 inputs from N(0, 1));
  dQ, dK, dV: relative Frobenius error <= 2e-2.
"""

import numpy as np
import torch

import oracle
from exact_tiled_attention_41_b200 import attention as A

O_TOL = 1e-2
LSE_TOL = 1e-3
GRAD_TOL = 2e-2


def f64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def check_o(o_gpu, o_ref, tol=O_TOL):
    o = f64(o_gpu)
    assert np.isfinite(o).all(), "non-finite output"
    err = np.abs(o - o_ref).max() if o.size else 0.0
    assert err <= tol, f"O max-abs error {err:.3e} > {tol}"
    return err


def check_lse(l_gpu, l_ref, tol=LSE_TOL):
    lg = f64(l_gpu)
    ninf_ref = np.isneginf(l_ref)
    assert np.array_equal(np.isneginf(lg), ninf_ref), "LSE -inf pattern differs"
    fin = ~ninf_ref
    err = np.abs(lg[fin] - l_ref[fin]).max() if fin.any() else 0.0
    assert err <= tol, f"LSE max-abs error {err:.3e} > {tol}"
    return err


def rel_fro(x_gpu, ref):
    x = f64(x_gpu)
    assert np.isfinite(x).all(), "non-finite gradient"
    den = np.linalg.norm(ref)
    num = np.linalg.norm(x - ref)
    return num / den if den > 0 else num


def check_grad(x_gpu, ref, name, tol=GRAD_TOL):
    e = rel_fro(x_gpu, ref)
    assert e <= tol, f"{name} relative Frobenius error {e:.3e} > {tol}"
    return e


def run_dense(w, backward=True, deterministic=False):
    t = w.tensors
    q, k, v = t["q"].cuda(), t["k"].cuda(), t["v"].cuda()
    out, lse = A.flash_attn_func(q, k, v, w.scale, w.causal, w.window)
    res = dict(out=out, lse=lse)
    if backward:
        do = t["do"].cuda()
        res["dq"], res["dk"], res["dv"] = A.flash_attn_backward(do, q, k, v, out, lse, w.scale, w.causal, w.window,
                                                                deterministic)
    torch.cuda.synchronize()
    return res


def check_dense(w, backward=True, deterministic=False, o_tol=O_TOL):
    res = run_dense(w, backward, deterministic)
    t = w.tensors
    qn, kn, vn = f64(t["q"]), f64(t["k"]), f64(t["v"])
    o_ref, l_ref = oracle.mha_forward(qn, kn, vn, w.scale, w.causal, w.window)
    errs = dict(o=check_o(res["out"], o_ref, o_tol), lse=check_lse(res["lse"], l_ref))
    if backward:
        dq, dk, dv = oracle.mha_backward(qn, kn, vn, f64(t["do"]), w.scale, w.causal, w.window)
        errs["dq"] = check_grad(res["dq"], dq, "dQ")
        errs["dk"] = check_grad(res["dk"], dk, "dK")
        errs["dv"] = check_grad(res["dv"], dv, "dV")
    return errs


def check_varlen(w, backward=True, deterministic=False, o_tol=O_TOL):
    t = w.tensors
    m = w.meta
    q, k, v = t["q"].cuda(), t["k"].cuda(), t["v"].cuda()
    cq, ck = t["cu_q"].cuda(), t["cu_k"].cuda()
    out, lse = A.flash_attn_varlen_func(q, k, v, cq, ck, m["max_q"], m["max_k"], w.scale, w.causal, w.window)
    qn, kn, vn = f64(t["q"]), f64(t["k"]), f64(t["v"])
    cu_q, cu_k = t["cu_q"].numpy(), t["cu_k"].numpy()
    o_ref, l_ref = oracle.varlen_forward(qn, kn, vn, cu_q, cu_k, w.scale, w.causal, w.window)
    errs = dict(o=check_o(out, o_ref, o_tol), lse=check_lse(lse, l_ref))
    if backward:
        do = t["do"].cuda()
        dq, dk, dv = A.flash_attn_varlen_backward(do, q, k, v, out, lse, cq, ck, m["max_q"], m["max_k"], w.scale,
                                                  w.causal, w.window, deterministic)
        rq, rk, rv = oracle.varlen_backward(qn, kn, vn, f64(t["do"]), cu_q, cu_k, w.scale, w.causal, w.window)
        errs["dq"] = check_grad(dq, rq, "dQ")
        errs["dk"] = check_grad(dk, rk, "dK")
        errs["dv"] = check_grad(dv, rv, "dV")
    return errs


def run_kvcache(w, num_splits=0):
    t = w.tensors
    out, lse = A.flash_attn_with_kvcache(t["q"].cuda(), t["k_cache"].cuda(), t["v_cache"].cuda(),
                                         t["cache_seqlens"].cuda(), w.scale, False, num_splits)
    torch.cuda.synchronize()
    return out, lse
