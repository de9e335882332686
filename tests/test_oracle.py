"""Pins for the fp64 oracle, checked against things other than the oracle itself.

* masks and head mapping printed on the pages (tests/golden, cited there);
* torch's fp64 scaled_dot_product_attention and autograd (a library routine the
  problem reduces to);
* central finite differences on tiny inputs;
* closed forms and invariants (P rows sum to 1, identical keys give mean(V),
  joint key/value permutation invariance, causal row 0 gives v0, Sk = 1 gives
  v0, LSE = log sum exp by math.fsum, sum_j dK_j = 0, sum_j dV_j = sum_i dO_i).
"""

import math

import numpy as np
import pytest
import torch

import oracle
from tests.conftest import read_golden

RNG = np.random.default_rng(1234)


def rnd(*shape):
    return RNG.standard_normal(shape)


# ----------------------------------------------------------------------------- masks / GQA


def test_causal_mask_matches_pages_q2_k5():
    want = np.array(read_golden("causal_mask_q2_k5.txt"), dtype=bool)
    assert np.array_equal(oracle.allowed_mask(2, 5, True), want)


def test_causal_mask_matches_pages_q5_k2():
    want = np.array(read_golden("causal_mask_q5_k2.txt"), dtype=bool)
    assert np.array_equal(oracle.allowed_mask(5, 2, True), want)


def test_noncausal_mask_is_full():
    assert oracle.allowed_mask(3, 7, False).all()


def test_gqa_mapping_matches_pages():
    for qh, kh in read_golden("gqa_6_over_2.txt"):
        assert oracle.kv_head_of(qh, 6, 2) == kh


def test_gqa_forward_uses_mapped_kv_head():
    B, S, Hq, Hkv, D = 1, 9, 6, 2, 8
    q, k, v = rnd(B, S, Hq, D), rnd(B, S, Hkv, D), rnd(B, S, Hkv, D)
    o, lse = oracle.mha_forward(q, k, v, 0.3, False)
    for qh, kh in read_golden("gqa_6_over_2.txt"):
        # same query head run as plain MHA against the KV head the pages name
        o1, l1 = oracle.mha_forward(q[:, :, qh:qh + 1], k[:, :, kh:kh + 1], v[:, :, kh:kh + 1], 0.3, False)
        np.testing.assert_allclose(o[:, :, qh], o1[:, :, 0], rtol=0, atol=1e-14)
        np.testing.assert_allclose(lse[:, qh], l1[:, 0], rtol=0, atol=1e-14)


def test_gqa_rejects_indivisible_heads():
    with pytest.raises(ValueError):
        oracle.mha_forward(rnd(1, 4, 3, 8), rnd(1, 4, 2, 8), rnd(1, 4, 2, 8), 1.0, False)


# ----------------------------------------------------------------------------- forward vs torch


def sdpa64(q, k, v, scale, mask):
    """torch fp64 SDPA on (B, S, H, D) numpy arrays with explicit boolean mask; GQA by repetition."""
    g = q.shape[2] // k.shape[2]
    tq = torch.from_numpy(q).permute(0, 2, 1, 3)
    tk = torch.from_numpy(k).permute(0, 2, 1, 3).repeat_interleave(g, dim=1)
    tv = torch.from_numpy(v).permute(0, 2, 1, 3).repeat_interleave(g, dim=1)
    m = torch.from_numpy(mask)
    o = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=m, scale=scale)
    return o.permute(0, 2, 1, 3).numpy()


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("Sq,Sk", [(16, 16), (7, 13), (13, 13), (1, 9)])
@pytest.mark.parametrize("Hq,Hkv", [(2, 2), (4, 1), (6, 2)])
def test_forward_matches_torch_sdpa(causal, Sq, Sk, Hq, Hkv):
    D = 16
    q, k, v = rnd(2, Sq, Hq, D), rnd(2, Sk, Hkv, D), rnd(2, Sk, Hkv, D)
    scale = 1 / math.sqrt(D)
    o, _ = oracle.mha_forward(q, k, v, scale, causal)
    mask = oracle.allowed_mask(Sq, Sk, causal)
    np.testing.assert_allclose(o, sdpa64(q, k, v, scale, mask), rtol=1e-12, atol=1e-12)


def test_forward_causal_square_matches_torch_is_causal():
    # torch's is_causal is top-left aligned, which coincides with the pages' rule when Sq == Sk
    q, k, v = rnd(1, 11, 2, 8), rnd(1, 11, 2, 8), rnd(1, 11, 2, 8)
    o, _ = oracle.mha_forward(q, k, v, 0.5, True)
    t = torch.nn.functional.scaled_dot_product_attention(
        *(torch.from_numpy(x).permute(0, 2, 1, 3) for x in (q, k, v)), is_causal=True, scale=0.5)
    np.testing.assert_allclose(o, t.permute(0, 2, 1, 3).numpy(), rtol=1e-12, atol=1e-12)


def test_default_scale_value_in_configs():
    # README: softmax_scale defaults to 1/sqrt(headdim)
    from exact_tiled_attention_41_b200 import workloads
    w = workloads.tiny(False)
    assert w.scale == 1 / math.sqrt(64)


# ----------------------------------------------------------------------------- forward invariants


def test_probability_rows_sum_to_one():
    q, k, v = rnd(9, 8), rnd(12, 8), rnd(12, 8)
    for causal in (False, True):
        _, _, p = oracle.head_forward(q, k, v, 0.7, oracle.allowed_mask(9, 12, causal))
        np.testing.assert_allclose(p.sum(axis=1), 1.0, rtol=0, atol=1e-14)
        assert (p >= 0).all()


def test_identical_keys_give_mean_of_values():
    q, v = rnd(5, 8), rnd(10, 8)
    k = np.tile(rnd(1, 8), (10, 1))
    o, _, _ = oracle.head_forward(q, k, v, 1.0, oracle.allowed_mask(5, 10, False))
    np.testing.assert_allclose(o, np.tile(v.mean(axis=0), (5, 1)), rtol=0, atol=1e-13)


def test_joint_key_value_permutation_invariance():
    q, k, v = rnd(6, 8), rnd(11, 8), rnd(11, 8)
    perm = RNG.permutation(11)
    full = oracle.allowed_mask(6, 11, False)
    o1, l1, _ = oracle.head_forward(q, k, v, 0.4, full)
    o2, l2, _ = oracle.head_forward(q, k[perm], v[perm], 0.4, full)
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-13)
    np.testing.assert_allclose(l1, l2, rtol=0, atol=1e-13)


def test_causal_row_zero_returns_v0_exactly():
    q, k, v = rnd(1, 8, 1, 4), rnd(1, 8, 1, 4), rnd(1, 8, 1, 4)
    o, lse = oracle.mha_forward(q, k, v, 0.5, True)
    assert np.array_equal(o[0, 0, 0], v[0, 0, 0])
    assert lse[0, 0, 0] == pytest.approx(0.5 * float(q[0, 0, 0] @ k[0, 0, 0]), abs=1e-15)


def test_single_key_returns_v0_for_every_row():
    q, k, v = rnd(1, 5, 2, 4), rnd(1, 1, 2, 4), rnd(1, 1, 2, 4)
    o, _ = oracle.mha_forward(q, k, v, 0.5, False)
    for h in range(2):
        np.testing.assert_allclose(o[0, :, h], np.tile(v[0, 0, h], (5, 1)), rtol=0, atol=1e-15)


def test_lse_is_log_sum_exp_fsum():
    q, k, v = rnd(4, 6), rnd(7, 6), rnd(7, 6)
    scale = 0.9
    for causal in (False, True):
        mask = oracle.allowed_mask(4, 7, causal)
        _, lse, _ = oracle.head_forward(q, k, v, scale, mask)
        for i in range(4):
            terms = [math.exp(scale * float(q[i] @ k[j])) for j in range(7) if mask[i, j]]
            assert lse[i] == pytest.approx(math.log(math.fsum(terms)), rel=1e-13, abs=1e-13)


def test_empty_rows_give_zero_output_and_minus_inf_lse():
    # README: "If the row of the mask is all zero, the output will be zero" (Sq=5, Sk=2 example)
    q, k, v = rnd(1, 5, 1, 4), rnd(1, 2, 1, 4), rnd(1, 2, 1, 4)
    o, lse = oracle.mha_forward(q, k, v, 1.0, True)
    assert np.array_equal(o[0, :3], np.zeros((3, 1, 4)))
    assert np.all(np.isneginf(lse[0, 0, :3]))
    assert np.isfinite(lse[0, 0, 3:]).all()
    do = rnd(1, 5, 1, 4)
    dq, dk, dv = oracle.mha_backward(q, k, v, do, 1.0, True)
    assert np.array_equal(dq[0, :3], np.zeros((3, 1, 4)))


def test_large_scores_do_not_overflow():
    q, k, v = 300 * rnd(3, 4), 300 * rnd(5, 4), rnd(5, 4)
    o, lse, p = oracle.head_forward(q, k, v, 1.0, oracle.allowed_mask(3, 5, False))
    assert np.isfinite(o).all() and np.isfinite(lse).all()


# ----------------------------------------------------------------------------- backward


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("Sq,Sk,Hq,Hkv", [(9, 9, 2, 2), (6, 9, 4, 2), (9, 5, 3, 1)])
def test_backward_matches_torch_autograd(causal, Sq, Sk, Hq, Hkv):
    D = 8
    q, k, v, do = rnd(2, Sq, Hq, D), rnd(2, Sk, Hkv, D), rnd(2, Sk, Hkv, D), rnd(2, Sq, Hq, D)
    scale = 0.35
    mask = oracle.allowed_mask(Sq, Sk, causal)
    if not mask.any(axis=1).all():
        pytest.skip("torch SDPA returns NaN on fully masked rows")
    g = Hq // Hkv
    tq = torch.from_numpy(q).permute(0, 2, 1, 3).clone().requires_grad_()
    tk = torch.from_numpy(k).permute(0, 2, 1, 3).clone().requires_grad_()
    tv = torch.from_numpy(v).permute(0, 2, 1, 3).clone().requires_grad_()
    o = torch.nn.functional.scaled_dot_product_attention(
        tq, tk.repeat_interleave(g, 1), tv.repeat_interleave(g, 1), attn_mask=torch.from_numpy(mask), scale=scale)
    (o * torch.from_numpy(do).permute(0, 2, 1, 3)).sum().backward()
    dq, dk, dv = oracle.mha_backward(q, k, v, do, scale, causal)
    np.testing.assert_allclose(dq, tq.grad.permute(0, 2, 1, 3).numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dk, tk.grad.permute(0, 2, 1, 3).numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dv, tv.grad.permute(0, 2, 1, 3).numpy(), rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_backward_matches_central_finite_differences(causal):
    B, Sq, Sk, Hq, Hkv, D = 1, 5, 7, 2, 1, 4
    q, k, v, do = rnd(B, Sq, Hq, D), rnd(B, Sk, Hkv, D), rnd(B, Sk, Hkv, D), rnd(B, Sq, Hq, D)
    scale = 0.6

    def loss(qq, kk, vv):
        o, _ = oracle.mha_forward(qq, kk, vv, scale, causal)
        return float((o * do).sum())

    dq, dk, dv = oracle.mha_backward(q, k, v, do, scale, causal)
    h = 1e-6
    for x, grad, which in ((q, dq, 0), (k, dk, 1), (v, dv, 2)):
        num = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args_p = [q, k, v]
            args_m = [q, k, v]
            args_p[which], args_m[which] = xp, xm
            num[idx] = (loss(*args_p) - loss(*args_m)) / (2 * h)
        np.testing.assert_allclose(grad, num, rtol=1e-6, atol=1e-8)


@pytest.mark.parametrize("causal", [False, True])
def test_backward_invariants(causal):
    S, D = 12, 8
    q, k, v, do = rnd(S, D), rnd(S, D), rnd(S, D), rnd(S, D)
    mask = oracle.allowed_mask(S, S, causal)
    dq, dk, dv = oracle.head_backward(q, k, v, do, 0.5, mask)
    # softmax rows are invariant to a shift of the scores, so sum_j dS_ij = 0 -> sum_j dK_j = 0
    np.testing.assert_allclose(dk.sum(axis=0), 0.0, atol=1e-12)
    # sum_j P_ij = 1 -> sum_j dV_j = sum_i dO_i
    np.testing.assert_allclose(dv.sum(axis=0), do.sum(axis=0), atol=1e-12)
    # Delta = rowsum(dO * O) equals sum_j P dP
    o, _, p = oracle.head_forward(q, k, v, 0.5, mask)
    np.testing.assert_allclose((do * o).sum(axis=1), (p * (do @ v.T)).sum(axis=1), atol=1e-12)


# ----------------------------------------------------------------------------- varlen / cache / merge


@pytest.mark.parametrize("causal", [False, True])
def test_varlen_equals_per_sequence_dense(causal):
    lens = [5, 1, 9, 3]
    Hq, Hkv, D = 4, 2, 8
    cu = np.concatenate([[0], np.cumsum(lens)])
    T = cu[-1]
    q, k, v, do = rnd(T, Hq, D), rnd(T, Hkv, D), rnd(T, Hkv, D), rnd(T, Hq, D)
    o, lse = oracle.varlen_forward(q, k, v, cu, cu, 0.3, causal)
    dq, dk, dv = oracle.varlen_backward(q, k, v, do, cu, cu, 0.3, causal)
    for s in range(len(lens)):
        a, b = cu[s], cu[s + 1]
        od, ld = oracle.mha_forward(q[None, a:b], k[None, a:b], v[None, a:b], 0.3, causal)
        gq, gk, gv = oracle.mha_backward(q[None, a:b], k[None, a:b], v[None, a:b], do[None, a:b], 0.3, causal)
        np.testing.assert_allclose(o[a:b], od[0], atol=1e-14)
        np.testing.assert_allclose(lse[:, a:b], ld[0], atol=1e-14)
        np.testing.assert_allclose(dq[a:b], gq[0], atol=1e-14)
        np.testing.assert_allclose(dk[a:b], gk[0], atol=1e-14)
        np.testing.assert_allclose(dv[a:b], gv[0], atol=1e-14)


def test_kvcache_equals_dense_on_valid_prefix():
    B, cap, Hq, Hkv, D = 3, 20, 4, 2, 8
    lens = np.array([20, 1, 7])
    q = rnd(B, 1, Hq, D)
    kc, vc = np.full((B, cap, Hkv, D), np.nan), np.full((B, cap, Hkv, D), np.nan)
    for b in range(B):
        kc[b, :lens[b]] = rnd(lens[b], Hkv, D)
        vc[b, :lens[b]] = rnd(lens[b], Hkv, D)
    o, lse = oracle.kvcache_forward(q, kc, vc, lens, 0.4, False)
    assert np.isfinite(o).all()
    for b in range(B):
        L = lens[b]
        od, ld = oracle.mha_forward(q[b:b + 1], kc[b:b + 1, :L], vc[b:b + 1, :L], 0.4, False)
        np.testing.assert_allclose(o[b], od[0], atol=1e-14)
        np.testing.assert_allclose(lse[b], ld[0], atol=1e-14)
    # with one query, bottom-right causal keeps every valid key
    o2, _ = oracle.kvcache_forward(q, kc, vc, lens, 0.4, True)
    np.testing.assert_allclose(o, o2, atol=0)


def test_merge_of_key_blocks_equals_full_attention():
    q, k, v = rnd(3, 8), rnd(40, 8), rnd(40, 8)
    full = oracle.allowed_mask(3, 40, False)
    o, lse, _ = oracle.head_forward(q, k, v, 0.5, full)
    edges = [0, 7, 8, 30, 40]
    parts_o, parts_l = [], []
    for a, b in zip(edges[:-1], edges[1:]):
        oo, ll, _ = oracle.head_forward(q, k[a:b], v[a:b], 0.5, oracle.allowed_mask(3, b - a, False))
        parts_o.append(oo)
        parts_l.append(ll)
    # an empty block (LSE = -inf) must not change the result
    parts_o.append(np.zeros_like(o))
    parts_l.append(np.full(3, -np.inf))
    om, lm = oracle.merge_lse_partials(parts_l, parts_o)
    np.testing.assert_allclose(om, o, atol=1e-13)
    np.testing.assert_allclose(lm, lse, atol=1e-13)


# ----------------------------------------------------------------------------- sliding window


@pytest.mark.parametrize("name,Lq,Lk,window", [
    ("window_mask_q4_k6_l1_r0.txt", 4, 6, (1, 0)),
    ("window_mask_q5_k3_l0_r1.txt", 5, 3, (0, 1)),
    ("window_mask_q5_k5_l2_unbounded.txt", 5, 5, (2, -1)),
])
def test_window_mask_matches_hand_derived_interval(name, Lq, Lk, window):
    want = np.array(read_golden(name), dtype=bool)
    assert np.array_equal(oracle.allowed_mask(Lq, Lk, False, window), want)


def test_window_reduces_to_causal_and_full_masks():
    for Lq, Lk in ((2, 5), (5, 2), (7, 7)):
        # right side 0 with an unbounded left side is the bottom-right causal mask the pages print
        assert np.array_equal(oracle.allowed_mask(Lq, Lk, False, (-1, 0)), oracle.allowed_mask(Lq, Lk, True))
        assert oracle.allowed_mask(Lq, Lk, False, (-1, -1)).all()
        assert oracle.allowed_mask(Lq, Lk, False, (Lq + Lk, Lq + Lk)).all()
    want = np.array(read_golden("causal_mask_q2_k5.txt"), dtype=bool)
    assert np.array_equal(oracle.allowed_mask(2, 5, False, (-1, 0)), want)


def test_causal_with_window_keeps_the_intersection():
    # the reading taken where the pages are silent: both rules apply
    for Lq, Lk, w in ((6, 9, (2, 3)), (9, 6, (1, 0)), (8, 8, (3, -1))):
        both = oracle.allowed_mask(Lq, Lk, True, w)
        assert np.array_equal(both, oracle.allowed_mask(Lq, Lk, True) & oracle.allowed_mask(Lq, Lk, False, w))


def _row_interval(i, Lq, Lk, window):
    # the docstring's interval for query i, clipped to the keys that exist
    off = Lk - Lq
    lo = 0 if window[0] < 0 else max(0, i + off - window[0])
    hi = Lk - 1 if window[1] < 0 else min(Lk - 1, i + off + window[1])
    return lo, hi


def _sliced_rows(q, k, v, scale, window):
    """Each query row attends, with no mask at all, to the slice of keys its window names
    (torch fp64 SDPA per row); rows whose slice is empty give 0 / -inf."""
    Lq, Lk = q.shape[0], k.shape[0]
    outs, lses = [], []
    for i in range(Lq):
        lo, hi = _row_interval(i, Lq, Lk, window)
        if hi < lo:
            outs.append(torch.zeros(v.shape[1], dtype=torch.float64))
            lses.append(torch.tensor(-math.inf, dtype=torch.float64))
            continue
        ks, vs = k[lo:hi + 1], v[lo:hi + 1]
        o = torch.nn.functional.scaled_dot_product_attention(q[i:i + 1][None], ks[None], vs[None], scale=scale)
        outs.append(o[0, 0])
        lses.append(torch.logsumexp(scale * (ks @ q[i]), dim=0))
    return torch.stack(outs), torch.stack(lses)


@pytest.mark.parametrize("Lq,Lk,window", [(13, 13, (3, 0)), (9, 14, (2, 1)), (14, 9, (0, 2)),
                                          (11, 11, (-1, 2)), (10, 10, (4, -1)), (6, 6, (0, 0))])
def test_window_forward_matches_sliced_sdpa(Lq, Lk, window):
    q, k, v = rnd(Lq, 8), rnd(Lk, 8), rnd(Lk, 8)
    o, lse, _ = oracle.head_forward(q, k, v, 0.4, oracle.allowed_mask(Lq, Lk, False, window))
    o_ref, lse_ref = _sliced_rows(*(torch.from_numpy(x) for x in (q, k, v)), 0.4, window)
    np.testing.assert_allclose(o, o_ref.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_array_equal(np.isneginf(lse), np.isneginf(lse_ref.numpy()))
    fin = np.isfinite(lse)
    np.testing.assert_allclose(lse[fin], lse_ref.numpy()[fin], rtol=0, atol=1e-12)


@pytest.mark.parametrize("Lq,Lk,window", [(12, 12, (3, 0)), (8, 13, (2, 1)), (13, 8, (1, 3))])
def test_window_backward_matches_sliced_autograd(Lq, Lk, window):
    B, Hq, Hkv, D = 1, 4, 2, 8
    q, k, v, do = rnd(B, Lq, Hq, D), rnd(B, Lk, Hkv, D), rnd(B, Lk, Hkv, D), rnd(B, Lq, Hq, D)
    dq, dk, dv = oracle.mha_backward(q, k, v, do, 0.35, False, window)
    tq, tk, tv = (torch.from_numpy(x.copy()).requires_grad_() for x in (q, k, v))
    loss = 0
    for h in range(Hq):
        hk = h // (Hq // Hkv)
        o, _ = _sliced_rows(tq[0, :, h], tk[0, :, hk], tv[0, :, hk], 0.35, window)
        loss = loss + (o * torch.from_numpy(do[0, :, h])).sum()
    loss.backward()
    for got, ref in ((dq, tq.grad), (dk, tk.grad), (dv, tv.grad)):
        np.testing.assert_allclose(got, ref.numpy(), rtol=0, atol=1e-11)


def test_window_varlen_equals_per_sequence_dense():
    lens = [5, 17, 1, 9]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T = int(cu[-1])
    q, k, v, do = rnd(T, 2, 8), rnd(T, 1, 8), rnd(T, 1, 8), rnd(T, 2, 8)
    w = (3, 1)
    o, lse = oracle.varlen_forward(q, k, v, cu, cu, 0.3, True, w)
    dq, dk, dv = oracle.varlen_backward(q, k, v, do, cu, cu, 0.3, True, w)
    for a, b in zip(cu[:-1], cu[1:]):
        od, ld = oracle.mha_forward(q[None, a:b], k[None, a:b], v[None, a:b], 0.3, True, w)
        gq, gk, gv = oracle.mha_backward(q[None, a:b], k[None, a:b], v[None, a:b], do[None, a:b], 0.3, True, w)
        np.testing.assert_array_equal(o[a:b], od[0])
        np.testing.assert_array_equal(lse[:, a:b], ld[0])
        np.testing.assert_array_equal(dq[a:b], gq[0])
        np.testing.assert_array_equal(dk[a:b], gk[0])
        np.testing.assert_array_equal(dv[a:b], gv[0])


# ----------------------------------------------------------------------------- KV cache: append, paging, Sq > 1


def test_paged_cache_address_matches_hand_derived_rows():
    want = read_golden("paged_cache_rows_page2.txt")
    cache = np.zeros((4, 2, 1, 1))
    for blk in range(4):
        for r in range(2):
            cache[blk, r, 0, 0] = 10 * blk + r
    table = np.array([[2, 0], [3, 1]])
    for b in range(2):
        _, rows = oracle.logical_cache_rows(cache, b, 4, block_table=table)
        assert rows[:, 0, 0].tolist() == want[b]


def _cache(B, cap, Hkv, D, lens):
    kc, vc = np.full((B, cap, Hkv, D), np.nan), np.full((B, cap, Hkv, D), np.nan)
    for b in range(B):
        kc[b, :lens[b]] = rnd(lens[b], Hkv, D)
        vc[b, :lens[b]] = rnd(lens[b], Hkv, D)
    return kc, vc


def test_kvcache_update_equals_dense_on_the_concatenation():
    # append k_new / v_new at cache_seqlens, then attend causally with several queries: the dense
    # function on the concatenated keys, bottom-right aligned
    B, cap, Hq, Hkv, D, Sq, Sn = 3, 24, 4, 2, 8, 5, 3
    lens = np.array([0, 9, 21])
    kc, vc = _cache(B, cap, Hkv, D, lens)
    q, kn, vn = rnd(B, Sq, Hq, D), rnd(B, Sn, Hkv, D), rnd(B, Sn, Hkv, D)
    for causal, window in ((True, (-1, -1)), (False, (-1, -1)), (True, (4, -1)), (False, (2, 1))):
        o, lse, ka, va = oracle.kvcache_update_forward(q, kc, vc, lens, 0.4, causal, window, kn, vn)
        for b in range(B):
            L = lens[b]
            kk = np.concatenate([kc[b, :L], kn[b]])[None]
            vv = np.concatenate([vc[b, :L], vn[b]])[None]
            od, ld = oracle.mha_forward(q[b:b + 1], kk, vv, 0.4, causal, window)
            np.testing.assert_allclose(o[b], od[0], rtol=0, atol=1e-14)
            np.testing.assert_array_equal(np.isneginf(lse[b]), np.isneginf(ld[0]))
            np.testing.assert_allclose(lse[b][np.isfinite(ld[0])], ld[0][np.isfinite(ld[0])], rtol=0, atol=1e-14)
            # the caches were updated in place at rows L .. L + Sn - 1 and nowhere else
            np.testing.assert_array_equal(ka[b, L:L + Sn], kn[b])
            np.testing.assert_array_equal(va[b, L:L + Sn], vn[b])
            np.testing.assert_array_equal(np.isnan(ka[b, L + Sn:]), np.isnan(kc[b, L + Sn:]))


def test_kvcache_update_paged_equals_contiguous():
    # scatter a contiguous cache into pages through a random block table: same result, and the append
    # lands in the right physical rows
    B, cap, Hq, Hkv, D, page = 3, 16, 2, 1, 8, 4
    lens = np.array([5, 12, 0])
    kc, vc = _cache(B, cap, Hkv, D, lens)
    nblk = B * cap // page
    perm = np.random.default_rng(5).permutation(nblk)
    table = perm.reshape(B, cap // page)
    kp, vp = np.zeros((nblk, page, Hkv, D)), np.zeros((nblk, page, Hkv, D))
    for b in range(B):
        for i in range(cap // page):
            kp[table[b, i]] = kc[b, i * page:(i + 1) * page]
            vp[table[b, i]] = vc[b, i * page:(i + 1) * page]
    q, kn, vn = rnd(B, 3, Hq, D), rnd(B, 2, Hkv, D), rnd(B, 2, Hkv, D)
    o1, l1, ka1, _ = oracle.kvcache_update_forward(q, kc, vc, lens, 0.3, True, (-1, -1), kn, vn)
    o2, l2, ka2, _ = oracle.kvcache_update_forward(q, kp, vp, lens, 0.3, True, (-1, -1), kn, vn, block_table=table)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)
    for b in range(B):
        for i in range(cap // page):
            np.testing.assert_array_equal(ka2[table[b, i]], ka1[b, i * page:(i + 1) * page])


def test_kvcache_update_with_batch_index_reads_the_indexed_rows():
    B, cap, Hq, Hkv, D = 3, 10, 2, 2, 8
    kc, vc = _cache(4, cap, Hkv, D, [10, 10, 10, 10])
    idx = np.array([3, 0, 2])
    lens = np.array([4, 10, 7])
    q = rnd(B, 2, Hq, D)
    o, lse, _, _ = oracle.kvcache_update_forward(q, kc, vc, lens, 0.5, True, cache_batch_idx=idx)
    o_ref, l_ref = oracle.kvcache_forward(q, kc[idx], vc[idx], lens, 0.5, True)
    np.testing.assert_array_equal(o, o_ref)
    np.testing.assert_array_equal(lse, l_ref)


def test_kvcache_update_without_new_keys_is_kvcache_forward():
    B, cap, Hq, Hkv, D = 2, 12, 4, 1, 8
    lens = np.array([12, 3])
    kc, vc = _cache(B, cap, Hkv, D, lens)
    q = rnd(B, 4, Hq, D)
    for causal in (False, True):
        o, lse, ka, _ = oracle.kvcache_update_forward(q, kc, vc, lens, 0.5, causal)
        o_ref, l_ref = oracle.kvcache_forward(q, kc, vc, lens, 0.5, causal)
        np.testing.assert_array_equal(o, o_ref)
        np.testing.assert_array_equal(lse, l_ref)
        np.testing.assert_array_equal(np.isnan(ka), np.isnan(kc))
