"""GPU parity of the deterministic backward (flash-attention README, flash_attn_func docstring:
deterministic backward pass; the forward is always deterministic).  dq comes from a
query-tile-stationary pass that sums the key tiles in a fixed order, so repeated runs on the
same inputs give bit-identical dq, dk and dv; the values match the fp64 oracle within the
same tolerances as the default backward."""

import pytest
import torch

from exact_tiled_attention_41_b200 import workloads as W
from tests import gpu_helpers as H

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("D", [64, 128, 256])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("Sq,Sk", [(300, 300), (200, 333), (333, 200)])
def test_deterministic_dense_matches_oracle(D, causal, Sq, Sk):
    w = W.dense(2, Sq, Sk, 4, 2, D, causal, seed=Sq * 5 + Sk + D)
    H.check_dense(w, deterministic=True)


@pytest.mark.parametrize("D", [64, 128, 256])
def test_deterministic_window_and_varlen(D):
    w = W.dense(1, 517, 517, 4, 1, D, True, seed=D)
    w.window = (130, -1)
    H.check_dense(w, deterministic=True)
    lens = [1, 127, 128, 129, 300, 64, 2]
    wv = W.varlen(lens, lens, 4, 2, D, True, seed=D + 1)
    H.check_varlen(wv, deterministic=True)
    wv.window = (40, 3)
    H.check_varlen(wv, deterministic=True)


def test_deterministic_rows_without_keys():
    w = W.dense(1, 300, 100, 2, 2, 128, True, seed=5)
    H.check_dense(w, deterministic=True)
    res = H.run_dense(w, deterministic=True)
    assert torch.all(res["dq"][0, :200] == 0)


@pytest.mark.parametrize("D", [64, 128, 256])
def test_deterministic_backward_is_bit_reproducible(D):
    # large enough that many key tiles add into every query row's dq
    w = W.dense(2, 2048, 2048, 8, 2, D, True, seed=31)
    runs = [H.run_dense(w, deterministic=True) for _ in range(3)]
    for r in runs[1:]:
        for n in ("dq", "dk", "dv"):
            assert torch.equal(runs[0][n], r[n]), n


@pytest.mark.parametrize("D", [64, 128, 256])
def test_deterministic_dk_dv_equal_default_backward(D):
    # only the dq path differs between the two modes
    w = W.dense(1, 700, 700, 4, 2, D, True, seed=32)
    a = H.run_dense(w, deterministic=True)
    b = H.run_dense(w, deterministic=False)
    assert torch.equal(a["dk"], b["dk"]) and torch.equal(a["dv"], b["dv"])
    dq_err = (a["dq"].float() - b["dq"].float()).norm() / b["dq"].float().norm()
    assert dq_err.item() <= 1e-2


def test_deterministic_gqa_long_context_full_size():
    # the long-context GQA workload (B=2, Hq=32, Hkv=8, S=8192, D=128, causal), sampled KV group
    import oracle
    w = W.gqa_long(seed=0)
    res = H.run_dense(w, deterministic=True)
    t = w.tensors
    f = H.f64
    b, hk = 1, 6
    qs = slice(4 * hk, 4 * hk + 4)
    q, do = f(t["q"][b:b + 1, :, qs]), f(t["do"][b:b + 1, :, qs])
    k, v = f(t["k"][b:b + 1, :, hk:hk + 1]), f(t["v"][b:b + 1, :, hk:hk + 1])
    dq, dk, dv = oracle.mha_backward(q, k, v, do, w.scale, True)
    H.check_grad(res["dq"][b:b + 1, :, qs], dq, "dQ")
    H.check_grad(res["dk"][b:b + 1, :, hk:hk + 1], dk, "dK")
    H.check_grad(res["dv"][b:b + 1, :, hk:hk + 1], dv, "dV")
    again = H.run_dense(w, deterministic=True)
    assert torch.equal(res["dq"], again["dq"])
