"""Pins for the oracle's reverse-KL self-distillation ("Geometric-AI Kernels",
section "Reverse KL"): closed forms, an independent library route, invariants
and finite differences.  No GPU."""
import math

import numpy as np
import pytest
import scipy.special as sp
import torch

import oracle


def test_two_logit_closed_form():
    # p = (1/4, 3/4) from logits (0, ln 3); q uniform: KL = 3/4 ln(3/2) - 1/4 ln 2
    s = torch.tensor([[0.0, math.log(3.0)]], dtype=torch.float64)
    t = torch.zeros(1, 2, dtype=torch.float64)
    out = oracle.reverse_kl(s, t)
    want = 0.75 * math.log(1.5) - 0.25 * math.log(2.0)
    assert abs(out["loss"] - want) < 1e-15
    # d KL / d s_1 for two logits: p1 p0 (log(p1/q1) - log(p0/q0)) = 3/16 ln 3
    assert abs(out["grad"][0, 1] - 3.0 / 16.0 * math.log(3.0)) < 1e-15
    assert abs(out["grad"][0, 0] + 3.0 / 16.0 * math.log(3.0)) < 1e-15


def test_matches_scipy_relative_entropy():
    rng = np.random.default_rng(3)
    s = rng.normal(0, 2, (6, 97))
    t = rng.normal(0, 2, (6, 97))
    out = oracle.reverse_kl(torch.from_numpy(s), torch.from_numpy(t), want_grad=False)
    want = sp.rel_entr(sp.softmax(s, axis=1), sp.softmax(t, axis=1)).sum(axis=1)
    assert np.allclose(out["kl_rows"], want, rtol=1e-12, atol=1e-14)
    assert abs(out["loss"] - want.mean()) < 1e-12


def test_uniform_teacher_is_log_v_minus_entropy():
    rng = np.random.default_rng(4)
    s = rng.normal(0, 1, (3, 50))
    out = oracle.reverse_kl(torch.from_numpy(s), torch.full((3, 50), 0.7, dtype=torch.float64))
    p = sp.softmax(s, axis=1)
    assert np.allclose(out["kl_rows"], math.log(50) + (p * np.log(p)).sum(axis=1), rtol=1e-12)


def test_shift_invariance_and_identity():
    rng = np.random.default_rng(5)
    s = torch.from_numpy(rng.normal(0, 1, (4, 33)))
    t = torch.from_numpy(rng.normal(0, 1, (4, 33)))
    a = oracle.reverse_kl(s, t)
    b = oracle.reverse_kl(s + torch.tensor([[3.0], [-7.0], [0.5], [11.0]], dtype=torch.float64),
                          t + torch.tensor([[-2.0], [1.0], [40.0], [0.0]], dtype=torch.float64))
    assert np.allclose(a["kl_rows"], b["kl_rows"], rtol=1e-10)
    assert np.allclose(a["grad"], b["grad"], rtol=1e-9, atol=1e-15)
    same = oracle.reverse_kl(s, s.clone())
    assert same["loss"] == 0.0 and np.all(same["kl_rows"] == 0.0) and np.all(same["grad"] == 0.0)
    assert np.all(a["kl_rows"] > 0.0)   # Gibbs' inequality


def test_gradient_matches_finite_differences_and_sums_to_zero():
    rng = np.random.default_rng(6)
    s = rng.normal(0, 1.5, (3, 7))
    t = rng.normal(0, 1.5, (3, 7))
    mask = torch.tensor([1, 0, 1], dtype=torch.uint8)
    g = oracle.reverse_kl(torch.from_numpy(s), torch.from_numpy(t), mask)["grad"]
    h = 1e-6
    for r in range(3):
        for v in range(7):
            sp_, sm_ = s.copy(), s.copy()
            sp_[r, v] += h
            sm_[r, v] -= h
            lp = oracle.reverse_kl(torch.from_numpy(sp_), torch.from_numpy(t), mask, want_grad=False)["loss"]
            lm = oracle.reverse_kl(torch.from_numpy(sm_), torch.from_numpy(t), mask, want_grad=False)["loss"]
            assert abs((lp - lm) / (2 * h) - g[r, v]) < 1e-8, (r, v)
    assert np.all(g[1] == 0.0)
    assert np.allclose(g.sum(axis=1), 0.0, atol=1e-15)


def test_mask_mean_and_all_masked():
    rng = np.random.default_rng(7)
    s = torch.from_numpy(rng.normal(0, 1, (2, 3, 11)))
    t = torch.from_numpy(rng.normal(0, 1, (2, 3, 11)))
    m = torch.tensor([[1, 1, 0], [0, 1, 0]], dtype=torch.bool)
    out = oracle.reverse_kl(s, t, m)
    assert out["n_valid"] == 3
    assert abs(out["loss"] - out["kl_rows"][m.numpy()].mean()) < 1e-14
    none = oracle.reverse_kl(s, t, torch.zeros(2, 3, dtype=torch.bool))
    assert none["loss"] == 0.0 and none["n_valid"] == 0 and np.all(none["grad"] == 0.0)
    full = oracle.reverse_kl(s, t, None)
    assert full["n_valid"] == 6 and abs(full["loss"] - full["kl_rows"].mean()) < 1e-14


@pytest.mark.parametrize("dt", [torch.bfloat16, torch.float16, torch.float32])
def test_low_precision_inputs_are_decoded_exactly(dt):
    g = torch.Generator().manual_seed(8)
    s = torch.randn(5, 40, generator=g).to(dt)
    t = torch.randn(5, 40, generator=g).to(dt)
    a = oracle.reverse_kl(s, t)
    b = oracle.reverse_kl(s.double(), t.double())
    assert a["loss"] == b["loss"] and np.array_equal(a["grad"], b["grad"])
