"""Pins of the CPU oracle against facts fixed by the pages and by mathematics.

Nothing here compares the oracle with itself: each check is a hand-worked value,
a closed form, an invariant, a library routine the oracle does not use, or a
finite difference.  CPU only.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import BNPO, GRPO

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_tokens.txt")
EPS_LO, EPS_HI = 0.2, 0.28


def _one_token(ratio, A, two_sided, beta=0.0, ref_minus_lp=0.0):
    lp = torch.tensor([[-1.0]], dtype=torch.float64)
    old = lp - math.log(ratio)
    ref = lp + ref_minus_lp
    return oracle.policy_loss(lp, old, ref, torch.tensor([A], dtype=torch.float64),
                              torch.ones(1, 1, dtype=torch.int8), eps_lo=EPS_LO, eps_hi=EPS_HI,
                              beta=beta, reduction=BNPO, two_sided=two_sided)


def _golden_rows():
    rows = []
    with open(GOLDEN) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            r, a, form, pt, g = line.split()
            rows.append((float(r), float(a), form, float(pt), float(g)))
    return rows


@pytest.mark.parametrize("row", _golden_rows())
def test_hand_worked_tokens(row):
    r, A, form, pt, g = row
    for red in (BNPO, GRPO):  # one valid token: both reductions equal the token's term
        out = _one_token(r, A, form == "two_sided")
        assert out["loss"] == pytest.approx(pt, abs=1e-6)
        assert out["grad"][0, 0] == pytest.approx(g, abs=1e-6)
        assert out["n_valid"] == 1


def test_decode_binary16_all_codes():
    codes = np.arange(65536, dtype=np.uint16)
    want = codes.view(np.float16).astype(np.float64)
    got = oracle.decode(torch.from_numpy(codes.view(np.int16).copy()).view(torch.float16))
    finite = np.isfinite(want)
    assert np.array_equal(got[finite], want[finite])
    assert np.array_equal(np.isnan(got), np.isnan(want))
    assert np.array_equal(got[np.isinf(want)], want[np.isinf(want)])


def test_decode_bfloat16_all_codes():
    codes = torch.arange(-32768, 32768, dtype=torch.int32).to(torch.int16)
    t = codes.view(torch.bfloat16)
    want = (codes.to(torch.int32).bitwise_and(0xFFFF) << 16).numpy().astype(np.uint32).view(np.float32)
    want = want.astype(np.float64)
    got = oracle.decode(t)
    finite = np.isfinite(want)
    assert np.array_equal(got[finite], want[finite])
    assert np.array_equal(np.isnan(got), np.isnan(want))


def test_kl_zero_when_ref_equals_policy():
    out = _one_token(1.0, 0.0, False, beta=1.0, ref_minus_lp=0.0)
    assert out["loss"] == 0.0 and out["grad"][0, 0] == 0.0


def test_kl_at_ln2():
    # e = ref - lp = ln 2: kl = 2 - ln2 - 1 = 1 - ln 2, d kl / d lp = -(e^e - 1) = -1
    beta = 0.5
    out = _one_token(1.0, 0.0, False, beta=beta, ref_minus_lp=math.log(2.0))
    assert out["loss"] == pytest.approx(beta * 0.30685281944005469, abs=1e-15)
    assert out["grad"][0, 0] == pytest.approx(-beta, abs=1e-15)


def _rand_loss_inputs(bs, seq, seed, dtype=torch.float64, lens=None):
    g = torch.Generator().manual_seed(seed)
    lp = -2 * torch.randn(bs, seq, generator=g, dtype=torch.float64).abs()
    old = lp + 0.3 * torch.randn(bs, seq, generator=g, dtype=torch.float64)
    ref = lp + 0.2 * torch.randn(bs, seq, generator=g, dtype=torch.float64)
    adv = torch.randn(bs, generator=g, dtype=torch.float64)
    if lens is None:
        lens = torch.randint(1, seq + 1, (bs,), generator=g)
    mask = (torch.arange(seq)[None, :] < torch.as_tensor(lens)[:, None]).to(torch.int8)
    return lp.to(dtype), old.to(dtype), ref.to(dtype), adv.to(dtype), mask


@pytest.mark.parametrize("red", [BNPO, GRPO])
@pytest.mark.parametrize("two_sided", [False, True])
def test_beta_zero_ignores_ref(red, two_sided):
    lp, old, ref, adv, mask = _rand_loss_inputs(4, 33, 1)
    a = oracle.policy_loss(lp, old, ref, adv, mask, eps_lo=EPS_LO, eps_hi=EPS_HI, beta=0.0,
                           reduction=red, two_sided=two_sided)
    b = oracle.policy_loss(lp, old, None, adv, mask, eps_lo=EPS_LO, eps_hi=EPS_HI, beta=0.0,
                           reduction=red, two_sided=two_sided)
    c = oracle.policy_loss(lp, old, ref + 5.0, adv, mask, eps_lo=EPS_LO, eps_hi=EPS_HI,
                           beta=0.0, reduction=red, two_sided=two_sided)
    assert a["loss"] == b["loss"] == c["loss"]
    assert np.array_equal(a["grad"], b["grad"]) and np.array_equal(a["grad"], c["grad"])


@pytest.mark.parametrize("red", [BNPO, GRPO])
def test_all_masked_batch(red):
    lp, old, ref, adv, _ = _rand_loss_inputs(3, 17, 2)
    mask = torch.zeros(3, 17, dtype=torch.int8)
    out = oracle.policy_loss(lp, old, ref, adv, mask, eps_lo=EPS_LO, eps_hi=EPS_HI, beta=0.04,
                             reduction=red)
    assert out["loss"] == 0.0 and out["n_valid"] == 0
    assert np.all(out["grad"] == 0.0)


@pytest.mark.parametrize("red", [BNPO, GRPO])
def test_masked_tokens_have_zero_grad(red):
    lp, old, ref, adv, mask = _rand_loss_inputs(5, 29, 3)
    out = oracle.policy_loss(lp, old, ref, adv, mask, eps_lo=EPS_LO, eps_hi=EPS_HI, beta=0.04,
                             reduction=red)
    assert np.all(out["grad"][mask.numpy() == 0] == 0.0)
    # masked tokens do not influence the loss either
    lp2 = lp.clone()
    lp2[mask == 0] += 3.0
    out2 = oracle.policy_loss(lp2, old, ref, adv, mask, eps_lo=EPS_LO, eps_hi=EPS_HI, beta=0.04,
                              reduction=red)
    assert out2["loss"] == out["loss"]


def test_grpo_equals_bnpo_for_equal_lengths():
    lp, old, ref, adv, mask = _rand_loss_inputs(4, 20, 4, lens=[13, 13, 13, 13])
    a = oracle.policy_loss(lp, old, ref, adv, mask, eps_lo=EPS_LO, eps_hi=EPS_HI, beta=0.04,
                           reduction=BNPO)
    b = oracle.policy_loss(lp, old, ref, adv, mask, eps_lo=EPS_LO, eps_hi=EPS_HI, beta=0.04,
                           reduction=GRPO)
    assert a["loss"] == pytest.approx(b["loss"], rel=1e-13, abs=1e-15)
    np.testing.assert_allclose(a["grad"], b["grad"], rtol=1e-13, atol=0)


def test_ratio_one_closed_forms():
    # old == lp => ratio 1 (inside the clip band), beta = 0: per_token = -A.
    bs, seq = 6, 40
    lens = [0, 1, 7, 40, 23, 5]
    g = torch.Generator().manual_seed(5)
    lp = -torch.rand(bs, seq, generator=g, dtype=torch.float64)
    adv = torch.randn(bs, generator=g, dtype=torch.float64)
    mask = (torch.arange(seq)[None, :] < torch.tensor(lens)[:, None]).to(torch.int8)
    n = np.array(lens, dtype=np.float64)
    A = adv.numpy()
    bn = oracle.policy_loss(lp, lp, None, adv, mask, eps_lo=EPS_LO, eps_hi=EPS_HI, beta=0.0,
                            reduction=BNPO)
    assert bn["loss"] == pytest.approx(-(A * n).sum() / n.sum(), rel=1e-14)
    gr = oracle.policy_loss(lp, lp, None, adv, mask, eps_lo=EPS_LO, eps_hi=EPS_HI, beta=0.0,
                            reduction=GRPO)
    assert gr["loss"] == pytest.approx(-(A[n > 0]).sum() / bs, rel=1e-14)
    assert bn["n_valid"] == sum(lens) and list(gr["row_valid"]) == lens


def test_loss_linear_in_advantage_when_beta_zero():
    lp, old, ref, adv, mask = _rand_loss_inputs(4, 25, 6)
    for red in (BNPO, GRPO):
        a = oracle.policy_loss(lp, old, None, adv, mask, eps_lo=EPS_LO, eps_hi=EPS_HI, beta=0.0,
                               reduction=red)
        b = oracle.policy_loss(lp, old, None, 2.5 * adv, mask, eps_lo=EPS_LO, eps_hi=EPS_HI,
                               beta=0.0, reduction=red)
        assert b["loss"] == pytest.approx(2.5 * a["loss"], rel=1e-13)


def test_two_sided_matches_literal_for_nonnegative_advantage():
    lp, old, ref, adv, mask = _rand_loss_inputs(6, 31, 7)
    adv = adv.abs()
    for red in (BNPO, GRPO):
        a = oracle.policy_loss(lp, old, ref, adv, mask, eps_lo=EPS_LO, eps_hi=EPS_HI, beta=0.04,
                               reduction=red, two_sided=False)
        b = oracle.policy_loss(lp, old, ref, adv, mask, eps_lo=EPS_LO, eps_hi=EPS_HI, beta=0.04,
                               reduction=red, two_sided=True)
        assert a["loss"] == b["loss"]
        assert np.array_equal(a["grad"], b["grad"])


def _near_kink(lp, old, tol):
    hi = float(np.float32(1.0) + np.float32(EPS_HI))
    lo = float(np.float32(1.0) - np.float32(EPS_LO))
    r = np.exp(oracle.decode(lp) - oracle.decode(old))
    return np.any(np.abs(r - hi) < tol) or np.any(np.abs(r - lo) < tol)


@pytest.mark.parametrize("red", [BNPO, GRPO])
@pytest.mark.parametrize("two_sided", [False, True])
def test_loss_gradient_matches_finite_differences(red, two_sided):
    lp, old, ref, adv, mask = _rand_loss_inputs(3, 11, 8)
    assert not _near_kink(lp, old, 1e-4)
    kw = dict(eps_lo=EPS_LO, eps_hi=EPS_HI, beta=0.04, reduction=red, two_sided=two_sided)
    base = oracle.policy_loss(lp, old, ref, adv, mask, **kw)
    h = 1e-6
    fd = np.zeros_like(base["grad"])
    for b in range(3):
        for t in range(11):
            p, m = lp.clone(), lp.clone()
            p[b, t] += h
            m[b, t] -= h
            fd[b, t] = (oracle.policy_loss(p, old, ref, adv, mask, **kw)["loss"]
                        - oracle.policy_loss(m, old, ref, adv, mask, **kw)["loss"]) / (2 * h)
    np.testing.assert_allclose(base["grad"], fd, atol=1e-8, rtol=1e-6)


def test_logsumexp_against_brute_force():
    g = torch.Generator().manual_seed(9)
    N, H, V = 5, 64, 512
    X = torch.randn(N, H, generator=g, dtype=torch.float64)
    W = 0.3 * torch.randn(V, H, generator=g, dtype=torch.float64)
    b = 0.1 * torch.randn(V, generator=g, dtype=torch.float64)
    tg = torch.randint(0, V, (N,), generator=g)
    lse, logp, zt = oracle.lm_head_logprob(X, W, b, tg)
    z = (X.numpy() @ W.numpy().T + b.numpy()).astype(np.longdouble)
    brute = np.log(np.exp(z).sum(axis=1))
    np.testing.assert_allclose(lse, brute.astype(np.float64), rtol=0, atol=1e-12)
    want = torch.log_softmax(torch.from_numpy(z.astype(np.float64)), dim=1)[torch.arange(N), tg]
    np.testing.assert_allclose(logp, want.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(zt, z[np.arange(N), tg.numpy()].astype(np.float64), atol=1e-12)


def test_logprob_bf16_inputs_decoded_exactly():
    g = torch.Generator().manual_seed(10)
    X = torch.randn(3, 48, generator=g).to(torch.bfloat16)
    W = (0.5 * torch.randn(40, 48, generator=g)).to(torch.bfloat16)
    tg = torch.randint(0, 40, (3,), generator=g)
    a = oracle.lm_head_logprob(X, W, None, tg)
    b = oracle.lm_head_logprob(X.double(), W.double(), None, tg)
    for x, y in zip(a, b):
        np.testing.assert_allclose(x, y, rtol=0, atol=1e-13)


def _tiny_fused(seed, red, bias=True, beta=0.04):
    g = torch.Generator().manual_seed(seed)
    bs, T, H, V = 2, 3, 5, 7
    N = bs * T
    X = torch.randn(N, H, generator=g, dtype=torch.float64)
    W = 0.5 * torch.randn(V, H, generator=g, dtype=torch.float64)
    bvec = 0.1 * torch.randn(V, generator=g, dtype=torch.float64) if bias else None
    Xr = X + 0.05 * torch.randn(N, H, generator=g, dtype=torch.float64)
    Wr = W + 0.05 * torch.randn(V, H, generator=g, dtype=torch.float64)
    tg = torch.randint(0, V, (N,), generator=g)
    adv = torch.randn(bs, generator=g, dtype=torch.float64)
    mask = torch.tensor([[1, 1, 0], [1, 1, 1]], dtype=torch.int8)
    _, logp, _ = oracle.lm_head_logprob(X, W, bvec, tg)
    old = torch.from_numpy(logp) + 0.2 * torch.randn(N, generator=g, dtype=torch.float64)
    kw = dict(eps_lo=EPS_LO, eps_hi=EPS_HI, beta=beta, reduction=red)
    return dict(X=X, W=W, bias=bvec, targets=tg, Xref=Xr, Wref=Wr, old_lp=old.reshape(bs, T),
                adv=adv, mask=mask), kw


@pytest.mark.parametrize("red", [BNPO, GRPO])
@pytest.mark.parametrize("beta", [0.0, 0.04])
def test_fused_gradients_match_finite_differences(red, beta):
    inp, kw = _tiny_fused(11, red, beta=beta)
    base = oracle.fused_grpo(**inp, **kw)
    r = np.exp(base["logp"] - inp["old_lp"].reshape(-1).numpy())
    hi = float(np.float32(1.0) + np.float32(EPS_HI))
    assert np.all(np.abs(r - hi) > 1e-4)

    def loss_with(**over):
        d = dict(inp)
        d.update(over)
        return oracle.fused_grpo(**d, **kw, dx_rows=[], dw_rows=[])["loss"]

    h = 1e-6
    N, H = inp["X"].shape
    V = inp["W"].shape[0]
    fdX = np.zeros((N, H))
    for i in range(N):
        for k in range(H):
            p, m = inp["X"].clone(), inp["X"].clone()
            p[i, k] += h
            m[i, k] -= h
            fdX[i, k] = (loss_with(X=p) - loss_with(X=m)) / (2 * h)
    np.testing.assert_allclose(base["dX"], fdX, atol=1e-8, rtol=1e-5)
    fdW = np.zeros((V, H))
    for v in range(V):
        for k in range(H):
            p, m = inp["W"].clone(), inp["W"].clone()
            p[v, k] += h
            m[v, k] -= h
            fdW[v, k] = (loss_with(W=p) - loss_with(W=m)) / (2 * h)
    np.testing.assert_allclose(base["dW"], fdW, atol=1e-8, rtol=1e-5)
    fdb = np.zeros(V)
    for v in range(V):
        p, m = inp["bias"].clone(), inp["bias"].clone()
        p[v] += h
        m[v] -= h
        fdb[v] = (loss_with(bias=p) - loss_with(bias=m)) / (2 * h)
    np.testing.assert_allclose(base["dbias"], fdb, atol=1e-8, rtol=1e-5)
    # the per-row loss gradient matches a difference taken through the log-prob
    assert base["n_valid"] == 5


def test_fused_invariants():
    inp, kw = _tiny_fused(12, GRPO)
    out = oracle.fused_grpo(**inp, **kw)
    # sum_v dz[i, v] = g_i (1 - sum_v p_v) = 0  =>  columns of dW and dbias sum to 0
    np.testing.assert_allclose(out["dW"].sum(axis=0), 0.0, atol=1e-13)
    assert abs(out["dbias"].sum()) < 1e-13
    # masked row (sequence 0, position 2) has an exactly zero dX row and zero g
    assert out["g"][2] == 0.0 and np.all(out["dX"][2] == 0.0)


def test_fused_beta_zero_skips_reference():
    inp, kw = _tiny_fused(13, BNPO, beta=0.0)
    a = oracle.fused_grpo(**inp, **kw)
    inp2 = dict(inp, Xref=None, Wref=None)
    b = oracle.fused_grpo(**inp2, **kw)
    assert a["loss"] == b["loss"] and np.array_equal(a["dX"], b["dX"])


@pytest.mark.parametrize("tau", [0.6, 1.7])
def test_temperature_equals_scaled_weights(tau):
    # logits (X W^T + b) / tau are the logits of the weights W / tau and bias b / tau
    g = torch.Generator().manual_seed(21)
    X = torch.randn(6, 40, generator=g, dtype=torch.float64)
    W = 0.4 * torch.randn(90, 40, generator=g, dtype=torch.float64)
    b = 0.1 * torch.randn(90, generator=g, dtype=torch.float64)
    tg = torch.randint(0, 90, (6,), generator=g)
    lse_t, lp_t, zt_t = oracle.lm_head_logprob(X, W, b, tg, temperature=tau)
    lse_s, lp_s, zt_s = oracle.lm_head_logprob(X, W / tau, b / tau, tg)
    np.testing.assert_allclose(lp_t, lp_s, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse_t, lse_s, rtol=0, atol=1e-12)
    # temperature 1 is the untempered path
    a = oracle.lm_head_logprob(X, W, b, tg, temperature=1.0)
    c = oracle.lm_head_logprob(X, W, b, tg)
    for x, y in zip(a, c):
        assert np.array_equal(x, y)


@pytest.mark.parametrize("tau", [0.7, 1.5])
def test_tempered_gradients_match_finite_differences(tau):
    inp, kw = _tiny_fused(14, GRPO)
    base = oracle.fused_grpo(**inp, **kw, temperature=tau)
    r = np.exp(base["logp"] - inp["old_lp"].reshape(-1).numpy())
    hi = float(np.float32(1.0) + np.float32(EPS_HI))
    assert np.all(np.abs(r - hi) > 1e-4)

    def loss_with(**over):
        d = dict(inp)
        d.update(over)
        return oracle.fused_grpo(**d, **kw, dx_rows=[], dw_rows=[], temperature=tau)["loss"]

    h = 1e-6
    N, H = inp["X"].shape
    V = inp["W"].shape[0]
    for (name, t, grad) in (("X", inp["X"], base["dX"]), ("W", inp["W"], base["dW"])):
        fd = np.zeros(tuple(t.shape))
        for idx in np.ndindex(*t.shape):
            p, m = t.clone(), t.clone()
            p[idx] += h
            m[idx] -= h
            fd[idx] = (loss_with(**{name: p}) - loss_with(**{name: m})) / (2 * h)
        np.testing.assert_allclose(grad, fd, atol=1e-8, rtol=1e-5)
    fdb = np.zeros(V)
    for v in range(V):
        p, m = inp["bias"].clone(), inp["bias"].clone()
        p[v] += h
        m[v] -= h
        fdb[v] = (loss_with(bias=p) - loss_with(bias=m)) / (2 * h)
    np.testing.assert_allclose(base["dbias"], fdb, atol=1e-8, rtol=1e-5)


# ---- row groups of at most four rows ----
# The oracle's contractions take 32 rows per pass over a weight row and a short
# branch for a group of at most 4 rows: every N <= 4, and the remainder group of
# N = 33 and N = 36.  These pins reach that branch in the forward and in both
# halves of the backward.
SMALL_GROUP_N = [1, 2, 3, 4, 33, 36]


def _longdouble_logits(X, W, b):
    Xl = X.numpy().astype(np.longdouble)
    Wl = W.numpy().astype(np.longdouble)
    z = np.einsum("ih,vh->iv", Xl, Wl)  # a plain sum per element, no BLAS, in long double
    return z + b.numpy().astype(np.longdouble)


@pytest.mark.parametrize("N", SMALL_GROUP_N)
def test_small_row_groups_logprob_against_brute_force(N):
    g = torch.Generator().manual_seed(100 + N)
    H, V = 24, 300
    X = torch.randn(N, H, generator=g, dtype=torch.float64)
    W = 0.3 * torch.randn(V, H, generator=g, dtype=torch.float64)
    b = 0.1 * torch.randn(V, generator=g, dtype=torch.float64)
    tg = torch.randint(0, V, (N,), generator=g)
    lse, logp, zt = oracle.lm_head_logprob(X, W, b, tg)
    z = _longdouble_logits(X, W, b)
    brute = np.log(np.exp(z).sum(axis=1))
    rows = np.arange(N)
    np.testing.assert_allclose(lse, brute.astype(np.float64), rtol=0, atol=1e-12)
    np.testing.assert_allclose(zt, z[rows, tg.numpy()].astype(np.float64), rtol=0, atol=1e-12)
    np.testing.assert_allclose(logp, (z[rows, tg.numpy()] - brute).astype(np.float64), rtol=0, atol=1e-12)


@pytest.mark.parametrize("N", SMALL_GROUP_N)
def test_small_row_groups_backward_against_brute_force(N):
    # dz = g (onehot - softmax), dX = dz W, dW = dz^T X, dbias = column sums of dz,
    # each written out element by element in long double
    g = torch.Generator().manual_seed(200 + N)
    H, V = 16, 90
    X = torch.randn(N, H, generator=g, dtype=torch.float64)
    W = 0.3 * torch.randn(V, H, generator=g, dtype=torch.float64)
    b = 0.1 * torch.randn(V, generator=g, dtype=torch.float64)
    tg = torch.randint(0, V, (N,), generator=g)
    gv = torch.randn(N, generator=g, dtype=torch.float64).numpy()
    if N > 2:
        gv[N // 2] = 0.0  # a row with no gradient
    z = _longdouble_logits(X, W, b)
    lse = np.log(np.exp(z).sum(axis=1))
    onehot = np.zeros((N, V), dtype=np.longdouble)
    onehot[np.arange(N), tg.numpy()] = 1
    dz = gv.astype(np.longdouble)[:, None] * (onehot - np.exp(z - lse[:, None]))
    want_dX = np.einsum("iv,vh->ih", dz, W.numpy().astype(np.longdouble))
    want_dW = np.einsum("iv,ih->vh", dz, X.numpy().astype(np.longdouble))
    want_db = dz.sum(axis=0)
    dx_rows = np.arange(N)[::-1].copy()  # any order: rows are gathered by index
    dw_rows = np.array([0, 5, V - 1] + [int(t) for t in tg[:3]])
    dX, dW, db = oracle.lm_head_backward(X, W, b, tg, lse.astype(np.float64), gv, dx_rows, dw_rows)
    np.testing.assert_allclose(dX, want_dX[dx_rows].astype(np.float64), rtol=1e-11, atol=1e-14)
    np.testing.assert_allclose(dW, want_dW[dw_rows].astype(np.float64), rtol=1e-11, atol=1e-14)
    np.testing.assert_allclose(db, want_db[dw_rows].astype(np.float64), rtol=1e-11, atol=1e-14)


@pytest.mark.parametrize("N", SMALL_GROUP_N)
def test_small_row_groups_fused_gradients_match_finite_differences(N):
    bs = {1: 1, 2: 1, 3: 1, 4: 2, 33: 3, 36: 4}[N]
    T = N // bs
    g = torch.Generator().manual_seed(300 + N)
    H, V = 4, 6
    X = torch.randn(N, H, generator=g, dtype=torch.float64)
    W = 0.5 * torch.randn(V, H, generator=g, dtype=torch.float64)
    bvec = 0.1 * torch.randn(V, generator=g, dtype=torch.float64)
    Xr = X + 0.05 * torch.randn(N, H, generator=g, dtype=torch.float64)
    Wr = W + 0.05 * torch.randn(V, H, generator=g, dtype=torch.float64)
    tg = torch.randint(0, V, (N,), generator=g)
    adv = torch.randn(bs, generator=g, dtype=torch.float64)
    mask = torch.ones(bs, T, dtype=torch.int8)
    if T > 1:
        mask[0, T - 1] = 0
    _, logp, _ = oracle.lm_head_logprob(X, W, bvec, tg)
    old = torch.from_numpy(logp) + 0.2 * torch.randn(N, generator=g, dtype=torch.float64)
    # keep every ratio clear of the kink at 1 + eps_hi (finite differences straddle it otherwise)
    ln_hi = math.log(float(np.float32(1.0) + np.float32(EPS_HI)))
    d = torch.from_numpy(logp) - old - ln_hi
    old[d.abs() < 1e-3] -= 2e-3
    inp = dict(X=X, W=W, bias=bvec, targets=tg, Xref=Xr, Wref=Wr, old_lp=old.reshape(bs, T), adv=adv, mask=mask)
    kw = dict(eps_lo=EPS_LO, eps_hi=EPS_HI, beta=0.04, reduction=GRPO)
    base = oracle.fused_grpo(**inp, **kw)

    def loss_with(**over):
        dd = dict(inp)
        dd.update(over)
        return oracle.fused_grpo(**dd, **kw, dx_rows=[], dw_rows=[])["loss"]

    h = 1e-6
    for name, grad in (("X", base["dX"]), ("W", base["dW"]), ("bias", base["dbias"])):
        t = inp[name]
        fd = np.zeros(tuple(t.shape))
        for idx in np.ndindex(*t.shape):
            p, m = t.clone(), t.clone()
            p[idx] += h
            m[idx] -= h
            fd[idx] = (loss_with(**{name: p}) - loss_with(**{name: m})) / (2 * h)
        np.testing.assert_allclose(grad, fd, atol=1e-8, rtol=1e-5, err_msg=name)
