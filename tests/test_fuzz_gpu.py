"""Property-based parity with the oracle over random shapes and settings
(hypothesis, derandomized so every run draws the same examples).

Loss-only kernel: bs, seq, dtype, reduction, beta, clip form, clip bounds,
advantage dtype, arbitrary (non-prefix) masks and misaligned pointers.  Fused
linear path: batch and sequence sizes, hidden sizes down to one 16-byte row,
vocabularies smaller than one tile and ragged ones, bias, beta, reduction and
chunking.  Reverse KL: rows (across several 512-row blocks of the row
dealing), vocabulary sizes, dtypes, mask densities including none and all,
cluster sizes and the forward-only form.  Tolerances as in the dedicated
tests; tokens within rounding of a clip bound may take either side of the
min() and are left out of the element-wise loss-gradient comparison
(loss-only) or moved off the bound in the input recipe (fused).
"""
import numpy as np
import pytest
import torch
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

import oracle
import synth

pytestmark = pytest.mark.gpu

SETTINGS = dict(max_examples=50, derandomize=True, deadline=None,
                suppress_health_check=[HealthCheck.too_slow, HealthCheck.function_scoped_fixture])


def _ulp(x, dtype):
    mant, emin = {torch.bfloat16: (7, -126), torch.float16: (10, -14)}[dtype]
    e = np.maximum(np.floor(np.log2(np.where(np.abs(x) > 0, np.abs(x), 1.0))), emin)
    return np.exp2(e - mant)


@settings(**SETTINGS)
@given(bs=st.integers(1, 40), seq=st.integers(1, 700),
       dtype=st.sampled_from([torch.bfloat16, torch.float16, torch.float32]),
       red=st.sampled_from([0, 1]), beta=st.sampled_from([0.0, 0.04, 0.3]), two_sided=st.booleans(),
       eps_lo=st.sampled_from([0.1, 0.2]), eps_hi=st.sampled_from([0.2, 0.28]), adv_lp=st.booleans(),
       offset=st.sampled_from([0, 1]), seed=st.integers(0, 2 ** 20), keep=st.floats(0.0, 1.0))
def test_loss_kernel_random_settings(bs, seq, dtype, red, beta, two_sided, eps_lo, eps_hi, adv_lp, offset, seed,
                                     keep):
    import rl_post_policy_b200 as pl
    # alternate the two loss kernels (every drawn size here is small enough for either)
    assert pl.pl_debug_set_loss_path(1 + (seed & 1)) == 0
    dev = torch.device("cuda")
    inp = synth.loss_inputs(bs, seq, torch.float32, seed, len_lo=1, len_hi=seq)
    g = torch.Generator().manual_seed(seed + 1)
    inp["mask"] = (torch.rand(bs, seq, generator=g) < keep).to(torch.int8)   # arbitrary, not a prefix

    def up(t, dt=None):
        t = t.to(dt) if dt is not None else t
        buf = torch.empty(t.numel() + offset, dtype=t.dtype, device=dev)
        v = buf[offset:].view(t.shape)
        v.copy_(t)
        return v

    def want_for(a):
        return oracle.policy_loss(inp["policy_lp"].to(dtype), inp["old_lp"].to(dtype),
                                  inp["ref_lp"].to(dtype) if beta != 0 else None,
                                  a.to(dtype) if adv_lp else a, inp["mask"], eps_lo=eps_lo,
                                  eps_hi=eps_hi, beta=beta, reduction=red, two_sided=two_sided)

    want = want_for(inp["adv"])
    if abs(want["loss"]) < 0.05 * want["abs_sum"]:
        # +/-A cancellation brought the loss near zero, where a relative error says
        # nothing: draw same-sign advantages instead (the input recipe, not the bound)
        inp["adv"] = inp["adv"].abs() + 0.1
        want = want_for(inp["adv"])
    lp, old = up(inp["policy_lp"], dtype), up(inp["old_lp"], dtype)
    ref = up(inp["ref_lp"], dtype) if beta != 0.0 else None
    adv = up(inp["adv"], dtype if adv_lp else torch.float32)
    mask = up(inp["mask"])
    loss = torch.full((1,), float("nan"), device=dev)
    grad = torch.full((bs, seq), float("nan"), dtype=dtype, device=dev)
    nv = torch.full((1,), -1, dtype=torch.int64, device=dev)
    wsb = pl.pl_loss_workspace_bytes(bs, seq)
    ws = torch.zeros(wsb, dtype=torch.uint8, device=dev)
    mode = pl.dtype_mode(dtype) | red | (pl.PL_CLIP_TWO_SIDED if two_sided else 0) | (pl.PL_ADV_LP_DTYPE if adv_lp else 0)
    pl.check(pl.pl_loss_ex(lp, old, ref, adv, mask, bs, seq, eps_lo, eps_hi, beta, mode, loss, grad, nv, None,
                           ws, wsb))
    torch.cuda.synchronize()
    assert pl.pl_device_status(ws) == 0

    assert int(nv.item()) == want["n_valid"]
    tol = 1e-5 if dtype == torch.float32 else 1e-3
    if want["loss"] == 0.0:
        assert loss.item() == 0.0
    else:
        assert abs(loss.item() - want["loss"]) <= tol * abs(want["loss"])
    # gradient element by element, except within rounding of a clip bound
    lpd, oldd = oracle.decode(inp["policy_lp"].to(dtype)), oracle.decode(inp["old_lp"].to(dtype))
    r = np.exp(lpd - oldd)
    lo_b, hi_b = float(np.float32(1) - np.float32(eps_lo)), float(np.float32(1) + np.float32(eps_hi))
    kink = (np.abs(r - hi_b) <= 8 * np.spacing(np.float32(hi_b))) | (np.abs(r - lo_b) <= 8 * np.spacing(np.float32(lo_b)))
    gg = grad.float().cpu().double().numpy()
    w = want["grad"]
    if dtype == torch.float32:
        err, bound = np.abs(gg - w), 1e-6
    else:
        wr = torch.from_numpy(w).to(dtype).double().numpy()
        err, bound = np.abs(gg - wr) / _ulp(wr, dtype), 1.0
    bad = (err > bound) & ~kink
    assert not bad.any(), (int(bad.sum()), float(err[~kink].max()))
    pl.pl_debug_set_loss_path(0)


@settings(**SETTINGS)
@given(bs=st.integers(1, 3), T=st.integers(1, 150), H=st.sampled_from([8, 64, 136, 200]),
       V=st.integers(10, 1500), dtype=st.sampled_from([torch.bfloat16, torch.float16]), bias=st.booleans(),
       beta=st.sampled_from([0.0, 0.04]), red=st.sampled_from([0, 1]), chunk=st.sampled_from([None, 128]),
       seed=st.integers(0, 2 ** 20))
def test_fused_path_random_shapes(bs, T, H, V, dtype, bias, beta, red, chunk, seed):
    import rl_post_policy_b200 as pl
    dev = "cuda"
    N = bs * T
    inp = synth.fused_inputs(bs, T, H, V, dtype, seed, bias=bias, len_lo=0, len_hi=T, need_ref=True)
    _, logp, _ = oracle.lm_head_logprob(inp["X"], inp["W"], inp["bias"], inp["targets"])
    old = torch.from_numpy(logp) + inp["old_noise"].double()
    for bound in (np.log(float(np.float32(1) + np.float32(0.28))), np.log(float(np.float32(1) - np.float32(0.2)))):
        d = torch.from_numpy(logp) - old - bound
        near = d.abs() < 2e-4
        old[near] -= torch.where(d[near] >= 0, 2e-4, -2e-4).double()
    inp["old_lp"] = old.float()

    def want_for(a):
        return oracle.fused_grpo(inp["X"], inp["W"], inp["bias"], inp["targets"], inp["Xref"], inp["Wref"],
                                 inp["old_lp"].reshape(bs, T), a, inp["mask"], eps_lo=0.2, eps_hi=0.28,
                                 beta=beta, reduction=red)

    want = want_for(inp["adv"])
    if abs(want["loss"]) < 0.05 * want["abs_sum"]:
        # +/-A cancellation brought the loss near zero: same-sign advantages instead
        inp["adv"] = inp["adv"].abs() + 0.1
        want = want_for(inp["adv"])
    g = {k: (inp[k].to(dev) if inp.get(k) is not None else None)
         for k in ("X", "W", "bias", "targets", "Xref", "Wref", "old_lp", "adv", "mask")}
    if beta == 0:
        g["Xref"] = g["Wref"] = None
    loss = torch.full((1,), float("nan"), device=dev)
    dX = torch.full((N, H), float("nan"), dtype=dtype, device=dev)
    dW = torch.full((V, H), float("nan"), dtype=dtype, device=dev)
    db = torch.full((V,), float("nan"), dtype=dtype, device=dev) if bias else None
    lp = torch.empty(N, device=dev)
    nv = torch.zeros(1, dtype=torch.int64, device=dev)
    mode = pl.dtype_mode(dtype) | red | (pl.PL_CHUNK_ROWS(chunk) if chunk else 0)
    wsb = pl.pl_fused_linear_grpo_workspace_bytes(bs, T, H, V, mode, 1, int(bias))
    ws = torch.zeros(wsb, dtype=torch.uint8, device=dev)
    pl.check(pl.pl_fused_linear_grpo(g["X"], g["W"], g["bias"], g["targets"], g["Xref"], g["Wref"], g["old_lp"],
                                     g["adv"], g["mask"], bs, T, H, V, 0.2, 0.28, beta, mode, loss, dX, dW, db, lp,
                                     None, nv, ws, wsb))
    torch.cuda.synchronize()
    assert pl.pl_device_status(ws) == 0
    assert int(nv.item()) == want["n_valid"]
    assert np.max(np.abs(lp.cpu().double().numpy() - want["logp"])) <= 2e-3
    if want["loss"] == 0.0:
        assert loss.item() == 0.0
    else:
        assert abs(loss.item() - want["loss"]) <= 1e-3 * abs(want["loss"])

    def rel(a, w):
        a = a.float().cpu().double().numpy()
        nw = np.linalg.norm(w)
        return np.linalg.norm(a - w) / nw if nw > 0 else np.linalg.norm(a)

    for k, t in (("dX", dX), ("dW", dW), ("dbias", db)):
        if t is not None:
            assert rel(t, want[k]) <= 1e-2, k


@settings(**dict(SETTINGS, max_examples=40))
@given(N=st.integers(1, 1400), V=st.integers(1, 2500),
       dtype=st.sampled_from([torch.bfloat16, torch.float16, torch.float32]),
       keep=st.sampled_from([0.0, 0.05, 0.5, 0.9, 1.0, None]), cl=st.sampled_from([0, 1, 2, 4, 8]),
       grad=st.booleans(), seed=st.integers(0, 2 ** 20))
def test_reverse_kl_random_shapes(N, V, dtype, keep, cl, grad, seed):
    # valid rows are dealt to the clusters by their rank among the valid rows, in
    # blocks of 512 rows, and masked rows after them: any count, density and order
    import rl_post_policy_b200 as pl
    dev = torch.device("cuda")
    inp = synth.reverse_kl_inputs(1, N, V, dtype, seed)
    s, t = inp["student"].reshape(N, V), inp["teacher"].reshape(N, V)
    if keep is None:
        mask = None
    else:
        g = torch.Generator().manual_seed(seed + 7)
        mask = (torch.rand(N, generator=g) < keep).to(torch.uint8)
    want = oracle.reverse_kl(s, t, mask, want_grad=grad)
    assert pl.pl_debug_set_rkl_cluster(cl) == 0
    try:
        S, T = s.to(dev), t.to(dev)
        G = torch.full_like(S, float("nan")) if grad else None
        M = mask.to(dev) if mask is not None else None
        loss = torch.full((1,), float("nan"), device=dev)
        kl = torch.full((N,), float("nan"), device=dev)
        nv = torch.full((1,), -1, dtype=torch.int64, device=dev)
        wsb = pl.pl_reverse_kl_workspace_bytes(N, V)
        ws = torch.zeros(wsb, dtype=torch.uint8, device=dev)
        pl.check(pl.pl_reverse_kl(S, T, M, N, V, pl.dtype_mode(dtype), loss, G, kl, nv, ws, wsb))
        torch.cuda.synchronize()
        assert pl.pl_device_status(ws) == 0
    finally:
        pl.pl_debug_set_rkl_cluster(0)
    valid = np.ones(N, bool) if mask is None else mask.numpy() != 0
    assert int(nv.item()) == int(valid.sum())
    wl = float(want["loss"])
    assert abs(loss.item() - wl) <= 1e-4 * abs(wl) + 1e-7, (loss.item(), wl)
    wk = np.asarray(want["kl_rows"]).reshape(-1)
    gk = kl.cpu().double().numpy()
    assert np.all(np.abs(gk[valid] - wk[valid]) <= 1e-5 + 1e-4 * np.abs(wk[valid]))
    assert np.all(gk[~valid] == 0.0)
    if grad:
        gg = G.float().cpu().double().numpy()
        wg = np.asarray(want["grad"]).reshape(N, V)
        err = np.linalg.norm(gg - wg) / max(np.linalg.norm(wg), 1e-300)
        assert err <= (1e-4 if dtype == torch.float32 else 1e-2), err
        assert np.all(gg[~valid] == 0.0)
