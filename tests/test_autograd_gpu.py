"""The autograd-aware wrappers: loss.backward() through the fused loss kernel
and through the fused selective log-prob, against the C entry points and the
CPU oracle."""
import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("which", ["bnpo", "grpo"])
@pytest.mark.parametrize("outer", [1.0, -2.5])
def test_loss_autograd_matches_direct_kernel(which, outer):
    from rl_post_policy_b200 import autograd as ag
    import rl_post_policy_b200 as pl
    inp = synth.loss_inputs(8, 256, torch.float32, 901)
    dt = torch.bfloat16
    lp = inp["policy_lp"].to(dt).cuda().requires_grad_(True)
    old, ref = inp["old_lp"].to(dt).cuda(), inp["ref_lp"].to(dt).cuda()
    adv, mask = inp["adv"].cuda(), inp["mask"].cuda()
    f = ag.bnpo_loss_autograd if which == "bnpo" else ag.grpo_loss_autograd
    loss = f(lp, old, ref, adv, mask, epsilon=0.2, epsilon_high=0.28, beta=0.04)
    (outer * loss).backward()
    want = oracle.policy_loss(inp["policy_lp"].to(dt), inp["old_lp"].to(dt), inp["ref_lp"].to(dt),
                              inp["adv"], inp["mask"], eps_lo=0.2, eps_hi=0.28, beta=0.04,
                              reduction=0 if which == "bnpo" else 1)
    assert abs(loss.item() - want["loss"]) <= 1e-3 * abs(want["loss"])
    # direct entry point on the same inputs: same kernel, gradient scaled by `outer`
    g = torch.empty_like(lp)
    l2 = torch.empty(1, device="cuda")
    wsb = pl.pl_loss_workspace_bytes(8, 256)
    ws = torch.zeros(wsb, dtype=torch.uint8, device="cuda")
    pl.check(pl.pl_loss_ex(lp.detach(), old, ref, adv, mask, 8, 256, 0.2, 0.28, 0.04,
                           pl.PL_BF16 | (pl.PL_BNPO if which == "bnpo" else pl.PL_GRPO), l2, g, None, None,
                           ws, wsb))
    ref_grad = (g.float() * outer).to(dt)
    assert torch.equal(lp.grad, ref_grad)


def test_selective_logprob_autograd():
    from rl_post_policy_b200 import autograd as ag
    inp = synth.fused_inputs(2, 64, 128, 700, torch.bfloat16, 902, bias=True, need_ref=False)
    X = inp["X"].cuda().requires_grad_(True)
    W = inp["W"].cuda().requires_grad_(True)
    b = inp["bias"].cuda().requires_grad_(True)
    tg = inp["targets"].cuda()
    logp = ag.fused_selective_logprob(X, W, tg, bias=b)
    c = synth.normal((128,), 903, std=1e-2).cuda()
    (logp * c).sum().backward()
    lse, want_lp, _ = oracle.lm_head_logprob(inp["X"], inp["W"], inp["bias"], inp["targets"])
    assert np.max(np.abs(logp.detach().cpu().double().numpy() - want_lp)) <= 2e-3
    wX, wW, wb = oracle.lm_head_backward(inp["X"], inp["W"], inp["bias"], inp["targets"], lse,
                                         c.cpu().double().numpy(), np.arange(128), np.arange(700))

    def rel(a, w):
        a = a.detach().cpu().double().numpy()
        return np.linalg.norm(a - w) / np.linalg.norm(w)

    assert rel(X.grad, wX) <= 1e-2
    assert rel(W.grad, wW) <= 1e-2
    assert rel(b.grad, wb) <= 1e-2
