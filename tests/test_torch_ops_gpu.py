"""The custom operators (rl_post_policy_b200.torch_ops) on the GPU: eager
results equal the autograd.Function wrappers bit for bit (same kernels), the
oracle agrees within the usual tolerances, torch.compile(fullgraph=True)
traces them without graph breaks and reproduces the eager values, and
torch.library.opcheck accepts their schemas, shape functions and autograd
registrations."""
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu


def _loss_inputs(dt):
    inp = synth.loss_inputs(6, 200, torch.float32, 1717, len_lo=1, len_hi=200)
    lp = inp["policy_lp"].to(dt).cuda()
    old, ref = inp["old_lp"].to(dt).cuda(), inp["ref_lp"].to(dt).cuda()
    return inp, lp, old, ref, inp["adv"].cuda(), inp["mask"].cuda()


@pytest.mark.parametrize("which", ["bnpo", "grpo"])
def test_policy_loss_op_eager_and_compiled(which):
    from rl_post_policy_b200 import autograd as ag
    from rl_post_policy_b200 import torch_ops as ops
    inp, lp, old, ref, adv, mask = _loss_inputs(torch.bfloat16)
    f_op = ops.bnpo_loss if which == "bnpo" else ops.grpo_loss
    f_ag = ag.bnpo_loss_autograd if which == "bnpo" else ag.grpo_loss_autograd
    kw = dict(epsilon=0.2, epsilon_high=0.28, beta=0.04)

    def run(f):
        x = lp.clone().requires_grad_(True)
        loss = f(x, old, ref, adv, mask, **kw)
        (-1.5 * loss).backward()
        return loss.detach(), x.grad

    l_op, g_op = run(f_op)
    l_ag, g_ag = run(f_ag)
    assert torch.equal(l_op.reshape(1), l_ag.reshape(1)) and torch.equal(g_op, g_ag)
    want = oracle.policy_loss(inp["policy_lp"].to(torch.bfloat16), inp["old_lp"].to(torch.bfloat16),
                              inp["ref_lp"].to(torch.bfloat16), inp["adv"], inp["mask"], eps_lo=0.2, eps_hi=0.28,
                              beta=0.04, reduction=0 if which == "bnpo" else 1)
    # these inputs keep the loss well away from a +/-A cancellation (|loss| > 0.1 sum|terms|),
    # so the plain relative bound of bf16 inputs applies
    assert abs(want["loss"]) > 0.1 * want["abs_sum"]
    assert abs(l_op.item() - want["loss"]) <= 1e-3 * abs(want["loss"])

    torch._dynamo.reset()
    compiled = torch.compile(lambda *a, **k: f_op(*a, **k), backend="aot_eager", fullgraph=True)
    l_c, g_c = run(compiled)
    assert torch.equal(l_c.reshape(1), l_op.reshape(1)) and torch.equal(g_c, g_op)


def test_reverse_kl_op_eager_and_compiled():
    from rl_post_policy_b200 import autograd as ag
    from rl_post_policy_b200 import torch_ops as ops
    inp = synth.reverse_kl_inputs(2, 9, 3000, torch.bfloat16, synth.seed_for(48))
    s, t, m = inp["student"].cuda(), inp["teacher"].cuda(), inp["mask"].cuda()

    def run(f):
        x = s.clone().requires_grad_(True)
        loss = f(x, t, m)
        (0.5 * loss).backward()
        return loss.detach(), x.grad

    l_op, g_op = run(ops.reverse_kl_loss)
    l_ag, g_ag = run(ag.reverse_kl_autograd)
    assert torch.equal(l_op.reshape(1), l_ag.reshape(1)) and torch.equal(g_op, g_ag)
    want = oracle.reverse_kl(inp["student"], inp["teacher"], inp["mask"])
    assert abs(l_op.item() - want["loss"]) <= 1e-4 * abs(want["loss"]) + 1e-7
    torch._dynamo.reset()
    l_c, g_c = run(torch.compile(ops.reverse_kl_loss, backend="aot_eager", fullgraph=True))
    assert torch.equal(l_c.reshape(1), l_op.reshape(1)) and torch.equal(g_c, g_op)


@pytest.mark.parametrize("bias", [False, True])
def test_selective_logprob_op_eager_and_compiled(bias):
    from rl_post_policy_b200 import autograd as ag
    from rl_post_policy_b200 import torch_ops as ops
    inp = synth.fused_inputs(2, 40, 64, 700, torch.bfloat16, 3131, bias=bias, need_ref=False)
    X, W = inp["X"].cuda(), inp["W"].cuda()
    b = inp["bias"].cuda() if bias else None
    tg = inp["targets"].cuda()
    w_out = torch.linspace(-1, 1, X.shape[0], device="cuda")

    def run(f):
        x, w = X.clone().requires_grad_(True), W.clone().requires_grad_(True)
        bb = b.clone().requires_grad_(True) if b is not None else None
        logp = f(x, w, tg, bias=bb)
        (logp * w_out).sum().backward()
        return logp.detach(), x.grad, w.grad, (bb.grad if bb is not None else None)

    r_op = run(ops.selective_logprob)
    r_ag = run(ag.fused_selective_logprob)
    for a_, b_ in zip(r_op, r_ag):
        assert (a_ is None and b_ is None) or torch.equal(a_, b_)
    torch._dynamo.reset()
    r_c = run(torch.compile(ops.selective_logprob, backend="aot_eager", fullgraph=True))
    for a_, b_ in zip(r_c, r_op):
        assert (a_ is None and b_ is None) or torch.equal(a_, b_)


def test_opcheck():
    from rl_post_policy_b200 import torch_ops  # noqa: F401
    ops = torch.ops.rl_post_policy_b200
    _, lp, old, ref, adv, mask = _loss_inputs(torch.float32)
    lp.requires_grad_(True)
    torch.library.opcheck(ops.policy_loss.default, (lp, old, ref, adv, mask, 0.2, 0.28, 0.04, 1, False),
                          test_utils=("test_schema", "test_faketensor", "test_autograd_registration"))
    s = torch.randn(5, 300, device="cuda", requires_grad=True)
    torch.library.opcheck(ops.reverse_kl.default, (s, torch.randn(5, 300, device="cuda"), None),
                          test_utils=("test_schema", "test_faketensor", "test_autograd_registration"))
    x = torch.randn(4, 8, device="cuda", dtype=torch.bfloat16)
    torch.library.opcheck(ops.scale.default, (x, torch.tensor([0.5], device="cuda")),
                          test_utils=("test_schema", "test_faketensor"))


@pytest.mark.parametrize("chunk", [0, 64], ids=["one_chunk", "chunks64"])
def test_fused_linear_grpo_autograd_and_op(chunk):
    # loss.backward() through the fused linear path: the gradients equal the
    # direct entry point's scaled by the outer factor, for the autograd.Function
    # and the custom operator alike, eager and compiled
    import rl_post_policy_b200 as pl
    from rl_post_policy_b200 import autograd as ag
    from rl_post_policy_b200 import torch_ops as ops
    bs, T, H, V = 2, 96, 64, 700
    inp = synth.fused_inputs(bs, T, H, V, torch.bfloat16, 6262, bias=True, need_ref=True)
    inp["old_lp"] = (inp["old_noise"] - 6.5).float()
    g = {k: v.cuda() for k, v in inp.items() if isinstance(v, torch.Tensor)}
    kw = dict(bias=None, Xref=g["Xref"], Wref=g["Wref"], epsilon=0.2, epsilon_high=0.28, beta=0.04,
              reduction="bnpo", temperature=0.9, chunk_rows=chunk)
    outer = -0.75

    def run(f):
        x, w = g["X"].clone().requires_grad_(True), g["W"].clone().requires_grad_(True)
        b = g["bias"].clone().requires_grad_(True)
        loss = f(x, w, g["targets"], g["old_lp"], g["adv"], g["mask"], **dict(kw, bias=b))
        (outer * loss).backward()
        return loss.detach().reshape(1), x.grad, w.grad, b.grad

    # the direct entry point, unscaled
    N = bs * T
    mode = pl.PL_BF16 | pl.PL_BNPO | (pl.PL_CHUNK_ROWS(chunk) if chunk else 0)
    loss = torch.empty(1, device="cuda")
    dX, dW, db = torch.empty_like(g["X"]), torch.empty_like(g["W"]), torch.empty_like(g["bias"])
    wsb = pl.pl_fused_linear_grpo_workspace_bytes(bs, T, H, V, mode, 1, 1)
    ws = torch.zeros(wsb, dtype=torch.uint8, device="cuda")
    pl.check(pl.pl_fused_linear_grpo_temp(g["X"], g["W"], g["bias"], g["targets"], g["Xref"], g["Wref"],
                                          g["old_lp"], g["adv"], g["mask"], bs, T, H, V, 0.2, 0.28, 0.04, 0.9, mode,
                                          loss, dX, dW, db, None, None, None, ws, wsb))
    want = (loss, (dX.float() * outer).to(dX.dtype), (dW.float() * outer).to(dW.dtype),
            (db.float() * outer).to(db.dtype))
    for f in (ag.fused_linear_grpo_loss, ops.fused_linear_grpo_loss):
        got = run(f)
        for a_, b_ in zip(got, want):
            assert torch.equal(a_, b_)
    torch._dynamo.reset()
    got = run(torch.compile(ops.fused_linear_grpo_loss, backend="aot_eager", fullgraph=True))
    for a_, b_ in zip(got, want):
        assert torch.equal(a_, b_)
