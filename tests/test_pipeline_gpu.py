"""InputPrefetcher: inputs copied one step ahead on a copy stream must give the
same results as inputs copied on the compute stream, batch for batch."""
import pytest
import torch

pytestmark = pytest.mark.gpu


def test_prefetched_inputs_match_direct_copies():
    from rl_post_policy_b200.pipeline import InputPrefetcher
    g = torch.Generator().manual_seed(5)
    batches = [{"a": torch.randn(1 << 20, generator=g).pin_memory(),
                "b": torch.randint(0, 100, (4096,), generator=g).pin_memory()} for _ in range(6)]
    templates = {k: v.cuda() for k, v in batches[0].items()}
    pf = InputPrefetcher(templates)
    outs = []
    pf.prefetch(batches[0])
    for i in range(len(batches)):
        dev = pf.next()
        if i + 1 < len(batches):
            pf.prefetch(batches[i + 1])
        # a compute step that reads the inputs (long enough to overlap the next copy)
        r = (dev["a"] * 2.0).sum() + dev["b"].sum().float()
        for _ in range(20):
            r = r + dev["a"].mul(1e-9).sum()
        outs.append(r)
        pf.release()
    pf.finish()
    torch.cuda.synchronize()
    for i, bt in enumerate(batches):
        a, b = bt["a"].cuda(), bt["b"].cuda()
        want = (a * 2.0).sum() + b.sum().float()
        for _ in range(20):
            want = want + a.mul(1e-9).sum()
        assert torch.equal(outs[i], want), i


def test_prefetcher_guards():
    from rl_post_policy_b200.pipeline import InputPrefetcher
    t = {"x": torch.zeros(8, device="cuda")}
    pf = InputPrefetcher(t)
    with pytest.raises(RuntimeError):
        pf.next()
    h = {"x": torch.ones(8).pin_memory()}
    pf.prefetch(h)
    pf.prefetch(h)
    with pytest.raises(RuntimeError):
        pf.prefetch(h)


def test_graphed_fused_step_matches_eager_calls():
    # the tiny fused workload: count, two GEMM launches, combine, dlogits, finalize in one graph
    import rl_post_policy_b200 as pl
    from rl_post_policy_b200.pipeline import GraphedCall
    import synth
    w = synth.WORKLOADS[0]
    bs, T, H, V = w["bs"], w["T"], w["H"], w["V"]
    inp = synth.fused_inputs(bs, T, H, V, torch.bfloat16, synth.seed_for(0), len_lo=1, len_hi=T, need_ref=True)
    g = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    g["old_lp"] = (g["old_noise"] - 5.0).float()
    N = bs * T
    mode = pl.PL_BF16 | pl.PL_GRPO
    wsb = pl.pl_fused_linear_grpo_workspace_bytes(bs, T, H, V, mode, 1, 0)
    ws = torch.zeros(wsb, dtype=torch.uint8, device="cuda")
    loss = torch.zeros(1, device="cuda")
    dX = torch.empty(N, H, dtype=torch.bfloat16, device="cuda")
    dW = torch.empty(V, H, dtype=torch.bfloat16, device="cuda")
    lp = torch.empty(N, device="cuda")

    def step():
        pl.check(pl.pl_fused_linear_grpo(g["X"], g["W"], None, g["targets"], g["Xref"], g["Wref"], g["old_lp"],
                                         g["adv"], g["mask"], bs, T, H, V, 0.2, 0.28, 0.04, mode, loss, dX, dW,
                                         None, lp, None, None, ws, wsb))

    step()
    torch.cuda.synchronize()
    want = (loss.clone(), dX.clone(), dW.clone(), lp.clone())
    gc = GraphedCall(step)
    loss.zero_(); dX.zero_(); dW.zero_(); lp.zero_()
    for _ in range(3):
        gc.replay()
    torch.cuda.synchronize()
    assert pl.pl_device_status(ws) == 0
    for a, b in zip((loss, dX, dW, lp), want):
        assert torch.equal(a, b)
    # new inputs copied into the captured buffers are picked up by the replay
    g["adv"].mul_(-1.0)
    gc.replay()
    torch.cuda.synchronize()
    got = (loss.clone(), dX.clone(), dW.clone())
    step()
    torch.cuda.synchronize()
    assert not torch.equal(got[0], want[0])
    for a, b in zip(got, (loss, dX, dW)):
        assert torch.equal(a, b)


def test_graphed_loss_kernel_matches_eager_calls():
    # the cooperative single-launch loss kernel captured in a graph
    import rl_post_policy_b200 as pl
    from rl_post_policy_b200.pipeline import GraphedCall
    import synth
    inp = synth.loss_inputs(16, 1024, torch.bfloat16, synth.seed_for(1), len_lo=64, len_hi=1024)
    d = {k: inp[k].cuda() for k in ("policy_lp", "old_lp", "ref_lp", "adv", "mask")}
    loss = torch.zeros(1, device="cuda")
    grad = torch.empty_like(d["policy_lp"])
    wsb = pl.pl_loss_workspace_bytes(16, 1024)
    ws = torch.zeros(wsb, dtype=torch.uint8, device="cuda")

    def call():
        pl.check(pl.pl_loss_ex(d["policy_lp"], d["old_lp"], d["ref_lp"], d["adv"], d["mask"], 16, 1024, 0.2,
                               0.28, 0.04, pl.PL_BF16 | pl.PL_BNPO, loss, grad, None, None, ws, wsb))

    call()
    torch.cuda.synchronize()
    want_loss, want_grad = loss.clone(), grad.clone()
    gc = GraphedCall(call)
    loss.zero_(); grad.zero_()
    for _ in range(5):
        gc.replay()
    torch.cuda.synchronize()
    assert pl.pl_device_status(ws) == 0
    assert torch.equal(loss, want_loss) and torch.equal(grad, want_grad)


def test_pl_init_lets_the_first_library_scratch_call_be_captured():
    # pl_init creates the per-stream scratch up front, so the very first pl_loss call
    # on that stream allocates nothing and can be captured into a graph
    import rl_post_policy_b200 as pl
    import synth
    s = torch.cuda.Stream()
    assert pl.pl_init(16, s) == 0
    inp = synth.loss_inputs(16, 512, torch.bfloat16, synth.seed_for(1, 3), len_lo=32, len_hi=512)
    d = {k: inp[k].cuda() for k in ("policy_lp", "old_lp", "ref_lp", "adv", "mask")}
    loss = torch.zeros(1, device="cuda")
    grad = torch.empty_like(d["policy_lp"])
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        pl.check(pl.pl_loss(d["policy_lp"], d["old_lp"], d["ref_lp"], d["adv"], d["mask"], 16, 512, 0.2, 0.28,
                            0.04, pl.PL_BF16 | pl.PL_GRPO, loss, grad))
    g.replay()
    torch.cuda.synchronize()
    lossb = torch.zeros(1, device="cuda")
    gradb = torch.empty_like(grad)
    wsb = pl.pl_loss_workspace_bytes(16, 512)
    ws = torch.zeros(wsb, dtype=torch.uint8, device="cuda")
    pl.check(pl.pl_loss_ex(d["policy_lp"], d["old_lp"], d["ref_lp"], d["adv"], d["mask"], 16, 512, 0.2, 0.28,
                           0.04, pl.PL_BF16 | pl.PL_GRPO, lossb, gradb, None, None, ws, wsb))
    torch.cuda.synchronize()
    assert torch.equal(loss, lossb) and torch.equal(grad, gradb)
