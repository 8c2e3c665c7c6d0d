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
