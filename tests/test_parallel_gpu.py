"""The data-parallel step on one GPU (an NCCL group of one rank): the library's
per-rank operations (pl_fused_linear_grpo_temp, pl_count_ratio, pl_scale) in
the order dp_fused_linear_grpo runs them must give the single-GPU result, and
pl_count_ratio / pl_scale must apply a share that is not 1."""
import os
import socket

import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


@pytest.fixture(scope="module")
def group():
    import torch.distributed as dist
    os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
    os.environ["MASTER_PORT"] = str(_free_port())
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device("cuda:0"))
    yield dist.group.WORLD
    dist.destroy_process_group()


@pytest.mark.parametrize("red", [0, 1], ids=["bnpo", "grpo"])
def test_one_rank_equals_single_gpu_call(group, red):
    import rl_post_policy_b200 as pl
    from rl_post_policy_b200 import parallel
    bs, T, H, V = 3, 64, 128, 1000
    inp = synth.fused_inputs(bs, T, H, V, torch.bfloat16, 5150, bias=True, need_ref=True)
    inp["old_lp"] = (inp["old_noise"] - 7.0).float()
    g = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    out = parallel.dp_fused_linear_grpo(g["X"], g["W"], g["bias"], g["targets"], g["Xref"], g["Wref"],
                                        g["old_lp"], g["adv"], g["mask"], eps_lo=0.2, eps_hi=0.28, beta=0.04,
                                        reduction=red, group=group)
    ref = parallel.LibraryOps().local_step(g["X"], g["W"], g["bias"], g["targets"], g["Xref"], g["Wref"],
                                           g["old_lp"], g["adv"], g["mask"], 0.2, 0.28, 0.04, red)
    torch.cuda.synchronize()
    assert torch.equal(out["loss"], ref["loss"])
    for k in ("dX", "dW", "dbias"):
        assert torch.equal(out[k], ref[k]), k
    assert int(out["count"].item()) == (int(ref["n_valid"].item()) if red == pl.PL_BNPO else bs)


@pytest.mark.parametrize("red", [0, 1], ids=["bnpo", "grpo"])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32], ids=["bf16", "fp32"])
def test_one_rank_loss_step_equals_oracle(group, red, dtype):
    # dp_policy_loss on one rank: the share is exactly 1, so loss and gradient
    # are the loss kernel's own, and they match the oracle
    import numpy as np
    import oracle
    from rl_post_policy_b200 import parallel
    bs, seq = 6, 700
    inp = synth.loss_inputs(bs, seq, dtype, 6061, len_lo=1, len_hi=seq)
    g = {k: v.cuda() for k, v in inp.items()}
    out = parallel.dp_policy_loss(g["policy_lp"], g["old_lp"], g["ref_lp"], g["adv"], g["mask"], eps_lo=0.2,
                                  eps_hi=0.28, beta=0.04, reduction=red, group=group)
    torch.cuda.synchronize()
    want = oracle.policy_loss(inp["policy_lp"], inp["old_lp"], inp["ref_lp"], inp["adv"], inp["mask"],
                              eps_lo=0.2, eps_hi=0.28, beta=0.04, reduction=red)
    tol = 1e-5 if dtype == torch.float32 else 1e-3
    # these inputs keep the loss well away from a +/-A cancellation (|loss| > 0.5 sum|terms|)
    assert abs(want["loss"]) > 0.5 * want["abs_sum"]
    assert abs(out["loss"].item() - want["loss"]) <= tol * abs(want["loss"])
    w = want["grad"]
    # fp32: max abs 1e-6; bf16: one unit in the last place of the rounded oracle value.
    # A token whose ratio lies within 8 fp32 ulps of 1 + eps_hi may take either side of
    # the min() in fp32 (both are correct), so it is left out, as in the loss-kernel tests.
    lp_d, old_d = oracle.decode(inp["policy_lp"]), oracle.decode(inp["old_lp"])
    hi = np.float32(1.0) + np.float32(0.28)
    kink = np.abs(np.exp(lp_d - old_d) - float(hi)) <= 8 * float(np.spacing(hi))
    got = out["grad"].double().cpu().numpy()
    if dtype == torch.float32:
        err, bound = np.abs(got - w), 1e-6
    else:
        wr = torch.from_numpy(w).to(dtype).double().numpy()
        ax = np.abs(wr)
        ulp = np.exp2(np.maximum(np.floor(np.log2(np.where(ax > 0, ax, 1.0))), -126) - 7)
        err, bound = np.abs(got - wr) / ulp, 1.0
    bad = (err > bound) & ~kink
    assert not bad.any(), (int(bad.sum()), float(err[~kink].max()))
    assert int(out["count"].item()) == (want["n_valid"] if red == 0 else bs)


def test_count_ratio_and_scale():
    import rl_post_policy_b200 as pl
    from rl_post_policy_b200 import parallel
    ops = parallel.LibraryOps()
    for local, total, want in ((3, 12, 0.25), (0, 5, 0.2), (0, 0, 1.0), (7, 7, 1.0)):
        f = ops.ratio(torch.tensor([local], dtype=torch.int64, device="cuda"),
                      torch.tensor([total], dtype=torch.int64, device="cuda"))
        assert f.item() == pytest.approx(want, rel=1e-7)
    x = torch.linspace(-3, 3, 1001, device="cuda").to(torch.bfloat16)
    y = x.clone()
    ops.scale(y, torch.tensor([0.25], device="cuda"))
    assert torch.equal(y, (x.float() * 0.25).to(torch.bfloat16))
