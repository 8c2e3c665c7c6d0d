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
    assert abs(out["loss"].item() - want["loss"]) <= tol * max(abs(want["loss"]), 1e-3 * want["abs_sum"])
    w = torch.from_numpy(want["grad"]).to(dtype).double().numpy()
    err = np.abs(out["grad"].double().cpu().numpy() - w)
    # fp32: the loss kernel's 1e-6; bf16: two units in the last place of the rounded oracle.
    # At most one token within rounding of a clip bound may take the other side of the min.
    bound = 1e-6 if dtype == torch.float32 else 2.0 ** -7 * np.abs(w) + 1e-9
    assert np.count_nonzero(err > bound) <= 1, float(err.max())
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
