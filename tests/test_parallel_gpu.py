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
