"""The data-parallel steps (rl_post_policy_b200.parallel) on two and three
`gloo` CPU ranks.

Each rank takes its share of the sequences of one seeded batch (2 + 3, or
2 + 1 + 2, of 5 for the fused step).  The per-rank
operations are the CPU oracle (the fused loss and gradients of the rank's
shard, normalised by the shard's own count) and plain tensor arithmetic for
the ratio and the scale, so what is under test is the host-side sequence: the
count all-reduce, each rank's share and the loss / dW / dbias all-reduce.  The
result must equal the oracle on the whole batch, for BNPO (global valid-token
denominator) and GRPO (global sequence mean), with unequal shard sizes and a
fully masked sequence.
"""
import os
import socket
import subprocess
import sys
import textwrap

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


SCRIPT = textwrap.dedent("""
    import os, sys
    sys.path.insert(0, {root!r})
    import numpy as np
    import torch
    import torch.distributed as dist
    import oracle, synth
    from rl_post_policy_b200 import parallel
    import rl_post_policy_b200.binding as pl

    rank, ws = int(os.environ["RANK"]), int(os.environ["WORLD_SIZE"])
    dist.init_process_group("gloo", rank=rank, world_size=ws)
    red = {red}
    bs, T, H, V = 5, 12, 32, 96
    inp = synth.fused_inputs(bs, T, H, V, torch.float32, 4711, bias=True, len_lo=0, len_hi=T,
                             fully_masked_last=True, need_ref=True)
    _, logp, _ = oracle.lm_head_logprob(inp["X"], inp["W"], inp["bias"], inp["targets"])
    inp["old_lp"] = (torch.from_numpy(logp) + inp["old_noise"].double()).float()
    want = oracle.fused_grpo(inp["X"], inp["W"], inp["bias"], inp["targets"], inp["Xref"], inp["Wref"],
                             inp["old_lp"].reshape(bs, T), inp["adv"], inp["mask"], eps_lo=0.2, eps_hi=0.28,
                             beta=0.04, reduction=red)
    seqs = {shards}[rank]                               # unequal shards; the last holds the empty sequence
    rows = [r * T + t for r in seqs for t in range(T)]

    class OracleOps:
        def local_step(self, X, W, bias, targets, Xref, Wref, old_lp, adv, mask, eps_lo, eps_hi, beta,
                       reduction, **kw):
            o = oracle.fused_grpo(X, W, bias, targets, Xref, Wref, old_lp.reshape(mask.shape), adv, mask,
                                  eps_lo=eps_lo, eps_hi=eps_hi, beta=beta, reduction=reduction)
            t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).double()
            return {{"loss": torch.tensor([o["loss"]], dtype=torch.float64), "dX": t(o["dX"]),
                    "dW": t(o["dW"]), "dbias": t(o["dbias"]),
                    "n_valid": torch.tensor([o["n_valid"]], dtype=torch.int64)}}
        def ratio(self, local, total):
            return (local.clamp(min=1).double() / total.clamp(min=1).double())
        def scale(self, t, f):
            t.mul_(f)

    got = parallel.dp_fused_linear_grpo(
        inp["X"][rows], inp["W"], inp["bias"], inp["targets"][rows], inp["Xref"][rows], inp["Wref"],
        inp["old_lp"][rows], inp["adv"][list(seqs)], inp["mask"][list(seqs)], eps_lo=0.2, eps_hi=0.28,
        beta=0.04, reduction=red, ops=OracleOps())
    rel = lambda a, b: float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))
    assert abs(got["loss"].item() - want["loss"]) <= 1e-12 * max(1.0, abs(want["loss"])), (got["loss"], want["loss"])
    assert rel(got["dW"].numpy(), want["dW"]) <= 1e-12
    assert rel(got["dbias"].numpy(), want["dbias"]) <= 1e-12
    assert rel(got["dX"].numpy(), want["dX"][rows]) <= 1e-12
    expect_count = want["n_valid"] if red == pl.PL_BNPO else bs
    assert int(got["count"].item()) == expect_count
    print("RANK_OK", rank, flush=True)
    dist.destroy_process_group()
""")


SHARDS = {2: "[range(0, 2), range(2, 5)]", 3: "[range(0, 2), range(2, 3), range(3, 5)]"}


@pytest.mark.parametrize("world", [2, 3], ids=["2ranks", "3ranks"])
@pytest.mark.parametrize("red", [0, 1], ids=["bnpo", "grpo"])
def test_dp_step_matches_whole_batch_oracle(red, world):
    script = SCRIPT.format(root=ROOT, red=red, shards=SHARDS[world])
    port = _free_port()
    procs = []
    for r in range(world):
        env = dict(os.environ, RANK=str(r), LOCAL_RANK=str(r), WORLD_SIZE=str(world), MASTER_ADDR="127.0.0.1",
                   MASTER_PORT=str(port), CUDA_VISIBLE_DEVICES="")
        procs.append(subprocess.Popen([sys.executable, "-c", script], env=env, stdout=subprocess.PIPE,
                                      stderr=subprocess.PIPE, text=True))
    for p in procs:
        out, err = p.communicate(timeout=180)
        assert p.returncode == 0, err[-3000:]
        assert "RANK_OK" in out


LOSS_SCRIPT = textwrap.dedent("""
    import os, sys
    sys.path.insert(0, {root!r})
    import numpy as np
    import torch
    import torch.distributed as dist
    import oracle, synth
    from rl_post_policy_b200 import parallel

    rank, ws = int(os.environ["RANK"]), int(os.environ["WORLD_SIZE"])
    dist.init_process_group("gloo", rank=rank, world_size=ws)
    red, two_sided = {red}, {two_sided}
    bs, seq = 7, 40
    inp = synth.loss_inputs(bs, seq, torch.float32, 99, len_lo=1, len_hi=seq)
    inp["mask"][5] = 0                                  # a fully masked sequence
    kw = dict(eps_lo=0.2, eps_hi=0.28, beta=0.04, reduction=red, two_sided=two_sided)
    want = oracle.policy_loss(inp["policy_lp"], inp["old_lp"], inp["ref_lp"], inp["adv"], inp["mask"], **kw)
    seqs = {shards}[rank]                               # unequal shards; the last holds the empty sequence

    class OracleOps:
        def local_loss(self, lp, old, ref, adv, mask, eps_lo, eps_hi, beta, reduction, two_sided=False,
                       want_grad=True):
            o = oracle.policy_loss(lp, old, ref, adv, mask, eps_lo=eps_lo, eps_hi=eps_hi, beta=beta,
                                   reduction=reduction, two_sided=two_sided)
            return {{"loss": torch.tensor([o["loss"]], dtype=torch.float64),
                    "grad": torch.from_numpy(o["grad"]).double(),
                    "n_valid": torch.tensor([o["n_valid"]], dtype=torch.int64)}}
        def ratio(self, local, total):
            return local.clamp(min=1).double() / total.clamp(min=1).double()
        def scale(self, t, f):
            t.mul_(f)

    got = parallel.dp_policy_loss(inp["policy_lp"][seqs], inp["old_lp"][seqs], inp["ref_lp"][seqs],
                                  inp["adv"][seqs], inp["mask"][seqs], ops=OracleOps(), **kw)
    assert abs(got["loss"].item() - want["loss"]) <= 1e-12 * max(1.0, abs(want["loss"])), (got["loss"], want["loss"])
    err = np.abs(got["grad"].numpy() - want["grad"][seqs]).max()
    assert err <= 1e-15, err
    assert int(got["count"].item()) == (want["n_valid"] if red == 0 else bs)
    print("RANK_OK", rank, flush=True)
    dist.destroy_process_group()
""")


LOSS_SHARDS = {2: "[[0, 1, 2], [3, 4, 5, 6]]", 3: "[[0, 1], [2, 3, 4], [5, 6]]"}


@pytest.mark.parametrize("world", [2, 3], ids=["2ranks", "3ranks"])
@pytest.mark.parametrize("red,two_sided", [(0, False), (1, False), (1, True)], ids=["bnpo", "grpo", "grpo_two_sided"])
def test_dp_loss_step_matches_whole_batch_oracle(red, two_sided, world):
    script = LOSS_SCRIPT.format(root=ROOT, red=red, two_sided=two_sided, shards=LOSS_SHARDS[world])
    port = _free_port()
    procs = []
    for r in range(world):
        env = dict(os.environ, RANK=str(r), LOCAL_RANK=str(r), WORLD_SIZE=str(world), MASTER_ADDR="127.0.0.1",
                   MASTER_PORT=str(port), CUDA_VISIBLE_DEVICES="")
        procs.append(subprocess.Popen([sys.executable, "-c", script], env=env, stdout=subprocess.PIPE,
                                      stderr=subprocess.PIPE, text=True))
    for p in procs:
        out, err = p.communicate(timeout=180)
        assert p.returncode == 0, err[-3000:]
        assert "RANK_OK" in out
