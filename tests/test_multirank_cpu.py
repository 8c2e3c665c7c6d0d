"""The multi-process side of bench.py on CPU, on two `gloo` ranks: the ranks
must agree on the max of their times and on the summed token count, the
barrier must pair up, and the bench's data-parallel step (one batch sharded by
sequences, the count and gradient all-reduces) must give the oracle's result on
the whole batch."""
import os
import socket
import subprocess
import sys
import textwrap

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def test_two_gloo_ranks_reduce_like_the_bench():
    script = textwrap.dedent(f"""
        import os, sys
        sys.path.insert(0, {ROOT!r})
        import torch
        import bench
        class A: pass
        ws, rank = bench.dist_init(A())
        assert ws == 2
        bench.barrier(ws)
        t = bench.max_over_ranks(10.0 + rank, ws)          # rank 1 is the slower one
        n = bench.sum_over_ranks(1024.0 * (rank + 1), ws)  # per-rank tokens
        print(f"RESULT {{rank}} {{t}} {{n}}", flush=True)
        import torch.distributed as dist
        dist.destroy_process_group()
    """)
    port = _free_port()
    procs = []
    for r in range(2):
        env = dict(os.environ, RANK=str(r), LOCAL_RANK=str(r), WORLD_SIZE="2", MASTER_ADDR="127.0.0.1",
                   MASTER_PORT=str(port), CUDA_VISIBLE_DEVICES="")
        procs.append(subprocess.Popen([sys.executable, "-c", script], env=env, stdout=subprocess.PIPE,
                                      stderr=subprocess.PIPE, text=True))
    outs = []
    for p in procs:
        out, err = p.communicate(timeout=120)
        assert p.returncode == 0, err
        outs.append(out)
    for r, out in enumerate(outs):
        line = [l for l in out.splitlines() if l.startswith("RESULT")][0].split()
        assert int(line[1]) == r
        assert float(line[2]) == 11.0
        assert float(line[3]) == 3072.0


DP_SCRIPT = textwrap.dedent("""
    import os, sys
    sys.path.insert(0, {root!r})
    import numpy as np
    import torch
    import torch.distributed as dist
    import bench, oracle, synth

    class A: pass
    ws, rank = bench.dist_init(A())
    assert ws == 2
    bs, T, H, V = 2, 6, 16, 40
    d = dict(bs=bs, T=T, H=H, V=V, N=bs * T, beta=0.04, dtype=torch.float32)

    def rank_inputs(r):
        inp = synth.fused_inputs(bs, T, H, V, torch.float32, 777 + r, bias=True, len_lo=0, len_hi=T,
                                 need_ref=True)
        _, lp, _ = oracle.lm_head_logprob(inp["X"], inp["W"], inp["bias"], inp["targets"])
        inp["old_lp"] = (torch.from_numpy(lp) + inp["old_noise"].double()).float()
        return inp

    inp = rank_inputs(rank)
    bench.broadcast_weights(inp, ws)           # rank 0's weights everywhere
    w0 = rank_inputs(0)
    assert torch.equal(inp["W"], w0["W"]) and torch.equal(inp["bias"], w0["bias"])

    class OracleOps:                            # the per-rank operations on the CPU
        def local_step(self, X, W, bias, targets, Xref, Wref, old_lp, adv, mask, eps_lo, eps_hi, beta,
                       reduction, **kw):
            o = oracle.fused_grpo(X, W, bias, targets, Xref, Wref, old_lp.reshape(mask.shape), adv, mask,
                                  eps_lo=eps_lo, eps_hi=eps_hi, beta=beta, reduction=reduction)
            t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).double()
            return {{"loss": torch.tensor([o["loss"]], dtype=torch.float64), "dX": t(o["dX"]),
                    "dW": t(o["dW"]), "dbias": t(o["dbias"]),
                    "n_valid": torch.tensor([o["n_valid"]], dtype=torch.int64)}}
        def ratio(self, local, total):
            return local.clamp(min=1).double() / total.clamp(min=1).double()
        def scale(self, t, f):
            t.mul_(f)

    step = bench.DataParallelStep(d, inp, ops=OracleOps())
    out = step()
    # the whole batch: both ranks' rows and old_lp as each rank drew them, rank 0's weights
    parts = [rank_inputs(r) for r in range(ws)]
    cat = lambda k: torch.cat([p[k] for p in parts])
    old = cat("old_lp")
    want = oracle.fused_grpo(cat("X"), w0["W"], w0["bias"], cat("targets"), cat("Xref"), w0["Wref"],
                             old.reshape(ws * bs, T), cat("adv"), cat("mask"), eps_lo=bench.EPS_LO,
                             eps_hi=bench.EPS_HI, beta=0.04, reduction=bench.GRPO)
    rel = lambda a, b: float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))
    assert abs(out["loss"].item() - want["loss"]) <= 1e-12 * max(1.0, abs(want["loss"]))
    assert rel(out["dW"].numpy(), want["dW"]) <= 1e-12
    assert rel(out["dbias"].numpy(), want["dbias"]) <= 1e-12
    rows = slice(rank * bs * T, (rank + 1) * bs * T)
    assert rel(out["dX"].numpy(), want["dX"][rows]) <= 1e-12
    assert int(out["count"].item()) == ws * bs
    print(f"RESULT {{rank}} {{out['loss'].item()!r}}", flush=True)
    dist.destroy_process_group()
""")


def test_data_parallel_step_of_the_bench_on_two_gloo_ranks():
    """bench.DataParallelStep (the multi-GPU arm of bench.py) on two gloo ranks,
    with the CPU oracle as each rank's local step: the rank count, the weight
    broadcast, the count all-reduce and the loss / dW / dbias all-reduce give the
    oracle's result on the whole batch."""
    script = DP_SCRIPT.format(root=ROOT)
    port = _free_port()
    procs = []
    for r in range(2):
        env = dict(os.environ, RANK=str(r), LOCAL_RANK=str(r), WORLD_SIZE="2", MASTER_ADDR="127.0.0.1",
                   MASTER_PORT=str(port), CUDA_VISIBLE_DEVICES="")
        procs.append(subprocess.Popen([sys.executable, "-c", script], env=env, stdout=subprocess.PIPE,
                                      stderr=subprocess.PIPE, text=True))
    outs = []
    for p in procs:
        out, err = p.communicate(timeout=300)
        assert p.returncode == 0, err[-3000:]
        outs.append(out)
    losses = []
    for r, out in enumerate(outs):
        line = [l for l in out.splitlines() if l.startswith("RESULT")][0].split()
        assert int(line[1]) == r
        losses.append(float(line[2]))
    assert losses[0] == losses[1]
